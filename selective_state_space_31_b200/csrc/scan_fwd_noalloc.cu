// scan_fwd_noalloc.cu -- ssm_scan_fwd_noalloc: the chunked forward scan for
// callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at all: code that runs inside a
// memory-capped or pre-partitioned allocator (an inference server that owns
// every byte of the device up front), plugins loaded into a host process
// whose allocator must not be bypassed, and code paths that must not
// synchronise the device (cudaMalloc/cudaFree can).  They cannot create an
// ssm_scan_plan, whose workspace is allocated by ssm_scan_create.  This entry
// point runs the same chunked forward kernel with its scratch (the carried
// states between chunks, the per-chunk flags and the work counter) in a
// fixed file-scope device array instead, so it allocates nothing.
//
// The scratch array lives in every device that loads this library, until
// the process exits: kNoAllocScratchBytes (4 MiB).  All calls share it and it
// keeps the previous call's contents, so:
//   * calls that overlap on the GPU (two streams, or two host threads) race
//     on it and give wrong results: order them;
//   * the finished-CTA counter starts at zero (static initialisation) and
//     every launch returns it to zero when its last CTA finishes; the
//     per-chunk flags carry a launch counter that the same CTA advances, so
//     stale flags from an earlier call never match.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstddef>
#include <cstdint>
#include <mutex>

#include "ssm_scan.h"
#include "scan_params.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;
constexpr size_t kCtlBytes = 256;
constexpr int kMaxDevices = 64;
constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Test hook (ssm_scan_noalloc_set_debug): wait bound and dropped hand-over.
std::atomic<uint64_t> g_timeout_ns{kDefaultTimeoutNs};
std::atomic<int64_t> g_drop_unit{-1};

PFN_cuCtxGetCurrent_v4000 ctx_getter() {
  static PFN_cuCtxGetCurrent_v4000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 4000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
  });
  return fn;
}

// Device address of g_noalloc_scratch in the current context of `device`
// (host code must not use the symbol itself as an address).  Looked up with
// that device current and cached per device together with the context it was
// taken in: a new primary context (after cudaDeviceReset) reloads the module,
// so the address is looked up again.
void *scratch_address(int device) {
  static std::mutex mu;
  static void *addr[kMaxDevices] = {};
  static CUcontext ctx_of[kMaxDevices] = {};
  if (device < 0 || device >= kMaxDevices) return nullptr;
  CUcontext ctx = nullptr;
  auto get_ctx = ctx_getter();
  if (!get_ctx || get_ctx(&ctx) != CUDA_SUCCESS || !ctx) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[device] || ctx_of[device] != ctx) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    addr[device] = p;
    ctx_of[device] = ctx;
  }
  return addr[device];
}

// Launch shapes chosen before, per device and problem: repeat calls only
// encode tensor maps and launch.
struct ShapeKey {
  int device, in_dtype, out_dtype, ns;
  int64_t batch, seqlen, dim;
  bool zoh;
  bool operator==(const ShapeKey &o) const {
    return device == o.device && in_dtype == o.in_dtype && out_dtype == o.out_dtype &&
           ns == o.ns && batch == o.batch && seqlen == o.seqlen && dim == o.dim && zoh == o.zoh;
  }
};
constexpr int kShapeCache = 16;

bool cached_shape(const ShapeKey &key, int num_sms, ssm::FwdShape *out) {
  static std::mutex mu;
  static ShapeKey keys[kShapeCache];
  static ssm::FwdShape shapes[kShapeCache];
  static int used = 0, next = 0;
  {
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < used; ++i)
      if (keys[i] == key) {
        *out = shapes[i];
        return true;
      }
  }
  ssm::FwdShape fs;
  ssm::FwdOverrides o{0, 0, 0, 0};
  o.segments = 1;  // no carry pass: its maps would need more scratch
  if (ssm::choose_fwd_shape(key.in_dtype, key.out_dtype, key.batch, key.seqlen, key.dim, key.ns,
                            key.zoh, false, num_sms, o, &fs) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  std::lock_guard<std::mutex> lock(mu);
  keys[next] = key;
  shapes[next] = fs;
  next = (next + 1) % kShapeCache;
  used = std::min(used + 1, kShapeCache);
  *out = fs;
  return true;
}

PFN_cuTensorMapEncodeTiled_v12000 encoder_na() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool encode_na(CUtensorMap *m, ssm_dtype dt, const void *base, uint64_t d0, uint64_t d1,
               uint64_t d2, uint32_t box0, uint32_t box1) {
  auto enc = encoder_na();
  if (!enc) return false;
  const uint64_t es = dt == SSM_BF16 ? 2 : 4;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * es, d0 * d1 * es};
  cuuint32_t box[3] = {box0, box1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, dt == SSM_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
             3, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool al16(const void *p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

extern "C" SSM_API ssm_status ssm_scan_fwd_noalloc(
    const ssm_scan_desc *desc, const void *x, const void *delta, const float *delta_bias,
    const float *A, const void *B, const void *C, const float *D, const void *z,
    const float *h0, void *y, float *h_last, ssm_stream_t stream_) {
  if (!desc) return SSM_ERR_INVALID_ARG;
  const ssm_scan_desc &d = *desc;
  const uint32_t f = d.flags;
  if (d.batch < 1 || d.seqlen < 1 || d.dim < 1 || d.dstate < 1) return SSM_ERR_INVALID_ARG;
  if (d.batch > INT32_MAX || d.seqlen > INT32_MAX || d.dim > INT32_MAX) return SSM_ERR_UNSUPPORTED;
  if ((d.in_dtype != SSM_F32 && d.in_dtype != SSM_BF16) ||
      (d.out_dtype != SSM_F32 && d.out_dtype != SSM_BF16))
    return SSM_ERR_INVALID_ARG;
  constexpr uint32_t known = SSM_HAS_Z | SSM_HAS_D | SSM_DELTA_SOFTPLUS | SSM_HAS_DELTA_BIAS |
                             SSM_HAS_H0 | SSM_WANT_HLAST | SSM_ZOH;
  if (f & ~known) return SSM_ERR_INVALID_ARG;
  // the fast-path shape rules of the chunked kernel (dstate checked before
  // it is narrowed)
  if (d.dstate != 4 && d.dstate != 8 && d.dstate != 16) return SSM_ERR_UNSUPPORTED;
  const int ns = (int)d.dstate;
  const size_t ei = d.in_dtype == SSM_BF16 ? 2 : 4, eo = d.out_dtype == SSM_BF16 ? 2 : 4;
  if (ns == 4 && d.in_dtype == SSM_BF16) return SSM_ERR_UNSUPPORTED;
  if (d.in_dtype == SSM_F32 && d.out_dtype == SSM_BF16) return SSM_ERR_UNSUPPORTED;
  if ((d.dim * ei) % 16 || (ns * ei) % 16 || (d.dim * eo) % 16) return SSM_ERR_UNSUPPORTED;
  if (!x || !delta || !A || !B || !C || !y) return SSM_ERR_INVALID_ARG;
  if (((f & SSM_HAS_Z) != 0) != (z != nullptr) || ((f & SSM_HAS_D) != 0) != (D != nullptr) ||
      ((f & SSM_HAS_DELTA_BIAS) != 0) != (delta_bias != nullptr) ||
      ((f & SSM_HAS_H0) != 0) != (h0 != nullptr) ||
      ((f & SSM_WANT_HLAST) != 0) != (h_last != nullptr))
    return SSM_ERR_INVALID_ARG;
  if (!al16(x) || !al16(delta) || !al16(z) || !al16(B) || !al16(C) || !al16(y))
    return SSM_ERR_MISALIGNED;

  int device = 0, num_sms = 0;
  if (cudaGetDevice(&device) != cudaSuccess ||
      cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess) {
    cudaGetLastError();
    return SSM_ERR_CUDA;
  }
  // launch shape: the same choice a plan makes by default (cached)
  ssm::FwdShape fs;
  const ShapeKey key{device, (int)d.in_dtype, (int)d.out_dtype, ns, d.batch, d.seqlen, d.dim,
                     (f & SSM_ZOH) != 0};
  if (!cached_shape(key, num_sms, &fs)) return SSM_ERR_UNSUPPORTED;
  const int DT = fs.DT, warps = fs.ls.warps, TT = fs.ls.tt;
  const int nDT = (int)((d.dim + DT - 1) / DT);
  const int64_t rows = fs.rows;
  // scratch layout: [Control | flags rows*warps u64 | states rows*DT*N f32]
  const size_t fl_bytes = (size_t)rows * warps * sizeof(unsigned long long);
  const size_t st_off = (kCtlBytes + fl_bytes + 255) / 256 * 256;
  const size_t need = st_off + (size_t)rows * DT * ns * sizeof(float);
  if (need > kNoAllocScratchBytes) return SSM_ERR_UNSUPPORTED;  // beyond the fixed scratch
  const ssm::LaunchShape ls = fs.ls;

  unsigned char *base = static_cast<unsigned char *>(scratch_address(device));
  if (!base) return SSM_ERR_CUDA;

  ssm::TmaMaps maps;
  const uint64_t Bn = d.batch, L = d.seqlen, Dm = d.dim, N = (uint64_t)ns;
  if (!encode_na(&maps.x, d.in_dtype, x, Dm, L, Bn, DT, TT) ||
      !encode_na(&maps.dt, d.in_dtype, delta, Dm, L, Bn, DT, TT) ||
      !encode_na(&maps.z, d.in_dtype, z ? z : x, Dm, L, Bn, DT, TT) ||
      !encode_na(&maps.B, d.in_dtype, B, N, L, Bn, (uint32_t)N, TT) ||
      !encode_na(&maps.C, d.in_dtype, C, N, L, Bn, (uint32_t)N, TT))
    return SSM_ERR_CUDA;

  ssm::FwdParams p{};
  p.Bsz = (int)d.batch; p.L = (int)d.seqlen; p.D = (int)d.dim; p.N = ns;
  p.DT = DT; p.nDT = nDT; p.rows = (int)rows; p.S = fs.S;
  p.M = 1; p.SPS = fs.S; p.nq = 0; p.nsub_row = 0;
  p.agg_h = nullptr; p.agg_s = nullptr;
  p.conv_w = nullptr; p.conv_b = nullptr; p.xconv = nullptr;
  p.PL = fs.PL; p.items = (int)(rows * fs.parts);
  p.softplus = (f & SSM_DELTA_SOFTPLUS) != 0;
  p.has_z = (f & SSM_HAS_Z) != 0;
  p.has_D = (f & SSM_HAS_D) != 0;
  p.has_bias = (f & SSM_HAS_DELTA_BIAS) != 0;
  p.has_h0 = (f & SSM_HAS_H0) != 0;
  p.want_hlast = (f & SSM_WANT_HLAST) != 0;
  p.zoh = (f & SSM_ZOH) != 0;
  p.A = A; p.Dv = D; p.bias = delta_bias; p.h0 = h0; p.h_last = h_last; p.y = y;
  p.ctl = reinterpret_cast<ssm::Control *>(base);
  p.ws_flags = reinterpret_cast<unsigned long long *>(base + kCtlBytes);
  p.ws_state = reinterpret_cast<float *>(base + st_off);
  p.timeout_ns = g_timeout_ns.load();
  p.drop_unit = g_drop_unit.load();
  const cudaError_t e = ssm::launch_fwd_tma((int)d.in_dtype, (int)d.out_dtype, ls, maps, p,
                                            reinterpret_cast<cudaStream_t>(stream_));
  return e == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

extern "C" SSM_API ssm_status ssm_scan_noalloc_status(void) {
  int device = 0;
  if (cudaGetDevice(&device) != cudaSuccess) {
    cudaGetLastError();
    return SSM_ERR_CUDA;
  }
  if (!scratch_address(device)) return SSM_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return SSM_ERR_CUDA;
  const size_t off = offsetof(ssm::Control, status);
  int st = 0;
  if (cudaMemcpyFromSymbol(&st, g_noalloc_scratch, sizeof(int), off) != cudaSuccess)
    return SSM_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_noalloc_scratch, &zero, sizeof(int), off) != cudaSuccess)
    return SSM_ERR_CUDA;
  return (ssm_status)st;
}

extern "C" SSM_API ssm_status ssm_scan_noalloc_set_debug(uint64_t wait_timeout_ns,
                                                          int64_t drop_unit) {
  g_timeout_ns.store(wait_timeout_ns ? wait_timeout_ns : kDefaultTimeoutNs);
  g_drop_unit.store(drop_unit);
  return SSM_OK;
}
