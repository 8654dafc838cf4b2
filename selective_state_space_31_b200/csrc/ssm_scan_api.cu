// ssm_scan_api.cu -- the C ABI declared in include/ssm_scan.h: argument
// validation, plan (launch shape + workspace), tensor-map encoding and
// dispatch to the kernels.  Host code only; every step of the scan runs in
// the CUDA kernels of this library.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <new>

#include "ssm_scan.h"
#include "scan_params.h"
#include "scan_bwd.h"

namespace {

constexpr uint32_t kKnownFlags = SSM_HAS_Z | SSM_HAS_D | SSM_DELTA_SOFTPLUS | SSM_HAS_DELTA_BIAS |
                                 SSM_HAS_H0 | SSM_WANT_HLAST | SSM_A_DIRECT | SSM_ZOH;
constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;
constexpr int kMaxDstate = 64;

enum Path { PATH_TMA = 0, PATH_GENERAL = 1, PATH_DIRECT = 2 };

size_t dtype_size(ssm_dtype t) { return t == SSM_BF16 ? 2 : 4; }

// Restores the caller's current device on scope exit.
struct DeviceGuard {
  int prev = -1;
  bool ok = false;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) return;
    ok = prev == dev || cudaSetDevice(dev) == cudaSuccess;
  }
  ~DeviceGuard() {
    if (ok && prev >= 0) cudaSetDevice(prev);
  }
};

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
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

// 3-d tiled map over a row-major (d2, d1, d0) tensor, d0 innermost.
bool encode3d(CUtensorMap *m, ssm_dtype dt, const void *base, uint64_t d0, uint64_t d1,
              uint64_t d2, uint32_t box0, uint32_t box1) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  const uint64_t es = dtype_size(dt);
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * es, d0 * d1 * es};
  cuuint32_t box[3] = {box0, box1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUtensorMapDataType t =
      dt == SSM_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  return enc(m, t, 3, const_cast<void *>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void *p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

struct ssm_scan_plan {
  ssm_scan_desc desc{};
  int device = 0;
  int num_sms = 0;
  int path = PATH_GENERAL;
  ssm::LaunchShape ls{};
  int DT = 0, nDT = 0, S = 0, PL = 0, parts = 0;
  int64_t rows = 0, units = 0;
  ssm_scan_config cfg{};  // user overrides
  ssm::Control *ctl = nullptr;
  int ring = 0;  // stage slots of the fused kernel's TMA ring
  float *ws_ck = nullptr;  // backward checkpoints (allocated by the first ssm_scan_bwd)
  size_t ws_ck_bytes = 0;
  float *ws_state = nullptr;
  unsigned long long *ws_flags = nullptr;
  size_t ws_state_bytes = 0, ws_flag_bytes = 0;
  uint64_t timeout_ns = kDefaultTimeoutNs;
  int64_t drop_unit = -1;
};

namespace {

ssm_status validate_desc(const ssm_scan_desc *d) {
  if (!d) return SSM_ERR_INVALID_ARG;
  if (d->batch < 0 || d->seqlen < 0 || d->dim < 0 || d->dstate < 1) return SSM_ERR_INVALID_ARG;
  if (d->batch > INT32_MAX || d->seqlen > INT32_MAX || d->dim > INT32_MAX) return SSM_ERR_UNSUPPORTED;
  if ((d->in_dtype != SSM_F32 && d->in_dtype != SSM_BF16) ||
      (d->out_dtype != SSM_F32 && d->out_dtype != SSM_BF16))
    return SSM_ERR_INVALID_ARG;
  if (d->flags & ~kKnownFlags) return SSM_ERR_INVALID_ARG;
  if (d->flags & SSM_A_DIRECT) {
    if (d->dstate != 1) return SSM_ERR_INVALID_ARG;
    if (d->flags & (SSM_HAS_Z | SSM_HAS_D | SSM_DELTA_SOFTPLUS | SSM_HAS_DELTA_BIAS | SSM_ZOH))
      return SSM_ERR_INVALID_ARG;
  }
  if (d->dstate > kMaxDstate) return SSM_ERR_UNSUPPORTED;
  return SSM_OK;
}

bool tma_eligible(const ssm_scan_desc &d) {
  if (d.flags & SSM_A_DIRECT) return false;
  if (d.batch == 0 || d.seqlen == 0 || d.dim == 0) return false;
  const size_t ei = dtype_size(d.in_dtype);
  if (d.in_dtype == SSM_F32 && d.out_dtype == SSM_BF16) return false;  // no such variant
  if (d.dstate != 4 && d.dstate != 8 && d.dstate != 16) return false;
  if (d.dstate == 4 && d.in_dtype == SSM_BF16) return false;
  if ((d.dim * ei) % 16 != 0 || (d.dstate * ei) % 16 != 0) return false;
  if ((d.dim * dtype_size(d.out_dtype)) % 16 != 0) return false;
  return true;
}

// Choose the launch shape of the fused kernel (shared with the
// allocation-free entry point) and size the workspace.
ssm_status plan_tma(ssm_scan_plan *pl) {
  const ssm_scan_desc &d = pl->desc;
  const int ns = (int)d.dstate;
  if (pl->cfg.tile_t && pl->cfg.tile_t != 16 && pl->cfg.tile_t != 32 && pl->cfg.tile_t != 64)
    return SSM_ERR_INVALID_ARG;
  const ssm::FwdOverrides o{pl->cfg.lanes_per_chan, pl->cfg.warps_per_cta, pl->cfg.tile_t,
                            pl->cfg.grid};
  ssm::FwdShape fs;
  if (ssm::choose_fwd_shape((int)d.in_dtype, (int)d.out_dtype, d.batch, d.seqlen, d.dim, ns,
                            (d.flags & SSM_ZOH) != 0, pl->num_sms, o, &fs) != cudaSuccess) {
    cudaGetLastError();
    return SSM_ERR_UNSUPPORTED;  // no variant fits (or bad override)
  }
  // workspace: carried state per (row, channel, n) and a flag per (row, warp)
  const size_t st_bytes = (size_t)fs.rows * fs.DT * ns * sizeof(float);
  const size_t fl_bytes = (size_t)fs.rows * fs.ls.warps * sizeof(unsigned long long);
  if (st_bytes > pl->ws_state_bytes) {
    if (pl->ws_state) cudaFree(pl->ws_state);
    pl->ws_state = nullptr;
    pl->ws_state_bytes = 0;
    if (cudaMalloc(&pl->ws_state, st_bytes) != cudaSuccess) return SSM_ERR_OOM;
    pl->ws_state_bytes = st_bytes;
  }
  if (fl_bytes > pl->ws_flag_bytes) {
    if (pl->ws_flags) cudaFree(pl->ws_flags);
    pl->ws_flags = nullptr;
    pl->ws_flag_bytes = 0;
    if (cudaMalloc(&pl->ws_flags, fl_bytes) != cudaSuccess) return SSM_ERR_OOM;
    pl->ws_flag_bytes = fl_bytes;
  }
  // flags start below every epoch tag (epochs start at 1)
  if (cudaMemset(pl->ws_flags, 0, pl->ws_flag_bytes) != cudaSuccess) return SSM_ERR_CUDA;
  pl->ls = fs.ls;
  pl->DT = fs.DT;
  pl->nDT = (int)((d.dim + fs.DT - 1) / fs.DT);
  pl->S = fs.S;
  pl->PL = fs.PL;
  pl->parts = fs.parts;
  pl->ring = fs.ring;
  pl->rows = fs.rows;
  pl->units = fs.rows * fs.S;
  return SSM_OK;
}

ssm_status make_plan(ssm_scan_plan *pl) {
  if (pl->desc.flags & SSM_A_DIRECT) {
    pl->path = PATH_DIRECT;
    return SSM_OK;
  }
  if (tma_eligible(pl->desc)) {
    pl->path = PATH_TMA;
    return plan_tma(pl);
  }
  pl->path = PATH_GENERAL;
  return SSM_OK;
}

ssm_status map_cuda(cudaError_t e) { return e == cudaSuccess ? SSM_OK : SSM_ERR_CUDA; }

}  // namespace

extern "C" {

const char *ssm_status_string(ssm_status s) {
  switch (s) {
    case SSM_OK: return "success";
    case SSM_ERR_INVALID_ARG: return "invalid argument";
    case SSM_ERR_UNSUPPORTED: return "unsupported problem";
    case SSM_ERR_MISALIGNED: return "misaligned pointer";
    case SSM_ERR_CUDA: return "CUDA runtime error";
    case SSM_ERR_TIMEOUT: return "device-side wait timed out";
    case SSM_ERR_OOM: return "out of device memory";
    default: return "unknown status";
  }
}

int ssm_scan_version(void) { return 100; }

ssm_status ssm_scan_create(ssm_scan_plan **plan, const ssm_scan_desc *desc, int device) {
  if (!plan) return SSM_ERR_INVALID_ARG;
  *plan = nullptr;
  const ssm_status v = validate_desc(desc);
  if (v != SSM_OK) return v;
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || device < 0 || device >= ndev) {
    cudaGetLastError();
    return SSM_ERR_CUDA;
  }
  DeviceGuard guard(device);
  if (!guard.ok) return SSM_ERR_CUDA;
  ssm_scan_plan *pl = new (std::nothrow) ssm_scan_plan();
  if (!pl) return SSM_ERR_OOM;
  pl->desc = *desc;
  pl->device = device;
  if (cudaDeviceGetAttribute(&pl->num_sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess) {
    delete pl;
    return SSM_ERR_CUDA;
  }
  if (cudaMalloc(&pl->ctl, sizeof(ssm::Control)) != cudaSuccess) {
    delete pl;
    return SSM_ERR_OOM;
  }
  ssm::Control init{};
  init.epoch = 1;
  if (cudaMemcpy(pl->ctl, &init, sizeof(init), cudaMemcpyHostToDevice) != cudaSuccess) {
    cudaFree(pl->ctl);
    delete pl;
    return SSM_ERR_CUDA;
  }
  const ssm_status s = make_plan(pl);
  if (s != SSM_OK) {
    ssm_scan_destroy(pl);
    return s;
  }
  *plan = pl;
  return SSM_OK;
}

ssm_status ssm_scan_destroy(ssm_scan_plan *pl) {
  if (!pl) return SSM_ERR_INVALID_ARG;
  {
    DeviceGuard guard(pl->device);
    cudaDeviceSynchronize();
    if (pl->ctl) cudaFree(pl->ctl);
    if (pl->ws_ck) cudaFree(pl->ws_ck);
    if (pl->ws_state) cudaFree(pl->ws_state);
    if (pl->ws_flags) cudaFree(pl->ws_flags);
  }
  delete pl;
  return SSM_OK;
}

ssm_status ssm_scan_get_info(const ssm_scan_plan *pl, ssm_scan_info *info) {
  if (!pl || !info) return SSM_ERR_INVALID_ARG;
  std::memset(info, 0, sizeof(*info));
  info->path = pl->path;
  if (pl->path == PATH_TMA) {
    info->lanes_per_chan = pl->ls.lpc;
    info->warps_per_cta = pl->ls.warps;
    info->tile_t = pl->ls.tt;
    info->stages = pl->ring;
    info->stages_per_row = pl->S;
    info->chans_per_cta = pl->DT;
    info->grid = pl->ls.grid;
    info->rows = pl->rows;
    info->units = pl->units;
    info->parts_per_row = pl->parts;
    info->stages_per_part = pl->PL;
    info->smem_bytes = pl->ls.smem;
  }
  info->workspace_bytes = pl->ws_state_bytes + pl->ws_flag_bytes + sizeof(ssm::Control);
  return SSM_OK;
}

ssm_status ssm_scan_set_config(ssm_scan_plan *pl, const ssm_scan_config *cfg) {
  if (!pl || !cfg) return SSM_ERR_INVALID_ARG;
  if (cfg->lanes_per_chan < 0 || cfg->warps_per_cta < 0 || cfg->grid < 0 || cfg->tile_t < 0)
    return SSM_ERR_INVALID_ARG;
  DeviceGuard guard(pl->device);
  if (!guard.ok) return SSM_ERR_CUDA;
  const ssm_scan_config old = pl->cfg;
  pl->cfg = *cfg;
  if (pl->path != PATH_TMA) return SSM_OK;
  if (cudaDeviceSynchronize() != cudaSuccess) return SSM_ERR_CUDA;
  const ssm_status s = plan_tma(pl);
  if (s != SSM_OK) {
    pl->cfg = old;
    plan_tma(pl);
  }
  return s;
}

ssm_status ssm_scan_set_debug(ssm_scan_plan *pl, uint64_t wait_timeout_ns, int64_t drop_unit) {
  if (!pl) return SSM_ERR_INVALID_ARG;
  pl->timeout_ns = wait_timeout_ns ? wait_timeout_ns : kDefaultTimeoutNs;
  pl->drop_unit = drop_unit;
  return SSM_OK;
}

ssm_status ssm_scan_get_status(ssm_scan_plan *pl) {
  if (!pl) return SSM_ERR_INVALID_ARG;
  DeviceGuard guard(pl->device);
  if (!guard.ok) return SSM_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return SSM_ERR_CUDA;
  int st = 0;
  if (cudaMemcpy(&st, &pl->ctl->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return SSM_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpy(&pl->ctl->status, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
    return SSM_ERR_CUDA;
  return (ssm_status)st;
}

ssm_status ssm_scan_fwd(ssm_scan_plan *pl, const void *x, const void *delta,
                        const float *delta_bias, const void *A, const void *B, const void *C,
                        const float *D, const void *z, const float *h0, void *y, float *h_last,
                        ssm_stream_t stream_) {
  if (!pl) return SSM_ERR_INVALID_ARG;
  const ssm_scan_desc &d = pl->desc;
  const uint32_t f = d.flags;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  // Pointer checks apply to tensors that have elements: a zero-size tensor
  // may legitimately be passed as NULL.
  const bool has_tokens = d.batch * d.seqlen * d.dim != 0;  // x, delta, z, y, B, C
  const bool has_chans = d.batch * d.dim != 0;              // h0, h_last, A, D, bias
  if (has_chans) {
    if (((f & SSM_HAS_H0) != 0) != (h0 != nullptr)) return SSM_ERR_INVALID_ARG;
    if (((f & SSM_WANT_HLAST) != 0) != (h_last != nullptr)) return SSM_ERR_INVALID_ARG;
  }
  if (has_tokens && (!x || !A || !B || !C || !y)) return SSM_ERR_INVALID_ARG;
  if (f & SSM_A_DIRECT) {
    if (delta || delta_bias || D || z) return SSM_ERR_INVALID_ARG;
  } else {
    if (has_tokens && !delta) return SSM_ERR_INVALID_ARG;
    if (has_tokens && (((f & SSM_HAS_Z) != 0) != (z != nullptr))) return SSM_ERR_INVALID_ARG;
    if (has_chans) {
      if (!A) return SSM_ERR_INVALID_ARG;
      if (((f & SSM_HAS_D) != 0) != (D != nullptr)) return SSM_ERR_INVALID_ARG;
      if (((f & SSM_HAS_DELTA_BIAS) != 0) != (delta_bias != nullptr)) return SSM_ERR_INVALID_ARG;
    }
  }
  if (d.batch == 0 || d.dim == 0) return SSM_OK;
  DeviceGuard guard(pl->device);
  if (!guard.ok) return SSM_ERR_CUDA;

  if (pl->path == PATH_DIRECT) {
    ssm::DirectParams p{};
    p.Bsz = (int)d.batch; p.L = (int)d.seqlen; p.D = (int)d.dim;
    p.in_bf16 = d.in_dtype == SSM_BF16;
    p.out_bf16 = d.out_dtype == SSM_BF16;
    p.x = x; p.A = A; p.B = B; p.C = C; p.h0 = h0; p.y = y; p.h_last = h_last;
    return map_cuda(ssm::launch_direct(p, stream));
  }

  const bool aligned = aligned16(x) && aligned16(delta) && aligned16(z) && aligned16(B) &&
                       aligned16(C) && aligned16(y);
  if (pl->path == PATH_TMA && aligned) {
    ssm::TmaMaps maps;
    const uint64_t Bn = d.batch, L = d.seqlen, Dm = d.dim, N = d.dstate;
    const uint32_t DT = (uint32_t)pl->DT, TT = (uint32_t)pl->ls.tt;
    if (!encode3d(&maps.x, d.in_dtype, x, Dm, L, Bn, DT, TT) ||
        !encode3d(&maps.dt, d.in_dtype, delta, Dm, L, Bn, DT, TT) ||
        !encode3d(&maps.z, d.in_dtype, z ? z : x, Dm, L, Bn, DT, TT) ||
        !encode3d(&maps.B, d.in_dtype, B, N, L, Bn, (uint32_t)N, TT) ||
        !encode3d(&maps.C, d.in_dtype, C, N, L, Bn, (uint32_t)N, TT))
      return SSM_ERR_CUDA;
    ssm::FwdParams p{};
    p.Bsz = (int)d.batch; p.L = (int)d.seqlen; p.D = (int)d.dim; p.N = (int)d.dstate;
    p.DT = pl->DT; p.nDT = pl->nDT; p.rows = (int)pl->rows; p.S = pl->S;
    p.PL = pl->PL; p.items = (int)(pl->rows * pl->parts);
    p.softplus = (f & SSM_DELTA_SOFTPLUS) != 0;
    p.has_z = (f & SSM_HAS_Z) != 0;
    p.has_D = (f & SSM_HAS_D) != 0;
    p.has_bias = (f & SSM_HAS_DELTA_BIAS) != 0;
    p.has_h0 = (f & SSM_HAS_H0) != 0;
    p.want_hlast = (f & SSM_WANT_HLAST) != 0;
    p.zoh = (f & SSM_ZOH) != 0;
    p.A = static_cast<const float *>(A);
    p.Dv = D; p.bias = delta_bias; p.h0 = h0; p.h_last = h_last; p.y = y;
    p.ws_state = pl->ws_state; p.ws_flags = pl->ws_flags; p.ctl = pl->ctl;
    p.timeout_ns = pl->timeout_ns;
    p.drop_unit = pl->drop_unit;
    return map_cuda(ssm::launch_fwd_tma((int)d.in_dtype, (int)d.out_dtype, pl->ls, maps, p, stream));
  }

  ssm::GenericParams p{};
  p.Bsz = (int)d.batch; p.L = (int)d.seqlen; p.D = (int)d.dim; p.N = (int)d.dstate;
  p.softplus = f & SSM_DELTA_SOFTPLUS;
  p.has_z = f & SSM_HAS_Z;
  p.has_D = f & SSM_HAS_D;
  p.has_bias = f & SSM_HAS_DELTA_BIAS;
  p.has_h0 = f & SSM_HAS_H0;
  p.want_hlast = f & SSM_WANT_HLAST;
  p.zoh = f & SSM_ZOH;
  p.in_bf16 = d.in_dtype == SSM_BF16;
  p.out_bf16 = d.out_dtype == SSM_BF16;
  p.x = x; p.dt = delta; p.z = z; p.B = B; p.C = C;
  p.A = static_cast<const float *>(A);
  p.Dv = D; p.bias = delta_bias; p.h0 = h0; p.y = y; p.h_last = h_last;
  return map_cuda(ssm::launch_fwd_general(p, stream));
}

ssm_status ssm_scan_bwd(ssm_scan_plan *pl, const void *x, const void *delta,
                        const float *delta_bias, const float *A, const void *B, const void *C,
                        const float *D, const void *z, const float *h0, const void *dy,
                        const float *dh_last, float *dx, float *ddelta, float *ddelta_bias,
                        float *dA, float *dB, float *dC, float *dD, float *dz, float *dh0,
                        ssm_stream_t stream_) {
  if (!pl) return SSM_ERR_INVALID_ARG;
  const ssm_scan_desc &d = pl->desc;
  const uint32_t f = d.flags;
  if (f & (SSM_ZOH | SSM_A_DIRECT)) return SSM_ERR_UNSUPPORTED;
  const bool has_tokens = d.batch * d.seqlen * d.dim != 0;
  const bool has_chans = d.batch * d.dim != 0;
  if (has_tokens && (!x || !delta || !B || !C || !dy || !dx || !ddelta || !dB || !dC))
    return SSM_ERR_INVALID_ARG;
  if (d.dim != 0 && (!A || !dA)) return SSM_ERR_INVALID_ARG;
  if (has_tokens && (((f & SSM_HAS_Z) != 0) != (z != nullptr) ||
                     ((f & SSM_HAS_Z) != 0) != (dz != nullptr)))
    return SSM_ERR_INVALID_ARG;
  if (d.dim != 0 && (((f & SSM_HAS_D) != 0) != (D != nullptr) ||
                     ((f & SSM_HAS_D) != 0) != (dD != nullptr) ||
                     ((f & SSM_HAS_DELTA_BIAS) != 0) != (delta_bias != nullptr) ||
                     ((f & SSM_HAS_DELTA_BIAS) != 0) != (ddelta_bias != nullptr)))
    return SSM_ERR_INVALID_ARG;
  if (has_chans && ((f & SSM_HAS_H0) != 0) != (h0 != nullptr)) return SSM_ERR_INVALID_ARG;
  if (d.dim == 0) return SSM_OK;
  DeviceGuard guard(pl->device);
  if (!guard.ok) return SSM_ERR_CUDA;
  const int64_t nck = (d.seqlen + ssm::kBwdChunk - 1) / ssm::kBwdChunk;
  const size_t need = (size_t)(d.batch * d.dim * nck * d.dstate) * sizeof(float);
  if (need > pl->ws_ck_bytes) {
    if (pl->ws_ck) cudaFree(pl->ws_ck);
    pl->ws_ck = nullptr;
    pl->ws_ck_bytes = 0;
    if (cudaMalloc(&pl->ws_ck, need) != cudaSuccess) {
      cudaGetLastError();
      return SSM_ERR_OOM;
    }
    pl->ws_ck_bytes = need;
  }
  ssm::BwdParams p{};
  p.Bsz = (int)d.batch; p.L = (int)d.seqlen; p.D = (int)d.dim; p.N = (int)d.dstate;
  p.softplus = f & SSM_DELTA_SOFTPLUS;
  p.has_z = f & SSM_HAS_Z;
  p.has_D = f & SSM_HAS_D;
  p.has_bias = f & SSM_HAS_DELTA_BIAS;
  p.has_h0 = f & SSM_HAS_H0;
  p.in_bf16 = d.in_dtype == SSM_BF16;
  p.out_bf16 = d.out_dtype == SSM_BF16;
  p.x = x; p.dt = delta; p.z = z; p.B = B; p.C = C; p.dy = dy;
  p.A = A; p.Dv = D; p.bias = delta_bias; p.h0 = h0; p.dh_last = dh_last;
  p.dx = dx; p.ddelta = ddelta; p.dz = dz; p.dB = dB; p.dC = dC; p.dA = dA; p.dD = dD;
  p.dbias = ddelta_bias; p.dh0 = dh0; p.ws_ck = pl->ws_ck;
  return map_cuda(ssm::launch_bwd(p, reinterpret_cast<cudaStream_t>(stream_)));
}

ssm_status ssm_scan_step(ssm_scan_plan *pl, const void *x, const void *delta,
                         const float *delta_bias, const float *A, const void *B, const void *C,
                         const float *D, const void *z, float *state, void *y,
                         ssm_stream_t stream_) {
  if (!pl) return SSM_ERR_INVALID_ARG;
  const ssm_scan_desc &d = pl->desc;
  const uint32_t f = d.flags;
  if (f & SSM_A_DIRECT) return SSM_ERR_INVALID_ARG;
  const bool empty = d.batch * d.dim == 0;
  if (!empty && (!x || !delta || !A || !B || !C || !state || !y)) return SSM_ERR_INVALID_ARG;
  if (((f & SSM_HAS_Z) != 0) != (z != nullptr)) return SSM_ERR_INVALID_ARG;
  if (((f & SSM_HAS_D) != 0) != (D != nullptr)) return SSM_ERR_INVALID_ARG;
  if (((f & SSM_HAS_DELTA_BIAS) != 0) != (delta_bias != nullptr)) return SSM_ERR_INVALID_ARG;
  if (empty) return SSM_OK;
  DeviceGuard guard(pl->device);
  if (!guard.ok) return SSM_ERR_CUDA;
  ssm::StepParams p{};
  p.Bsz = (int)d.batch; p.D = (int)d.dim; p.N = (int)d.dstate;
  p.softplus = f & SSM_DELTA_SOFTPLUS;
  p.has_z = f & SSM_HAS_Z;
  p.has_D = f & SSM_HAS_D;
  p.has_bias = f & SSM_HAS_DELTA_BIAS;
  p.zoh = f & SSM_ZOH;
  p.in_bf16 = d.in_dtype == SSM_BF16;
  p.out_bf16 = d.out_dtype == SSM_BF16;
  p.x = x; p.dt = delta; p.z = z; p.B = B; p.C = C;
  p.A = A; p.Dv = D; p.bias = delta_bias; p.state = state; p.y = y;
  return map_cuda(ssm::launch_step(p, reinterpret_cast<cudaStream_t>(stream_)));
}

}  // extern "C"
