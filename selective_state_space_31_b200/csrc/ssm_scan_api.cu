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
                                 SSM_HAS_H0 | SSM_WANT_HLAST | SSM_A_DIRECT | SSM_ZOH |
                                 SSM_CONV_X;
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

namespace {
struct HostPipe;
void host_pipe_free(HostPipe *hp);
}  // namespace

struct ssm_scan_plan {
  ssm_scan_desc desc{};
  int device = 0;
  int num_sms = 0;
  int path = PATH_GENERAL;
  ssm::FwdShape fs{};  // launch shape of the fused kernel (and of its carry pass)
  ssm::LaunchShape ls{};
  int DT = 0, nDT = 0, S = 0, PL = 0, parts = 0;
  int64_t rows = 0, units = 0;
  float *ws_agg = nullptr;  // carry-pass maps: (B, nsub, D, N) states then (B, nsub, D) sums
  size_t ws_agg_bytes = 0;
  float *ws_map = nullptr;  // sub-chunk maps of ssm_scan_seq_map (allocated by its first call)
  size_t ws_map_bytes = 0;
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
  HostPipe *pipe = nullptr;       // staging of ssm_scan_fwd_host (allocated by its first call)
  HostPipe *step_pipe = nullptr;  // staging of ssm_scan_step_host (allocated by its first call)
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
    if (d->flags & (SSM_HAS_Z | SSM_HAS_D | SSM_DELTA_SOFTPLUS | SSM_HAS_DELTA_BIAS | SSM_ZOH |
                    SSM_CONV_X))
      return SSM_ERR_INVALID_ARG;
  }
  if ((d->flags & SSM_CONV_X) && (d->flags & SSM_ZOH)) return SSM_ERR_UNSUPPORTED;
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
  if (pl->cfg.chans_per_lane && pl->cfg.chans_per_lane != 1 && pl->cfg.chans_per_lane != 2)
    return SSM_ERR_INVALID_ARG;
  if (pl->cfg.segments && pl->cfg.segments != 1 && pl->cfg.segments != 2 &&
      pl->cfg.segments != 4 && pl->cfg.segments != 8 &&
      pl->cfg.segments != 16)
    return SSM_ERR_INVALID_ARG;
  ssm::FwdOverrides o{pl->cfg.lanes_per_chan, pl->cfg.warps_per_cta, pl->cfg.tile_t,
                      pl->cfg.grid};
  o.kc = pl->cfg.chans_per_lane;
  o.segments = pl->cfg.segments;
  o.opt = pl->cfg.scan_loop;
  o.carry_lpc = pl->cfg.carry_lanes_per_chan;
  o.carry_opt = pl->cfg.carry_loop;
  o.carry_kc = pl->cfg.carry_chans_per_lane;
  ssm::FwdShape fs;
  if (ssm::choose_fwd_shape((int)d.in_dtype, (int)d.out_dtype, d.batch, d.seqlen, d.dim, ns,
                            (d.flags & SSM_ZOH) != 0, (d.flags & SSM_CONV_X) != 0, pl->num_sms, o,
                            &fs) != cudaSuccess) {
    cudaGetLastError();
    return SSM_ERR_UNSUPPORTED;  // no variant fits (or bad override)
  }
  // workspace: carried state per (row, segment, channel, n), a flag per
  // (row, segment, warp), and the carry pass's maps per (batch, sub-chunk, channel)
  const int64_t vrows = fs.rows * fs.M;
  const size_t st_bytes = (size_t)vrows * fs.DT * ns * sizeof(float);
  const size_t fl_bytes = (size_t)vrows * fs.ls.warps * sizeof(unsigned long long);
  const int64_t nsub = fs.M > 1 ? (int64_t)(fs.M - 1) * fs.nq : 0;
  const size_t agg_bytes = (size_t)(d.batch * nsub * d.dim * (ns + 1)) * sizeof(float);
  if (agg_bytes > pl->ws_agg_bytes) {
    if (pl->ws_agg) cudaFree(pl->ws_agg);
    pl->ws_agg = nullptr;
    pl->ws_agg_bytes = 0;
    if (cudaMalloc(&pl->ws_agg, agg_bytes) != cudaSuccess) return SSM_ERR_OOM;
    pl->ws_agg_bytes = agg_bytes;
  }
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
  pl->fs = fs;
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

int ssm_scan_version(void) { return 200; }

int ssm_scan_list_variants(ssm_dtype in_dtype, ssm_dtype out_dtype, ssm_scan_variant *out,
                           int max) {
  constexpr int kMax = 512;
  ssm::VariantDesc v[kMax];
  const int n = std::min(kMax, ssm::fwd_variants((int)in_dtype, (int)out_dtype, v, kMax));
  if (out)
    for (int i = 0; i < n && i < max; ++i)
      out[i] = ssm_scan_variant{v[i].ns, v[i].lpc, v[i].kc, v[i].warps, v[i].tt,
                                v[i].zoh ? 1 : 0, v[i].carry ? 1 : 0, v[i].conv ? 1 : 0,
                                v[i].opt};
  return n;
}

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
    if (pl->ws_agg) cudaFree(pl->ws_agg);
    if (pl->ws_map) cudaFree(pl->ws_map);
    host_pipe_free(pl->pipe);
    host_pipe_free(pl->step_pipe);
  }
  delete pl;
  return SSM_OK;
}

ssm_status ssm_scan_get_info(const ssm_scan_plan *pl, ssm_scan_info *info) {
  if (!pl || !info) return SSM_ERR_INVALID_ARG;
  std::memset(info, 0, sizeof(*info));
  const ssm_scan_desc &d = pl->desc;
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
    info->chans_per_lane = pl->ls.kc;
    info->segments = pl->fs.M;
    info->stages_per_segment = pl->fs.SPS;
    info->carry_grid = pl->fs.M > 1 ? pl->fs.cls.grid : 0;
    info->scan_loop = 1 + pl->ls.opt;
    info->carry_lanes_per_chan = pl->fs.M > 1 ? pl->fs.cls.lpc : 0;
    info->carry_loop = pl->fs.M > 1 ? 1 + pl->fs.cls.opt : 0;
    info->carry_chans_per_lane = pl->fs.M > 1 ? pl->fs.cls.kc : 0;
  }
  info->launches_per_call = pl->path == PATH_TMA && pl->fs.M > 1 ? 2 : 1;
  ssm::BwdShape bs;
  info->bwd_warps_per_cta =
      pl->path == PATH_TMA &&
              ssm::choose_bwd_shape((int)d.in_dtype, (int)d.out_dtype, d.batch, d.seqlen, d.dim,
                                    (int)d.dstate, pl->cfg.bwd_warps_per_cta,
                                    pl->cfg.bwd_segments, pl->num_sms, &bs)
          ? bs.warps
          : 0;
  info->bwd_segments = info->bwd_warps_per_cta ? bs.M : 0;
  info->workspace_bytes =
      pl->ws_state_bytes + pl->ws_flag_bytes + pl->ws_agg_bytes + sizeof(ssm::Control);
  return SSM_OK;
}

ssm_status ssm_scan_set_config(ssm_scan_plan *pl, const ssm_scan_config *cfg) {
  if (!pl || !cfg) return SSM_ERR_INVALID_ARG;
  if (cfg->lanes_per_chan < 0 || cfg->warps_per_cta < 0 || cfg->grid < 0 || cfg->tile_t < 0 ||
      cfg->chans_per_lane < 0 || cfg->segments < 0 || cfg->scan_loop < 0 || cfg->scan_loop > 32 ||
      cfg->carry_lanes_per_chan < 0 || cfg->carry_loop < 0 || cfg->carry_loop > 32 ||
      (cfg->bwd_warps_per_cta != 0 && cfg->bwd_warps_per_cta != 2 && cfg->bwd_warps_per_cta != 4) ||
      (cfg->bwd_segments != 0 && cfg->bwd_segments != 1 && cfg->bwd_segments != 2 &&
       cfg->bwd_segments != 4 && cfg->bwd_segments != 8 && cfg->bwd_segments != 16) ||
      cfg->carry_chans_per_lane < 0 || cfg->carry_chans_per_lane > 2)
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

}  // extern "C"

namespace {

// Both forward entry points: conv_w non-null selects the conv front-end (x
// then holds the raw x branch).
ssm_status fwd_impl(ssm_scan_plan *pl, const void *x, const float *conv_w, const float *conv_b,
                    void *xconv, const void *delta, const float *delta_bias, const void *A,
                    const void *B, const void *C, const float *D, const void *z, const float *h0,
                    void *y, float *h_last, ssm_stream_t stream_) {
  const ssm_scan_desc &d = pl->desc;
  const bool conv = conv_w != nullptr;
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
                       aligned16(C) && aligned16(y) && aligned16(xconv);
  if (pl->path == PATH_TMA && aligned) {
    const ssm::FwdShape &fs = pl->fs;
    ssm::TmaMaps maps;
    const uint64_t Bn = d.batch, L = d.seqlen, Dm = d.dim, N = d.dstate;
    const uint32_t DT = (uint32_t)pl->DT, TT = (uint32_t)pl->ls.tt;
    // the conv front-end's x tiles carry kConvWidth earlier tokens
    const uint32_t XT = TT + (conv ? (uint32_t)ssm::kConvWidth : 0u);
    if (!encode3d(&maps.x, d.in_dtype, x, Dm, L, Bn, DT, XT) ||
        !encode3d(&maps.dt, d.in_dtype, delta, Dm, L, Bn, DT, TT) ||
        !encode3d(&maps.z, d.in_dtype, z ? z : x, Dm, L, Bn, DT, TT) ||
        !encode3d(&maps.B, d.in_dtype, B, N, L, Bn, (uint32_t)N, TT) ||
        !encode3d(&maps.C, d.in_dtype, C, N, L, Bn, (uint32_t)N, TT))
      return SSM_ERR_CUDA;
    ssm::FwdParams p{};
    p.Bsz = (int)d.batch; p.L = (int)d.seqlen; p.D = (int)d.dim; p.N = (int)d.dstate;
    p.DT = pl->DT; p.nDT = pl->nDT; p.rows = (int)pl->rows; p.S = pl->S;
    p.M = fs.M; p.SPS = fs.SPS;
    p.PL = pl->PL; p.items = (int)(pl->rows * fs.M * pl->parts);
    p.nq = fs.nq; p.nsub_row = fs.M > 1 ? (fs.M - 1) * fs.nq : 0;
    const size_t nagg = (size_t)d.batch * p.nsub_row * d.dim;
    p.agg_h = pl->ws_agg;
    p.agg_s = pl->ws_agg ? pl->ws_agg + nagg * d.dstate : nullptr;
    p.softplus = (f & SSM_DELTA_SOFTPLUS) != 0;
    p.has_z = (f & SSM_HAS_Z) != 0;
    p.has_D = (f & SSM_HAS_D) != 0;
    p.has_bias = (f & SSM_HAS_DELTA_BIAS) != 0;
    p.has_h0 = (f & SSM_HAS_H0) != 0;
    p.want_hlast = (f & SSM_WANT_HLAST) != 0;
    p.zoh = (f & SSM_ZOH) != 0;
    p.A = static_cast<const float *>(A);
    p.Dv = D; p.bias = delta_bias; p.h0 = h0; p.h_last = h_last; p.y = y;
    p.conv_w = conv_w; p.conv_b = conv_b; p.xconv = xconv;
    p.ws_state = pl->ws_state; p.ws_flags = pl->ws_flags; p.ctl = pl->ctl;
    p.timeout_ns = pl->timeout_ns;
    p.drop_unit = pl->drop_unit;
    if (fs.M > 1) {
      // carry pass: the map of every sub-chunk of segments 0 .. M-2, from 0
      ssm::TmaMaps cmaps = maps;
      const uint32_t cDT = (uint32_t)fs.cDT;
      if (cDT != DT && (!encode3d(&cmaps.x, d.in_dtype, x, Dm, L, Bn, cDT, XT) ||
                        !encode3d(&cmaps.dt, d.in_dtype, delta, Dm, L, Bn, cDT, TT)))
        return SSM_ERR_CUDA;
      ssm::FwdParams c = p;
      c.DT = fs.cDT;
      c.nDT = (int)((d.dim + fs.cDT - 1) / fs.cDT);
      c.rows = (int)fs.crows;
      c.M = 1;
      c.SPS = pl->S;
      c.PL = fs.Q;
      c.items = (int)(fs.crows * p.nsub_row);
      c.drop_unit = -1;
      c.xconv = nullptr;
      const cudaError_t e =
          ssm::launch_fwd_tma((int)d.in_dtype, (int)d.out_dtype, fs.cls, cmaps, c, stream);
      if (e != cudaSuccess) return SSM_ERR_CUDA;
    }
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
  p.conv_w = conv_w; p.conv_b = conv_b; p.xconv = xconv;
  return map_cuda(ssm::launch_fwd_general(p, stream));
}

}  // namespace

extern "C" {

ssm_status ssm_scan_fwd(ssm_scan_plan *pl, const void *x, const void *delta,
                        const float *delta_bias, const void *A, const void *B, const void *C,
                        const float *D, const void *z, const float *h0, void *y, float *h_last,
                        ssm_stream_t stream) {
  if (!pl) return SSM_ERR_INVALID_ARG;
  if (pl->desc.flags & SSM_CONV_X) return SSM_ERR_INVALID_ARG;  // needs ssm_scan_fwd_conv
  return fwd_impl(pl, x, nullptr, nullptr, nullptr, delta, delta_bias, A, B, C, D, z, h0, y,
                  h_last, stream);
}

ssm_status ssm_scan_seq_map(ssm_scan_plan *pl, const void *x, const void *delta,
                            const float *delta_bias, const float *A, const void *B, float *map_h,
                            float *map_s, ssm_stream_t stream_) {
  if (!pl) return SSM_ERR_INVALID_ARG;
  const ssm_scan_desc &d = pl->desc;
  const uint32_t f = d.flags;
  if (f & (SSM_A_DIRECT | SSM_CONV_X)) return SSM_ERR_UNSUPPORTED;
  const bool has_chans = d.batch * d.dim != 0;
  if (has_chans && (!A || !map_h || !map_s)) return SSM_ERR_INVALID_ARG;
  if (d.batch * d.seqlen * d.dim != 0 && (!x || !delta || !B)) return SSM_ERR_INVALID_ARG;
  if (has_chans && ((f & SSM_HAS_DELTA_BIAS) != 0) != (delta_bias != nullptr))
    return SSM_ERR_INVALID_ARG;
  if (!has_chans) return SSM_OK;
  DeviceGuard guard(pl->device);
  if (!guard.ok) return SSM_ERR_CUDA;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  const uint64_t Bn = d.batch, L = d.seqlen, Dm = d.dim, N = d.dstate;
  const bool aligned = aligned16(x) && aligned16(delta) && aligned16(B);
  ssm::MapShape ms{};
  if (pl->path == PATH_TMA && aligned && d.seqlen > 0 &&
      ssm::choose_map_shape((int)d.in_dtype, (int)d.out_dtype, d.batch, d.dim, pl->fs,
                            pl->num_sms, &ms) == cudaSuccess) {
    const size_t nagg = (size_t)d.batch * ms.nsub * d.dim;
    const size_t need = nagg * (d.dstate + 1) * sizeof(float);
    if (need > pl->ws_map_bytes) {
      if (pl->ws_map) cudaFree(pl->ws_map);
      pl->ws_map = nullptr;
      pl->ws_map_bytes = 0;
      if (cudaMalloc(&pl->ws_map, need) != cudaSuccess) {
        cudaGetLastError();
        return SSM_ERR_OOM;
      }
      pl->ws_map_bytes = need;
    }
    const uint32_t TT = (uint32_t)pl->fs.ls.tt, cDT = (uint32_t)ms.DT;
    ssm::TmaMaps maps;
    if (!encode3d(&maps.x, d.in_dtype, x, Dm, L, Bn, cDT, TT) ||
        !encode3d(&maps.dt, d.in_dtype, delta, Dm, L, Bn, cDT, TT) ||
        !encode3d(&maps.z, d.in_dtype, x, Dm, L, Bn, cDT, TT) ||
        !encode3d(&maps.B, d.in_dtype, B, N, L, Bn, (uint32_t)N, TT) ||
        !encode3d(&maps.C, d.in_dtype, B, N, L, Bn, (uint32_t)N, TT))
      return SSM_ERR_CUDA;
    ssm::FwdParams c{};
    c.Bsz = (int)d.batch; c.L = (int)d.seqlen; c.D = (int)d.dim; c.N = (int)d.dstate;
    c.DT = ms.DT; c.nDT = (int)((d.dim + ms.DT - 1) / ms.DT); c.rows = (int)ms.rows;
    c.S = pl->fs.S; c.M = 1; c.SPS = pl->fs.S; c.PL = ms.Q;
    c.items = (int)(ms.rows * ms.nsub);
    c.nq = ms.nsub; c.nsub_row = ms.nsub;
    c.agg_h = pl->ws_map;
    c.agg_s = pl->ws_map + nagg * d.dstate;
    c.softplus = (f & SSM_DELTA_SOFTPLUS) != 0;
    c.has_bias = (f & SSM_HAS_DELTA_BIAS) != 0;
    c.zoh = (f & SSM_ZOH) != 0;
    c.A = A; c.bias = delta_bias;
    c.ws_state = pl->ws_state; c.ws_flags = pl->ws_flags; c.ctl = pl->ctl;
    c.timeout_ns = pl->timeout_ns;
    c.drop_unit = -1;
    if (ssm::launch_fwd_tma((int)d.in_dtype, (int)d.out_dtype, ms.ls, maps, c, stream) !=
        cudaSuccess)
      return SSM_ERR_CUDA;
    ssm::FoldParams fp{};
    fp.Bsz = (int)d.batch; fp.D = (int)d.dim; fp.N = (int)d.dstate; fp.count = ms.nsub;
    fp.stride_b = (long long)ms.nsub * d.dim;
    fp.stride_j = d.dim;
    fp.A = A; fp.maps_h = c.agg_h; fp.maps_s = c.agg_s; fp.h0 = nullptr;
    fp.h_out = map_h; fp.s_out = map_s;
    return map_cuda(ssm::launch_fold_maps(fp, stream));
  }
  ssm::MapParams mp{};
  mp.Bsz = (int)d.batch; mp.L = (int)d.seqlen; mp.D = (int)d.dim; mp.N = (int)d.dstate;
  mp.softplus = (f & SSM_DELTA_SOFTPLUS) != 0;
  mp.zoh = (f & SSM_ZOH) != 0;
  mp.in_bf16 = d.in_dtype == SSM_BF16;
  mp.x = x; mp.dt = delta; mp.B = B; mp.A = A; mp.bias = delta_bias;
  mp.map_h = map_h; mp.map_s = map_s;
  return map_cuda(ssm::launch_map_general(mp, stream));
}

ssm_status ssm_scan_fold_maps(ssm_scan_plan *pl, int count, const float *maps_h,
                              const float *maps_s, const float *A, const float *h0, float *h_out,
                              ssm_stream_t stream) {
  if (!pl || count < 0) return SSM_ERR_INVALID_ARG;
  const ssm_scan_desc &d = pl->desc;
  if (d.flags & SSM_A_DIRECT) return SSM_ERR_UNSUPPORTED;
  if (d.batch * d.dim == 0) return SSM_OK;
  if (!A || !h_out || (count > 0 && (!maps_h || !maps_s))) return SSM_ERR_INVALID_ARG;
  DeviceGuard guard(pl->device);
  if (!guard.ok) return SSM_ERR_CUDA;
  ssm::FoldParams fp{};
  fp.Bsz = (int)d.batch; fp.D = (int)d.dim; fp.N = (int)d.dstate; fp.count = count;
  fp.stride_b = d.dim;
  fp.stride_j = d.batch * d.dim;
  fp.A = A; fp.maps_h = maps_h; fp.maps_s = maps_s; fp.h0 = h0; fp.h_out = h_out;
  fp.s_out = nullptr;
  return map_cuda(ssm::launch_fold_maps(fp, reinterpret_cast<cudaStream_t>(stream)));
}

ssm_status ssm_scan_fwd_conv(ssm_scan_plan *pl, const void *x_in, const float *conv_w,
                             const float *conv_b, const void *delta, const float *delta_bias,
                             const float *A, const void *B, const void *C, const float *D,
                             const void *z, const float *h0, void *y, float *h_last,
                             void *x_conv, ssm_stream_t stream) {
  if (!pl) return SSM_ERR_INVALID_ARG;
  if (!(pl->desc.flags & SSM_CONV_X)) return SSM_ERR_INVALID_ARG;
  if (!conv_w && pl->desc.dim * pl->desc.batch * pl->desc.seqlen != 0) return SSM_ERR_INVALID_ARG;
  return fwd_impl(pl, x_in, conv_w, conv_b, x_conv, delta, delta_bias, A, B, C, D, z, h0, y,
                  h_last, stream);
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
  if (f & (SSM_ZOH | SSM_A_DIRECT | SSM_CONV_X)) return SSM_ERR_UNSUPPORTED;
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
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  ssm::BwdShape bs;
  const bool fused = has_tokens && pl->path == PATH_TMA &&
                     ssm::choose_bwd_shape((int)d.in_dtype, (int)d.out_dtype, d.batch, d.seqlen,
                                           d.dim, (int)d.dstate, pl->cfg.bwd_warps_per_cta,
                                           pl->cfg.bwd_segments, pl->num_sms, &bs) &&
                     aligned16(x) && aligned16(delta) && aligned16(z) && aligned16(B) &&
                     aligned16(C) && aligned16(dy) && aligned16(dB) && aligned16(dC) &&
                     aligned16(dh0);
  if (fused) {
    const size_t need = (bs.ws_ck_floats + bs.ws_bc_floats + 2 * bs.ws_map_floats) * sizeof(float);
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
    ssm::BwdMaps maps;
    const uint64_t Bn = d.batch, L = d.seqlen, Dm = d.dim, N = d.dstate;
    const uint32_t DT = (uint32_t)bs.DT, TT = (uint32_t)ssm::kBwdStage;
    if (!encode3d(&maps.x, d.in_dtype, x, Dm, L, Bn, DT, TT) ||
        !encode3d(&maps.dt, d.in_dtype, delta, Dm, L, Bn, DT, TT) ||
        !encode3d(&maps.z, d.in_dtype, z ? z : x, Dm, L, Bn, DT, TT) ||
        !encode3d(&maps.dy, d.out_dtype, dy, Dm, L, Bn, DT, TT) ||
        !encode3d(&maps.B, d.in_dtype, B, N, L, Bn, (uint32_t)N, TT) ||
        !encode3d(&maps.C, d.in_dtype, C, N, L, Bn, (uint32_t)N, TT))
      return SSM_ERR_CUDA;
    ssm::BwdTmaParams p{};
    p.Bsz = (int)d.batch; p.L = (int)d.seqlen; p.D = (int)d.dim; p.N = (int)d.dstate;
    p.DT = bs.DT; p.nDT = bs.nDT; p.S = bs.S; p.rows = (int)bs.rows;
    p.M = bs.M; p.SPS = bs.SPS;
    p.softplus = f & SSM_DELTA_SOFTPLUS;
    p.has_z = f & SSM_HAS_Z;
    p.has_D = f & SSM_HAS_D;
    p.has_bias = f & SSM_HAS_DELTA_BIAS;
    p.has_h0 = f & SSM_HAS_H0;
    p.A = A; p.Dv = D; p.bias = delta_bias; p.h0 = h0; p.dh_last = dh_last;
    p.dx = dx; p.ddelta = ddelta; p.dz = dz; p.dB = dB; p.dC = dC; p.dA = dA; p.dD = dD;
    p.dbias = ddelta_bias; p.dh0 = dh0;
    p.ws_ck = pl->ws_ck;
    p.ws_bc = pl->ws_ck + bs.ws_ck_floats;
    p.ws_fmap = bs.M > 1 ? p.ws_bc + bs.ws_bc_floats : nullptr;
    p.ws_amap = bs.M > 1 ? p.ws_fmap + bs.ws_map_floats : nullptr;
    p.ctl = pl->ctl;
    p.timeout_ns = pl->timeout_ns;
    return map_cuda(ssm::launch_bwd_tma((int)d.in_dtype, (int)d.out_dtype, bs, maps, p, stream));
  }
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
  return map_cuda(ssm::launch_bwd(p, stream));
}

ssm_status ssm_scan_step(ssm_scan_plan *pl, const void *x, const void *delta,
                         const float *delta_bias, const float *A, const void *B, const void *C,
                         const float *D, const void *z, float *state, void *y,
                         ssm_stream_t stream_) {
  if (!pl) return SSM_ERR_INVALID_ARG;
  const ssm_scan_desc &d = pl->desc;
  const uint32_t f = d.flags;
  if (f & SSM_A_DIRECT) return SSM_ERR_INVALID_ARG;
  if (f & SSM_CONV_X) return SSM_ERR_UNSUPPORTED;  // the conv's token history is not kept
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

// ---------------------------------------------------------------------------
// ssm_scan_fwd_host: the sequence streamed through the device in chunks of
// tokens, copies and scans overlapping on three streams
// ---------------------------------------------------------------------------

namespace {

constexpr int kPipeSlots = 3;  // chunks in flight: copy-in, scan, copy-out

struct HostPipe {
  int64_t Lc = 0;                                  // tokens per chunk
  ssm_scan_plan *body = nullptr, *tail = nullptr;  // plans for Lc and the last chunk's length
  cudaStream_t s_in = nullptr, s_out = nullptr;
  cudaEvent_t ev_start = nullptr, ev_done = nullptr;
  cudaEvent_t ev_in[kPipeSlots] = {}, ev_comp[kPipeSlots] = {}, ev_out[kPipeSlots] = {};
  unsigned char *slots = nullptr;  // kPipeSlots x [x | delta | z | B | C | y] of one chunk
  size_t off_dt = 0, off_z = 0, off_B = 0, off_C = 0, off_y = 0, slot_bytes = 0;
  float *params = nullptr;  // A (D x N), D (D), delta_bias (D)
  float *hbuf = nullptr;    // 2 x (B, D, N): the state handed from chunk to chunk
};

void host_pipe_free(HostPipe *hp) {
  if (!hp) return;
  if (hp->body) ssm_scan_destroy(hp->body);
  if (hp->tail) ssm_scan_destroy(hp->tail);
  for (cudaEvent_t e : {hp->ev_start, hp->ev_done})
    if (e) cudaEventDestroy(e);
  for (int i = 0; i < kPipeSlots; ++i)
    for (cudaEvent_t e : {hp->ev_in[i], hp->ev_comp[i], hp->ev_out[i]})
      if (e) cudaEventDestroy(e);
  if (hp->s_in) cudaStreamDestroy(hp->s_in);
  if (hp->s_out) cudaStreamDestroy(hp->s_out);
  if (hp->slots) cudaFree(hp->slots);
  if (hp->params) cudaFree(hp->params);
  if (hp->hbuf) cudaFree(hp->hbuf);
  delete hp;
}

size_t align256(size_t v) { return (v + 255) / 256 * 256; }

// A chunk plan: the parent's problem over `len` tokens, always with a
// starting state and a final state (they carry the sequence across chunks).
ssm_status make_chunk_plan(const ssm_scan_plan *pl, int64_t len, ssm_scan_plan **out) {
  ssm_scan_desc d = pl->desc;
  d.seqlen = len;
  d.flags |= SSM_HAS_H0 | SSM_WANT_HLAST;
  ssm_status st = ssm_scan_create(out, &d, pl->device);
  if (st == SSM_OK) (*out)->timeout_ns = pl->timeout_ns;
  return st;
}

ssm_status host_pipe_build(ssm_scan_plan *pl, int64_t Lc, HostPipe **out) {
  const ssm_scan_desc &d = pl->desc;
  HostPipe *hp = new (std::nothrow) HostPipe;
  if (!hp) return SSM_ERR_OOM;
  hp->Lc = Lc;
  auto fail = [&](ssm_status st) {
    cudaGetLastError();
    host_pipe_free(hp);
    return st;
  };
  const int64_t L = d.seqlen, nch = (L + Lc - 1) / Lc, tail = L - (nch - 1) * Lc;
  ssm_status st = make_chunk_plan(pl, Lc, &hp->body);
  if (st != SSM_OK) return fail(st);
  if (tail != Lc && (st = make_chunk_plan(pl, tail, &hp->tail)) != SSM_OK) return fail(st);
  const size_t ei = dtype_size(d.in_dtype), eo = dtype_size(d.out_dtype);
  const size_t tok = (size_t)(d.batch * Lc);
  const size_t xb = align256(tok * d.dim * ei), bb = align256(tok * d.dstate * ei);
  hp->off_dt = xb;
  hp->off_z = 2 * xb;
  hp->off_B = 3 * xb;
  hp->off_C = 3 * xb + bb;
  hp->off_y = 3 * xb + 2 * bb;
  hp->slot_bytes = hp->off_y + align256(tok * d.dim * eo);
  const size_t nparam = (size_t)(d.dim * d.dstate + 2 * d.dim);
  const size_t nstate = (size_t)(d.batch * d.dim * d.dstate);
  if (cudaMalloc(&hp->slots, kPipeSlots * hp->slot_bytes) != cudaSuccess ||
      cudaMalloc(&hp->params, nparam * sizeof(float)) != cudaSuccess ||
      cudaMalloc(&hp->hbuf, 2 * std::max<size_t>(nstate, 1) * sizeof(float)) != cudaSuccess)
    return fail(SSM_ERR_OOM);
  if (cudaStreamCreateWithFlags(&hp->s_in, cudaStreamNonBlocking) != cudaSuccess ||
      cudaStreamCreateWithFlags(&hp->s_out, cudaStreamNonBlocking) != cudaSuccess ||
      cudaEventCreateWithFlags(&hp->ev_start, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&hp->ev_done, cudaEventDisableTiming) != cudaSuccess)
    return fail(SSM_ERR_CUDA);
  for (int i = 0; i < kPipeSlots; ++i)
    if (cudaEventCreateWithFlags(&hp->ev_in[i], cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&hp->ev_comp[i], cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&hp->ev_out[i], cudaEventDisableTiming) != cudaSuccess)
      return fail(SSM_ERR_CUDA);
  *out = hp;
  return SSM_OK;
}

// Tokens [l0, l0 + len) of every batch element of a (B, L, W) host tensor
// into a contiguous (B, len, W) device buffer, or back.
cudaError_t copy_tokens_in(void *dst, const void *src, const ssm_scan_desc &d, int64_t W,
                           size_t es, int64_t l0, int64_t len, cudaStream_t s) {
  const size_t row = (size_t)(len * W) * es;
  return cudaMemcpy2DAsync(dst, row, static_cast<const unsigned char *>(src) + (size_t)(l0 * W) * es,
                           (size_t)(d.seqlen * W) * es, row, (size_t)d.batch,
                           cudaMemcpyHostToDevice, s);
}
cudaError_t copy_tokens_out(void *dst, const void *src, const ssm_scan_desc &d, int64_t W,
                            size_t es, int64_t l0, int64_t len, cudaStream_t s) {
  const size_t row = (size_t)(len * W) * es;
  return cudaMemcpy2DAsync(static_cast<unsigned char *>(dst) + (size_t)(l0 * W) * es,
                           (size_t)(d.seqlen * W) * es, src, row, row, (size_t)d.batch,
                           cudaMemcpyDeviceToHost, s);
}

}  // namespace

extern "C" {

ssm_status ssm_scan_fwd_host(ssm_scan_plan *pl, const void *x, const void *delta,
                             const float *delta_bias, const float *A, const void *B,
                             const void *C, const float *D, const void *z, const float *h0,
                             void *y, float *h_last, int64_t chunk_tokens, ssm_stream_t stream_) {
  if (!pl || chunk_tokens < 0) return SSM_ERR_INVALID_ARG;
  const ssm_scan_desc &d = pl->desc;
  const uint32_t f = d.flags;
  if (f & (SSM_A_DIRECT | SSM_CONV_X)) return SSM_ERR_UNSUPPORTED;
  const bool has_tokens = d.batch * d.seqlen * d.dim != 0;
  if (has_tokens && (!x || !delta || !B || !C || !y)) return SSM_ERR_INVALID_ARG;
  if (d.dim != 0 && !A) return SSM_ERR_INVALID_ARG;
  if (((f & SSM_HAS_Z) != 0) != (z != nullptr) || ((f & SSM_HAS_D) != 0) != (D != nullptr) ||
      ((f & SSM_HAS_DELTA_BIAS) != 0) != (delta_bias != nullptr) ||
      ((f & SSM_HAS_H0) != 0) != (h0 != nullptr) ||
      ((f & SSM_WANT_HLAST) != 0) != (h_last != nullptr))
    return SSM_ERR_INVALID_ARG;
  if (d.batch * d.dim == 0) return SSM_OK;
  DeviceGuard guard(pl->device);
  if (!guard.ok) return SSM_ERR_CUDA;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  const int64_t L = d.seqlen;
  const size_t ei = dtype_size(d.in_dtype), eo = dtype_size(d.out_dtype);
  const size_t nstate = (size_t)(d.batch * d.dim * d.dstate);
  if (L == 0) {  // no tokens: h_last = h0 (or 0)
    if (!h_last) return SSM_OK;
    if (h0) return map_cuda(cudaMemcpyAsync(h_last, h0, nstate * 4, cudaMemcpyHostToHost, stream));
    return map_cuda(cudaMemsetAsync(h_last, 0, nstate * 4, stream));
  }
  int64_t Lc = chunk_tokens;
  if (!Lc) {  // about twelve chunks, none under ~8 MB of copies (below that, per-copy overheads rule)
    const int64_t per_token = d.batch * (d.dim * (3 * (int64_t)ei + (int64_t)eo) + 2 * d.dstate * (int64_t)ei);
    const int64_t min_tokens = ((int64_t)8 << 20) / std::max<int64_t>(per_token, 1) + 1;
    Lc = (std::max((L + 11) / 12, min_tokens) + 63) / 64 * 64;
  }
  Lc = std::min(Lc, L);
  if (!pl->pipe || pl->pipe->Lc != Lc) {
    host_pipe_free(pl->pipe);
    pl->pipe = nullptr;
    const ssm_status st = host_pipe_build(pl, Lc, &pl->pipe);
    if (st != SSM_OK) return st;
  }
  HostPipe &hp = *pl->pipe;
  const int64_t nch = (L + Lc - 1) / Lc;
  float *dA = hp.params, *dD = hp.params + d.dim * d.dstate, *dbias = dD + d.dim;
  auto ck = [](cudaError_t e) { return e == cudaSuccess; };
  // everything is enqueued by `run`; whatever it returns, the caller's stream
  // then waits for both copy streams, so no copy outlives the call's stream
  // order (the host buffers may be released after a synchronisation)
  auto run = [&]() -> ssm_status {
    // the copies start behind the caller's earlier work on `stream`
    if (!ck(cudaEventRecord(hp.ev_start, stream)) || !ck(cudaStreamWaitEvent(hp.s_in, hp.ev_start, 0)) ||
        !ck(cudaStreamWaitEvent(hp.s_out, hp.ev_start, 0)))
      return SSM_ERR_CUDA;
    // parameters once; the state before the first chunk into hbuf[1]
    if (!ck(cudaMemcpyAsync(dA, A, (size_t)(d.dim * d.dstate) * 4, cudaMemcpyHostToDevice, hp.s_in)) ||
        (D && !ck(cudaMemcpyAsync(dD, D, (size_t)d.dim * 4, cudaMemcpyHostToDevice, hp.s_in))) ||
        (delta_bias &&
         !ck(cudaMemcpyAsync(dbias, delta_bias, (size_t)d.dim * 4, cudaMemcpyHostToDevice, hp.s_in))))
      return SSM_ERR_CUDA;
    float *hprev0 = hp.hbuf + nstate;
    if (!ck(h0 ? cudaMemcpyAsync(hprev0, h0, nstate * 4, cudaMemcpyHostToDevice, hp.s_in)
               : cudaMemsetAsync(hprev0, 0, nstate * 4, hp.s_in)))
      return SSM_ERR_CUDA;
    for (int64_t c = 0; c < nch; ++c) {
      const int s = (int)(c % kPipeSlots);
      const int64_t l0 = c * Lc, len = std::min(Lc, L - l0);
      unsigned char *sb = hp.slots + s * hp.slot_bytes;
      // copy-in of chunk c once the scan of chunk c - kPipeSlots has left the slot
      if (c >= kPipeSlots && !ck(cudaStreamWaitEvent(hp.s_in, hp.ev_comp[s], 0))) return SSM_ERR_CUDA;
      if (!ck(copy_tokens_in(sb, x, d, d.dim, ei, l0, len, hp.s_in)) ||
          !ck(copy_tokens_in(sb + hp.off_dt, delta, d, d.dim, ei, l0, len, hp.s_in)) ||
          (z && !ck(copy_tokens_in(sb + hp.off_z, z, d, d.dim, ei, l0, len, hp.s_in))) ||
          !ck(copy_tokens_in(sb + hp.off_B, B, d, d.dstate, ei, l0, len, hp.s_in)) ||
          !ck(copy_tokens_in(sb + hp.off_C, C, d, d.dstate, ei, l0, len, hp.s_in)) ||
          !ck(cudaEventRecord(hp.ev_in[s], hp.s_in)))
        return SSM_ERR_CUDA;
      // the scan of chunk c on the caller's stream, from the state chunk c - 1 left
      if (!ck(cudaStreamWaitEvent(stream, hp.ev_in[s], 0)) ||
          (c >= kPipeSlots && !ck(cudaStreamWaitEvent(stream, hp.ev_out[s], 0))))
        return SSM_ERR_CUDA;
      float *hprev = hp.hbuf + ((c + 1) % 2) * nstate, *hnext = hp.hbuf + (c % 2) * nstate;
      ssm_scan_plan *cp = len == Lc ? hp.body : hp.tail;
      const ssm_status st =
          ssm_scan_fwd(cp, sb, sb + hp.off_dt, delta_bias ? dbias : nullptr, dA, sb + hp.off_B,
                       sb + hp.off_C, D ? dD : nullptr, z ? sb + hp.off_z : nullptr, hprev,
                       sb + hp.off_y, hnext, stream_);
      if (st != SSM_OK) return st;
      if (!ck(cudaEventRecord(hp.ev_comp[s], stream))) return SSM_ERR_CUDA;
      // copy-out of chunk c's y
      if (!ck(cudaStreamWaitEvent(hp.s_out, hp.ev_comp[s], 0)) ||
          !ck(copy_tokens_out(y, sb + hp.off_y, d, d.dim, eo, l0, len, hp.s_out)) ||
          !ck(cudaEventRecord(hp.ev_out[s], hp.s_out)))
        return SSM_ERR_CUDA;
    }
    if (h_last && !ck(cudaMemcpyAsync(h_last, hp.hbuf + ((nch - 1) % 2) * nstate, nstate * 4,
                                      cudaMemcpyDeviceToHost, hp.s_out)))
      return SSM_ERR_CUDA;
    return SSM_OK;
  };
  const ssm_status st = run();
  const bool joined = ck(cudaEventRecord(hp.ev_done, hp.s_out)) &&
                      ck(cudaStreamWaitEvent(stream, hp.ev_done, 0)) &&
                      ck(cudaEventRecord(hp.ev_start, hp.s_in)) &&
                      ck(cudaStreamWaitEvent(stream, hp.ev_start, 0));
  if (st != SSM_OK) return st;
  return joined ? SSM_OK : SSM_ERR_CUDA;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// ssm_scan_step_host: one decode step with the token's inputs and y in host
// memory, the batch streamed through the device in chunks of rows
// ---------------------------------------------------------------------------

namespace {

ssm_status step_pipe_build(ssm_scan_plan *pl, int64_t R, HostPipe **out) {
  const ssm_scan_desc &d = pl->desc;
  HostPipe *hp = new (std::nothrow) HostPipe;
  if (!hp) return SSM_ERR_OOM;
  hp->Lc = R;  // rows per chunk
  auto fail = [&](ssm_status st) {
    cudaGetLastError();
    host_pipe_free(hp);
    return st;
  };
  const size_t ei = dtype_size(d.in_dtype), eo = dtype_size(d.out_dtype);
  const size_t xb = align256((size_t)(R * d.dim) * ei), bb = align256((size_t)(R * d.dstate) * ei);
  hp->off_dt = xb;
  hp->off_z = 2 * xb;
  hp->off_B = 3 * xb;
  hp->off_C = 3 * xb + bb;
  hp->off_y = 3 * xb + 2 * bb;
  hp->slot_bytes = hp->off_y + align256((size_t)(R * d.dim) * eo);
  if (cudaMalloc(&hp->slots, kPipeSlots * hp->slot_bytes) != cudaSuccess) return fail(SSM_ERR_OOM);
  if (cudaStreamCreateWithFlags(&hp->s_in, cudaStreamNonBlocking) != cudaSuccess ||
      cudaStreamCreateWithFlags(&hp->s_out, cudaStreamNonBlocking) != cudaSuccess ||
      cudaEventCreateWithFlags(&hp->ev_start, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&hp->ev_done, cudaEventDisableTiming) != cudaSuccess)
    return fail(SSM_ERR_CUDA);
  for (int i = 0; i < kPipeSlots; ++i)
    if (cudaEventCreateWithFlags(&hp->ev_in[i], cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&hp->ev_comp[i], cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&hp->ev_out[i], cudaEventDisableTiming) != cudaSuccess)
      return fail(SSM_ERR_CUDA);
  *out = hp;
  return SSM_OK;
}

}  // namespace

extern "C" {

ssm_status ssm_scan_step_host(ssm_scan_plan *pl, const void *x, const void *delta,
                              const float *delta_bias, const float *A, const void *B,
                              const void *C, const float *D, const void *z, float *state,
                              void *y, int64_t chunk_rows, ssm_stream_t stream_) {
  if (!pl || chunk_rows < 0) return SSM_ERR_INVALID_ARG;
  const ssm_scan_desc &d = pl->desc;
  const uint32_t f = d.flags;
  if (f & SSM_A_DIRECT) return SSM_ERR_INVALID_ARG;
  if (f & SSM_CONV_X) return SSM_ERR_UNSUPPORTED;
  const bool empty = d.batch * d.dim == 0;
  if (!empty && (!x || !delta || !A || !B || !C || !state || !y)) return SSM_ERR_INVALID_ARG;
  if (((f & SSM_HAS_Z) != 0) != (z != nullptr) || ((f & SSM_HAS_D) != 0) != (D != nullptr) ||
      ((f & SSM_HAS_DELTA_BIAS) != 0) != (delta_bias != nullptr))
    return SSM_ERR_INVALID_ARG;
  if (empty) return SSM_OK;
  DeviceGuard guard(pl->device);
  if (!guard.ok) return SSM_ERR_CUDA;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  const int64_t Bn = d.batch;
  const size_t ei = dtype_size(d.in_dtype), eo = dtype_size(d.out_dtype);
  int64_t R = chunk_rows;
  if (!R) {  // two chunks, none under ~2 MB of copies (measured best on (256, 5120, 16))
    const int64_t per_row = d.dim * (3 * (int64_t)ei + (int64_t)eo) + 2 * d.dstate * (int64_t)ei;
    R = std::max((Bn + 1) / 2, ((int64_t)2 << 20) / std::max<int64_t>(per_row, 1) + 1);
  }
  R = std::min(R, Bn);
  if (!pl->step_pipe || pl->step_pipe->Lc != R) {
    host_pipe_free(pl->step_pipe);
    pl->step_pipe = nullptr;
    const ssm_status st = step_pipe_build(pl, R, &pl->step_pipe);
    if (st != SSM_OK) return st;
  }
  HostPipe &hp = *pl->step_pipe;
  const int64_t nch = (Bn + R - 1) / R;
  auto ck = [](cudaError_t e) { return e == cudaSuccess; };
  auto run = [&]() -> ssm_status {
    if (!ck(cudaEventRecord(hp.ev_start, stream)) || !ck(cudaStreamWaitEvent(hp.s_in, hp.ev_start, 0)) ||
        !ck(cudaStreamWaitEvent(hp.s_out, hp.ev_start, 0)))
      return SSM_ERR_CUDA;
    for (int64_t c = 0; c < nch; ++c) {
      const int s = (int)(c % kPipeSlots);
      const int64_t b0 = c * R, rows = std::min(R, Bn - b0);
      unsigned char *sb = hp.slots + s * hp.slot_bytes;
      const size_t xo = (size_t)(b0 * d.dim) * ei, xn = (size_t)(rows * d.dim) * ei;
      const size_t bo = (size_t)(b0 * d.dstate) * ei, bn = (size_t)(rows * d.dstate) * ei;
      auto in = [&](size_t off, const void *src, size_t so, size_t n) {
        return ck(cudaMemcpyAsync(sb + off, static_cast<const unsigned char *>(src) + so, n,
                                  cudaMemcpyHostToDevice, hp.s_in));
      };
      if (c >= kPipeSlots && !ck(cudaStreamWaitEvent(hp.s_in, hp.ev_comp[s], 0))) return SSM_ERR_CUDA;
      if (!in(0, x, xo, xn) || !in(hp.off_dt, delta, xo, xn) || (z && !in(hp.off_z, z, xo, xn)) ||
          !in(hp.off_B, B, bo, bn) || !in(hp.off_C, C, bo, bn) ||
          !ck(cudaEventRecord(hp.ev_in[s], hp.s_in)))
        return SSM_ERR_CUDA;
      if (!ck(cudaStreamWaitEvent(stream, hp.ev_in[s], 0)) ||
          (c >= kPipeSlots && !ck(cudaStreamWaitEvent(stream, hp.ev_out[s], 0))))
        return SSM_ERR_CUDA;
      ssm::StepParams p{};
      p.Bsz = (int)rows; p.D = (int)d.dim; p.N = (int)d.dstate;
      p.softplus = f & SSM_DELTA_SOFTPLUS;
      p.has_z = f & SSM_HAS_Z;
      p.has_D = f & SSM_HAS_D;
      p.has_bias = f & SSM_HAS_DELTA_BIAS;
      p.zoh = f & SSM_ZOH;
      p.in_bf16 = d.in_dtype == SSM_BF16;
      p.out_bf16 = d.out_dtype == SSM_BF16;
      p.x = sb; p.dt = sb + hp.off_dt; p.z = z ? sb + hp.off_z : nullptr;
      p.B = sb + hp.off_B; p.C = sb + hp.off_C;
      p.A = A; p.Dv = D; p.bias = delta_bias;
      p.state = state + (size_t)(b0 * d.dim * d.dstate);
      p.y = sb + hp.off_y;
      if (ssm::launch_step(p, stream) != cudaSuccess) return SSM_ERR_CUDA;
      if (!ck(cudaEventRecord(hp.ev_comp[s], stream)) ||
          !ck(cudaStreamWaitEvent(hp.s_out, hp.ev_comp[s], 0)) ||
          !ck(cudaMemcpyAsync(static_cast<unsigned char *>(y) + (size_t)(b0 * d.dim) * eo,
                              sb + hp.off_y, (size_t)(rows * d.dim) * eo, cudaMemcpyDeviceToHost,
                              hp.s_out)) ||
          !ck(cudaEventRecord(hp.ev_out[s], hp.s_out)))
        return SSM_ERR_CUDA;
    }
    return SSM_OK;
  };
  const ssm_status st = run();
  const bool joined = ck(cudaEventRecord(hp.ev_done, hp.s_out)) &&
                      ck(cudaStreamWaitEvent(stream, hp.ev_done, 0)) &&
                      ck(cudaEventRecord(hp.ev_start, hp.s_in)) &&
                      ck(cudaStreamWaitEvent(stream, hp.ev_start, 0));
  if (st != SSM_OK) return st;
  return joined ? SSM_OK : SSM_ERR_CUDA;
}

}  // extern "C"
