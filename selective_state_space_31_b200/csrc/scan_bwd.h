// scan_bwd.h -- parameter blocks of the backward kernels (internal to the
// library).
#pragma once

#include "scan_params.h"

namespace ssm {

// General backward kernel (scan_bwd.cu): tokens per recomputation chunk.
constexpr int kBwdChunk = 16;
struct BwdParams {
  int Bsz, L, D, N;
  bool softplus, has_z, has_D, has_bias, has_h0;
  int in_bf16, out_bf16;                 // inputs / dy dtypes
  const void *x, *dt, *z, *B, *C, *dy;
  const float *A, *Dv, *bias, *h0, *dh_last;
  float *dx, *ddelta, *dz, *dB, *dC, *dA, *dD, *dbias, *dh0;
  float *ws_ck;                          // B * D * ceil(L / kBwdChunk) * N checkpoints
  bool warp_uniform_b;                   // every warp's channels share one batch element
};
cudaError_t launch_bwd(const BwdParams &p, cudaStream_t stream);

// Fused backward kernel (scan_bwd_tma.cu): TMA-fed tiles of DT channels x
// kBwdStage tokens, a load warp and W scan warps of 32 / LPC channels each.
constexpr int kBwdStage = 8;
struct BwdMaps {
  CUtensorMap x, dt, z, dy, B, C;  // boxes (DT, kBwdStage) and (N, kBwdStage)
};
struct BwdShape {
  int lpc = 0, warps = 0;  // lanes per channel, scan warps per CTA
  int DT = 0, nDT = 0;     // channels per row tile, row tiles per batch element
  int64_t rows = 0;        // B * nDT: one CTA each
  int S = 0;               // stages of kBwdStage tokens
  int M = 1, SPS = 0;      // segments per row tile (scanned at once) and their stages
  size_t smem = 0;
  int occ = 0;              // resident CTAs per SM
  size_t ws_ck_floats = 0;  // (rows, S, DT, N): the state at the start of each stage
  size_t ws_bc_floats = 0;  // (B, nDT, L, 2N): each row tile's sums of dC and dB
  size_t ws_map_floats = 0; // segments: (rows, M, DT, N + 4) twice: forward and adjoint maps
};
struct BwdTmaParams {
  int Bsz, L, D, N, DT, nDT, S;
  int rows;
  int M, SPS;  // segments per row tile and stages per segment (M = 1: none)
  bool softplus, has_z, has_D, has_bias, has_h0;
  const float *A, *Dv, *bias, *h0, *dh_last;
  float *dx, *ddelta, *dz, *dB, *dC, *dA, *dD, *dbias, *dh0;
  float *ws_ck, *ws_bc;
  // segments: per (row, segment, channel) the forward map (state reached
  // from 0, then sum of Delta) and the adjoint map (dL/dh carried from 0
  // across the segment, then sum of Delta), N + 4 floats apart
  float *ws_fmap, *ws_amap;
  Control *ctl;  // status (timeouts) only
  unsigned long long timeout_ns;
};
// Is there a fused variant for this problem, and with which shape?
// (dtypes as ssm_dtype values; `warps` 0 = free choice)
bool choose_bwd_shape(int in_dtype, int out_dtype, int64_t batch, int64_t seqlen, int64_t dim,
                      int ns, int warps, int segments, int sms, BwdShape *out);
cudaError_t launch_bwd_tma(int in_dtype, int out_dtype, const BwdShape &s, const BwdMaps &maps,
                           const BwdTmaParams &p, cudaStream_t stream);

}  // namespace ssm
