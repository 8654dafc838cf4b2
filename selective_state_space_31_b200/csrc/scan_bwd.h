// scan_bwd.h -- parameter block of the backward kernel (internal to the
// library).
#pragma once

#include "scan_params.h"

namespace ssm {

// Backward pass (scan_bwd.cu): tokens per recomputation chunk.
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

}  // namespace ssm
