// scan_bwd.cu -- backward pass of the selective scan (reverse-mode gradient
// of the forward kernels' arithmetic: "Selective Scan trong Mamba ...",
// sections "Selection pha vo convolution kernel co dinh" and "Vi du Python";
// the pages' third pillar, recomputation instead of storing the (B, L, D, N)
// states, "Tai sao chi parallel scan van chua du nhanh?").
//
// One thread owns one channel (b, d) and all of its N states.  Pass 1 runs
// the recurrence forward and checkpoints the state at the start of every
// chunk of K tokens (the only state written to HBM: B*D*ceil(L/K)*N floats).
// Pass 2 walks the chunks backwards: it recomputes the chunk's K + 1 states
// from its checkpoint, then applies the chain rule token by token from the
// chunk's end, carrying g = dL/dh_t (g <- g * Abar_t after each token).
// Gradients of per-channel parameters (A, D, bias) are summed in registers
// and added once per thread; gradients of the per-token B_t, C_t (shared by
// every channel) are added with atomics.  This is the correctness-first form
// of the backward: it costs three exps per state update (forward pass,
// recomputation, reverse) and keeps the chunk's states in local memory.
#include "device_common.cuh"
#include "scan_bwd.h"

namespace ssm {

template <typename T>
__device__ __forceinline__ float ldb(const void *base, size_t i) {
  return to_f32(reinterpret_cast<const T *>(base)[i]);
}

template <typename InT, typename GradT, int NMAX, int K>
__global__ void __launch_bounds__(32) bwd_kernel(const BwdParams p) {
  const long long chn = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (chn >= (long long)p.Bsz * p.D) return;
  const int b = (int)(chn / p.D), d = (int)(chn % p.D);
  const int N = p.N, L = p.L;
  const int nck = (L + K - 1) / K;
  float A2[NMAX], An[NMAX], h[NMAX];
#pragma unroll
  for (int n = 0; n < NMAX; ++n) {
    const bool on = n < N;
    An[n] = on ? p.A[(size_t)d * N + n] : 0.f;
    A2[n] = An[n] * kLog2e;
    h[n] = (on && p.has_h0) ? p.h0[((size_t)b * p.D + d) * N + n] : 0.f;
  }
  const float Dd = p.has_D ? p.Dv[d] : 0.f;
  const float bias = p.has_bias ? p.bias[d] : 0.f;
  float *ck = p.ws_ck + (size_t)chn * nck * N;
  auto delta_of = [&](float v) { return p.softplus ? softplus_f(v) : v; };

  // pass 1: forward with a checkpoint at the start of every chunk
  for (int c = 0; c < nck; ++c) {
#pragma unroll
    for (int n = 0; n < NMAX; ++n)
      if (n < N) ck[(size_t)c * N + n] = h[n];
    const int t1 = min(L, (c + 1) * K);
    for (int t = c * K; t < t1; ++t) {
      const size_t i = ((size_t)b * L + t) * p.D + d, j = ((size_t)b * L + t) * N;
      const float xv = ldb<InT>(p.x, i);
      const float dt = delta_of(ldb<InT>(p.dt, i) + bias);
#pragma unroll
      for (int n = 0; n < NMAX; ++n)
        if (n < N) h[n] = fmaf(ex2_approx(dt * A2[n]), h[n], dt * ldb<InT>(p.B, j + n) * xv);
    }
  }

  // pass 2: chunks from the last, tokens from the chunk's end
  float g[NMAX], dA_acc[NMAX];
#pragma unroll
  for (int n = 0; n < NMAX; ++n) {
    g[n] = (n < N && p.dh_last) ? p.dh_last[((size_t)b * p.D + d) * N + n] : 0.f;
    dA_acc[n] = 0.f;
  }
  float dD_acc = 0.f, dbias_acc = 0.f;
  float hs[K + 1][NMAX];  // states h_{t0} .. h_{t1} of the chunk
  for (int c = nck - 1; c >= 0; --c) {
    const int t0 = c * K, t1 = min(L, t0 + K);
#pragma unroll
    for (int n = 0; n < NMAX; ++n) hs[0][n] = n < N ? ck[(size_t)c * N + n] : 0.f;
    for (int t = t0; t < t1; ++t) {
      const size_t i = ((size_t)b * L + t) * p.D + d, j = ((size_t)b * L + t) * N;
      const float xv = ldb<InT>(p.x, i);
      const float dt = delta_of(ldb<InT>(p.dt, i) + bias);
      const int k = t - t0;
#pragma unroll
      for (int n = 0; n < NMAX; ++n)
        hs[k + 1][n] = n < N ? fmaf(ex2_approx(dt * A2[n]), hs[k][n],
                                    dt * ldb<InT>(p.B, j + n) * xv)
                             : 0.f;
    }
    for (int t = t1 - 1; t >= t0; --t) {
      const size_t i = ((size_t)b * L + t) * p.D + d, j = ((size_t)b * L + t) * N;
      const int k = t - t0;
      const float xv = ldb<InT>(p.x, i);
      const float v = ldb<InT>(p.dt, i) + bias;
      const float dt = delta_of(v);
      float s = Dd * xv;
#pragma unroll
      for (int n = 0; n < NMAX; ++n)
        if (n < N) s = fmaf(ldb<InT>(p.C, j + n), hs[k + 1][n], s);
      const float dyv = ldb<GradT>(p.dy, i);
      float ds = dyv;
      if (p.has_z) {
        const float zv = ldb<InT>(p.z, i);
        const float sig = __fdividef(1.f, 1.f + __expf(-zv));
        ds = dyv * zv * sig;                                      // dy * silu(z)
        p.dz[i] = dyv * s * sig * fmaf(zv, 1.f - sig, 1.f);       // dy * s * silu'(z)
      }
      float dxi = ds * Dd;
      dD_acc = fmaf(ds, xv, dD_acc);
      float ddt = 0.f;
#pragma unroll
      for (int n = 0; n < NMAX; ++n) {
        if (n < N) {
          const float Cn = ldb<InT>(p.C, j + n), Bn = ldb<InT>(p.B, j + n);
          const float abar = ex2_approx(dt * A2[n]);
          atomicAdd(p.dC + j + n, ds * hs[k + 1][n]);
          g[n] = fmaf(ds, Cn, g[n]);
          const float dabar = g[n] * hs[k][n];
          ddt += dabar * abar * An[n] + g[n] * Bn * xv;
          dA_acc[n] = fmaf(dabar * abar, dt, dA_acc[n]);
          atomicAdd(p.dB + j + n, g[n] * dt * xv);
          dxi = fmaf(g[n] * dt, Bn, dxi);
          g[n] *= abar;
        }
      }
      p.dx[i] = dxi;
      const float dv = p.softplus ? ddt * __fdividef(1.f, 1.f + __expf(-v)) : ddt;
      p.ddelta[i] = dv;
      dbias_acc += dv;
    }
  }
  if (p.dh0) {
#pragma unroll
    for (int n = 0; n < NMAX; ++n)
      if (n < N) p.dh0[((size_t)b * p.D + d) * N + n] = g[n];
  }
#pragma unroll
  for (int n = 0; n < NMAX; ++n)
    if (n < N) atomicAdd(p.dA + (size_t)d * N + n, dA_acc[n]);
  if (p.has_D) atomicAdd(p.dD + d, dD_acc);
  if (p.has_bias) atomicAdd(p.dbias + d, dbias_acc);
}

// One warp per CTA: a layer has only B*D channels (12288 for the 130M
// layer), so small CTAs spread them over every SM.
constexpr int kBwdThreads = 32;

template <typename InT, typename GradT>
static cudaError_t bwd_by_n(const BwdParams &p, cudaStream_t stream) {
  const long long chans = (long long)p.Bsz * p.D;
  const unsigned grid = (unsigned)((chans + kBwdThreads - 1) / kBwdThreads);
  if (p.N <= 4) bwd_kernel<InT, GradT, 4, kBwdChunk><<<grid, kBwdThreads, 0, stream>>>(p);
  else if (p.N <= 16) bwd_kernel<InT, GradT, 16, kBwdChunk><<<grid, kBwdThreads, 0, stream>>>(p);
  else bwd_kernel<InT, GradT, 64, kBwdChunk><<<grid, kBwdThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_bwd(const BwdParams &p, cudaStream_t stream) {
  // the accumulated gradients start from zero
  const size_t bln = (size_t)p.Bsz * p.L * p.N * sizeof(float);
  cudaError_t e = cudaSuccess;
  if (bln) {
    if ((e = cudaMemsetAsync(p.dB, 0, bln, stream)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(p.dC, 0, bln, stream)) != cudaSuccess) return e;
  }
  if ((e = cudaMemsetAsync(p.dA, 0, (size_t)p.D * p.N * sizeof(float), stream)) != cudaSuccess)
    return e;
  if (p.has_D && (e = cudaMemsetAsync(p.dD, 0, (size_t)p.D * sizeof(float), stream)) != cudaSuccess)
    return e;
  if (p.has_bias &&
      (e = cudaMemsetAsync(p.dbias, 0, (size_t)p.D * sizeof(float), stream)) != cudaSuccess)
    return e;
  if ((long long)p.Bsz * p.D == 0) return cudaSuccess;
  if (!p.in_bf16 && !p.out_bf16) return bwd_by_n<float, float>(p, stream);
  if (p.in_bf16 && p.out_bf16) return bwd_by_n<__nv_bfloat16, __nv_bfloat16>(p, stream);
  if (p.in_bf16) return bwd_by_n<__nv_bfloat16, float>(p, stream);
  return bwd_by_n<float, __nv_bfloat16>(p, stream);
}

}  // namespace ssm
