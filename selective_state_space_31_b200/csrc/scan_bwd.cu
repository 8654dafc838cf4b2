// scan_bwd.cu -- backward pass of the selective scan (reverse-mode gradient
// of the forward kernels' arithmetic: "Selective Scan trong Mamba ...",
// sections "Selection pha vo convolution kernel co dinh" and "Vi du Python";
// the pages' third pillar, recomputation instead of storing the (B, L, D, N)
// states, "Tai sao chi parallel scan van chua du nhanh?").
//
// Four lanes share one channel (b, d) and split its N states.  The chunk's
// states stay in registers (its loops are unrolled).  Pass 1 runs
// the recurrence forward and checkpoints the state at the start of every
// chunk of K tokens (the only state written to HBM: B*D*ceil(L/K)*N floats).
// Pass 2 walks the chunks backwards: it recomputes the chunk's K + 1 states
// from its checkpoint, then applies the chain rule token by token from the
// chunk's end, carrying g = dL/dh_t (g <- g * Abar_t after each token).
// Gradients of per-channel parameters (A, D, bias) are summed in registers
// and added once per thread; gradients of the per-token B_t, C_t (shared by
// every channel) are first summed over the warp's channels by a shuffle
// reduce-scatter, then added with one atomic per (token, state) and warp.
// It costs three exps per state update (forward pass, recomputation,
// reverse).
#include "device_common.cuh"
#include "scan_bwd.h"

namespace ssm {

template <typename T>
__device__ __forceinline__ float ldb(const void *base, size_t i) {
  return to_f32(reinterpret_cast<const T *>(base)[i]);
}

// Sum over the TPC lanes that share a channel (xor butterfly; every lane of
// the group ends with the total).
template <int TPC>
__device__ __forceinline__ float group_sum(float v) {
#pragma unroll
  for (int m = TPC / 2; m >= 1; m >>= 1) v += __shfl_xor_sync(FULL_MASK, v, m);
  return v;
}

// Reduce-scatter over the G = 32 / TPC channels of a warp that hold the same
// state group: on entry every lane holds V values (its channel's
// contributions to V per-token sums), on exit lane (channel c) holds the sum
// over the warp's channels of value c (c < V).  log2(G) rounds of shuffles
// across lanes TPC, 2 TPC, ... apart.
template <int TPC, int V>
__device__ __forceinline__ float channel_reduce_scatter(float (&v)[V], int c) {
  constexpr int G = 32 / TPC;
  static_assert(V == G, "one value per channel of the warp");
#pragma unroll
  for (int m = G / 2; m >= 1; m >>= 1) {
    const bool upper = (c & m) != 0;
#pragma unroll
    for (int i = 0; i < m; ++i) {
      const float send = upper ? v[i] : v[i + m];
      const float keep = upper ? v[i + m] : v[i];
      v[i] = keep + __shfl_xor_sync(FULL_MASK, send, m * TPC);
    }
  }
  return v[0];
}

template <typename InT, typename GradT, int NPL, int TPC, int K>
__global__ void __launch_bounds__(128) bwd_kernel(const BwdParams p) {
  // TPC lanes per channel, lane q owns states q*NPL .. q*NPL + NPL-1; lanes
  // past the last channel run along (they take part in the shuffles) but
  // touch no memory
  const long long gt = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long chn = gt / TPC;
  const int q = (int)(gt % TPC);
  const bool active = chn < (long long)p.Bsz * p.D;
  const int b = active ? (int)(chn / p.D) : 0, d = active ? (int)(chn % p.D) : 0;
  const int N = p.N, L = p.L;
  const int nck = (L + K - 1) / K;
  float A2[NPL], An[NPL], h[NPL];
  bool on[NPL];
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    const int n = q * NPL + i;
    on[i] = active && n < N;
    An[i] = on[i] ? p.A[(size_t)d * N + n] : 0.f;
    A2[i] = An[i] * kLog2e;
    h[i] = (on[i] && p.has_h0) ? p.h0[((size_t)b * p.D + d) * N + n] : 0.f;
  }
  const float Dd = (active && p.has_D) ? p.Dv[d] : 0.f;
  const float bias = (active && p.has_bias) ? p.bias[d] : 0.f;
  float *ck = p.ws_ck + (size_t)(active ? chn : 0) * nck * N + q * NPL;
  auto delta_of = [&](float v) { return p.softplus ? softplus_f(v) : v; };
  auto idx = [&](int t) { return ((size_t)b * L + t) * p.D + d; };
  auto tok = [&](int t) { return ((size_t)b * L + t) * N + q * NPL; };

  // pass 1: forward with a checkpoint at the start of every chunk
  for (int c = 0; c < nck; ++c) {
#pragma unroll
    for (int i = 0; i < NPL; ++i)
      if (on[i]) ck[(size_t)c * N + i] = h[i];
    const int t1 = min(L, (c + 1) * K);
    if (active) {
      for (int t = c * K; t < t1; ++t) {
        const float xv = ldb<InT>(p.x, idx(t));
        const float dt = delta_of(ldb<InT>(p.dt, idx(t)) + bias);
#pragma unroll
        for (int i = 0; i < NPL; ++i)
          if (on[i]) h[i] = fmaf(ex2_approx(dt * A2[i]), h[i], dt * ldb<InT>(p.B, tok(t) + i) * xv);
      }
    }
  }

  // pass 2: chunks from the last, tokens from the chunk's end
  float g[NPL], dA_acc[NPL];
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    g[i] = (on[i] && p.dh_last) ? p.dh_last[((size_t)b * p.D + d) * N + q * NPL + i] : 0.f;
    dA_acc[i] = 0.f;
  }
  float dD_acc = 0.f, dbias_acc = 0.f;
  // channel of this lane within the warp, for the dB / dC reduction
  constexpr int G = 32 / TPC;
  constexpr bool kWarpRed = 2 * NPL <= G;  // the warp's channels reduce dB, dC first
  const int cw = (threadIdx.x & 31) / TPC;
  float hs[K + 1][NPL];  // this lane's states h_{t0} .. h_{t1} of the chunk (registers:
                         // the chunk loops are unrolled, tokens past the end skipped)
  for (int c = nck - 1; c >= 0; --c) {
    const int t0 = c * K, t1 = min(L, t0 + K);
#pragma unroll
    for (int i = 0; i < NPL; ++i) hs[0][i] = on[i] ? ck[(size_t)c * N + i] : 0.f;
#pragma unroll
    for (int k = 0; k < K; ++k) {
      const int t = t0 + k;
      if (t < t1) {
        const float xv = active ? ldb<InT>(p.x, idx(t)) : 0.f;
        const float dt = active ? delta_of(ldb<InT>(p.dt, idx(t)) + bias) : 0.f;
#pragma unroll
        for (int i = 0; i < NPL; ++i)
          hs[k + 1][i] = on[i] ? fmaf(ex2_approx(dt * A2[i]), hs[k][i],
                                      dt * ldb<InT>(p.B, tok(t) + i) * xv)
                               : 0.f;
      }
    }
#pragma unroll
    for (int k = K - 1; k >= 0; --k) {
      const int t = t0 + k;
      if (t >= t1) continue;  // (uniform over the warp: every lane has the same t1)
      const size_t i0 = idx(t), j = tok(t);
      const float xv = active ? ldb<InT>(p.x, i0) : 0.f;
      const float v = active ? ldb<InT>(p.dt, i0) + bias : 0.f;
      const float dt = delta_of(v);
      float sp = 0.f;
#pragma unroll
      for (int i = 0; i < NPL; ++i)
        if (on[i]) sp = fmaf(ldb<InT>(p.C, j + i), hs[k + 1][i], sp);
      const float s = group_sum<TPC>(sp) + Dd * xv;
      const float dyv = active ? ldb<GradT>(p.dy, i0) : 0.f;
      float ds = dyv;
      if (p.has_z) {
        const float zv = active ? ldb<InT>(p.z, i0) : 0.f;
        const float sig = __fdividef(1.f, 1.f + __expf(-zv));
        ds = dyv * zv * sig;                                          // dy * silu(z)
        if (active && q == 0) p.dz[i0] = dyv * s * sig * fmaf(zv, 1.f - sig, 1.f);
      }
      dD_acc = fmaf(ds, xv, dD_acc);
      float dxp = 0.f, ddtp = 0.f;
      // this channel's shares of dC_t and dB_t (NPL states each); summed over
      // the warp's channels below, then one atomic per (token, state) and warp
      float red[kWarpRed ? G : 2 * NPL];
#pragma unroll
      for (int i = 0; i < (kWarpRed ? G : 2 * NPL); ++i) red[i] = 0.f;
#pragma unroll
      for (int i = 0; i < NPL; ++i) {
        if (on[i]) {
          const float Cn = ldb<InT>(p.C, j + i), Bn = ldb<InT>(p.B, j + i);
          const float abar = ex2_approx(dt * A2[i]);
          red[i] = ds * hs[k + 1][i];
          g[i] = fmaf(ds, Cn, g[i]);
          const float dabar = g[i] * hs[k][i];
          ddtp += dabar * abar * An[i] + g[i] * Bn * xv;
          dA_acc[i] = fmaf(dabar * abar, dt, dA_acc[i]);
          red[NPL + i] = g[i] * dt * xv;
          dxp = fmaf(g[i] * dt, Bn, dxp);
          g[i] *= abar;
        }
      }
      bool reduced = false;
      if constexpr (kWarpRed) {
        if (p.warp_uniform_b) {
          // lane of channel cw ends with value cw summed over the warp's
          // channels (values 0..NPL-1 are dC, NPL..2NPL-1 are dB of its
          // states); every channel of the warp belongs to one batch element
          const float tot = channel_reduce_scatter<TPC, G>(red, cw);
          const int i = cw < NPL ? cw : cw - NPL;
          if (active && cw < 2 * NPL && q * NPL + i < N)
            atomicAdd((cw < NPL ? p.dC : p.dB) + j + i, tot);
          reduced = true;
        }
      }
      if (!reduced) {
#pragma unroll
        for (int i = 0; i < NPL; ++i)
          if (on[i]) {
            atomicAdd(p.dC + j + i, red[i]);
            atomicAdd(p.dB + j + i, red[NPL + i]);
          }
      }
      const float dxi = group_sum<TPC>(dxp) + ds * Dd;
      const float ddt = group_sum<TPC>(ddtp);
      const float dv = p.softplus ? ddt * __fdividef(1.f, 1.f + __expf(-v)) : ddt;
      dbias_acc += dv;
      if (active && q == 0) {
        p.dx[i0] = dxi;
        p.ddelta[i0] = dv;
      }
    }
  }
  if (p.dh0) {
#pragma unroll
    for (int i = 0; i < NPL; ++i)
      if (on[i]) p.dh0[((size_t)b * p.D + d) * N + q * NPL + i] = g[i];
  }
#pragma unroll
  for (int i = 0; i < NPL; ++i)
    if (on[i]) atomicAdd(p.dA + (size_t)d * N + q * NPL + i, dA_acc[i]);
  if (active && q == 0) {
    if (p.has_D) atomicAdd(p.dD + d, dD_acc);
    if (p.has_bias) atomicAdd(p.dbias + d, dbias_acc);
  }
}

template <typename InT, typename GradT, int NPL, int TPC>
static void launch_bwd_variant(BwdParams p, cudaStream_t stream) {
  const long long threads = (long long)p.Bsz * p.D * TPC;
  // a warp holds 32 / TPC consecutive channels: one batch element when D is
  // a multiple of that
  p.warp_uniform_b = p.D % (32 / TPC) == 0;
  bwd_kernel<InT, GradT, NPL, TPC, kBwdChunk>
      <<<(unsigned)((threads + 127) / 128), 128, 0, stream>>>(p);
}

// Four lanes per channel (N <= 16: up to 4 states each; larger N: 16 each),
// so a layer's B*D channels fill the SMs four times as densely as one
// thread per channel.
template <typename InT, typename GradT>
static cudaError_t bwd_by_n(const BwdParams &p, cudaStream_t stream) {
  if (p.N <= 4) launch_bwd_variant<InT, GradT, 1, 4>(p, stream);
  else if (p.N <= 16) launch_bwd_variant<InT, GradT, 4, 4>(p, stream);
  else launch_bwd_variant<InT, GradT, 16, 4>(p, stream);
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
