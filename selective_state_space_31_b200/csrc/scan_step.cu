// scan_step.cu -- single-token decode step ("Selective Scan trong Mamba ...",
// section "Selective Scan thay doi inference chuoi dai nhu the nao?": the
// fixed-size state of a layer is updated once per new token, no re-scan).
//
// The step is bandwidth-bound: the (B, D, N) fp32 state is read and written
// once per token (2 x 4 bytes per state) while the per-token inputs are
// (B, D) and (B, N) vectors.  Threads own NPT consecutive states of one
// channel (128-bit loads/stores of the state), TPC = N / NPT threads share a
// channel and combine their partial readouts with xor shuffles.  The
// per-channel scalars (x, delta, z) are re-read by the TPC threads of a
// channel from the same cache line and softplus/silu are recomputed by each;
// both are free next to the state traffic.
#include "device_common.cuh"
#include "scan_params.h"

#ifndef SSM_STEP_MINB
#define SSM_STEP_MINB 1
#endif
#ifndef SSM_STEP_ITEMS
#define SSM_STEP_ITEMS 1
#endif

namespace ssm {

template <typename T>
__device__ __forceinline__ float ld1(const void *base, size_t i) {
  return to_f32(reinterpret_cast<const T *>(base)[i]);
}

// Four consecutive values (a 16-byte-aligned group of states) as fp32.
__device__ __forceinline__ void ldg4(const float *src, float *v) {
  const float4 w = __ldg(reinterpret_cast<const float4 *>(src));
  v[0] = w.x; v[1] = w.y; v[2] = w.z; v[3] = w.w;
}
__device__ __forceinline__ void ldg4(const __nv_bfloat16 *src, float *v) {
  const uint2 w = __ldg(reinterpret_cast<const uint2 *>(src));
  v[0] = __uint_as_float(w.x << 16);  // a bf16 is the upper half of the equal fp32
  v[1] = __uint_as_float(w.x & 0xffff0000u);
  v[2] = __uint_as_float(w.y << 16);
  v[3] = __uint_as_float(w.y & 0xffff0000u);
}

// TPC threads share a channel; thread q owns the 4-state groups q, q + TPC,
// q + 2 TPC, ... (NPT states), so each of its 16-byte state accesses, taken
// over the warp, covers whole 32-byte sectors.
template <typename InT, typename OutT, int NPT, int TPC, int ITEMS, bool ZOH>
__global__ void __launch_bounds__(256, SSM_STEP_MINB) step_kernel(const StepParams p) {
  // ITEMS work items per thread, a grid apart: every item's state reads are
  // issued before any of them is used
  constexpr int G = NPT / 4;  // state groups per thread
  const long long total = (long long)gridDim.x * blockDim.x;
  const long long g0 = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long nch = (long long)p.Bsz * p.D;
  constexpr int N = NPT * TPC;
  const int q = (int)(g0 % TPC);  // the same for every item (total is a multiple of TPC)
  float4 s4[ITEMS][G];
#pragma unroll
  for (int it = 0; it < ITEMS; ++it) {
    const long long chn = (g0 + it * total) / TPC;
    if (chn < nch) {
      const float4 *sp = reinterpret_cast<const float4 *>(p.state + (size_t)chn * N);
#pragma unroll
      for (int i = 0; i < G; ++i) s4[it][i] = __ldcs(sp + i * TPC + q);
    }
  }
#pragma unroll
  for (int it = 0; it < ITEMS; ++it) {
    const long long chn = (g0 + it * total) / TPC;
    const bool active = chn < nch;
    float acc = 0.f, xv = 0.f, zv = 0.f, Dd = 0.f;
    if (active) {
      const int b = (int)(chn / p.D), d = (int)(chn % p.D);
      float Av[NPT], Bv[NPT], Cv[NPT];
#pragma unroll
      for (int i = 0; i < G; ++i) {
        const int n0 = 4 * (i * TPC + q);
        ldg4(p.A + (size_t)d * N + n0, Av + 4 * i);
        ldg4(reinterpret_cast<const InT *>(p.B) + (size_t)b * N + n0, Bv + 4 * i);
        ldg4(reinterpret_cast<const InT *>(p.C) + (size_t)b * N + n0, Cv + 4 * i);
      }
      xv = ld1<InT>(p.x, (size_t)chn);
      const float v = ld1<InT>(p.dt, (size_t)chn) + (p.has_bias ? __ldg(p.bias + d) : 0.f);
      if (p.has_z) zv = ld1<InT>(p.z, (size_t)chn);
      if (p.has_D) Dd = __ldg(p.Dv + d);
      const float dlt = p.softplus ? softplus_f(v) : v;
      const float dtx = dlt * xv;
      float h[NPT];
#pragma unroll
      for (int i = 0; i < G; ++i) {
        h[4 * i] = s4[it][i].x; h[4 * i + 1] = s4[it][i].y;
        h[4 * i + 2] = s4[it][i].z; h[4 * i + 3] = s4[it][i].w;
      }
#pragma unroll
      for (int n = 0; n < NPT; ++n) {
        const float arg = dlt * (Av[n] * kLog2e);
        const float a = ex2_approx(arg);
        // Bbar x: Delta B x, or (e^{Delta A} - 1) / A * B x under zero-order hold
        float bx = dtx * Bv[n];
        if constexpr (ZOH)
          bx = zoh_coef(arg * kLn2, a, dlt, Av[n] != 0.f ? 1.f / Av[n] : 0.f) * xv * Bv[n];
        h[n] = fmaf(a, h[n], bx);
        acc = fmaf(Cv[n], h[n], acc);
      }
      float4 *sp = reinterpret_cast<float4 *>(p.state + (size_t)chn * N);
#pragma unroll
      for (int i = 0; i < G; ++i)
        __stcs(sp + i * TPC + q, make_float4(h[4 * i], h[4 * i + 1], h[4 * i + 2], h[4 * i + 3]));
    }
#pragma unroll
    for (int m = TPC / 2; m >= 1; m >>= 1) acc += __shfl_xor_sync(FULL_MASK, acc, m);
    if (active && q == 0) {
      float yv = fmaf(Dd, xv, acc);
      if (p.has_z) yv *= silu_f(zv);
      reinterpret_cast<OutT *>(p.y)[chn] = from_f32<OutT>(yv);
    }
  }
}

// Any dstate: one thread per channel, plain loads.
template <typename InT, typename OutT>
__global__ void __launch_bounds__(128) step_general_kernel(const StepParams p) {
  const long long chn = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (chn >= (long long)p.Bsz * p.D) return;
  const int b = (int)(chn / p.D), d = (int)(chn % p.D), N = p.N;
  const float xv = ld1<InT>(p.x, (size_t)chn);
  const float v = ld1<InT>(p.dt, (size_t)chn) + (p.has_bias ? p.bias[d] : 0.f);
  const float dlt = p.softplus ? softplus_f(v) : v;
  const float dtx = dlt * xv;
  float acc = 0.f;
  for (int n = 0; n < N; ++n) {
    float *sp = p.state + (size_t)chn * N + n;
    const float An = p.A[(size_t)d * N + n];
    const float arg = dlt * (An * kLog2e);
    const float a = ex2_approx(arg);
    const float Bn = ld1<InT>(p.B, (size_t)b * N + n);
    const float bx = p.zoh ? zoh_coef(arg * kLn2, a, dlt, An != 0.f ? 1.f / An : 0.f) * xv * Bn
                           : dtx * Bn;
    const float hn = fmaf(a, *sp, bx);
    *sp = hn;
    acc = fmaf(ld1<InT>(p.C, (size_t)b * N + n), hn, acc);
  }
  float yv = fmaf(p.has_D ? p.Dv[d] : 0.f, xv, acc);
  if (p.has_z) yv *= silu_f(ld1<InT>(p.z, (size_t)chn));
  reinterpret_cast<OutT *>(p.y)[chn] = from_f32<OutT>(yv);
}

template <typename InT, typename OutT>
static cudaError_t step_typed(const StepParams &p, bool vec_ok, cudaStream_t stream) {
  const long long chans = (long long)p.Bsz * p.D;
  if (chans == 0) return cudaSuccess;
  constexpr int IT = SSM_STEP_ITEMS;
  auto grid_for = [&](int tpc) { return (unsigned)((chans * tpc + 256 * IT - 1) / (256 * IT)); };
  if (vec_ok) {
    if (p.zoh) {
      switch (p.N) {
        case 4: step_kernel<InT, OutT, 4, 1, IT, true><<<grid_for(1), 256, 0, stream>>>(p); return cudaGetLastError();
        case 8: step_kernel<InT, OutT, 8, 1, IT, true><<<grid_for(1), 256, 0, stream>>>(p); return cudaGetLastError();
        case 16: step_kernel<InT, OutT, 8, 2, IT, true><<<grid_for(2), 256, 0, stream>>>(p); return cudaGetLastError();
        case 32: step_kernel<InT, OutT, 8, 4, IT, true><<<grid_for(4), 256, 0, stream>>>(p); return cudaGetLastError();
        case 64: step_kernel<InT, OutT, 8, 8, IT, true><<<grid_for(8), 256, 0, stream>>>(p); return cudaGetLastError();
        default: break;
      }
    } else {
      switch (p.N) {
        case 4: step_kernel<InT, OutT, 4, 1, IT, false><<<grid_for(1), 256, 0, stream>>>(p); return cudaGetLastError();
        case 8: step_kernel<InT, OutT, 8, 1, IT, false><<<grid_for(1), 256, 0, stream>>>(p); return cudaGetLastError();
        case 16: step_kernel<InT, OutT, 8, 2, IT, false><<<grid_for(2), 256, 0, stream>>>(p); return cudaGetLastError();
        case 32: step_kernel<InT, OutT, 8, 4, IT, false><<<grid_for(4), 256, 0, stream>>>(p); return cudaGetLastError();
        case 64: step_kernel<InT, OutT, 8, 8, IT, false><<<grid_for(8), 256, 0, stream>>>(p); return cudaGetLastError();
        default: break;
      }
    }
  }
  step_general_kernel<InT, OutT><<<(unsigned)((chans + 127) / 128), 128, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_step(const StepParams &p, cudaStream_t stream) {
  auto al16 = [](const void *q) { return (reinterpret_cast<uintptr_t>(q) % 16) == 0; };
  const bool vec_ok = al16(p.state) && al16(p.A) && al16(p.B) && al16(p.C);
  if (!p.in_bf16 && !p.out_bf16) return step_typed<float, float>(p, vec_ok, stream);
  if (p.in_bf16 && p.out_bf16) return step_typed<__nv_bfloat16, __nv_bfloat16>(p, vec_ok, stream);
  if (p.in_bf16) return step_typed<__nv_bfloat16, float>(p, vec_ok, stream);
  return step_typed<float, __nv_bfloat16>(p, vec_ok, stream);
}

}  // namespace ssm
