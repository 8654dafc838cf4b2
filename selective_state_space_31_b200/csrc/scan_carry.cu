// scan_carry.cu -- maps of whole sequences and their composition, the pieces
// of a scan whose L is split over several devices or calls.
//
// A sequence (or any run of tokens) acts on the state as one affine map per
// channel and state, h -> P h + e, with P = prod_t exp(Delta_t A) =
// exp(A sum_t Delta_t) and e the state reached from h = 0 ("Scan bien
// recurrence thanh phep toan co the song song hoa ra sao?": the per-token
// maps compose associatively, (A2,b2) (x) (A1,b1) = (A2 A1, A2 b1 + b2)).
// map_general_kernel computes (sum Delta, e) of a whole sequence for shapes
// the fused kernel does not take; fold_maps_kernel composes `count` such
// maps in order onto a starting state (also the last step of a fused-kernel
// sequence map, whose carry pass leaves one map per sub-chunk).
#include "device_common.cuh"
#include "scan_params.h"

namespace ssm {

namespace {

template <typename T>
__device__ __forceinline__ float ldc(const void *base, size_t i) {
  return to_f32(reinterpret_cast<const T *>(base)[i]);
}

// One thread per channel (b, d): Delta, the state from 0 and the sum of
// Delta over the whole sequence.
template <typename InT, int NMAX>
__global__ void __launch_bounds__(128) map_general_kernel(const MapParams p) {
  const long long chn = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (chn >= (long long)p.Bsz * p.D) return;
  const int b = (int)(chn / p.D), d = (int)(chn % p.D);
  const int N = p.N;
  float h[NMAX], A2[NMAX], invA[NMAX];
#pragma unroll
  for (int n = 0; n < NMAX; ++n) {
    const float a = n < N ? p.A[(size_t)d * N + n] : 0.f;
    h[n] = 0.f;
    A2[n] = a * kLog2e;
    invA[n] = a != 0.f ? 1.f / a : 0.f;
  }
  const float bias = p.bias ? p.bias[d] : 0.f;
  float sum = 0.f;
  for (int t = 0; t < p.L; ++t) {
    const size_t i = ((size_t)b * p.L + t) * p.D + d;
    const size_t j = ((size_t)b * p.L + t) * N;
    const float xv = ldc<InT>(p.x, i);
    const float v = ldc<InT>(p.dt, i) + bias;
    const float dlt = p.softplus ? softplus_f(v) : v;
    sum += dlt;
#pragma unroll
    for (int n = 0; n < NMAX; ++n) {
      if (n < N) {
        const float arg = dlt * A2[n];
        const float a = ex2_approx(arg);
        const float bx = p.zoh ? zoh_coef(arg * kLn2, a, dlt, invA[n]) * xv * ldc<InT>(p.B, j + n)
                               : dlt * xv * ldc<InT>(p.B, j + n);
        h[n] = fmaf(a, h[n], bx);
      }
    }
  }
#pragma unroll
  for (int n = 0; n < NMAX; ++n)
    if (n < N) p.map_h[((size_t)b * p.D + d) * N + n] = h[n];
  p.map_s[(size_t)b * p.D + d] = sum;
}

// One thread per (b, d, n): h = h0; for j < count: h = exp(A s_j) h + e_j.
// maps_h: (count, B, D, N); maps_s: (count, B, D), both with stride
// `map_stride` elements between consecutive maps of one channel (maps of a
// carry pass are (B, count, D, ...) instead: the strides say which).
__global__ void __launch_bounds__(256) fold_maps_kernel(const FoldParams p) {
  const long long k = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long total = (long long)p.Bsz * p.D * p.N;
  if (k >= total) return;
  const int n = (int)(k % p.N);
  const long long bd = k / p.N;
  const int d = (int)(bd % p.D), b = (int)(bd / p.D);
  const float A2 = p.A[(size_t)d * p.N + n] * kLog2e;
  float h = p.h0 ? p.h0[k] : 0.f;
  float s_total = 0.f;
  for (int j = 0; j < p.count; ++j) {
    const size_t base = (size_t)b * p.stride_b + (size_t)j * p.stride_j + d;
    const float s = p.maps_s[base];
    h = fmaf(ex2_approx(A2 * s), h, p.maps_h[base * p.N + n]);
    s_total += s;
  }
  p.h_out[k] = h;
  if (p.s_out && n == 0) p.s_out[bd] = s_total;
}

}  // namespace

cudaError_t launch_map_general(const MapParams &p, cudaStream_t stream) {
  const long long chans = (long long)p.Bsz * p.D;
  if (chans == 0) return cudaSuccess;
  const unsigned grid = (unsigned)((chans + 127) / 128);
  if (p.in_bf16) {
    if (p.N <= 16) map_general_kernel<__nv_bfloat16, 16><<<grid, 128, 0, stream>>>(p);
    else map_general_kernel<__nv_bfloat16, 64><<<grid, 128, 0, stream>>>(p);
  } else {
    if (p.N <= 16) map_general_kernel<float, 16><<<grid, 128, 0, stream>>>(p);
    else map_general_kernel<float, 64><<<grid, 128, 0, stream>>>(p);
  }
  return cudaGetLastError();
}

cudaError_t launch_fold_maps(const FoldParams &p, cudaStream_t stream) {
  const long long total = (long long)p.Bsz * p.D * p.N;
  if (total == 0) return cudaSuccess;
  fold_maps_kernel<<<(unsigned)((total + 255) / 256), 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace ssm
