// peak_probe.cu -- throughput probes for the roofline denominators of the
// scan: the special-function unit (ex2.approx, the exponential of every
// state update) and the FP32 FMA pipe.  Each thread runs several independent
// dependency chains so the unit under test, not latency, limits the rate.
// The benchmark times a launch with CUDA events and divides the operation
// count by it; the result is written to `sink` so nothing is optimised away.
#include <cuda_runtime.h>

#include <cstdint>

#include "ssm_scan.h"
#include "device_common.cuh"

namespace {

constexpr int kChains = 8;
constexpr int kUnroll = 8;
constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads) ex2_probe(int64_t iters, float *sink) {
  float v[kChains];
#pragma unroll
  for (int c = 0; c < kChains; ++c) v[c] = 0.25f + 0.01f * (threadIdx.x & 7) + 0.03f * c;
  for (int64_t i = 0; i < iters; ++i) {
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)
#pragma unroll
      for (int c = 0; c < kChains; ++c) v[c] = ssm::ex2_approx(-v[c]);  // stays in (0.5, 1)
  }
  float s = 0.f;
#pragma unroll
  for (int c = 0; c < kChains; ++c) s += v[c];
  if (s == 12345.f) sink[blockIdx.x] = s;  // never true; keeps the chains live
}

__global__ void __launch_bounds__(kThreads) ffma_probe(int64_t iters, float *sink) {
  float v[kChains];
#pragma unroll
  for (int c = 0; c < kChains; ++c) v[c] = 1.f + 0.001f * c;
  const float a = 0.999f + 1e-6f * (threadIdx.x & 3), b = 1e-3f;
  for (int64_t i = 0; i < iters; ++i) {
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)
#pragma unroll
      for (int c = 0; c < kChains; ++c) v[c] = fmaf(v[c], a, b);  // converges to b / (1 - a)
  }
  float s = 0.f;
#pragma unroll
  for (int c = 0; c < kChains; ++c) s += v[c];
  if (s == 12345.f) sink[blockIdx.x] = s;
}

// Both 2^x implementations of the kernels on the same inputs.
__global__ void __launch_bounds__(256) exp2_pair_kernel(const float *x, float *y_fma,
                                                        float *y_sfu, int64_t n) {
  const int64_t i = 2 * ((int64_t)blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float2 v = make_float2(x[i], i + 1 < n ? x[i + 1] : 0.f);
  const float2 f = ssm::exp2_fma2(v);
  y_fma[i] = f.x;
  y_sfu[i] = ssm::ex2_approx(v.x);
  if (i + 1 < n) {
    y_fma[i + 1] = f.y;
    y_sfu[i + 1] = ssm::ex2_approx(v.y);
  }
}

}  // namespace

extern "C" SSM_API ssm_status ssm_probe_exp2(const float *x, float *y_fma, float *y_sfu,
                                             int64_t n, ssm_stream_t stream) {
  if (n < 0 || (n > 0 && (!x || !y_fma || !y_sfu))) return SSM_ERR_INVALID_ARG;
  if (n == 0) return SSM_OK;
  const int64_t pairs = (n + 1) / 2;
  if ((pairs + 255) / 256 > INT32_MAX) return SSM_ERR_UNSUPPORTED;
  exp2_pair_kernel<<<(unsigned)((pairs + 255) / 256), 256, 0,
                     reinterpret_cast<cudaStream_t>(stream)>>>(x, y_fma, y_sfu, n);
  return cudaGetLastError() == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

extern "C" SSM_API ssm_status ssm_probe_peak(int kind, int64_t iters, int blocks,
                                             float *sink, int64_t *ops, ssm_stream_t stream) {
  if (iters < 1 || blocks < 1 || !sink || !ops || (kind != 0 && kind != 1))
    return SSM_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (kind == 0)
    ex2_probe<<<blocks, kThreads, 0, s>>>(iters, sink);
  else
    ffma_probe<<<blocks, kThreads, 0, s>>>(iters, sink);
  *ops = (int64_t)blocks * kThreads * iters * kUnroll * kChains;
  return cudaGetLastError() == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}
