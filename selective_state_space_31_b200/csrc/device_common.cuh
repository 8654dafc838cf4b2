// device_common.cuh -- sm_100a device helpers shared by the scan kernels:
// transcendental wrappers, bf16 conversion, mbarrier / TMA (cp.async.bulk)
// PTX wrappers, bounded waits and the global timer.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ssm {

constexpr unsigned FULL_MASK = 0xffffffffu;
constexpr float kLog2e = 1.4426950408889634f;

// status codes written by kernels into Control::status (match ssm_status)
constexpr int kStatusOk = 0;
constexpr int kStatusTimeout = 5;

// --- arithmetic -----------------------------------------------------------

// 2^x on the special-function unit (ex2.approx, flush-to-zero).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// --- packed fp32 pairs (sm_100 f32x2 instructions: two lanes of fp32 work per
// issued instruction; round-to-nearest like the scalar forms) -------------

// float2 is an 8-byte aligned pair: pass it to PTX as one 64-bit register.
#define SSM_U64(v) (*reinterpret_cast<unsigned long long *>(&(v)))
#define SSM_CU64(v) (*reinterpret_cast<const unsigned long long *>(&(v)))

// a * b + c, elementwise on the pair
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(SSM_U64(d)) : "l"(SSM_CU64(a)), "l"(SSM_CU64(b)), "l"(SSM_CU64(c)));
  return d;
}
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
  float2 d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(SSM_U64(d)) : "l"(SSM_CU64(a)), "l"(SSM_CU64(b)));
  return d;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  float2 d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(SSM_U64(d)) : "l"(SSM_CU64(a)), "l"(SSM_CU64(b)));
  return d;
}

// log1p(u) for u in [0, 1] as u * P(u), P of degree 8 fitted to log1p(u)/u
// by least squares on Chebyshev nodes (csrc/fit_log1p.py derives and checks
// the coefficients: max relative error 1.9e-7 in float32).  Never forms
// 1 + u, so small u keeps full relative accuracy.
__device__ __forceinline__ float log1p_unit(float u) {
  float p = 0.00525345793f;
  p = fmaf(p, u, -0.0295885075f);
  p = fmaf(p, u, 0.0783616677f);
  p = fmaf(p, u, -0.136747703f);
  p = fmaf(p, u, 0.191114306f);
  p = fmaf(p, u, -0.248443693f);
  p = fmaf(p, u, 0.333192706f);
  p = fmaf(p, u, -0.499995023f);
  p = fmaf(p, u, 1.0f);
  return u * p;
}

// 1/x on the special-function unit (rcp.approx, flush-to-zero).
__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// softplus(v) = log(1 + e^v) = max(v, 0) + log1p(e^{-|v|}), e^{-|v|} in (0, 1]
// on the special-function unit, log1p by the fitted polynomial.
__device__ __forceinline__ float softplus_f(float v) {
  return fmaxf(v, 0.f) + log1p_unit(ex2_approx(-fabsf(v) * kLog2e));
}

// silu(z) = z * sigmoid(z) = z / (1 + e^{-z}).
__device__ __forceinline__ float silu_f(float z) { return __fdividef(z, 1.f + __expf(-z)); }

// The same two functions on a pair of channels, with packed arithmetic.
__device__ __forceinline__ float2 log1p_unit2(float2 u) {
  float2 p = make_float2(0.00525345793f, 0.00525345793f);
  p = ffma2(p, u, make_float2(-0.0295885075f, -0.0295885075f));
  p = ffma2(p, u, make_float2(0.0783616677f, 0.0783616677f));
  p = ffma2(p, u, make_float2(-0.136747703f, -0.136747703f));
  p = ffma2(p, u, make_float2(0.191114306f, 0.191114306f));
  p = ffma2(p, u, make_float2(-0.248443693f, -0.248443693f));
  p = ffma2(p, u, make_float2(0.333192706f, 0.333192706f));
  p = ffma2(p, u, make_float2(-0.499995023f, -0.499995023f));
  p = ffma2(p, u, make_float2(1.0f, 1.0f));
  return fmul2(u, p);
}
__device__ __forceinline__ float2 softplus_f2(float2 v) {
  const float2 u = make_float2(ex2_approx(-fabsf(v.x) * kLog2e), ex2_approx(-fabsf(v.y) * kLog2e));
  return fadd2(make_float2(fmaxf(v.x, 0.f), fmaxf(v.y, 0.f)), log1p_unit2(u));
}
__device__ __forceinline__ float2 silu_f2(float2 z) {
  const float2 e = make_float2(ex2_approx(-z.x * kLog2e), ex2_approx(-z.y * kLog2e));
  const float2 den = fadd2(e, make_float2(1.f, 1.f));
  return fmul2(z, make_float2(rcp_approx(den.x), rcp_approx(den.y)));
}

// Zero-order hold ("Vi du Python" of the first page): Bbar / B = (e^u - 1) / A
// with u = Delta * A, given e = e^u from ex2.approx.  For |u| < 1/4 it is
// Delta * (expm1(u) / u), the Taylor series 1 + u/2 + u^2/6 + ... + u^6/5040
// (the next term is below 2e-9 relative), so a small or zero A needs neither
// a division nor the cancellation of e - 1; elsewhere (e - 1) * (1/A), where
// |e - 1| > 0.22 keeps ex2.approx's 2^-22 relative error below 1.2e-6.
__device__ __forceinline__ float zoh_coef(float u, float e, float dlt, float invA) {
  float p = 1.f / 5040.f;
  p = fmaf(p, u, 1.f / 720.f);
  p = fmaf(p, u, 1.f / 120.f);
  p = fmaf(p, u, 1.f / 24.f);
  p = fmaf(p, u, 1.f / 6.f);
  p = fmaf(p, u, 0.5f);
  p = fmaf(p, u, 1.f);
  return fabsf(u) < 0.25f ? dlt * p : (e - 1.f) * invA;
}
// The same for two states at once (packed polynomial).
__device__ __forceinline__ float2 zoh_coef2(float2 u, float2 e, float2 dlt, float2 invA) {
  float2 p = make_float2(1.f / 5040.f, 1.f / 5040.f);
  p = ffma2(p, u, make_float2(1.f / 720.f, 1.f / 720.f));
  p = ffma2(p, u, make_float2(1.f / 120.f, 1.f / 120.f));
  p = ffma2(p, u, make_float2(1.f / 24.f, 1.f / 24.f));
  p = ffma2(p, u, make_float2(1.f / 6.f, 1.f / 6.f));
  p = ffma2(p, u, make_float2(0.5f, 0.5f));
  p = ffma2(p, u, make_float2(1.f, 1.f));
  const float2 small = fmul2(dlt, p);
  const float2 large = fmul2(fadd2(e, make_float2(-1.f, -1.f)), invA);
  return make_float2(fabsf(u.x) < 0.25f ? small.x : large.x,
                     fabsf(u.y) < 0.25f ? small.y : large.y);
}
// 2^x for a pair on the FMA pipe instead of the special-function unit
// (Cody-Waite range reduction): x = n + f with n the nearest integer (adding
// 1.5 * 2^23 rounds x to an integer in the low mantissa bits) and f in
// [-1/2, 1/2]; 2^f = 1 + f * Q(f), Q of degree 4 fitted to (2^f - 1) / f for
// relative error (csrc/fit_exp2.py derives and checks the coefficients: max
// relative error 1.8e-7 in float32), so f = 0 gives exactly 1; 2^n is added
// to the exponent field.  x is first clamped to [-125, 127] so the exponent
// never wraps (below, the result is a number under 2^-124 where ex2.approx
// flushes to 0; above, it stays finite).
__device__ __forceinline__ float2 exp2_fma2(float2 x) {
  x = make_float2(fminf(fmaxf(x.x, -125.f), 127.f), fminf(fmaxf(x.y, -125.f), 127.f));
  const float2 t = fadd2(x, make_float2(12582912.f, 12582912.f));
  const float2 n = fadd2(t, make_float2(-12582912.f, -12582912.f));
  const float2 f = ffma2(n, make_float2(-1.f, -1.f), x);
  float2 q = ffma2(make_float2(0.00132186722f, 0.00132186722f), f,
                   make_float2(0.00967169832f, 0.00967169832f));
  q = ffma2(q, f, make_float2(0.0555089302f, 0.0555089302f));
  q = ffma2(q, f, make_float2(0.24022238f, 0.24022238f));
  q = ffma2(q, f, make_float2(0.693146884f, 0.693146884f));
  const float2 p = ffma2(q, f, make_float2(1.f, 1.f));
  return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23)),
                     __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23)));
}

constexpr float kLn2 = 0.6931471805599453f;

template <typename T> __device__ __forceinline__ float to_f32(T v);
template <> __device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}
template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// --- lane groups and bf16 tiles ---------------------------------------------

// Butterfly reduce-scatter over the LPC lanes of a channel group: on entry
// lane q holds partial sums v[j] (its NPL states) of the group's LPC tokens;
// on exit it returns the full sum (all N states) of token q.
template <int LPC>
__device__ __forceinline__ float reduce_scatter(float (&v)[LPC], int q) {
#pragma unroll
  for (int m = LPC / 2; m >= 1; m >>= 1) {
    const bool upper = (q & m) != 0;
#pragma unroll
    for (int i = 0; i < m; ++i) {
      const float send = upper ? v[i] : v[i + m];
      const float keep = upper ? v[i + m] : v[i];
      v[i] = keep + __shfl_xor_sync(FULL_MASK, send, m);
    }
  }
  return v[0];
}
// The same for a lane's two channels at once (.x and .y).
template <int LPC>
__device__ __forceinline__ float2 reduce_scatter2(float2 (&v)[LPC], int q) {
#pragma unroll
  for (int m = LPC / 2; m >= 1; m >>= 1) {
    const bool upper = (q & m) != 0;
#pragma unroll
    for (int i = 0; i < m; ++i) {
      const float2 send = upper ? v[i] : v[i + m];
      const float2 keep = upper ? v[i + m] : v[i];
      const float2 got = make_float2(__shfl_xor_sync(FULL_MASK, send.x, m),
                                     __shfl_xor_sync(FULL_MASK, send.y, m));
      v[i] = fadd2(keep, got);
    }
  }
  return v[0];
}

// A bf16 is the upper half of the fp32 of equal value.
__device__ __forceinline__ void widen_bf16x2(uint32_t w, float &lo, float &hi) {
  lo = __uint_as_float(w << 16);
  hi = __uint_as_float(w & 0xffff0000u);
}

// NPL consecutive B or C values of one token as fp32.
template <int NPL>
__device__ __forceinline__ void load_bc(const float *src, float (&dst)[NPL]) {
  if constexpr (NPL % 4 == 0) {
#pragma unroll
    for (int i = 0; i < NPL; i += 4) {
      const float4 v = *reinterpret_cast<const float4 *>(src + i);
      dst[i] = v.x; dst[i + 1] = v.y; dst[i + 2] = v.z; dst[i + 3] = v.w;
    }
  } else if constexpr (NPL == 2) {
    const float2 v = *reinterpret_cast<const float2 *>(src);
    dst[0] = v.x; dst[1] = v.y;
  } else {
#pragma unroll
    for (int i = 0; i < NPL; ++i) dst[i] = src[i];
  }
}
template <int NPL>
__device__ __forceinline__ void load_bc(const __nv_bfloat16 *src, float (&dst)[NPL]) {
  if constexpr (NPL % 8 == 0) {
#pragma unroll
    for (int i = 0; i < NPL; i += 8) {
      const uint4 w = *reinterpret_cast<const uint4 *>(src + i);
      widen_bf16x2(w.x, dst[i], dst[i + 1]);
      widen_bf16x2(w.y, dst[i + 2], dst[i + 3]);
      widen_bf16x2(w.z, dst[i + 4], dst[i + 5]);
      widen_bf16x2(w.w, dst[i + 6], dst[i + 7]);
    }
  } else if constexpr (NPL == 4) {
    const uint2 w = *reinterpret_cast<const uint2 *>(src);
    widen_bf16x2(w.x, dst[0], dst[1]);
    widen_bf16x2(w.y, dst[2], dst[3]);
  } else if constexpr (NPL == 2) {
    widen_bf16x2(*reinterpret_cast<const uint32_t *>(src), dst[0], dst[1]);
  } else {
    dst[0] = __bfloat162float(src[0]);
  }
}

// Widen a tile of `N` bf16 values (N a multiple of 4) to fp32 with the 32
// lanes of a warp: per round lane i turns the 4 values at 8-byte word i into
// one 16-byte store, so both the reads and the writes of a round are
// consecutive in the banks.
template <int N>
__device__ __forceinline__ void widen_tile(const __nv_bfloat16 *src, float *dst, int lane) {
  static_assert(N % 4 == 0, "whole 8-byte words");
  constexpr int WORDS = N / 4;
#pragma unroll
  for (int i = 0; i < (WORDS + 31) / 32; ++i) {
    const int w = i * 32 + lane;
    if (WORDS % 32 == 0 || w < WORDS) {
      const uint2 u = reinterpret_cast<const uint2 *>(src)[w];
      float4 f;
      widen_bf16x2(u.x, f.x, f.y);
      widen_bf16x2(u.y, f.z, f.w);
      reinterpret_cast<float4 *>(dst)[w] = f;
    }
  }
}

// --- time / ordering --------------------------------------------------------

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint64_t ld_acquire_u64(const unsigned long long *p) {
  uint64_t v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_release_u64(unsigned long long *p, uint64_t v) {
  asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// --- mbarrier ---------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(1000000u)
      : "memory");
  return ok != 0;
}

// Wait for the phase with `parity` to complete; gives up after `timeout_ns`.
// Returns false on timeout.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity,
                                                  uint64_t timeout_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer_ns() - t0 > timeout_ns) return false;
  }
}

// --- TMA (cp.async.bulk.tensor) into this CTA's own shared memory ----------

__device__ __forceinline__ void tma_load_3d(void *smem_dst, const void *tmap, uint64_t *bar,
                                            int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tma_store_3d(const void *tmap, const void *smem_src, int c0,
                                             int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%1, %2, %3}], [%4];" ::"l"(
          reinterpret_cast<uint64_t>(tmap)),
      "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(smem_src))
      : "memory");
}

__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

template <int N> __device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

template <int N> __device__ __forceinline__ void bulk_wait() {
  asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

// Make generic-proxy shared-memory writes visible to the async (TMA) proxy.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

}  // namespace ssm
