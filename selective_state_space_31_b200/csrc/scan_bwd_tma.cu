// scan_bwd_tma.cu -- the backward pass of the selective scan on the fused
// forward kernel's layout: the reverse-mode gradient of its arithmetic
// ("Selective Scan trong Mamba ...", sections "Selection pha vo convolution
// kernel co dinh" and "Vi du Python"), with the pages' third pillar,
// recomputation instead of storing the (B, L, D, N) states ("Tai sao chi
// parallel scan van chua du nhanh?").
//
// One CTA owns a row tile: DT channels of one batch element over the whole
// sequence.  A load warp streams stages of kBwdStage tokens with TMA into a
// ring of shared-memory slots (bf16 B and C are widened to fp32 there by the
// same warp); W scan warps hold LPC lanes per channel, four states per lane.
//   phase 1  stages 0 .. S-1: the recurrence, writing the state at the start
//            of every stage (the only state that reaches memory);
//   phase 2  stages S-1 .. 0: from the stage's start state the lane
//            recomputes the stage's states into registers, then walks the
//            tokens backwards carrying lam = dL/dh_t (lam <- lam * Abar_t).
// Per-channel sums over the N states (the readout C.h for dz, sum lam B for
// dx and dDelta, sum lam h Abar A for dDelta) are reduced over the LPC lanes
// by the forward kernel's butterfly reduce-scatter.  dB_t and dC_t sum over
// channels: each warp transposes its lanes' shares through shared memory
// and sums over its channel groups, the W warps' sums are added at the end
// of every stage and written per row tile; a second kernel adds the row
// tiles (fixed order: the result is deterministic).  Three exponentials per
// state update (phase 1, recomputation, reverse).
#include <type_traits>

#include "device_common.cuh"
#include "scan_bwd.h"

namespace ssm {

namespace {

constexpr int rup(int v, int a) { return (v + a - 1) / a * a; }

template <typename InT, typename GT, int NS, int LPC, int W>
struct BwdCfg {
  static constexpr int TT = kBwdStage;
  static constexpr int NPL = NS / LPC;    // states per lane
  static constexpr int GPW = 32 / LPC;    // channels per scan warp
  static constexpr int DT = W * GPW;      // channels per row tile
  static constexpr int TPL = TT / LPC;    // tokens a lane prepares and finishes per stage
  static constexpr int THREADS = (W + 1) * 32;
  static constexpr bool WIDEN = std::is_same<InT, __nv_bfloat16>::value;
  // slot: x, delta, z (TT x DT, InT), dy (TT x DT, GT), B, C (TT x NS, InT)
  // and, for bf16 inputs, B and C widened to fp32
  static constexpr int XTILE = rup(TT * DT * (int)sizeof(InT), 128);
  static constexpr int YTILE = rup(TT * DT * (int)sizeof(GT), 128);
  static constexpr int BCTILE = rup(TT * NS * (int)sizeof(InT), 128);
  static constexpr int BFTILE = WIDEN ? rup(TT * NS * 4, 128) : 0;
  static constexpr int OFF_DT = XTILE, OFF_Z = 2 * XTILE, OFF_DY = 3 * XTILE;
  static constexpr int OFF_B = OFF_DY + YTILE, OFF_C = OFF_B + BCTILE;
  static constexpr int OFF_BF = OFF_C + BCTILE, OFF_CF = OFF_BF + BFTILE;
  static constexpr int SLOT = OFF_CF + BFTILE;
  static constexpr int RAW = 4;
  // per warp: one row of TTP float4 (Delta, Delta*x, ds, x) per channel
  // group (the pad spreads the groups over the banks)
  static constexpr int TTP = TT + 1;
  static constexpr int PLANE = rup(GPW * TTP * 16, 128);
  // per warp: the lanes' dC / dB shares of LPC tokens, (token, block of 4
  // values, group) with a padded block row; a lane stores its group at
  // position (group + block) mod GPW of the row, so that the lanes' stores
  // as well as the per-block sums (which read whole rows) spread over the
  // banks
  static constexpr int VB = 2 * NS / 4;
  static constexpr int BSTR = GPW * 4 + 4;
  static constexpr int XPOSE = rup(LPC * VB * BSTR * 4, 128);
  // per warp and stage parity: the warp's channel sums (TT x 2NS floats)
  static constexpr int SLICE = TT * 2 * NS * 4;
  static constexpr int OFF_PLANE = RAW * SLOT;
  static constexpr int OFF_XP = OFF_PLANE + W * PLANE;
  static constexpr int OFF_SL = OFF_XP + W * XPOSE;
  static constexpr int OFF_BAR = OFF_SL + 2 * W * SLICE;
  static constexpr int OFF_ABORT = OFF_BAR + 3 * RAW * 8;
  static constexpr int SMEM = OFF_ABORT + 16;
  static_assert(NPL == 4, "four states per lane");
  static_assert(TT % LPC == 0, "LPC divides the stage");
  static_assert(LPC * VB <= 32, "one (token, block) per lane in the channel sum");
  static_assert(DT * sizeof(InT) % 16 == 0 && DT * sizeof(GT) % 16 == 0, "TMA rows");
  static_assert(SLOT % 128 == 0, "slot alignment");
};

// Wait for a phase; gives up when another warp has given up (the CTA's abort
// flag) or after `timeout_ns` (then raises the flag itself).
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, volatile int *abort,
                                              uint64_t timeout_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (globaltimer_ns() - t0 > timeout_ns) {
      *abort = 1;
      return false;
    }
  }
}

__device__ __forceinline__ void scan_warps_sync(int threads) {
  asm volatile("bar.sync 1, %0;" ::"r"(threads) : "memory");
}

__device__ __forceinline__ float sigmoid_f(float v) {
  return rcp_approx(1.f + ex2_approx(-v * kLog2e));
}

// Work item i: row tile i / M, segment i % M over stages [st_lo, st_hi);
// n1 forward steps (phase 1), then n2 reverse steps (phase 2).  The map pass
// walks a segment forward only if a later segment needs its forward map and
// backwards only if an earlier one needs its adjoint map.
struct BwdItem {
  int row, seg, st_lo, st_hi, n1, n2;
  __device__ __forceinline__ void set(int i, const BwdTmaParams &p, bool maps) {
    row = i / p.M;
    seg = i - row * p.M;
    st_lo = min(p.S, seg * p.SPS);
    st_hi = min(p.S, st_lo + p.SPS);
    const int n = st_hi - st_lo;
    n1 = maps ? (seg < p.M - 1 ? n : 0) : n;
    n2 = maps ? (seg > 0 ? n : 0) : n;
  }
};

// MAPS = false: the backward pass over each item (phase 1 from the segment's
// start state, phase 2 from the gradient flowing in from the later
// segments).  MAPS = true (segmented plans, launched first): per item the
// forward map (state reached from 0, sum of Delta) and the adjoint map
// (dL/dh carried from 0 backwards across the segment, sum of Delta).
template <typename InT, typename GT, int NS, int LPC, int W, bool MAPS>
__global__ void __launch_bounds__((W + 1) * 32, W == 4 ? 3 : 5)
    bwd_tma_kernel(const __grid_constant__ BwdMaps maps, const BwdTmaParams p) {
  using Cfg = BwdCfg<InT, GT, NS, LPC, W>;
  constexpr int TT = Cfg::TT, NPL = Cfg::NPL, GPW = Cfg::GPW, DT = Cfg::DT, RAW = Cfg::RAW,
                TPL = Cfg::TPL, VB = Cfg::VB, BSTR = Cfg::BSTR, TTP = Cfg::TTP;
  constexpr bool WIDEN = Cfg::WIDEN;
  extern __shared__ __align__(1024) unsigned char smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint64_t *rfull = reinterpret_cast<uint64_t *>(smem + Cfg::OFF_BAR);
  uint64_t *rempty = rfull + RAW;  // every scan warp is done with the slot
  uint64_t *rconv = rempty + RAW;  // B and C of the slot are widened (32 arrivals)
  volatile int *abort = reinterpret_cast<volatile int *>(smem + Cfg::OFF_ABORT);
  if (tid == 0) {
#pragma unroll
    for (int i = 0; i < RAW; ++i) {
      mbar_init(&rfull[i], 1);
      mbar_init(&rempty[i], W);
      mbar_init(&rconv[i], 32);
    }
    *abort = 0;
    fence_mbar_init();
  }
  __syncthreads();

  const int S = p.S;
  const int items = p.rows * p.M;

  if (warp == W) {
    // ===================== load warp =====================
    constexpr uint32_t XB = TT * DT * sizeof(InT), YB = TT * DT * sizeof(GT),
                       BB = TT * NS * sizeof(InT);
    auto widen = [&](int j) -> bool {  // B and C of step j's slot to fp32, then release it
      const int r = j % RAW;
      if (!__all_sync(FULL_MASK, wait_or_abort(&rfull[r], (uint32_t)((j / RAW) & 1), abort,
                                               p.timeout_ns)))
        return false;
      unsigned char *sb = smem + r * Cfg::SLOT;
      widen_tile<TT * NS>(reinterpret_cast<const __nv_bfloat16 *>(sb + Cfg::OFF_B),
                          reinterpret_cast<float *>(sb + Cfg::OFF_BF), lane);
      widen_tile<TT * NS>(reinterpret_cast<const __nv_bfloat16 *>(sb + Cfg::OFF_C),
                          reinterpret_cast<float *>(sb + Cfg::OFF_CF), lane);
      mbar_arrive(&rconv[r]);
      return true;
    };
    int issued = 0, k = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < items && ok; it += gridDim.x) {
      BwdItem I;
      I.set(it, p, MAPS);
      const int b = I.row / p.nDT, d0 = (I.row - b * p.nDT) * DT;
      for (int j = 0; j < I.n1 + I.n2; ++j, ++k) {
        const int r = k % RAW;
        const bool ph2 = j >= I.n1;
        const int st = ph2 ? I.st_hi - 1 - (j - I.n1) : I.st_lo + j;
        if (lane == 0) {
          if (k >= RAW &&
              !wait_or_abort(&rempty[r], (uint32_t)(((k / RAW) - 1) & 1), abort, p.timeout_ns)) {
            ok = false;
          } else {
            const int t0 = st * TT;
            const uint32_t tx = 2u * XB + BB + (ph2 ? (p.has_z ? XB : 0u) + YB + BB : 0u);
            unsigned char *sb = smem + r * Cfg::SLOT;
            mbar_arrive_expect_tx(&rfull[r], tx);
            tma_load_3d(sb, &maps.x, &rfull[r], d0, t0, b);
            tma_load_3d(sb + Cfg::OFF_DT, &maps.dt, &rfull[r], d0, t0, b);
            tma_load_3d(sb + Cfg::OFF_B, &maps.B, &rfull[r], 0, t0, b);
            if (ph2) {
              if (p.has_z) tma_load_3d(sb + Cfg::OFF_Z, &maps.z, &rfull[r], d0, t0, b);
              tma_load_3d(sb + Cfg::OFF_DY, &maps.dy, &rfull[r], d0, t0, b);
              tma_load_3d(sb + Cfg::OFF_C, &maps.C, &rfull[r], 0, t0, b);
            }
            issued = k + 1;
          }
        }
        ok = __shfl_sync(FULL_MASK, ok, 0);
        if (!ok) break;
        if constexpr (WIDEN) {  // the previous step's slot, while this one is in flight
          if (k > 0 && !widen(k - 1)) {
            ok = false;
            break;
          }
        }
      }
    }
    if constexpr (WIDEN) {
      if (ok && k > 0) ok = widen(k - 1);
    }
    if (!ok && lane == 0) {
      *abort = 1;
      atomicCAS(&p.ctl->status, 0, kStatusTimeout);
      // let the loads still in flight land before the CTA exits (bounded)
      for (int kk = (issued > RAW ? issued - RAW : 0); kk < issued; ++kk)
        (void)mbar_wait_bounded(&rfull[kk % RAW], (uint32_t)((kk / RAW) & 1), p.timeout_ns);
    }
    return;
  }

  // ===================== scan warps =====================
  const int g_loc = lane / LPC;  // channel group (channel) within the warp
  const int q = lane % LPC;      // state group: states q*NPL .. q*NPL + 3
  const int grp = warp * GPW + g_loc;
  float4 *plane = reinterpret_cast<float4 *>(smem + Cfg::OFF_PLANE + warp * Cfg::PLANE) +
                  g_loc * TTP;
  float *xp = reinterpret_cast<float *>(smem + Cfg::OFF_XP + warp * Cfg::XPOSE);
  // this lane's dC block q and dB block LPC + q of the first token, at its
  // rotated position (a rotation only permutes the groups within a row, and
  // the per-block sum reads the whole row)
  float *xp_c = xp + q * BSTR + ((g_loc + q) % GPW) * 4;
  float *xp_b = xp + (LPC + q) * BSTR + ((g_loc + LPC + q) % GPW) * 4;
  using BCT = typename std::conditional<WIDEN, float, InT>::type;
  bool ok = true;
  int k = 0;
  auto wait_slot = [&](int kk) -> bool {
    const int r = kk % RAW;
    const uint32_t par = (uint32_t)((kk / RAW) & 1);
    bool got = wait_or_abort(WIDEN ? &rconv[r] : &rfull[r], par, abort, p.timeout_ns);
    // (with widening, waiting on the slot's own barrier too makes the bulk
    // copy's data visible to this warp)
    if (WIDEN && got) got = wait_or_abort(&rfull[r], par, abort, p.timeout_ns);
    return __all_sync(FULL_MASK, got);
  };

  for (int it = blockIdx.x; it < items; it += gridDim.x) {
    BwdItem I;
    I.set(it, p, MAPS);
    const int row = I.row;
    const int b = row / p.nDT, dtile = row - b * p.nDT;
    const int d = dtile * DT + grp;
    const bool valid = d < p.D;
    float A2[NPL], An[NPL], h[NPL];
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
      An[i] = valid ? __ldg(p.A + (size_t)d * NS + q * NPL + i) : 0.f;
      A2[i] = An[i] * kLog2e;
      h[i] = (!MAPS && valid && p.has_h0)
                 ? __ldg(p.h0 + ((size_t)b * p.D + d) * NS + q * NPL + i) : 0.f;
    }
    const float bias = (valid && p.has_bias) ? __ldg(p.bias + d) : 0.f;
    const float Dd = (valid && p.has_D) ? __ldg(p.Dv + d) : 0.f;
    float *ckrow = p.ws_ck + (size_t)row * S * DT * NS + (size_t)grp * NS + q * NPL;
    // this channel's maps of (row, segment j): N states, then the sum of Delta
    // (a stride of N + 4 floats keeps every map 16-byte aligned)
    auto map_at = [&](float *base, int j) {
      return base + ((size_t)(row * p.M + j) * DT + grp) * (NS + 4);
    };
    if constexpr (!MAPS) {
      // the segment's start state: h0 carried through the forward maps of the
      // segments before it, h <- exp(A sum Delta) h + h_from_0
      for (int j = 0; j < I.seg; ++j) {
        const float *m = map_at(p.ws_fmap, j);
        const float sj = __ldcg(m + NS);
#pragma unroll
        for (int i = 0; i < NPL; ++i)
          h[i] = fmaf(ex2_approx(A2[i] * sj), h[i], __ldcg(m + q * NPL + i));
      }
    }
    float hstart[NPL];
#pragma unroll
    for (int i = 0; i < NPL; ++i) hstart[i] = h[i];
    float dsum = 0.f;  // sum of Delta over the segment (map pass)

    // ---------------- phase 1: forward, stage-start states ----------------
    for (int st = I.st_lo; st < I.st_lo + I.n1; ++st, ++k) {
      ok = ok && wait_slot(k);
      if (ok) {
        const unsigned char *sb = smem + (k % RAW) * Cfg::SLOT;
        const InT *xs = reinterpret_cast<const InT *>(sb);
        const InT *ds = reinterpret_cast<const InT *>(sb + Cfg::OFF_DT);
        const BCT *Bs = reinterpret_cast<const BCT *>(sb + (WIDEN ? Cfg::OFF_BF : Cfg::OFF_B));
        const int nvalid = min(TT, p.L - st * TT);
#pragma unroll
        for (int j = 0; j < TPL; ++j) {
          const int ta = j * LPC + q;
          const float v = to_f32(ds[ta * DT + grp]) + bias;
          float dl = p.softplus ? softplus_f(v) : v;
          if (ta >= nvalid) dl = 0.f;  // past the end: identity update
          *reinterpret_cast<float2 *>(plane + ta) = make_float2(dl, dl * to_f32(xs[ta * DT + grp]));
        }
        __syncwarp();
#pragma unroll
        for (int t = 0; t < TT; ++t) {
          const float2 pl = *reinterpret_cast<const float2 *>(plane + t);
          if constexpr (MAPS) dsum += pl.x;
          float bv[NPL];
          load_bc<NPL>(Bs + t * NS + q * NPL, bv);
#pragma unroll
          for (int i = 0; i < NPL; i += 2) {
            const float2 arg = fmul2(make_float2(pl.x, pl.x), make_float2(A2[i], A2[i + 1]));
            const float2 hn = ffma2(make_float2(ex2_approx(arg.x), ex2_approx(arg.y)),
                                    make_float2(h[i], h[i + 1]),
                                    fmul2(make_float2(pl.y, pl.y), make_float2(bv[i], bv[i + 1])));
            h[i] = hn.x;
            h[i + 1] = hn.y;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&rempty[k % RAW]);
        if (!MAPS && st + 1 < I.st_hi)
          *reinterpret_cast<float4 *>(ckrow + (size_t)(st + 1) * DT * NS) =
              make_float4(h[0], h[1], h[2], h[3]);
      }
    }
    if constexpr (MAPS) {
      if (ok && I.n1 > 0) {  // forward map of this segment
        float *m = map_at(p.ws_fmap, I.seg);
        *reinterpret_cast<float4 *>(m + q * NPL) = make_float4(h[0], h[1], h[2], h[3]);
        if (q == 0) m[NS] = dsum;
      }
    }

    // ---------------- phase 2: reverse ----------------
    float lam[NPL], dA[NPL];
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
      lam[i] = (!MAPS && valid && p.dh_last)
                   ? __ldg(p.dh_last + ((size_t)b * p.D + d) * NS + q * NPL + i) : 0.f;
      dA[i] = 0.f;
    }
    if constexpr (MAPS) {
      // adjoint map: dL/dh from 0 at the segment's end, carried back across
      // it (lam += ds C_t; lam <- lam Abar_t), and the sum of Delta
      dsum = 0.f;
      for (int st = I.st_hi - 1; st >= I.st_hi - I.n2; --st, ++k) {
        ok = ok && wait_slot(k);
        if (!ok) continue;
        const unsigned char *sb = smem + (k % RAW) * Cfg::SLOT;
        const InT *ds = reinterpret_cast<const InT *>(sb + Cfg::OFF_DT);
        const InT *zs = reinterpret_cast<const InT *>(sb + Cfg::OFF_Z);
        const GT *dys = reinterpret_cast<const GT *>(sb + Cfg::OFF_DY);
        const BCT *Cs = reinterpret_cast<const BCT *>(sb + (WIDEN ? Cfg::OFF_CF : Cfg::OFF_C));
        const int nvalid = min(TT, p.L - st * TT);
#pragma unroll
        for (int j = 0; j < TPL; ++j) {
          const int ta = j * LPC + q;
          const float v = to_f32(ds[ta * DT + grp]) + bias;
          float dl = p.softplus ? softplus_f(v) : v;
          float dsv = to_f32(dys[ta * DT + grp]);
          if (p.has_z) {
            const float zv = to_f32(zs[ta * DT + grp]);
            dsv *= zv * sigmoid_f(zv);
          }
          if (ta >= nvalid) {
            dl = 0.f;
            dsv = 0.f;
          }
          *reinterpret_cast<float2 *>(plane + ta) = make_float2(dl, dsv);
        }
        __syncwarp();
#pragma unroll
        for (int t = TT - 1; t >= 0; --t) {
          const float2 pl = *reinterpret_cast<const float2 *>(plane + t);  // (Delta, ds)
          dsum += pl.x;
          float cv[NPL];
          load_bc<NPL>(Cs + t * NS + q * NPL, cv);
#pragma unroll
          for (int i = 0; i < NPL; i += 2) {
            const float2 arg = fmul2(make_float2(pl.x, pl.x), make_float2(A2[i], A2[i + 1]));
            float2 lm = ffma2(make_float2(pl.y, pl.y), make_float2(cv[i], cv[i + 1]),
                              make_float2(lam[i], lam[i + 1]));
            lm = fmul2(lm, make_float2(ex2_approx(arg.x), ex2_approx(arg.y)));
            lam[i] = lm.x;
            lam[i + 1] = lm.y;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&rempty[k % RAW]);
      }
      if (ok && I.n2 > 0) {
        float *m = map_at(p.ws_amap, I.seg);
        *reinterpret_cast<float4 *>(m + q * NPL) = make_float4(lam[0], lam[1], lam[2], lam[3]);
        if (q == 0) m[NS] = dsum;
      }
      continue;
    } else {
      // the gradient flowing in from the later segments: dL/dh_last carried
      // back through their adjoint maps, lam <- exp(A sum Delta) lam + e
      for (int j = p.M - 1; j > I.seg; --j) {
        const float *m = map_at(p.ws_amap, j);
        const float sj = __ldcg(m + NS);
#pragma unroll
        for (int i = 0; i < NPL; ++i)
          lam[i] = fmaf(ex2_approx(A2[i] * sj), lam[i], __ldcg(m + q * NPL + i));
      }
    }
    float dD_acc = 0.f, dbias_acc = 0.f;
    for (int st = I.st_hi - 1; st >= I.st_hi - I.n2; --st, ++k) {
      const int par = st & 1;
      float *slice = reinterpret_cast<float *>(smem + Cfg::OFF_SL) + (par * W + warp) * TT * 2 * NS;
      const int t0 = st * TT;
      const int nvalid = min(TT, p.L - t0);
      // the stage's start state (the segment's start, or what this lane wrote
      // in phase 1)
      float hs[TT + 1][NPL];
      if (st == I.st_lo) {
#pragma unroll
        for (int i = 0; i < NPL; ++i) hs[0][i] = hstart[i];
      } else {
        const float4 c = *reinterpret_cast<const float4 *>(ckrow + (size_t)st * DT * NS);
        hs[0][0] = c.x; hs[0][1] = c.y; hs[0][2] = c.z; hs[0][3] = c.w;
      }
      ok = ok && wait_slot(k);
      if (ok) {
        const unsigned char *sb = smem + (k % RAW) * Cfg::SLOT;
        const InT *xs = reinterpret_cast<const InT *>(sb);
        const InT *ds = reinterpret_cast<const InT *>(sb + Cfg::OFF_DT);
        const InT *zs = reinterpret_cast<const InT *>(sb + Cfg::OFF_Z);
        const GT *dys = reinterpret_cast<const GT *>(sb + Cfg::OFF_DY);
        const BCT *Bs = reinterpret_cast<const BCT *>(sb + (WIDEN ? Cfg::OFF_BF : Cfg::OFF_B));
        const BCT *Cs = reinterpret_cast<const BCT *>(sb + (WIDEN ? Cfg::OFF_CF : Cfg::OFF_C));
        // -- per-token prologue of this lane's tokens j * LPC + q --
        float sig[TPL], dzf[TPL];
#pragma unroll
        for (int j = 0; j < TPL; ++j) {
          const int ta = j * LPC + q;
          const float v = to_f32(ds[ta * DT + grp]) + bias;
          float dl = v, sg = 1.f;
          if (p.softplus) {
            dl = softplus_f(v);
            sg = sigmoid_f(v);  // softplus' = sigmoid
          }
          const float xv = to_f32(xs[ta * DT + grp]);
          const float dyv = to_f32(dys[ta * DT + grp]);
          float dsv = dyv, zf = 0.f;
          if (p.has_z) {  // y = ypre * silu(z): ds = dy silu(z), dz = dy ypre silu'(z)
            const float zv = to_f32(zs[ta * DT + grp]);
            const float sz = sigmoid_f(zv);
            dsv = dyv * zv * sz;
            zf = dyv * sz * fmaf(zv, 1.f - sz, 1.f);
          }
          if (ta >= nvalid) {
            dl = 0.f;
            dsv = 0.f;
          }
          plane[ta] = make_float4(dl, dl * xv, dsv, xv);
          sig[j] = sg;
          dzf[j] = zf;
        }
        __syncwarp();
        // -- the stage's states from its start state --
#pragma unroll
        for (int t = 0; t < TT; ++t) {
          const float2 pl = *reinterpret_cast<const float2 *>(plane + t);
          float bv[NPL];
          load_bc<NPL>(Bs + t * NS + q * NPL, bv);
#pragma unroll
          for (int i = 0; i < NPL; i += 2) {
            const float2 arg = fmul2(make_float2(pl.x, pl.x), make_float2(A2[i], A2[i + 1]));
            const float2 hn = ffma2(make_float2(ex2_approx(arg.x), ex2_approx(arg.y)),
                                    make_float2(hs[t][i], hs[t][i + 1]),
                                    fmul2(make_float2(pl.y, pl.y), make_float2(bv[i], bv[i + 1])));
            hs[t + 1][i] = hn.x;
            hs[t + 1][i + 1] = hn.y;
          }
        }
        // -- tokens backwards, LPC at a time --
#pragma unroll
        for (int tt = TT - LPC; tt >= 0; tt -= LPC) {
          float yc[LPC], yg[LPC], yq[LPC];
#pragma unroll
          for (int jj = LPC - 1; jj >= 0; --jj) {
            const int t = tt + jj;
            const float4 pl = plane[t];  // (Delta, Delta*x, ds, x)
            float bv[NPL], cv[NPL];
            load_bc<NPL>(Bs + t * NS + q * NPL, bv);
            load_bc<NPL>(Cs + t * NS + q * NPL, cv);
            const float2 dl2 = make_float2(pl.x, pl.x), dx2 = make_float2(pl.y, pl.y),
                         ds2 = make_float2(pl.z, pl.z);
            float2 sc = make_float2(0.f, 0.f), sg = sc, sq = sc;
            float dCv[NPL], dBv[NPL];
#pragma unroll
            for (int i = 0; i < NPL; i += 2) {
              const float2 arg = fmul2(dl2, make_float2(A2[i], A2[i + 1]));
              const float2 ab = make_float2(ex2_approx(arg.x), ex2_approx(arg.y));
              const float2 hn = make_float2(hs[t + 1][i], hs[t + 1][i + 1]);
              const float2 hp = make_float2(hs[t][i], hs[t][i + 1]);
              const float2 cc = make_float2(cv[i], cv[i + 1]);
              const float2 bb = make_float2(bv[i], bv[i + 1]);
              float2 lm = ffma2(ds2, cc, make_float2(lam[i], lam[i + 1]));  // dL/dh_t
              sc = ffma2(cc, hn, sc);                                        // C . h_t
              const float2 dc = fmul2(ds2, hn);                              // dC share
              const float2 q1 = fmul2(fmul2(lm, hp), ab);  // dL/dAbar * Abar
              sq = ffma2(q1, make_float2(An[i], An[i + 1]), sq);
              float2 da = ffma2(q1, dl2, make_float2(dA[i], dA[i + 1]));
              sg = ffma2(lm, bb, sg);                                        // lam . B
              const float2 db = fmul2(lm, dx2);                              // dB share
              lm = fmul2(lm, ab);                                            // to h_{t-1}
              lam[i] = lm.x; lam[i + 1] = lm.y;
              dA[i] = da.x; dA[i + 1] = da.y;
              dCv[i] = dc.x; dCv[i + 1] = dc.y;
              dBv[i] = db.x; dBv[i + 1] = db.y;
            }
            *reinterpret_cast<float4 *>(xp_c + jj * VB * BSTR) =
                make_float4(dCv[0], dCv[1], dCv[2], dCv[3]);
            *reinterpret_cast<float4 *>(xp_b + jj * VB * BSTR) =
                make_float4(dBv[0], dBv[1], dBv[2], dBv[3]);
            yc[jj] = sc.x + sc.y;
            yg[jj] = sg.x + sg.y;
            yq[jj] = sq.x + sq.y;
          }
          __syncwarp();
          // this lane's token of the group: totals over the N states
          const float sC = reduce_scatter<LPC>(yc, q);
          const float sG = reduce_scatter<LPC>(yg, q);
          const float sQ = reduce_scatter<LPC>(yq, q);
          const int to = tt + q, j = tt / LPC;
          const float4 pl = plane[to];
          if (valid && to < nvalid) {
            const size_t idx = ((size_t)b * p.L + t0 + to) * p.D + d;
            if (p.has_z) p.dz[idx] = dzf[j] * fmaf(Dd, pl.w, sC);
            p.dx[idx] = fmaf(pl.x, sG, Dd * pl.z);
            const float dv = fmaf(pl.w, sG, sQ) * sig[j];
            p.ddelta[idx] = dv;
            dbias_acc += dv;
            dD_acc = fmaf(pl.z, pl.w, dD_acc);
          }
          // this warp's channel sums of dC and dB for the group's tokens
          if (lane < LPC * VB) {
            const int jl = lane / VB, vb = lane - jl * VB;
            const float *src = xp + (jl * VB + vb) * BSTR;
            float4 s = *reinterpret_cast<const float4 *>(src);
            float2 lo = make_float2(s.x, s.y), hi = make_float2(s.z, s.w);
#pragma unroll
            for (int gg = 1; gg < GPW; ++gg) {
              const float4 u = *reinterpret_cast<const float4 *>(src + gg * 4);
              lo = fadd2(lo, make_float2(u.x, u.y));
              hi = fadd2(hi, make_float2(u.z, u.w));
            }
            *reinterpret_cast<float4 *>(slice + (tt + jl) * 2 * NS + vb * 4) =
                make_float4(lo.x, lo.y, hi.x, hi.y);
          }
          __syncwarp();
        }
        if (lane == 0) mbar_arrive(&rempty[k % RAW]);
      }
      // stage end: add the W warps' sums, write them for this row tile
      scan_warps_sync(W * 32);
      if (ok) {
        const float *sl = reinterpret_cast<const float *>(smem + Cfg::OFF_SL) + par * W * TT * 2 * NS;
        float *dst = p.ws_bc + (((size_t)b * p.nDT + dtile) * p.L + t0) * 2 * NS;
        for (int i = warp * 32 + lane; i < TT * VB; i += W * 32) {
          const int t = i / VB;
          if (t >= nvalid) continue;
          const float4 s = *reinterpret_cast<const float4 *>(sl + i * 4);
          float2 lo = make_float2(s.x, s.y), hi = make_float2(s.z, s.w);
#pragma unroll
          for (int w = 1; w < W; ++w) {
            const float4 u = *reinterpret_cast<const float4 *>(sl + w * TT * 2 * NS + i * 4);
            lo = fadd2(lo, make_float2(u.x, u.y));
            hi = fadd2(hi, make_float2(u.z, u.w));
          }
          *reinterpret_cast<float4 *>(dst + (size_t)i * 4) = make_float4(lo.x, lo.y, hi.x, hi.y);
        }
      }
    }
    if (!ok) continue;  // (every remaining step gives up at once: the CTA's abort flag)
    // ---------------- per-row results ----------------
    if (valid) {
      if (p.dh0 && I.seg == 0) {
        *reinterpret_cast<float4 *>(p.dh0 + ((size_t)b * p.D + d) * NS + q * NPL) =
            make_float4(lam[0], lam[1], lam[2], lam[3]);
      }
#pragma unroll
      for (int i = 0; i < NPL; ++i) atomicAdd(p.dA + (size_t)d * NS + q * NPL + i, dA[i]);
    }
#pragma unroll
    for (int m = LPC / 2; m >= 1; m >>= 1) {
      dD_acc += __shfl_xor_sync(FULL_MASK, dD_acc, m);
      dbias_acc += __shfl_xor_sync(FULL_MASK, dbias_acc, m);
    }
    if (valid && q == 0) {
      if (p.has_D) atomicAdd(p.dD + d, dD_acc);
      if (p.has_bias) atomicAdd(p.dbias + d, dbias_acc);
    }
  }
  if (!ok && lane == 0) atomicCAS(&p.ctl->status, 0, kStatusTimeout);
}

// dC[b, t, :] and dB[b, t, :]: the row tiles' sums added in tile order.
template <int NS>
__global__ void __launch_bounds__(256) bwd_bc_sum_kernel(const BwdTmaParams p) {
  constexpr int VB = 2 * NS / 4;
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long total = (long long)p.Bsz * p.L * VB;
  if (i >= total) return;
  const int vb = (int)(i % VB);
  const long long bt = i / VB;
  const int t = (int)(bt % p.L), b = (int)(bt / p.L);
  const size_t tile = (size_t)p.L * 2 * NS;
  const float *src = p.ws_bc + ((size_t)b * p.nDT * p.L + t) * 2 * NS + vb * 4;
  float4 s = __ldcs(reinterpret_cast<const float4 *>(src));
  for (int k = 1; k < p.nDT; ++k) {
    const float4 u = __ldcs(reinterpret_cast<const float4 *>(src + k * tile));
    s.x += u.x; s.y += u.y; s.z += u.z; s.w += u.w;
  }
  float *dst = (vb < VB / 2 ? p.dC : p.dB) + ((size_t)b * p.L + t) * NS + (vb % (VB / 2)) * 4;
  *reinterpret_cast<float4 *>(dst) = s;
}

template <typename InT, typename GT, int NS, int LPC, int W>
cudaError_t run_bwd(const BwdShape &s, const BwdMaps &maps, const BwdTmaParams &p,
                    cudaStream_t stream, BwdShape *query) {
  using Cfg = BwdCfg<InT, GT, NS, LPC, W>;
  auto kern = bwd_tma_kernel<InT, GT, NS, LPC, W, false>;
  auto kmap = bwd_tma_kernel<InT, GT, NS, LPC, W, true>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(kmap, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
  if (e != cudaSuccess) return e;
  if (query) {  // what the variant needs and gets on the device
    query->smem = Cfg::SMEM;
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(&query->occ, kern, Cfg::THREADS,
                                                         Cfg::SMEM);
  }
  const unsigned grid = (unsigned)(s.rows * s.M);  // one CTA per (row tile, segment)
  if (s.M > 1) {  // the segments' maps first
    kmap<<<grid, Cfg::THREADS, Cfg::SMEM, stream>>>(maps, p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  kern<<<grid, Cfg::THREADS, Cfg::SMEM, stream>>>(maps, p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const long long total = (long long)p.Bsz * p.L * (2 * NS / 4);
  if (total > 0)
    bwd_bc_sum_kernel<NS><<<(unsigned)((total + 255) / 256), 256, 0, stream>>>(p);
  return cudaGetLastError();
}

// The compiled variants: N = 16 with 4 lanes per channel, N = 8 with 2 (four
// states per lane either way), 2 or 4 scan warps.
template <typename InT, typename GT>
cudaError_t bwd_by_shape(const BwdShape &s, const BwdMaps *maps, const BwdTmaParams *p,
                         cudaStream_t stream, BwdShape *query) {
  static const BwdMaps kNoMaps{};
  static const BwdTmaParams kNoParams{};
  const BwdMaps &m = maps ? *maps : kNoMaps;
  const BwdTmaParams &pp = p ? *p : kNoParams;
  if (s.lpc == 4 && s.warps == 4) return run_bwd<InT, GT, 16, 4, 4>(s, m, pp, stream, query);
  if (s.lpc == 4 && s.warps == 2) return run_bwd<InT, GT, 16, 4, 2>(s, m, pp, stream, query);
  if (s.lpc == 2 && s.warps == 4) return run_bwd<InT, GT, 8, 2, 4>(s, m, pp, stream, query);
  if (s.lpc == 2 && s.warps == 2) return run_bwd<InT, GT, 8, 2, 2>(s, m, pp, stream, query);
  return cudaErrorInvalidValue;
}

cudaError_t bwd_dispatch(int in_dtype, int out_dtype, const BwdShape &s, const BwdMaps *maps,
                         const BwdTmaParams *p, cudaStream_t stream, BwdShape *query) {
  constexpr int kF32 = 0, kBF16 = 1;  // ssm_dtype values
  if (in_dtype == kBF16 && out_dtype == kBF16)
    return bwd_by_shape<__nv_bfloat16, __nv_bfloat16>(s, maps, p, stream, query);
  if (in_dtype == kBF16 && out_dtype == kF32)
    return bwd_by_shape<__nv_bfloat16, float>(s, maps, p, stream, query);
  if (in_dtype == kF32 && out_dtype == kF32)
    return bwd_by_shape<float, float>(s, maps, p, stream, query);
  return cudaErrorInvalidValue;
}

}  // namespace

// Scan warps (2 or 4) and segments per row tile (1, 2, 4, 8, 16): each
// CTA walks one (row tile, segment) item, so the score is how well the items
// fill whole waves of resident CTAs, divided by the map pass's extra work
// for segments (about two more exponentials per update on (M-1)/M of the
// tokens, against the backward's 3.5: weight kBwdSegCost); ties go to fewer
// segments and then to four warps.
constexpr double kBwdSegCost = 0.8;

bool choose_bwd_shape(int in_dtype, int out_dtype, int64_t batch, int64_t seqlen, int64_t dim,
                      int ns, int warps, int segments, int sms, BwdShape *out) {
  if (ns != 16 && ns != 8) return false;
  if (warps != 0 && warps != 2 && warps != 4) return false;
  if (segments != 0 && segments != 1 && segments != 2 && segments != 4 && segments != 8 &&
      segments != 16)
    return false;
  if (batch <= 0 || seqlen <= 0 || dim <= 0) return false;
  const int es = in_dtype == 1 ? 2 : 4, gs = out_dtype == 1 ? 2 : 4;
  if (in_dtype == 0 && out_dtype == 1) return false;  // no such variant
  if ((dim * es) % 16 != 0 || (dim * gs) % 16 != 0 || (ns * es) % 16 != 0) return false;
  bool found = false;
  double best_score = -1.0;
  BwdShape best;
  for (int w : {4, 2}) {
    if (warps && w != warps) continue;
    BwdShape s;
    s.lpc = ns / 4;
    s.warps = w;
    s.DT = w * (32 / s.lpc);
    s.nDT = (int)((dim + s.DT - 1) / s.DT);
    s.rows = batch * s.nDT;
    s.S = (int)((seqlen + kBwdStage - 1) / kBwdStage);
    if (bwd_dispatch(in_dtype, out_dtype, s, nullptr, nullptr, nullptr, &s) != cudaSuccess ||
        s.occ < 1) {
      cudaGetLastError();
      continue;
    }
    const int64_t slots = (int64_t)s.occ * sms;
    for (int M : {1, 2, 4, 8, 16}) {
      if (segments && M != segments) continue;
      if (M > 1 && s.S < 4 * M) continue;  // each segment keeps a few stages
      BwdShape c = s;
      c.SPS = (s.S + M - 1) / M;
      c.M = (s.S + c.SPS - 1) / c.SPS;
      const int64_t units = c.rows * c.M;
      if (units > INT32_MAX || c.rows * (int64_t)c.S > INT32_MAX / 2) continue;
      const double fill = (double)units / (double)(((units + slots - 1) / slots) * slots);
      const double score = fill / (1.0 + kBwdSegCost * (c.M - 1) / c.M) - 1e-4 * c.M;
      if (!found || score > best_score + 1e-9) {
        found = true;
        best_score = score;
        best = c;
      }
    }
  }
  if (!found) return false;
  best.ws_ck_floats = (size_t)best.rows * best.S * best.DT * ns;
  best.ws_bc_floats = (size_t)best.rows * seqlen * 2 * ns;
  best.ws_map_floats = best.M > 1 ? (size_t)best.rows * best.M * best.DT * (ns + 4) : 0;
  *out = best;
  return true;
}

cudaError_t launch_bwd_tma(int in_dtype, int out_dtype, const BwdShape &s, const BwdMaps &maps,
                           const BwdTmaParams &p, cudaStream_t stream) {
  // dA, dD and dbias are sums over the batch (atomics onto zero)
  cudaError_t e;
  if ((e = cudaMemsetAsync(p.dA, 0, (size_t)p.D * p.N * sizeof(float), stream)) != cudaSuccess)
    return e;
  if (p.has_D && (e = cudaMemsetAsync(p.dD, 0, (size_t)p.D * sizeof(float), stream)) != cudaSuccess)
    return e;
  if (p.has_bias &&
      (e = cudaMemsetAsync(p.dbias, 0, (size_t)p.D * sizeof(float), stream)) != cudaSuccess)
    return e;
  return bwd_dispatch(in_dtype, out_dtype, s, &maps, &p, stream, nullptr);
}

}  // namespace ssm
