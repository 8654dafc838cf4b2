// scan_fwd_kernel.cuh -- fused selective-scan forward kernel for sm_100a.
//
// One kernel does everything the pages' "Kernel fusion" section lists after
// the projections: Delta = softplus(delta + bias), discretisation
// Abar = exp(Delta*A), Bbar*x = (Delta*x)*B_t, the recurrence
// h = Abar*h + Bbar*x, the readout C_t.h, the D skip and the silu(z) gate
// ("Selective Scan trong Mamba ...", sections "Selection pha vo convolution
// kernel co dinh", "Vi du Python", "Kernel fusion").  The (B, L, D, N) state
// lives only in registers ("Tai sao chi parallel scan van chua du nhanh?"):
// HBM sees the (B, L, D) inputs/outputs, the (B, L, N) B/C and the (B, D, N)
// h0/h_last only.
//
// Work decomposition
//   * A "row" is DT consecutive channels of one batch element; its L tokens
//     are cut into stages of TT tokens.  A channel's N states are split over
//     LPC lanes (NPL = N / LPC each); the lanes' partial readouts of a group
//     of LPC tokens are combined by a shuffle butterfly that leaves lane q with
//     token q, and lane q finishes that token.
//   * Strided item schedule.  Each row's S stages are cut into parts of PL
//     stages; item i = part * R + row.  CTA c runs items c, c + P, c + 2P, ...
//     in order (P = gridDim.x <= R).  The predecessor of an item (same row,
//     previous part) has index i - R <= i - P, so it belongs to an earlier
//     slot of some CTA: run in lock-step, no CTA waits, and every CTA gets the
//     same number of items (to within one).  A part hands its final state to
//     the next part through a per-(row, warp) flag carrying the stage index
//     and a launch epoch (release/acquire) -- the pages' associative carry
//     ("Scan bien recurrence ...": (A2,b2) (x) (A1,b1) = (A2A1, A2b1+b2)): the
//     state after one part is the exact starting state of the next.  Every
//     wait is bounded by a timer.
//   * Warp specialisation.  One producer warp per CTA issues the TMA loads
//     (cp.async.bulk.tensor, no multicast) of the [TT, DT] tiles of
//     x / delta / z and the [TT, N] tiles of B / C into a ring of raw slots,
//     turns each stage into fp32 (Delta, Delta, Delta*x, Delta*x) and
//     (g1, g2) per token and channel -- g1 = silu(z), g2 = D*x*g1, so that
//     y = (C.h)*g1 + g2 -- plus fp32 B / C, and writes finished y tiles out
//     with coalesced 16-byte stores.  The consumer warps only scan: they read
//     the fp32 tiles (Delta pairs feed packed fp32x2 instructions, two states
//     per instruction) and write y into the same ring slot.  Producer and
//     consumers meet on mbarriers (slot full / slot empty); no CTA-wide
//     barrier per stage.  Tokens past the end get Delta = 0, an identity
//     update, so carried states are exact for ragged tails.
#pragma once

#include "device_common.cuh"
#include "scan_params.h"

namespace ssm {

constexpr int align_up(int v, int a) { return (v + a - 1) / a * a; }

template <typename InT, typename OutT, int NS, int LPC, int WARPS, int TT>
struct FwdCfg {
  static constexpr int NPL = NS / LPC;    // states per lane
  static constexpr int DTW = 32 / LPC;    // channels per consumer warp
  static constexpr int DT = WARPS * DTW;  // channels per row tile
  static constexpr int PWARPS = WARPS >= 4 ? WARPS / 2 : 1;  // producer warps
  static constexpr int THREADS = (WARPS + PWARPS) * 32;
  // ring depths: ~96 tokens of TMA prefetch and 3 fp32 stage slots, halved
  // for wide tiles (>= 128 channels) so that the CTA still fits one SM
  static constexpr bool WIDE = DT * TT * 16 > 16384;
  static constexpr int RAW = TT >= 48 ? 2 : (WIDE ? 64 : 96) / TT;  // TMA slots
  static constexpr int PSLOTS = WIDE ? 2 : 3;                          // fp32 stage slots
  static constexpr bool BF16_IN = sizeof(InT) == 2;
  static constexpr int XTILE = align_up(TT * DT * (int)sizeof(InT), 128);
  static constexpr int BCTILE = align_up(TT * NS * (int)sizeof(InT), 128);
  static constexpr int SLOT = 3 * XTILE + 2 * BCTILE;
  static constexpr int PLANE_A = TT * DT * 16;  // (Delta, Delta, Delta*x, Delta*x)
  // (g1, g2) rows and y rows are padded so that the epilogue's access to LPC
  // consecutive tokens of 32/LPC channels spreads over the shared-memory banks
  static constexpr int GROW = DT + 8;           // float2 per (g1, g2) row
  static constexpr int PLANE_G = align_up(TT * GROW * 8, 128);
  static constexpr int BCF = align_up(2 * TT * NS * 4, 128);  // fp32 B then C
  static constexpr int YROW = DT * (int)sizeof(OutT) + 16;     // bytes per y row
  static constexpr int YT = align_up(TT * YROW, 128);
  static constexpr int OFF_G = PLANE_A;
  static constexpr int OFF_BC = OFF_G + PLANE_G;
  static constexpr int OFF_Y = OFF_BC + BCF;
  static constexpr int PSLOT = OFF_Y + YT;
  static constexpr int OFF_PREP = RAW * SLOT;
  static constexpr int OFF_BAR = OFF_PREP + PSLOTS * PSLOT;
  static constexpr int OFF_COORD = OFF_BAR + (2 * RAW + 2 * PSLOTS) * 8;
  static constexpr int SMEM = OFF_COORD + PSLOTS * 16;
  static constexpr int PAIRS = DT / 2;                  // channel pairs of the pre-pass
  static constexpr int YCHUNKS = DT * (int)sizeof(OutT) / 16;  // 16-byte chunks per y row
  static_assert(NS % LPC == 0, "LPC must divide N");
  static_assert(TT % LPC == 0, "LPC must divide the stage length");
  static constexpr int PTHREADS = PWARPS * 32;
  static_assert(PTHREADS % PAIRS == 0 && TT % (PTHREADS / PAIRS) == 0, "pre-pass mapping");
  static_assert(DT * (int)sizeof(InT) % 16 == 0, "TMA rows need 16-byte multiples");
  static_assert(DT * (int)sizeof(OutT) % 16 == 0, "y rows need 16-byte multiples");
  static_assert(PLANE_A % 128 == 0, "slot alignment");
};

// Butterfly reduce-scatter over the LPC lanes of a channel: on entry lane q
// holds partial sums v[j] (its NPL states) of the group's LPC tokens; on exit
// it returns the full sum (all N states) of token q.
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

template <int NPL>
__device__ __forceinline__ void load_vec(const float *src, float (&dst)[NPL]) {
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

template <typename InT>
__device__ __forceinline__ float2 load_pair(const InT *p);
template <>
__device__ __forceinline__ float2 load_pair<float>(const float *p) {
  return *reinterpret_cast<const float2 *>(p);
}
template <>
__device__ __forceinline__ float2 load_pair<__nv_bfloat16>(const __nv_bfloat16 *p) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(p));
}

// Walks one CTA's items (c, c + P, c + 2P, ...) stage by stage; a division
// happens only when a new item starts.
struct ItemCursor {
  int item, items, P, R, PL, S, nDT;
  int row, part, st, st_end, b, dtile;
  __device__ __forceinline__ void load() {
    if (item >= items) return;
    part = item / R;
    row = item - part * R;
    st = part * PL;
    st_end = min(S, st + PL);
    b = row / nDT;
    dtile = row - b * nDT;
  }
  __device__ __forceinline__ void init(int c, const FwdParams &p) {
    item = c; items = p.items; P = gridDim.x; R = p.rows; PL = p.PL; S = p.S; nDT = p.nDT;
    row = part = st = st_end = b = dtile = 0;
    load();
  }
  __device__ __forceinline__ void advance() {
    if (++st == st_end) { item += P; load(); }
  }
};

template <typename InT, typename OutT, int NS, int LPC, int WARPS, int TT>
__global__ void __launch_bounds__((WARPS + (WARPS >= 4 ? WARPS / 2 : 1)) * 32)
    fwd_kernel(const __grid_constant__ TmaMaps maps, const FwdParams p) {
  using Cfg = FwdCfg<InT, OutT, NS, LPC, WARPS, TT>;
  constexpr int NPL = Cfg::NPL, DTW = Cfg::DTW, DT = Cfg::DT, RAW = Cfg::RAW,
                PS = Cfg::PSLOTS;
  extern __shared__ __align__(1024) unsigned char smem[];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint64_t *rfull = reinterpret_cast<uint64_t *>(smem + Cfg::OFF_BAR);
  uint64_t *rdone = rfull + RAW;  // producers finished reading a raw slot
  uint64_t *pfull = rdone + RAW;
  uint64_t *pempty = pfull + PS;

  const unsigned int epoch = *reinterpret_cast<volatile unsigned int *>(&p.ctl->epoch);

  // ---- strided item schedule: stages this CTA runs ----
  const int S = p.S;
  int n = 0;
  for (int it = blockIdx.x; it < p.items; it += gridDim.x) {
    const int part = it / p.rows;
    n += min(S, (part + 1) * p.PL) - part * p.PL;
  }

  if (tid == 0) {
#pragma unroll
    for (int i = 0; i < RAW; ++i) {
      mbar_init(&rfull[i], 1);
      mbar_init(&rdone[i], Cfg::PWARPS);
    }
#pragma unroll
    for (int i = 0; i < PS; ++i) {
      mbar_init(&pfull[i], Cfg::PWARPS);
      mbar_init(&pempty[i], WARPS);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp >= WARPS) {
    // =================== producer warps ===================
    const int ptid = tid - WARPS * 32;
    const bool issuer = ptid == 0;
    const uint32_t tx_bytes =
        (p.has_z ? 3u : 2u) * TT * DT * sizeof(InT) + 2u * TT * NS * sizeof(InT);
    ItemCursor iss;  // next stage to load (issuer thread)
    iss.init(blockIdx.x, p);
    int iss_k = 0;
    auto issue = [&]() {
      const int r = iss_k % RAW;
      const int d0 = iss.dtile * DT, t0 = iss.st * TT, b = iss.b;
      unsigned char *sb = smem + r * Cfg::SLOT;
      mbar_arrive_expect_tx(&rfull[r], tx_bytes);
      tma_load_3d(sb, &maps.x, &rfull[r], d0, t0, b);
      tma_load_3d(sb + Cfg::XTILE, &maps.dt, &rfull[r], d0, t0, b);
      if (p.has_z) tma_load_3d(sb + 2 * Cfg::XTILE, &maps.z, &rfull[r], d0, t0, b);
      tma_load_3d(sb + 3 * Cfg::XTILE, &maps.B, &rfull[r], 0, t0, b);
      tma_load_3d(sb + 3 * Cfg::XTILE + Cfg::BCTILE, &maps.C, &rfull[r], 0, t0, b);
      iss.advance();
      ++iss_k;
    };
    if (issuer)
      for (int k = 0; k < n && k < RAW; ++k) issue();

    // y tile of slot s -> global, 16 bytes a thread; (b, d0, t0) of the stage
    // that last used each slot are kept in shared memory
    int4 *coord = reinterpret_cast<int4 *>(smem + Cfg::OFF_COORD);
    auto flush_y = [&](int s) {
      const int4 cs = coord[s];
      const int fbs = cs.x, fd0s = cs.y, ft0s = cs.z;
      const int nval = min(TT, p.L - ft0s);
      constexpr int EPC = 16 / sizeof(OutT);
      const unsigned char *src = smem + Cfg::OFF_PREP + s * Cfg::PSLOT + Cfg::OFF_Y;
      OutT *ybase = reinterpret_cast<OutT *>(p.y);
      for (int i = ptid; i < TT * Cfg::YCHUNKS; i += Cfg::PTHREADS) {
        const int t = i / Cfg::YCHUNKS, c = (i % Cfg::YCHUNKS) * EPC;
        if (t < nval && fd0s + c < p.D)
          *reinterpret_cast<uint4 *>(ybase + ((size_t)fbs * p.L + ft0s + t) * p.D + fd0s + c) =
              *reinterpret_cast<const uint4 *>(src + t * Cfg::YROW + c * sizeof(OutT));
      }
    };

    // pre-pass mapping: a fixed channel pair, tokens pt0, pt0 + PSTEP, ...
    constexpr int PSTEP = Cfg::PTHREADS / Cfg::PAIRS;
    const int pc = (ptid % Cfg::PAIRS) * 2;
    const int pt0 = ptid / Cfg::PAIRS;
    int pre_row = -1;
    float2 bias2 = make_float2(0.f, 0.f), dsk2 = make_float2(0.f, 0.f);

    ItemCursor cur;
    cur.init(blockIdx.x, p);
    bool ok = true;
    int k = 0;
    for (; k < n; ++k, cur.advance()) {
      const int r = k % RAW, s = k % PS;
      ok = mbar_wait_bounded(&rfull[r], (uint32_t)((k / RAW) & 1), p.timeout_ns);
      if (ok && k >= PS)  // consumers done with stage k - PS (its y tile is complete)
        ok = mbar_wait_bounded(&pempty[s], (uint32_t)(((k / PS) - 1) & 1), p.timeout_ns);
      if (!__all_sync(FULL_MASK, ok)) { ok = false; break; }
      if (k >= PS) flush_y(s);

      const int b = cur.b, d0 = cur.dtile * DT, t0 = cur.st * TT;
      const int nvalid = min(TT, p.L - t0);
      if (cur.row != pre_row) {  // per-row parameters of this thread's channel pair
        pre_row = cur.row;
        const int d = d0 + pc;  // D is even on this path, so d + 1 < D whenever d < D
        bias2 = (p.has_bias && d < p.D) ? make_float2(__ldg(p.bias + d), __ldg(p.bias + d + 1))
                                        : make_float2(0.f, 0.f);
        dsk2 = (p.has_D && d < p.D) ? make_float2(__ldg(p.Dv + d), __ldg(p.Dv + d + 1))
                                    : make_float2(0.f, 0.f);
      }
      const unsigned char *sb = smem + r * Cfg::SLOT;
      const InT *xs = reinterpret_cast<const InT *>(sb);
      const InT *ds = reinterpret_cast<const InT *>(sb + Cfg::XTILE);
      const InT *zs = reinterpret_cast<const InT *>(sb + 2 * Cfg::XTILE);
      unsigned char *ps = smem + Cfg::OFF_PREP + s * Cfg::PSLOT;
      float4 *planeA = reinterpret_cast<float4 *>(ps);
      float4 *planeG = reinterpret_cast<float4 *>(ps + Cfg::OFF_G);  // 2 channels a float4
      float *bcf = reinterpret_cast<float *>(ps + Cfg::OFF_BC);
#pragma unroll
      for (int t = pt0; t < TT; t += PSTEP) {
        const float2 xv = load_pair<InT>(xs + t * DT + pc);
        float2 v = fadd2(load_pair<InT>(ds + t * DT + pc), bias2);
        if (p.softplus) v = softplus_f2(v);
        if (t >= nvalid) v = make_float2(0.f, 0.f);  // past the end: identity update
        const float2 dx = fmul2(v, xv);
        float2 g = make_float2(1.f, 1.f);
        if (p.has_z) g = silu_f2(load_pair<InT>(zs + t * DT + pc));
        const float2 g2 = fmul2(fmul2(dsk2, xv), g);
        planeA[t * DT + pc] = make_float4(v.x, v.x, dx.x, dx.x);
        planeA[t * DT + pc + 1] = make_float4(v.y, v.y, dx.y, dx.y);
        planeG[(t * Cfg::GROW + pc) / 2] = make_float4(g.x, g2.x, g.y, g2.y);
      }
      if constexpr (Cfg::BF16_IN) {
        const __nv_bfloat162 *src = reinterpret_cast<const __nv_bfloat162 *>(sb + 3 * Cfg::XTILE);
        float2 *dst = reinterpret_cast<float2 *>(bcf);
        static_assert(!Cfg::BF16_IN || Cfg::BCTILE == TT * NS * 2, "B, C tiles contiguous");
        for (int i = ptid; i < TT * NS; i += Cfg::PTHREADS) dst[i] = __bfloat1622float2(src[i]);
      } else {
        const float4 *src = reinterpret_cast<const float4 *>(sb + 3 * Cfg::XTILE);
        float4 *dst = reinterpret_cast<float4 *>(bcf);
        static_assert(Cfg::BF16_IN || Cfg::BCTILE == TT * NS * 4, "B, C tiles contiguous");
        for (int i = ptid; i < TT * NS / 2; i += Cfg::PTHREADS) dst[i] = src[i];
      }
      if (ptid == 0) coord[s] = make_int4(b, d0, t0, 0);
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&pfull[s]);  // this warp's half of stage k is ready
        mbar_arrive(&rdone[r]);  // and it no longer reads raw slot r
      }
      if (issuer && iss_k < n) {  // refill raw slot r with stage k + RAW
        if (mbar_wait_bounded(&rdone[r], (uint32_t)((k / RAW) & 1), p.timeout_ns)) issue();
        else ok = false;
      }
    }
    if (ok) {  // write out the last tiles once the consumers are done with them
      for (int kk = (n > PS ? n - PS : 0); kk < n; ++kk) {
        const int s = kk % PS;
        if (!mbar_wait_bounded(&pempty[s], (uint32_t)((kk / PS) & 1), p.timeout_ns)) {
          ok = false;
          break;
        }
        flush_y(s);
      }
    }
    if (!__all_sync(FULL_MASK, ok) && lane == 0) {
      atomicCAS(&p.ctl->status, 0, kStatusTimeout);
      if (issuer)
        for (int kk = k; kk < iss_k; ++kk)  // let loads in flight land (bounded)
          (void)mbar_wait_bounded(&rfull[kk % RAW], (uint32_t)((kk / RAW) & 1), p.timeout_ns);
    }
  } else {
    // =================== consumer warps ===================
    const int c_loc = lane / LPC;       // channel within the warp
    const int q = lane % LPC;           // state group of this lane
    const int ch = warp * DTW + c_loc;  // channel within the row tile
    float h[NPL], A2[NPL];
#pragma unroll
    for (int i = 0; i < NPL; ++i) { h[i] = 0.f; A2[i] = 0.f; }
    ItemCursor cur;
    cur.init(blockIdx.x, p);
    for (int k = 0; k < n; ++k, cur.advance()) {
      const int s = k % PS;
      if (!__all_sync(FULL_MASK, mbar_wait_bounded(&pfull[s], (uint32_t)((k / PS) & 1),
                                                   p.timeout_ns))) {
        if (lane == 0) atomicCAS(&p.ctl->status, 0, kStatusTimeout);
        break;
      }
      const int row = cur.row, st = cur.st, b = cur.b;
      const int d = cur.dtile * DT + ch;
      const bool valid_ch = d < p.D;
      const bool run_start = st == cur.part * cur.PL;
      if (run_start) {
#pragma unroll
        for (int i = 0; i < NPL; ++i)
          A2[i] = valid_ch ? __ldg(p.A + (size_t)d * NS + q * NPL + i) * kLog2e : 0.f;
        if (st == 0) {
#pragma unroll
          for (int i = 0; i < NPL; ++i)
            h[i] = (p.has_h0 && valid_ch)
                       ? __ldg(p.h0 + ((size_t)b * p.D + d) * NS + q * NPL + i) : 0.f;
        } else {  // carried state of this row from the CTA that ran its head
          const unsigned long long want = ((unsigned long long)epoch << 32) | (unsigned)st;
          unsigned long long *flag = p.ws_flags + (size_t)row * WARPS + warp;
          bool got = ld_acquire_u64(flag) == want;
          if (!got) {
            const uint64_t tstart = globaltimer_ns();
            while (true) {
              __nanosleep(64);
              if (ld_acquire_u64(flag) == want) { got = true; break; }
              if (globaltimer_ns() - tstart > p.timeout_ns) break;
            }
          }
          if (!__all_sync(FULL_MASK, got) && lane == 0)
            atomicCAS(&p.ctl->status, 0, kStatusTimeout);
          const float *src = p.ws_state + ((size_t)row * DT + ch) * NS + q * NPL;
#pragma unroll
          for (int i = 0; i < NPL; ++i) h[i] = __ldcg(src + i);
        }
      }

      // -- the scan over TT tokens of this lane's channel --
      const unsigned char *ps = smem + Cfg::OFF_PREP + s * Cfg::PSLOT;
      const float4 *planeA = reinterpret_cast<const float4 *>(ps);
      const float2 *planeG = reinterpret_cast<const float2 *>(ps + Cfg::OFF_G);
      const float *Bf = reinterpret_cast<const float *>(ps + Cfg::OFF_BC);
      const float *Cf = Bf + TT * NS;
      unsigned char *yt = smem + Cfg::OFF_PREP + s * Cfg::PSLOT + Cfg::OFF_Y;
#pragma unroll
      for (int tt = 0; tt < TT; tt += LPC) {
        float yp[LPC];
#pragma unroll
        for (int j = 0; j < LPC; ++j) {
          const float4 dd = planeA[(tt + j) * DT + ch];
          float bv[NPL], cv[NPL];
          load_vec<NPL>(Bf + (tt + j) * NS + q * NPL, bv);
          load_vec<NPL>(Cf + (tt + j) * NS + q * NPL, cv);
          if constexpr (NPL % 2 == 0) {
            const float2 dA = make_float2(dd.x, dd.y), dX = make_float2(dd.z, dd.w);
            float2 acc = make_float2(0.f, 0.f);
#pragma unroll
            for (int i = 0; i < NPL; i += 2) {
              const float2 arg = fmul2(dA, make_float2(A2[i], A2[i + 1]));
              const float2 a = make_float2(ex2_approx(arg.x), ex2_approx(arg.y));
              const float2 bx = fmul2(dX, make_float2(bv[i], bv[i + 1]));
              const float2 hn = ffma2(a, make_float2(h[i], h[i + 1]), bx);
              h[i] = hn.x;
              h[i + 1] = hn.y;
              acc = ffma2(make_float2(cv[i], cv[i + 1]), hn, acc);
            }
            yp[j] = acc.x + acc.y;
          } else {
            const float a = ex2_approx(dd.x * A2[0]);
            h[0] = fmaf(a, h[0], dd.z * bv[0]);
            yp[j] = cv[0] * h[0];
          }
        }
        const float ys = reduce_scatter<LPC>(yp, q);
        const int to = tt + q;  // this lane's own token of the group
        const float2 gg = planeG[to * Cfg::GROW + ch];
        reinterpret_cast<OutT *>(yt + to * Cfg::YROW)[ch] = from_f32<OutT>(fmaf(ys, gg.x, gg.y));
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&pempty[s]);  // slot s consumed, y tile written

      const bool run_end = st + 1 == cur.st_end;
      if (run_end) {
        if (st == S - 1) {
          if (p.want_hlast && valid_ch) {
            float *dst = p.h_last + ((size_t)b * p.D + d) * NS + q * NPL;
#pragma unroll
            for (int i = 0; i < NPL; ++i) dst[i] = h[i];
          }
        } else if ((long long)row * S + st != p.drop_unit) {  // hand the state on
          float *dst = p.ws_state + ((size_t)row * DT + ch) * NS + q * NPL;
#pragma unroll
          for (int i = 0; i < NPL; ++i) __stcg(dst + i, h[i]);
          __threadfence();
          __syncwarp();
          if (lane == 0)
            st_release_u64(p.ws_flags + (size_t)row * WARPS + warp,
                           ((unsigned long long)epoch << 32) | (unsigned)(st + 1));
        }
      }
    }
  }

  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const unsigned int prev = atomicAdd(&p.ctl->done, 1u);
    if (prev == gridDim.x - 1) {  // last CTA of this launch: ready the next call
      p.ctl->done = 0u;
      p.ctl->epoch = epoch + 1u;
      __threadfence();
    }
  }
}

// ---------------------------------------------------------------------------
// host-side variant table (one translation unit per dtype pair)
// ---------------------------------------------------------------------------

constexpr int kStages = 2;

template <typename InT, typename OutT, int NS, int LPC, int WARPS, int TT>
static cudaError_t run_variant(const LaunchShape *ls, const TmaMaps *maps, const FwdParams *p,
                               cudaStream_t stream, size_t *smem_out, int *occ_out) {
  using Cfg = FwdCfg<InT, OutT, NS, LPC, WARPS, TT>;
  auto kern = fwd_kernel<InT, OutT, NS, LPC, WARPS, TT>;
  if (Cfg::SMEM > 227 * 1024) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return e;
  }
  if (smem_out) *smem_out = Cfg::SMEM;
  if (occ_out) {
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(occ_out, kern, Cfg::THREADS, Cfg::SMEM);
    if (e != cudaSuccess) return e;
  }
  if (!maps) return cudaSuccess;
  kern<<<ls->grid, Cfg::THREADS, Cfg::SMEM, stream>>>(*maps, *p);
  return cudaGetLastError();
}

template <typename InT, typename OutT, int NS, int LPC, int WARPS>
static cudaError_t by_tt(const LaunchShape *ls, const TmaMaps *maps, const FwdParams *p,
                         cudaStream_t st, size_t *sm, int *oc) {
  switch (ls->tt) {
    case 16:
      if constexpr (LPC <= 16) return run_variant<InT, OutT, NS, LPC, WARPS, 16>(ls, maps, p, st, sm, oc);
      return cudaErrorInvalidValue;
    case 32: return run_variant<InT, OutT, NS, LPC, WARPS, 32>(ls, maps, p, st, sm, oc);
    case 64: return run_variant<InT, OutT, NS, LPC, WARPS, 64>(ls, maps, p, st, sm, oc);
    default: return cudaErrorInvalidValue;
  }
}

template <typename InT, typename OutT, int NS, int LPC>
static cudaError_t by_warps(const LaunchShape *ls, const TmaMaps *maps, const FwdParams *p,
                            cudaStream_t st, size_t *sm, int *oc) {
  switch (ls->warps) {
    case 2: return by_tt<InT, OutT, NS, LPC, 2>(ls, maps, p, st, sm, oc);
    case 4: return by_tt<InT, OutT, NS, LPC, 4>(ls, maps, p, st, sm, oc);
    default: return cudaErrorInvalidValue;
  }
}

template <typename InT, typename OutT, int NS>
static cudaError_t by_lpc(const LaunchShape *ls, const TmaMaps *maps, const FwdParams *p,
                          cudaStream_t st, size_t *sm, int *oc) {
  switch (ls->lpc) {
    case 1: return by_warps<InT, OutT, NS, 1>(ls, maps, p, st, sm, oc);
    case 2: return by_warps<InT, OutT, NS, 2>(ls, maps, p, st, sm, oc);
    case 4: return by_warps<InT, OutT, NS, 4>(ls, maps, p, st, sm, oc);
    case 8:
      if constexpr (NS >= 8) return by_warps<InT, OutT, NS, 8>(ls, maps, p, st, sm, oc);
      return cudaErrorInvalidValue;
    default: return cudaErrorInvalidValue;
  }
}

template <typename InT, typename OutT>
static cudaError_t by_ns(const LaunchShape *ls, const TmaMaps *maps, const FwdParams *p,
                         cudaStream_t st, size_t *sm, int *oc) {
  if (ls->stages != kStages) return cudaErrorInvalidValue;
  switch (ls->ns) {
    case 4:
      if constexpr (sizeof(InT) == 4) return by_lpc<InT, OutT, 4>(ls, maps, p, st, sm, oc);
      return cudaErrorInvalidValue;
    case 8: return by_lpc<InT, OutT, 8>(ls, maps, p, st, sm, oc);
    case 16: return by_lpc<InT, OutT, 16>(ls, maps, p, st, sm, oc);
    default: return cudaErrorInvalidValue;
  }
}

// per-dtype entry points (defined in scan_fwd_<dtypes>.cu)
cudaError_t fwd_dispatch_f32(const LaunchShape *, const TmaMaps *, const FwdParams *, cudaStream_t,
                             size_t *, int *);
cudaError_t fwd_dispatch_bf16(const LaunchShape *, const TmaMaps *, const FwdParams *,
                              cudaStream_t, size_t *, int *);
cudaError_t fwd_dispatch_bf16_f32(const LaunchShape *, const TmaMaps *, const FwdParams *,
                                  cudaStream_t, size_t *, int *);

}  // namespace ssm
