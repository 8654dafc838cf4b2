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
//     are cut into stages of TT tokens.  A lane owns KC adjacent channels
//     (1 or 2) and NPL = N / LPC of their states, so LPC lanes share a
//     channel group; with two channels a lane loads and widens each B_t / C_t
//     value once for both.  The lanes' partial readouts of a group of LPC
//     tokens are combined by a shuffle butterfly that leaves lane q with
//     token q, and lane q finishes that token.
//   * Segments.  A row's stages may be cut into M segments that run at the
//     same time.  Segment k > 0 starts from the exact state at its first
//     token, obtained with the pages' associative composition ("Scan bien
//     recurrence ...": (A2,b2) (x) (A1,b1) = (A2A1, A2b1+b2)): a carry pass
//     (this kernel with CARRY set) scans every sub-chunk of the earlier
//     segments from h = 0 and records its map (prod Abar, h_end), where
//     prod_t exp(Delta_t A) = exp(A sum_t Delta_t) needs only the sum of
//     Delta; the segment's first part folds those maps onto h0.  Long
//     sequences gain parallelism this way at the cost of a second exponential
//     for the tokens of the earlier segments.
//   * Ticket schedule.  Each segment's stages are cut into parts of PL
//     stages; item i = part * VR + (row, segment) with VR = rows * M.  A
//     CTA's load warp takes item numbers in increasing order from a device
//     counter (one atomic per item), so the predecessor of an item (same row
//     and segment, previous part, number i - VR) always went to a CTA that
//     was already running: every wait for a carried state ends, however few
//     CTAs the device runs at once, and CTAs that finish early simply take
//     more items.  A part hands its final state to the next part through a
//     per-(row, segment, warp) flag carrying the stage index and a launch
//     epoch (release/acquire): the state after one part is the exact starting
//     state of the next.  Every wait is bounded by a timer.
//   * One load warp streams the stages' [TT, DT] tiles of x / delta / z and
//     [TT, N] tiles of B / C into a ring of RAW shared-memory slots with TMA
//     (cp.async.bulk.tensor, every CTA loads its own tiles); slot full / slot
//     empty mbarriers are the only coupling between warps.  Each scan warp
//     does all the per-token work of its own channels: lane q of a channel
//     group prepares tokens q, q + LPC, ... (Delta, Delta*x into a
//     warp-private plane that the group's LPC lanes read back; silu(z) and
//     D*x*silu(z) stay in the registers of the lane that finishes those very
//     tokens), scans, and stores y straight from registers.  B / C are read
//     as stored (bf16 words are widened with integer ops).  Tokens past the
//     end get Delta = 0, an identity update, so carried states are exact for
//     ragged tails.
#pragma once

#include <type_traits>

#include "device_common.cuh"
#include "scan_params.h"

namespace ssm {

constexpr int align_up(int v, int a) { return (v + a - 1) / a * a; }
constexpr int clamp_int(int v, int lo, int hi) { return v < lo ? lo : (v > hi ? hi : v); }

template <typename InT, typename OutT, int NS, int LPC, int KC, int WARPS, int TT,
          bool CONV = false, bool CARRY = false, bool BCF = false>
struct FwdCfg {
  static constexpr int NPL = NS / LPC;    // states per lane and channel
  static constexpr int GPW = 32 / LPC;    // channel groups per scan warp
  static constexpr int DTW = GPW * KC;    // channels per scan warp
  static constexpr int DT = WARPS * DTW;  // channels per row tile
  static constexpr int TPL = TT / LPC;    // tokens a lane prepares and finishes per stage
  static constexpr int THREADS = (WARPS + 1) * 32;  // scan warps + the load warp
  // the conv front-end reads the x branch from kConvWidth tokens before the
  // stage on (zero-filled by TMA before the sequence)
  static constexpr int XHALO = CONV ? kConvWidth : 0;
  static constexpr int XTILE = align_up(TT * DT * (int)sizeof(InT), 128);
  static constexpr int XTILE_X = align_up((TT + XHALO) * DT * (int)sizeof(InT), 128);
  static constexpr int BCTILE = align_up(TT * NS * (int)sizeof(InT), 128);
  // (the carry pass reads neither z nor C: its slots hold x, delta and B only)
  static constexpr int OFF_DT = XTILE_X, OFF_Z = XTILE_X + XTILE,
                       OFF_B = XTILE_X + (CARRY ? 1 : 2) * XTILE, OFF_C = OFF_B + BCTILE;
  // BCF: the load warp widens the stage's B (and C) to fp32 beside the bf16
  // tiles, once per CTA, so the scan warps read fp32 values
  static constexpr int OFF_BF = OFF_C + (CARRY ? 0 : BCTILE);
  static constexpr int BFTILE = BCF ? align_up(TT * NS * 4, 128) : 0;
  static constexpr int OFF_CF = OFF_BF + BFTILE;
  static constexpr int SLOT = OFF_BF + (CARRY ? 1 : 2) * BFTILE;
  // ring depth: ~128 tokens of prefetch, within ~64 KB (~40 KB with the
  // wider BCF slots, so that four CTAs still fit), at least 3 slots
  static constexpr int RAW =
      clamp_int((BCF ? 40960 : 65536) / SLOT, 3, 128 / TT > 3 ? 128 / TT : 3);
  // Per warp, channel-group-major plane of per-token values: KC = 1 keeps
  // (Delta, Delta*x) as a float2, KC = 2 (Delta0, Delta1, Delta*x0, Delta*x1)
  // as a float4.  Row g holds tokens 0..TT-1 of group g; the TTP - TT pad
  // spreads the rows and the prologue's writes over the shared-memory banks.
  static constexpr int ESZ = 8 * KC;  // bytes per token and group
  static constexpr int TTP = KC == 1 ? TT + (LPC > 2 ? LPC : 2) : TT + (LPC > 1 ? LPC : 2);
  static constexpr int PLANE = align_up(TTP * GPW * ESZ, 128);
  static constexpr int OFF_PLANE = RAW * SLOT;
  static constexpr int OFF_BAR = OFF_PLANE + WARPS * PLANE;
  static constexpr int SMEM = OFF_BAR + (BCF ? 3 : 2) * RAW * 8;
  static_assert(NS % LPC == 0, "LPC must divide N");
  static_assert(TT % LPC == 0, "LPC must divide the stage length");
  static_assert(KC == 1 || KC == 2, "one or two channels per lane");
  static_assert(KC == 1 || NPL % 2 == 0, "two channels per lane pair up their states");
  static_assert(DT * (int)sizeof(InT) % 16 == 0, "TMA rows need 16-byte multiples");
  static_assert(SLOT % 128 == 0 && OFF_PLANE % 128 == 0, "slot alignment");
};

// Two adjacent channels' values of one token (x, delta or z) as fp32.
__device__ __forceinline__ float2 load_pair(const float *src) {
  return *reinterpret_cast<const float2 *>(src);
}
__device__ __forceinline__ float2 load_pair(const __nv_bfloat16 *src) {
  float2 v;
  widen_bf16x2(*reinterpret_cast<const uint32_t *>(src), v.x, v.y);
  return v;
}
// Store two adjacent channels' outputs.
__device__ __forceinline__ void store_pair(float *dst, float2 v) {
  *reinterpret_cast<float2 *>(dst) = v;
}
__device__ __forceinline__ void store_pair(__nv_bfloat16 *dst, float2 v) {
  *reinterpret_cast<__nv_bfloat162 *>(dst) = __floats2bfloat162_rn(v.x, v.y);
}

// Position of one stage of work: item (row, segment, part) and its stages,
// derived from an item number once per item (divisions happen only there).
struct ItemPos {
  int item = -1, row = 0, seg = 0, vrow = 0, part = 0, b = 0, dtile = 0;
  int seg_begin = 0, seg_end = 0, st_begin = 0, st_end = 0;
  __device__ __forceinline__ void set(int it, const FwdParams &p) {
    const int VR = p.rows * p.M;
    item = it;
    part = it / VR;
    vrow = it - part * VR;
    row = vrow / p.M;
    seg = vrow - row * p.M;
    seg_begin = seg * p.SPS;
    seg_end = min(p.S, seg_begin + p.SPS);
    // a segment shorter than the others (the last) can end before some of
    // its parts begin: those parts are empty (st_begin == st_end)
    st_begin = min(seg_end, seg_begin + part * p.PL);
    st_end = min(seg_end, st_begin + p.PL);
    b = row / p.nDT;
    dtile = row - b * p.nDT;
  }
};

// CARRY = false: the fused forward scan.  CARRY = true: the carry pass over
// sub-chunks of PL stages (items independent, no readout): each item scans
// its stages from h = 0 and records (sum of Delta, h_end) per channel.
// OPT bit 0: software-pipelined scan loop (one channel per lane); bit 1:
// registers capped so that five CTAs fit on an SM (more warps in flight);
// bit 2 (bf16 inputs): the load warp widens each stage's B and C to fp32 in
// shared memory once for the CTA, instead of every lane widening the values
// it reads at every token; bit 3: a quarter of the state exponentials on the
// FMA pipe (one channel per lane, even states per lane); bit 4 (with bit 0):
// the pipelined loop prepares two tokens ahead instead of one.
template <typename InT, typename OutT, int NS, int LPC, int KC, int WARPS, int TT, bool ZOH,
          bool CARRY, bool CONV, int OPT>
__global__ void __launch_bounds__((WARPS + 1) * 32, (OPT & 2) ? 5 : 0)
    fwd_kernel(const __grid_constant__ TmaMaps maps, const FwdParams p) {
  constexpr bool BCF = (OPT & 4) != 0 && std::is_same<InT, __nv_bfloat16>::value;
  // OPT bit 3: one state pair in four (by token and pair index) takes its
  // exponentials on the FMA pipe (exp2_fma2) instead of the special-function
  // unit; the choice is fixed at compile time in the unrolled loops
  auto fma_exp = [](int pair_index) { return (OPT & 8) != 0 && pair_index % 4 == 0; };
  using Cfg = FwdCfg<InT, OutT, NS, LPC, KC, WARPS, TT, CONV, CARRY, BCF>;
  constexpr int NPL = Cfg::NPL, GPW = Cfg::GPW, DT = Cfg::DT, RAW = Cfg::RAW,
                TPL = Cfg::TPL;
  extern __shared__ __align__(1024) unsigned char smem[];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint64_t *rfull = reinterpret_cast<uint64_t *>(smem + Cfg::OFF_BAR);
  uint64_t *rempty = rfull + RAW;  // all scan warps are done with a slot
  uint64_t *rconv = rempty + RAW;  // BCF: the slot's B and C are widened (32 arrivals)

  // item and stage carried by each ring slot (written by the load warp
  // before the slot's full barrier completes; item -1 ends the CTA's work)
  __shared__ int2 slot_work[RAW];

  const unsigned int epoch = *reinterpret_cast<volatile unsigned int *>(&p.ctl->epoch);
  const int S = p.S;

  if (tid == 0) {
#pragma unroll
    for (int i = 0; i < RAW; ++i) {
      mbar_init(&rfull[i], 1);
      mbar_init(&rempty[i], WARPS);
      if constexpr (BCF) mbar_init(&rconv[i], 32);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == WARPS) {
    // ============ load warp (one thread issues; with BCF all 32 widen) ============
    const bool with_z = !CARRY && p.has_z;
    const uint32_t tx_bytes = (TT + Cfg::XHALO + (with_z ? 2u : 1u) * TT) * DT * sizeof(InT) +
                              (CARRY ? 1u : 2u) * TT * NS * sizeof(InT);
    ItemPos iss;
    int st = 0;
    int k = 0, issued = 0;
    int state = 0;  // 0: stage k issued, 1: no work left, 2: gave up waiting
    for (;; ++k) {
      const int r = k % RAW;
      if (lane == 0) {
        state = 0;
        if (k >= RAW &&
            !mbar_wait_bounded(&rempty[r], (uint32_t)(((k / RAW) - 1) & 1), p.timeout_ns)) {
          state = 2;
        } else {
          // next item when this one is done (parts past a short segment's end
          // have no stages and are skipped)
          while (iss.item < 0 || st >= iss.st_end) {
            const int it = (int)atomicAdd(&p.ctl->ticket, 1u);
            if (it >= p.items) {
              state = 1;
              break;
            }
            iss.set(it, p);
            st = iss.st_begin;
          }
          if (state == 1) {  // no work left: end marker, no data
            slot_work[r] = make_int2(-1, 0);
            if constexpr (!BCF) mbar_arrive(&rfull[r]);
          } else {
            slot_work[r] = make_int2(iss.item, st);
            const int d0 = iss.dtile * DT, t0 = st * TT, b = iss.b;
            unsigned char *sb = smem + r * Cfg::SLOT;
            mbar_arrive_expect_tx(&rfull[r], tx_bytes);
            tma_load_3d(sb, &maps.x, &rfull[r], d0, t0 - Cfg::XHALO, b);
            tma_load_3d(sb + Cfg::OFF_DT, &maps.dt, &rfull[r], d0, t0, b);
            if (with_z) tma_load_3d(sb + Cfg::OFF_Z, &maps.z, &rfull[r], d0, t0, b);
            tma_load_3d(sb + Cfg::OFF_B, &maps.B, &rfull[r], 0, t0, b);
            if (!CARRY) tma_load_3d(sb + Cfg::OFF_C, &maps.C, &rfull[r], 0, t0, b);
            ++st;
            issued = k + 1;
          }
        }
      }
      if constexpr (BCF) {
        // widen the previous stage while this one is in flight, then release
        // it to the scan warps (which wait on rconv, then on rfull)
        state = __shfl_sync(FULL_MASK, state, 0);
        if (state != 2 && k > 0) {
          const int rp = (k - 1) % RAW;
          if (!__all_sync(FULL_MASK, mbar_wait_bounded(&rfull[rp], (uint32_t)(((k - 1) / RAW) & 1),
                                                       p.timeout_ns))) {
            state = 2;
          } else {
            const unsigned char *sb = smem + rp * Cfg::SLOT;
            widen_tile<TT * NS>(reinterpret_cast<const __nv_bfloat16 *>(sb + Cfg::OFF_B),
                                reinterpret_cast<float *>(smem + rp * Cfg::SLOT + Cfg::OFF_BF),
                                lane);
            if constexpr (!CARRY)
              widen_tile<TT * NS>(reinterpret_cast<const __nv_bfloat16 *>(sb + Cfg::OFF_C),
                                  reinterpret_cast<float *>(smem + rp * Cfg::SLOT + Cfg::OFF_CF),
                                  lane);
            mbar_arrive(&rconv[rp]);
          }
        }
        if (state == 1) mbar_arrive(&rconv[r]);  // the end marker
      } else {
        state = __shfl_sync(FULL_MASK, state, 0);
      }
      if (state != 0) break;
    }
    if (lane == 0 && state == 2) {
      atomicCAS(&p.ctl->status, 0, kStatusTimeout);
      // let the loads still in flight land before the CTA exits (bounded)
      for (int kk = (issued > RAW ? issued - RAW : 0); kk < issued; ++kk)
        (void)mbar_wait_bounded(&rfull[kk % RAW], (uint32_t)((kk / RAW) & 1), p.timeout_ns);
    }
  } else {
    // =================== scan warps ===================
    const int g_loc = lane / LPC;        // channel group within the warp
    const int q = lane % LPC;            // state group of this lane
    const int grp = warp * GPW + g_loc;  // channel group within the row tile
    const int ch0 = grp * KC;            // first channel of this lane within the row tile
    unsigned char *plane_base = smem + Cfg::OFF_PLANE + warp * Cfg::PLANE;
    float h[KC][NPL], A2[KC][NPL], invA[KC][NPL];  // invA: 1/A (0 where A = 0), ZOH only
#pragma unroll
    for (int c = 0; c < KC; ++c)
#pragma unroll
      for (int i = 0; i < NPL; ++i) { h[c][i] = 0.f; A2[c][i] = 0.f; invA[c][i] = 0.f; }
    float bias[KC], dsk[KC], dsum[KC];
    float cw[KC][CONV ? kConvWidth : 1], cb[KC];  // conv taps and bias of each channel
#pragma unroll
    for (int c = 0; c < KC; ++c) {
      bias[c] = 0.f; dsk[c] = 0.f; dsum[c] = 0.f; cb[c] = 0.f;
#pragma unroll
      for (int k = 0; k < (CONV ? kConvWidth : 1); ++k) cw[c][k] = 0.f;
    }
    OutT *const ybase = reinterpret_cast<OutT *>(p.y);
    ItemPos cur;
    for (int k = 0;; ++k) {
      const int r = k % RAW;
      if (!__all_sync(FULL_MASK, mbar_wait_bounded(BCF ? &rconv[r] : &rfull[r],
                                                   (uint32_t)((k / RAW) & 1), p.timeout_ns))) {
        if (lane == 0) atomicCAS(&p.ctl->status, 0, kStatusTimeout);
        break;
      }
      const int2 work = slot_work[r];
      if (work.x < 0) break;  // end marker
      // (BCF: the load warp saw the tiles land before widening; waiting on
      // the slot's own barrier too makes the bulk copy's data visible here)
      if (BCF && !__all_sync(FULL_MASK, mbar_wait_bounded(&rfull[r], (uint32_t)((k / RAW) & 1),
                                                          p.timeout_ns))) {
        if (lane == 0) atomicCAS(&p.ctl->status, 0, kStatusTimeout);
        break;
      }
      if (work.x != cur.item) cur.set(work.x, p);
      const int st = work.y, b = cur.b;
      const int d = cur.dtile * DT + ch0;  // first channel (of KC) in the tensor
      const bool valid_ch = d < p.D;       // KC = 2: D is even there, so d + 1 < D too
      if (st == cur.st_begin) {  // per-item parameters and starting state of this lane
#pragma unroll
        for (int c = 0; c < KC; ++c) {
#pragma unroll
          for (int i = 0; i < NPL; ++i) {
            const float a = valid_ch ? __ldg(p.A + (size_t)(d + c) * NS + q * NPL + i) : 0.f;
            A2[c][i] = a * kLog2e;
            if constexpr (ZOH) invA[c][i] = a != 0.f ? 1.f / a : 0.f;
          }
          bias[c] = (p.has_bias && valid_ch) ? __ldg(p.bias + d + c) : 0.f;
          dsk[c] = (!CARRY && p.has_D && valid_ch) ? __ldg(p.Dv + d + c) : 0.f;
          dsum[c] = 0.f;
          if constexpr (CONV) {
#pragma unroll
            for (int k = 0; k < kConvWidth; ++k)
              cw[c][k] = valid_ch ? __ldg(p.conv_w + (size_t)(d + c) * kConvWidth + k) : 0.f;
            cb[c] = (valid_ch && p.conv_b) ? __ldg(p.conv_b + d + c) : 0.f;
          }
        }
        if (CARRY || st == cur.seg_begin) {
          // start of a carry sub-chunk (from 0) or of a segment: h0, then the
          // maps of all sub-chunks before this segment, in order
#pragma unroll
          for (int c = 0; c < KC; ++c)
#pragma unroll
            for (int i = 0; i < NPL; ++i)
              h[c][i] = (!CARRY && p.has_h0 && valid_ch)
                            ? __ldg(p.h0 + ((size_t)b * p.D + d + c) * NS + q * NPL + i) : 0.f;
          if (!CARRY && cur.seg > 0 && valid_ch) {
            const int nsub = cur.seg * p.nq;
            for (int j = 0; j < nsub; ++j) {
              const size_t base = ((size_t)b * p.nsub_row + j) * p.D + d;
#pragma unroll
              for (int c = 0; c < KC; ++c) {
                const float s = __ldcg(p.agg_s + base + c);
                const float *ah = p.agg_h + (base + c) * NS + q * NPL;
#pragma unroll
                for (int i = 0; i < NPL; ++i)
                  h[c][i] = fmaf(ex2_approx(A2[c][i] * s), h[c][i], __ldcg(ah + i));
              }
            }
          }
        } else {  // carried state of this (row, segment) from the CTA that ran the previous part
          const unsigned long long want = ((unsigned long long)epoch << 32) | (unsigned)st;
          unsigned long long *flag = p.ws_flags + (size_t)cur.vrow * WARPS + warp;
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
#pragma unroll
          for (int c = 0; c < KC; ++c) {
            const float *src = p.ws_state + ((size_t)cur.vrow * DT + ch0 + c) * NS + q * NPL;
#pragma unroll
            for (int i = 0; i < NPL; ++i) h[c][i] = __ldcg(src + i);
          }
        }
      }

      const unsigned char *sb = smem + r * Cfg::SLOT;
      // x rows: token t of the stage is row t + XHALO (conv front-end: rows
      // t + 1 .. t + 4 are tokens t - 3 .. t)
      const InT *xs = reinterpret_cast<const InT *>(sb);
      const InT *ds = reinterpret_cast<const InT *>(sb + Cfg::OFF_DT);
      const InT *zs = reinterpret_cast<const InT *>(sb + Cfg::OFF_Z);
      using BCT = typename std::conditional<BCF, float, InT>::type;  // B, C as the lanes read them
      const BCT *Bs = reinterpret_cast<const BCT *>(sb + (BCF ? Cfg::OFF_BF : Cfg::OFF_B));
      const BCT *Cs = reinterpret_cast<const BCT *>(sb + (BCF ? Cfg::OFF_CF : Cfg::OFF_C));
      const int t0 = st * TT;
      OutT *xcrow = CONV && p.xconv
                        ? reinterpret_cast<OutT *>(p.xconv) + ((size_t)b * p.L + t0) * p.D + d
                        : nullptr;
      const int nvalid = min(TT, p.L - t0);
      OutT *yrow = ybase + ((size_t)b * p.L + t0) * p.D + d;

      if constexpr (KC == 1) {
        float2 *plane = reinterpret_cast<float2 *>(plane_base);
        const int ch = ch0;
        // -- per-token prologue of this lane's tokens j * LPC + q --
        float g1[CARRY ? 1 : TPL], g2[CARRY ? 1 : TPL];
        if constexpr (TPL % 2 == 0) {
#pragma unroll
          for (int j = 0; j < TPL; j += 2) {
            const int ta = j * LPC + q, tb = ta + LPC;
            float2 xv;
            if constexpr (CONV) {
              float2 u = make_float2(cb[0], cb[0]);
#pragma unroll
              for (int k = 0; k < kConvWidth; ++k)
                u = ffma2(make_float2(cw[0][k], cw[0][k]),
                          make_float2(to_f32(xs[(ta + 1 + k) * DT + ch]),
                                      to_f32(xs[(tb + 1 + k) * DT + ch])), u);
              xv = silu_f2(u);
              if (xcrow && valid_ch && !CARRY) {
                if (ta < nvalid) xcrow[(size_t)ta * p.D] = from_f32<OutT>(xv.x);
                if (tb < nvalid) xcrow[(size_t)tb * p.D] = from_f32<OutT>(xv.y);
              }
            } else {
              xv = make_float2(to_f32(xs[ta * DT + ch]), to_f32(xs[tb * DT + ch]));
            }
            float2 v = fadd2(make_float2(to_f32(ds[ta * DT + ch]), to_f32(ds[tb * DT + ch])),
                             make_float2(bias[0], bias[0]));
            if (p.softplus) v = softplus_f2(v);
            if (ta >= nvalid) v.x = 0.f;  // past the end: identity update
            if (tb >= nvalid) v.y = 0.f;
            const float2 dx = fmul2(v, xv);
            // zero-order hold keeps x itself: its input term is not a multiple of Delta
            plane[g_loc * Cfg::TTP + ta] = make_float2(v.x, ZOH ? xv.x : dx.x);
            plane[g_loc * Cfg::TTP + tb] = make_float2(v.y, ZOH ? xv.y : dx.y);
            if constexpr (!CARRY) {
              float2 g = make_float2(1.f, 1.f);
              if (p.has_z)
                g = silu_f2(make_float2(to_f32(zs[ta * DT + ch]), to_f32(zs[tb * DT + ch])));
              const float2 gd = fmul2(fmul2(make_float2(dsk[0], dsk[0]), xv), g);
              g1[j] = g.x; g1[j + 1] = g.y;
              g2[j] = gd.x; g2[j + 1] = gd.y;
            }
          }
        } else {
#pragma unroll
          for (int j = 0; j < TPL; ++j) {
            const int ta = j * LPC + q;
            float xv;
            if constexpr (CONV) {
              float u = cb[0];
#pragma unroll
              for (int k = 0; k < kConvWidth; ++k)
                u = fmaf(cw[0][k], to_f32(xs[(ta + 1 + k) * DT + ch]), u);
              xv = silu_f(u);
              if (xcrow && valid_ch && !CARRY && ta < nvalid)
                xcrow[(size_t)ta * p.D] = from_f32<OutT>(xv);
            } else {
              xv = to_f32(xs[ta * DT + ch]);
            }
            float v = to_f32(ds[ta * DT + ch]) + bias[0];
            if (p.softplus) v = softplus_f(v);
            if (ta >= nvalid) v = 0.f;
            plane[g_loc * Cfg::TTP + ta] = make_float2(v, ZOH ? xv : v * xv);
            if constexpr (!CARRY) {
              const float g = p.has_z ? silu_f(to_f32(zs[ta * DT + ch])) : 1.f;
              g1[j] = g;
              g2[j] = dsk[0] * xv * g;
            }
          }
        }
        __syncwarp();

        // -- the scan over TT tokens of this lane's channel --
        const float2 *prow = plane + g_loc * Cfg::TTP;
        if constexpr ((OPT & 1) && !CARRY && !ZOH && NPL % 2 == 0) {
          // Software-pipelined form: the exponentials, input terms and C of
          // token t + 1 are formed (loads, ex2) before token t's state update
          // consumes those of token t, so the special-function latency and
          // the shared-memory loads overlap the update chain (option bit 4:
          // tokens t + 1 and t + 2, in registers: the special-function and
          // shared-memory latencies get two tokens' work to hide behind).
          constexpr int NP = NPL / 2;
          constexpr int PD = (OPT & 16) ? 2 : 1;  // tokens prepared ahead
          float2 an[PD][NP], bn[PD][NP], cn[PD][NP];
          auto prep = [&](int t, float2 (&a)[NP], float2 (&bx)[NP], float2 (&cc)[NP]) {
            const float4 dp = *reinterpret_cast<const float4 *>(prow + (t & ~1));
            const float2 dd = (t & 1) ? make_float2(dp.z, dp.w) : make_float2(dp.x, dp.y);
            float bv[NPL], cv[NPL];
            load_bc<NPL>(Bs + t * NS + q * NPL, bv);
            load_bc<NPL>(Cs + t * NS + q * NPL, cv);
            const float2 dA = make_float2(dd.x, dd.x), dX = make_float2(dd.y, dd.y);
#pragma unroll
            for (int k = 0; k < NP; ++k) {
              const float2 arg = fmul2(dA, make_float2(A2[0][2 * k], A2[0][2 * k + 1]));
              a[k] = fma_exp(t * NP + k) ? exp2_fma2(arg)
                                         : make_float2(ex2_approx(arg.x), ex2_approx(arg.y));
              bx[k] = fmul2(dX, make_float2(bv[2 * k], bv[2 * k + 1]));
              cc[k] = make_float2(cv[2 * k], cv[2 * k + 1]);
            }
          };
#pragma unroll
          for (int i = 0; i < PD; ++i) prep(i, an[i], bn[i], cn[i]);
#pragma unroll
          for (int tt = 0; tt < TT; tt += LPC) {
            float yp[LPC];
#pragma unroll
            for (int j = 0; j < LPC; ++j) {
              const int t = tt + j, sl = t % PD;
              float2 ac[NP], bc[NP], ccur[NP];
#pragma unroll
              for (int k = 0; k < NP; ++k) {
                ac[k] = an[sl][k];
                bc[k] = bn[sl][k];
                ccur[k] = cn[sl][k];
              }
              if (t + PD < TT) prep(t + PD, an[sl], bn[sl], cn[sl]);
              float2 acc = make_float2(0.f, 0.f);
#pragma unroll
              for (int k = 0; k < NP; ++k) {
                const float2 hn = ffma2(ac[k], make_float2(h[0][2 * k], h[0][2 * k + 1]), bc[k]);
                h[0][2 * k] = hn.x;
                h[0][2 * k + 1] = hn.y;
                acc = ffma2(ccur[k], hn, acc);
              }
              yp[j] = acc.x + acc.y;
            }
            const float ys = reduce_scatter<LPC>(yp, q);
            const int to = tt + q;
            if (to < nvalid && valid_ch)
              yrow[(size_t)to * p.D] = from_f32<OutT>(fmaf(ys, g1[tt / LPC], g2[tt / LPC]));
          }
        } else {
        float4 dpair;  // (Delta, Delta*x) of an even token and the next, one 16-byte load
#pragma unroll
        for (int tt = 0; tt < TT; tt += LPC) {
          float yp[LPC];
#pragma unroll
          for (int j = 0; j < LPC; ++j) {
            const int t = tt + j;
            if ((t & 1) == 0) dpair = *reinterpret_cast<const float4 *>(prow + t);
            const float2 dd =
                (t & 1) ? make_float2(dpair.z, dpair.w) : make_float2(dpair.x, dpair.y);
            if constexpr (CARRY) dsum[0] += dd.x;
            float bv[NPL], cv[NPL];
            load_bc<NPL>(Bs + t * NS + q * NPL, bv);
            if constexpr (!CARRY) load_bc<NPL>(Cs + t * NS + q * NPL, cv);
            if constexpr (NPL % 2 == 0) {
              const float2 dA = make_float2(dd.x, dd.x), dX = make_float2(dd.y, dd.y);
              float2 acc = make_float2(0.f, 0.f);
#pragma unroll
              for (int i = 0; i < NPL; i += 2) {
                const float2 arg = fmul2(dA, make_float2(A2[0][i], A2[0][i + 1]));
                const float2 a = fma_exp(t * (NPL / 2) + i / 2)
                                     ? exp2_fma2(arg)
                                     : make_float2(ex2_approx(arg.x), ex2_approx(arg.y));
                float2 bx = fmul2(dX, make_float2(bv[i], bv[i + 1]));
                if constexpr (ZOH)  // dX holds x: Bbar x = ((e^u - 1) / A) * (B x)
                  bx = fmul2(zoh_coef2(fmul2(arg, make_float2(kLn2, kLn2)), a, dA,
                                       make_float2(invA[0][i], invA[0][i + 1])),
                             bx);
                const float2 hn = ffma2(a, make_float2(h[0][i], h[0][i + 1]), bx);
                h[0][i] = hn.x;
                h[0][i + 1] = hn.y;
                if constexpr (!CARRY) acc = ffma2(make_float2(cv[i], cv[i + 1]), hn, acc);
              }
              yp[j] = acc.x + acc.y;
            } else {
              const float arg = dd.x * A2[0][0];
              const float a = ex2_approx(arg);
              float bx = dd.y * bv[0];
              if constexpr (ZOH) bx *= zoh_coef(arg * kLn2, a, dd.x, invA[0][0]);
              h[0][0] = fmaf(a, h[0][0], bx);
              yp[j] = CARRY ? 0.f : cv[0] * h[0][0];
            }
          }
          if constexpr (!CARRY) {
            const float ys = reduce_scatter<LPC>(yp, q);
            const int to = tt + q;  // this lane's own token of the group: prologue slot tt / LPC
            if (to < nvalid && valid_ch)
              yrow[(size_t)to * p.D] = from_f32<OutT>(fmaf(ys, g1[tt / LPC], g2[tt / LPC]));
          }
        }
        }
      } else {
        // ------------- two channels per lane: ch0 and ch0 + 1 -------------
        float4 *plane = reinterpret_cast<float4 *>(plane_base);
        float2 g1[CARRY ? 1 : TPL], g2[CARRY ? 1 : TPL];
#pragma unroll
        for (int j = 0; j < TPL; ++j) {
          const int ta = j * LPC + q;
          float2 xv;
          if constexpr (CONV) {
            float2 u = make_float2(cb[0], cb[1]);
#pragma unroll
            for (int k = 0; k < kConvWidth; ++k)
              u = ffma2(make_float2(cw[0][k], cw[1][k]), load_pair(xs + (ta + 1 + k) * DT + ch0),
                        u);
            xv = silu_f2(u);
            if (xcrow && valid_ch && !CARRY && ta < nvalid)
              store_pair(xcrow + (size_t)ta * p.D, xv);
          } else {
            xv = load_pair(xs + ta * DT + ch0);
          }
          float2 v = fadd2(load_pair(ds + ta * DT + ch0), make_float2(bias[0], bias[1]));
          if (p.softplus) v = softplus_f2(v);
          if (ta >= nvalid) v = make_float2(0.f, 0.f);  // past the end: identity update
          const float2 dx = ZOH ? xv : fmul2(v, xv);
          plane[g_loc * Cfg::TTP + ta] = make_float4(v.x, v.y, dx.x, dx.y);
          if constexpr (!CARRY) {
            const float2 g = p.has_z ? silu_f2(load_pair(zs + ta * DT + ch0))
                                     : make_float2(1.f, 1.f);
            g1[j] = g;
            g2[j] = fmul2(fmul2(make_float2(dsk[0], dsk[1]), xv), g);
          }
        }
        __syncwarp();

        const float4 *prow = plane + g_loc * Cfg::TTP;
#pragma unroll
        for (int tt = 0; tt < TT; tt += LPC) {
          float2 yp[LPC];
#pragma unroll
          for (int j = 0; j < LPC; ++j) {
            const int t = tt + j;
            const float4 dd = prow[t];  // (Delta0, Delta1, X0, X1)
            float bv[NPL], cv[NPL];
            load_bc<NPL>(Bs + t * NS + q * NPL, bv);
            if constexpr (!CARRY) load_bc<NPL>(Cs + t * NS + q * NPL, cv);
            float ypc[2];
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              const float dl = c ? dd.y : dd.x, xx = c ? dd.w : dd.z;
              if constexpr (CARRY) dsum[c] += dl;
              const float2 dA = make_float2(dl, dl), dX = make_float2(xx, xx);
              float2 acc = make_float2(0.f, 0.f);
#pragma unroll
              for (int i = 0; i < NPL; i += 2) {
                const float2 arg = fmul2(dA, make_float2(A2[c][i], A2[c][i + 1]));
                const float2 a = make_float2(ex2_approx(arg.x), ex2_approx(arg.y));
                float2 bx = fmul2(dX, make_float2(bv[i], bv[i + 1]));
                if constexpr (ZOH)
                  bx = fmul2(zoh_coef2(fmul2(arg, make_float2(kLn2, kLn2)), a, dA,
                                       make_float2(invA[c][i], invA[c][i + 1])),
                             bx);
                const float2 hn = ffma2(a, make_float2(h[c][i], h[c][i + 1]), bx);
                h[c][i] = hn.x;
                h[c][i + 1] = hn.y;
                if constexpr (!CARRY) acc = ffma2(make_float2(cv[i], cv[i + 1]), hn, acc);
              }
              ypc[c] = acc.x + acc.y;
            }
            yp[j] = make_float2(ypc[0], ypc[1]);
          }
          if constexpr (!CARRY) {
            const float2 ys = reduce_scatter2<LPC>(yp, q);
            const int to = tt + q;
            if (to < nvalid && valid_ch)
              store_pair(yrow + (size_t)to * p.D, ffma2(ys, g1[tt / LPC], g2[tt / LPC]));
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&rempty[r]);  // this warp is done with slot r

      if (st + 1 == cur.st_end) {  // end of this item's stages
        if constexpr (CARRY) {
          // the sub-chunk's map: (sum of Delta, state reached from 0)
          if (valid_ch) {
            const size_t base = ((size_t)b * p.nsub_row + cur.part) * p.D + d;
#pragma unroll
            for (int c = 0; c < KC; ++c) {
              float *dst = p.agg_h + (base + c) * NS + q * NPL;
#pragma unroll
              for (int i = 0; i < NPL; ++i) __stcg(dst + i, h[c][i]);
              if (q == 0) __stcg(p.agg_s + base + c, dsum[c]);
            }
          }
        } else if (st + 1 == cur.seg_end) {
          if (st == S - 1 && p.want_hlast && valid_ch) {  // the last segment's end
#pragma unroll
            for (int c = 0; c < KC; ++c) {
              float *dst = p.h_last + ((size_t)b * p.D + d + c) * NS + q * NPL;
#pragma unroll
              for (int i = 0; i < NPL; ++i) dst[i] = h[c][i];
            }
          }
        } else if ((long long)cur.row * S + st != p.drop_unit) {  // hand the state on
#pragma unroll
          for (int c = 0; c < KC; ++c) {
            float *dst = p.ws_state + ((size_t)cur.vrow * DT + ch0 + c) * NS + q * NPL;
#pragma unroll
            for (int i = 0; i < NPL; ++i) __stcg(dst + i, h[c][i]);
          }
          __threadfence();
          __syncwarp();
          if (lane == 0)
            st_release_u64(p.ws_flags + (size_t)cur.vrow * WARPS + warp,
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
      p.ctl->ticket = 0u;
      p.ctl->epoch = epoch + 1u;
      __threadfence();
    }
  }
}

// ---------------------------------------------------------------------------
// host side: one compiled variant
// ---------------------------------------------------------------------------

template <typename InT, typename OutT, int NS, int LPC, int KC, int WARPS, int TT, bool ZOH,
          bool CARRY, bool CONV, int OPT>
static cudaError_t run_variant(const LaunchShape *ls, const TmaMaps *maps, const FwdParams *p,
                               cudaStream_t stream, VariantInfo *vi) {
  constexpr bool BCF = (OPT & 4) != 0 && std::is_same<InT, __nv_bfloat16>::value;
  using Cfg = FwdCfg<InT, OutT, NS, LPC, KC, WARPS, TT, CONV, CARRY, BCF>;
  auto kern = fwd_kernel<InT, OutT, NS, LPC, KC, WARPS, TT, ZOH, CARRY, CONV, OPT>;
  if (Cfg::SMEM + 8 * Cfg::RAW > 227 * 1024) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return e;
  }
  if (vi) {
    vi->smem = Cfg::SMEM;
    vi->ring = Cfg::RAW;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&vi->occ, kern, Cfg::THREADS, Cfg::SMEM);
    if (e != cudaSuccess) return e;
  }
  if (!maps) return cudaSuccess;
  kern<<<ls->grid, Cfg::THREADS, Cfg::SMEM, stream>>>(*maps, *p);
  return cudaGetLastError();
}

// Does a launch shape ask for this compiled variant?
inline bool shape_is(const LaunchShape *ls, int ns, int lpc, int kc, int warps, int tt, bool zoh,
                     bool carry, bool conv, int opt) {
  return ls->ns == ns && ls->lpc == lpc && ls->kc == kc && ls->warps == warps && ls->tt == tt &&
         ls->zoh == zoh && ls->carry == carry && ls->conv == conv && ls->opt == opt;
}

}  // namespace ssm
