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
//   * Ticket schedule.  Each row's S stages are cut into parts of PL stages;
//     item i = part * R + row.  A CTA's load warp takes item numbers in
//     increasing order from a device counter (one atomic per item), so the
//     predecessor of an item (same row, previous part, number i - R) always
//     went to a CTA that was already running: every wait for a carried state
//     ends, however few CTAs the device runs at once, and CTAs that finish
//     early simply take more items.  A part hands its final state to the next
//     part through a per-(row, warp) flag carrying the stage index and a
//     launch epoch (release/acquire) -- the pages' associative carry ("Scan
//     bien recurrence ...": (A2,b2) (x) (A1,b1) = (A2A1, A2b1+b2)): the state
//     after one part is the exact starting state of the next.  Every wait is
//     bounded by a timer.
//   * One load warp streams the stages' [TT, DT] tiles of x / delta / z and
//     [TT, N] tiles of B / C into a ring of RAW shared-memory slots with TMA
//     (cp.async.bulk.tensor, every CTA loads its own tiles); slot full / slot
//     empty mbarriers are the only coupling between warps.  Each scan warp
//     does all the per-token work of its own channels: lane q of a channel
//     prepares tokens q, q + LPC, ... (Delta, Delta*x into a warp-private
//     plane that the channel's LPC lanes read back; silu(z) and D*x*silu(z)
//     stay in the registers of the lane that finishes those very tokens),
//     scans, and stores y straight from registers.  B / C are read as stored
//     (bf16 words are widened with integer ops), which halves the
//     shared-memory wavefronts of the scan loop against fp32 staging.
//     Tokens past the end get Delta = 0, an identity update, so carried
//     states are exact for ragged tails.
#pragma once

#include "device_common.cuh"
#include "scan_params.h"

namespace ssm {

constexpr int align_up(int v, int a) { return (v + a - 1) / a * a; }
constexpr int clamp_int(int v, int lo, int hi) { return v < lo ? lo : (v > hi ? hi : v); }

template <typename InT, typename OutT, int NS, int LPC, int WARPS, int TT>
struct FwdCfg {
  static constexpr int NPL = NS / LPC;    // states per lane
  static constexpr int DTW = 32 / LPC;    // channels per scan warp
  static constexpr int DT = WARPS * DTW;  // channels per row tile
  static constexpr int TPL = TT / LPC;    // tokens a lane prepares and finishes per stage
  static constexpr int THREADS = (WARPS + 1) * 32;  // scan warps + the load warp
  static constexpr int XTILE = align_up(TT * DT * (int)sizeof(InT), 128);
  static constexpr int BCTILE = align_up(TT * NS * (int)sizeof(InT), 128);
  static constexpr int SLOT = 3 * XTILE + 2 * BCTILE;
  // ring depth: ~128 tokens of prefetch, within ~64 KB, at least 3 slots
  static constexpr int RAW = clamp_int(65536 / SLOT, 3, 128 / TT > 3 ? 128 / TT : 3);
  // (Delta, Delta*x) per warp, channel-major: row c holds tokens 0..TT-1 of
  // channel c, rows TTP float2 apart (TTP - TT spreads the rows over the
  // shared-memory banks; TTP even keeps token pairs 16-byte aligned)
  static constexpr int TTP = TT + (LPC > 2 ? LPC : 2);
  static constexpr int PLANE = align_up(TTP * DTW * 8, 128);
  static constexpr int OFF_PLANE = RAW * SLOT;
  static constexpr int OFF_BAR = OFF_PLANE + WARPS * PLANE;
  static constexpr int SMEM = OFF_BAR + 2 * RAW * 8;
  static_assert(NS % LPC == 0, "LPC must divide N");
  static_assert(TT % LPC == 0, "LPC must divide the stage length");
  static_assert(DT * (int)sizeof(InT) % 16 == 0, "TMA rows need 16-byte multiples");
  static_assert(SLOT % 128 == 0 && OFF_PLANE % 128 == 0, "slot alignment");
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

// Position of one stage of work: item (row, part) and stage index, derived
// from an item number once per item (a division happens only there).
struct ItemPos {
  int item = -1, row = 0, part = 0, b = 0, dtile = 0, st_begin = 0, st_end = 0;
  __device__ __forceinline__ void set(int it, const FwdParams &p) {
    item = it;
    part = it / p.rows;
    row = it - part * p.rows;
    st_begin = part * p.PL;
    st_end = min(p.S, st_begin + p.PL);
    b = row / p.nDT;
    dtile = row - b * p.nDT;
  }
};

template <typename InT, typename OutT, int NS, int LPC, int WARPS, int TT, bool ZOH>
__global__ void __launch_bounds__((WARPS + 1) * 32)
    fwd_kernel(const __grid_constant__ TmaMaps maps, const FwdParams p) {
  using Cfg = FwdCfg<InT, OutT, NS, LPC, WARPS, TT>;
  constexpr int NPL = Cfg::NPL, DTW = Cfg::DTW, DT = Cfg::DT, RAW = Cfg::RAW, TPL = Cfg::TPL;
  extern __shared__ __align__(1024) unsigned char smem[];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint64_t *rfull = reinterpret_cast<uint64_t *>(smem + Cfg::OFF_BAR);
  uint64_t *rempty = rfull + RAW;  // all scan warps are done with a slot

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
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == WARPS) {
    // =================== load warp (one thread issues) ===================
    if (lane == 0) {
      const uint32_t tx_bytes =
          (p.has_z ? 3u : 2u) * TT * DT * sizeof(InT) + 2u * TT * NS * sizeof(InT);
      // Work items are handed out in increasing order from a device counter
      // (a ticket per item).  An item's predecessor (same row, previous part)
      // has a smaller number, so it went to a CTA that was already running
      // when this one took its ticket: waits on carried states always end,
      // whatever share of the device this launch gets.
      ItemPos iss;
      int st = 0;
      bool ok = true;
      int k = 0;
      for (;; ++k) {
        const int r = k % RAW;
        if (k >= RAW &&
            !mbar_wait_bounded(&rempty[r], (uint32_t)(((k / RAW) - 1) & 1), p.timeout_ns)) {
          ok = false;
          break;
        }
        if (iss.item < 0 || st == iss.st_end) {
          const int it = (int)atomicAdd(&p.ctl->ticket, 1u);
          if (it >= p.items) {  // no work left: end marker, no data
            slot_work[r] = make_int2(-1, 0);
            mbar_arrive(&rfull[r]);
            break;
          }
          iss.set(it, p);
          st = iss.st_begin;
        }
        slot_work[r] = make_int2(iss.item, st);
        const int d0 = iss.dtile * DT, t0 = st * TT, b = iss.b;
        unsigned char *sb = smem + r * Cfg::SLOT;
        mbar_arrive_expect_tx(&rfull[r], tx_bytes);
        tma_load_3d(sb, &maps.x, &rfull[r], d0, t0, b);
        tma_load_3d(sb + Cfg::XTILE, &maps.dt, &rfull[r], d0, t0, b);
        if (p.has_z) tma_load_3d(sb + 2 * Cfg::XTILE, &maps.z, &rfull[r], d0, t0, b);
        tma_load_3d(sb + 3 * Cfg::XTILE, &maps.B, &rfull[r], 0, t0, b);
        tma_load_3d(sb + 3 * Cfg::XTILE + Cfg::BCTILE, &maps.C, &rfull[r], 0, t0, b);
        ++st;
      }
      if (!ok) {
        atomicCAS(&p.ctl->status, 0, kStatusTimeout);
        // let the loads still in flight land before the CTA exits (bounded)
        for (int kk = (k > RAW ? k - RAW : 0); kk < k; ++kk)
          (void)mbar_wait_bounded(&rfull[kk % RAW], (uint32_t)((kk / RAW) & 1), p.timeout_ns);
      }
    }
  } else {
    // =================== scan warps ===================
    const int c_loc = lane / LPC;       // channel within the warp
    const int q = lane % LPC;           // state group of this lane
    const int ch = warp * DTW + c_loc;  // channel within the row tile
    float2 *plane = reinterpret_cast<float2 *>(smem + Cfg::OFF_PLANE + warp * Cfg::PLANE);
    float h[NPL], A2[NPL], invA[NPL];  // invA: 1/A (0 where A = 0), zero-order hold only
#pragma unroll
    for (int i = 0; i < NPL; ++i) { h[i] = 0.f; A2[i] = 0.f; invA[i] = 0.f; }
    float bias = 0.f, dsk = 0.f;
    OutT *const ybase = reinterpret_cast<OutT *>(p.y);
    ItemPos cur;
    for (int k = 0;; ++k) {
      const int r = k % RAW;
      if (!__all_sync(FULL_MASK, mbar_wait_bounded(&rfull[r], (uint32_t)((k / RAW) & 1),
                                                   p.timeout_ns))) {
        if (lane == 0) atomicCAS(&p.ctl->status, 0, kStatusTimeout);
        break;
      }
      const int2 work = slot_work[r];
      if (work.x < 0) break;  // end marker
      if (work.x != cur.item) cur.set(work.x, p);
      const int row = cur.row, st = work.y, b = cur.b;
      const int d = cur.dtile * DT + ch;
      const bool valid_ch = d < p.D;
      const bool run_start = st == cur.st_begin;
      if (run_start) {  // per-item parameters and starting state of this lane
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
          const float a = valid_ch ? __ldg(p.A + (size_t)d * NS + q * NPL + i) : 0.f;
          A2[i] = a * kLog2e;
          if constexpr (ZOH) invA[i] = a != 0.f ? 1.f / a : 0.f;
        }
        bias = (p.has_bias && valid_ch) ? __ldg(p.bias + d) : 0.f;
        dsk = (p.has_D && valid_ch) ? __ldg(p.Dv + d) : 0.f;
        if (st == 0) {
#pragma unroll
          for (int i = 0; i < NPL; ++i)
            h[i] = (p.has_h0 && valid_ch)
                       ? __ldg(p.h0 + ((size_t)b * p.D + d) * NS + q * NPL + i) : 0.f;
        } else {  // carried state of this row from the CTA that ran the previous part
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

      const unsigned char *sb = smem + r * Cfg::SLOT;
      const InT *xs = reinterpret_cast<const InT *>(sb);
      const InT *ds = reinterpret_cast<const InT *>(sb + Cfg::XTILE);
      const InT *zs = reinterpret_cast<const InT *>(sb + 2 * Cfg::XTILE);
      const InT *Bs = reinterpret_cast<const InT *>(sb + 3 * Cfg::XTILE);
      const InT *Cs = reinterpret_cast<const InT *>(sb + 3 * Cfg::XTILE + Cfg::BCTILE);
      const int t0 = st * TT;
      const int nvalid = min(TT, p.L - t0);

      // -- per-token prologue of this lane's tokens j * LPC + q --
      float g1[TPL], g2[TPL];
      if constexpr (TPL % 2 == 0) {
#pragma unroll
        for (int j = 0; j < TPL; j += 2) {
          const int ta = j * LPC + q, tb = ta + LPC;
          const float2 xv = make_float2(to_f32(xs[ta * DT + ch]), to_f32(xs[tb * DT + ch]));
          float2 v = fadd2(make_float2(to_f32(ds[ta * DT + ch]), to_f32(ds[tb * DT + ch])),
                           make_float2(bias, bias));
          if (p.softplus) v = softplus_f2(v);
          if (ta >= nvalid) v.x = 0.f;  // past the end: identity update
          if (tb >= nvalid) v.y = 0.f;
          const float2 dx = fmul2(v, xv);
          // zero-order hold keeps x itself: its input term is not a multiple of Delta
          plane[c_loc * Cfg::TTP + ta] = make_float2(v.x, ZOH ? xv.x : dx.x);
          plane[c_loc * Cfg::TTP + tb] = make_float2(v.y, ZOH ? xv.y : dx.y);
          float2 g = make_float2(1.f, 1.f);
          if (p.has_z) g = silu_f2(make_float2(to_f32(zs[ta * DT + ch]), to_f32(zs[tb * DT + ch])));
          const float2 gd = fmul2(fmul2(make_float2(dsk, dsk), xv), g);
          g1[j] = g.x; g1[j + 1] = g.y;
          g2[j] = gd.x; g2[j + 1] = gd.y;
        }
      } else {
#pragma unroll
        for (int j = 0; j < TPL; ++j) {
          const int ta = j * LPC + q;
          const float xv = to_f32(xs[ta * DT + ch]);
          float v = to_f32(ds[ta * DT + ch]) + bias;
          if (p.softplus) v = softplus_f(v);
          if (ta >= nvalid) v = 0.f;
          plane[c_loc * Cfg::TTP + ta] = make_float2(v, ZOH ? xv : v * xv);
          const float g = p.has_z ? silu_f(to_f32(zs[ta * DT + ch])) : 1.f;
          g1[j] = g;
          g2[j] = dsk * xv * g;
        }
      }
      __syncwarp();

      // -- the scan over TT tokens of this lane's channel --
      OutT *yrow = ybase + ((size_t)b * p.L + t0) * p.D + d;
      const float2 *prow = plane + c_loc * Cfg::TTP;
      float4 dpair;  // (Delta, Delta*x) of an even token and the next, one 16-byte load
#pragma unroll
      for (int tt = 0; tt < TT; tt += LPC) {
        float yp[LPC];
#pragma unroll
        for (int j = 0; j < LPC; ++j) {
          const int t = tt + j;
          if ((t & 1) == 0) dpair = *reinterpret_cast<const float4 *>(prow + t);
          const float2 dd = (t & 1) ? make_float2(dpair.z, dpair.w) : make_float2(dpair.x, dpair.y);
          float bv[NPL], cv[NPL];
          load_bc<NPL>(Bs + (tt + j) * NS + q * NPL, bv);
          load_bc<NPL>(Cs + (tt + j) * NS + q * NPL, cv);
          if constexpr (NPL % 2 == 0) {
            const float2 dA = make_float2(dd.x, dd.x), dX = make_float2(dd.y, dd.y);
            float2 acc = make_float2(0.f, 0.f);
#pragma unroll
            for (int i = 0; i < NPL; i += 2) {
              const float2 arg = fmul2(dA, make_float2(A2[i], A2[i + 1]));
              const float2 a = make_float2(ex2_approx(arg.x), ex2_approx(arg.y));
              float2 bx = fmul2(dX, make_float2(bv[i], bv[i + 1]));
              if constexpr (ZOH)  // dX holds x: Bbar x = ((e^u - 1) / A) * (B x)
                bx = fmul2(zoh_coef2(fmul2(arg, make_float2(kLn2, kLn2)), a, dA,
                                     make_float2(invA[i], invA[i + 1])),
                           bx);
              const float2 hn = ffma2(a, make_float2(h[i], h[i + 1]), bx);
              h[i] = hn.x;
              h[i + 1] = hn.y;
              acc = ffma2(make_float2(cv[i], cv[i + 1]), hn, acc);
            }
            yp[j] = acc.x + acc.y;
          } else {
            const float arg = dd.x * A2[0];
            const float a = ex2_approx(arg);
            float bx = dd.y * bv[0];
            if constexpr (ZOH) bx *= zoh_coef(arg * kLn2, a, dd.x, invA[0]);
            h[0] = fmaf(a, h[0], bx);
            yp[j] = cv[0] * h[0];
          }
        }
        const float ys = reduce_scatter<LPC>(yp, q);
        const int to = tt + q;  // this lane's own token of the group: prologue slot tt / LPC
        if (to < nvalid && valid_ch)
          yrow[(size_t)to * p.D] = from_f32<OutT>(fmaf(ys, g1[tt / LPC], g2[tt / LPC]));
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&rempty[r]);  // this warp is done with slot r

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
      p.ctl->ticket = 0u;
      p.ctl->epoch = epoch + 1u;
      __threadfence();
    }
  }
}

// ---------------------------------------------------------------------------
// host-side variant table (one translation unit per dtype pair)
// ---------------------------------------------------------------------------

template <typename InT, typename OutT, int NS, int LPC, int WARPS, int TT, bool ZOH>
static cudaError_t run_variant(const LaunchShape *ls, const TmaMaps *maps, const FwdParams *p,
                               cudaStream_t stream, VariantInfo *vi) {
  using Cfg = FwdCfg<InT, OutT, NS, LPC, WARPS, TT>;
  auto kern = fwd_kernel<InT, OutT, NS, LPC, WARPS, TT, ZOH>;
  if (Cfg::SMEM > 227 * 1024) return cudaErrorInvalidValue;
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

template <typename InT, typename OutT, int NS, int LPC, int WARPS, bool ZOH>
static cudaError_t by_tt(const LaunchShape *ls, const TmaMaps *maps, const FwdParams *p,
                         cudaStream_t st, VariantInfo *vi) {
  // a row tile's x / delta / z rows must be whole 16-byte TMA units
  if constexpr ((WARPS * (32 / LPC) * (int)sizeof(InT)) % 16 != 0) {
    return cudaErrorInvalidValue;
  } else {
    switch (ls->tt) {
      case 16:
        if constexpr (!ZOH) return run_variant<InT, OutT, NS, LPC, WARPS, 16, ZOH>(ls, maps, p, st, vi);
        return cudaErrorInvalidValue;
      case 32: return run_variant<InT, OutT, NS, LPC, WARPS, 32, ZOH>(ls, maps, p, st, vi);
      case 64: return run_variant<InT, OutT, NS, LPC, WARPS, 64, ZOH>(ls, maps, p, st, vi);
      default: return cudaErrorInvalidValue;
    }
  }
}

template <typename InT, typename OutT, int NS, int LPC, bool ZOH>
static cudaError_t by_warps(const LaunchShape *ls, const TmaMaps *maps, const FwdParams *p,
                            cudaStream_t st, VariantInfo *vi) {
  switch (ls->warps) {
    case 2: return by_tt<InT, OutT, NS, LPC, 2, ZOH>(ls, maps, p, st, vi);
    case 4: return by_tt<InT, OutT, NS, LPC, 4, ZOH>(ls, maps, p, st, vi);
    case 8: return by_tt<InT, OutT, NS, LPC, 8, ZOH>(ls, maps, p, st, vi);
    default: return cudaErrorInvalidValue;
  }
}

template <typename InT, typename OutT, int NS, bool ZOH>
static cudaError_t by_lpc(const LaunchShape *ls, const TmaMaps *maps, const FwdParams *p,
                          cudaStream_t st, VariantInfo *vi) {
  switch (ls->lpc) {
    case 1: return by_warps<InT, OutT, NS, 1, ZOH>(ls, maps, p, st, vi);
    case 2: return by_warps<InT, OutT, NS, 2, ZOH>(ls, maps, p, st, vi);
    case 4: return by_warps<InT, OutT, NS, 4, ZOH>(ls, maps, p, st, vi);
    case 8:
      if constexpr (NS >= 8) return by_warps<InT, OutT, NS, 8, ZOH>(ls, maps, p, st, vi);
      return cudaErrorInvalidValue;
    case 16:
      if constexpr (NS >= 16) return by_warps<InT, OutT, NS, 16, ZOH>(ls, maps, p, st, vi);
      return cudaErrorInvalidValue;
    default: return cudaErrorInvalidValue;
  }
}

template <typename InT, typename OutT, bool ZOH>
static cudaError_t by_ns_zoh(const LaunchShape *ls, const TmaMaps *maps, const FwdParams *p,
                             cudaStream_t st, VariantInfo *vi) {
  switch (ls->ns) {
    case 4:
      if constexpr (sizeof(InT) == 4) return by_lpc<InT, OutT, 4, ZOH>(ls, maps, p, st, vi);
      return cudaErrorInvalidValue;
    case 8: return by_lpc<InT, OutT, 8, ZOH>(ls, maps, p, st, vi);
    case 16: return by_lpc<InT, OutT, 16, ZOH>(ls, maps, p, st, vi);
    default: return cudaErrorInvalidValue;
  }
}

template <typename InT, typename OutT>
static cudaError_t by_ns(const LaunchShape *ls, const TmaMaps *maps, const FwdParams *p,
                         cudaStream_t st, VariantInfo *vi) {
  if (ls->stages != kStages) return cudaErrorInvalidValue;
  if (p && p->zoh != ls->zoh) return cudaErrorInvalidValue;
  return ls->zoh ? by_ns_zoh<InT, OutT, true>(ls, maps, p, st, vi)
                 : by_ns_zoh<InT, OutT, false>(ls, maps, p, st, vi);
}

// per-dtype entry points (defined in scan_fwd_<dtypes>.cu)
cudaError_t fwd_dispatch_f32(const LaunchShape *, const TmaMaps *, const FwdParams *, cudaStream_t,
                             VariantInfo *);
cudaError_t fwd_dispatch_bf16(const LaunchShape *, const TmaMaps *, const FwdParams *,
                              cudaStream_t, VariantInfo *);
cudaError_t fwd_dispatch_bf16_f32(const LaunchShape *, const TmaMaps *, const FwdParams *,
                                  cudaStream_t, VariantInfo *);

}  // namespace ssm
