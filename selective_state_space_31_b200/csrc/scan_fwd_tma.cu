// scan_fwd_tma.cu -- fused selective-scan forward kernel for sm_100a.
//
// One kernel does everything the pages' "Kernel fusion" section lists after
// the projections: Delta = softplus(delta + bias), discretisation
// Abar = exp(Delta*A), Bbar*x = (Delta*x)*B_t, the recurrence
// h = Abar*h + Bbar*x, the readout C_t.h, the D skip and the silu(z) gate
// ("Selective Scan trong Mamba ...", sections "Selection pha vo convolution
// kernel co dinh", "Vi du Python", "Kernel fusion").  The (B, L, D, N)
// state lives only in registers ("Tai sao chi parallel scan van chua du
// nhanh?"): HBM sees the (B, L, D) inputs/outputs, (B, L, N) B/C and the
// (B, D, N) h0/h_last only.
//
// Work decomposition
//   * A CTA owns DT consecutive channels of one batch element (a "row").
//     Inside the CTA a channel's N states are split over LPC lanes
//     (NPL = N / LPC states per lane); the LPC partial readouts of a token
//     are combined by a shuffle butterfly that leaves lane q holding token q
//     of each group of LPC tokens, and each lane does the per-token work
//     (softplus, gate, skip, store) for its own token only.
//   * A row's timeline is cut into chunks of Tseg tokens.  Work items
//     (row, chunk) are claimed in chunk-major order from an atomic counter by
//     persistent CTAs; the carried state of chunk c is handed to chunk c+1
//     through a small workspace with a release/acquire flag per (row, warp).
//     This is the pages' associative carry ("Scan bien recurrence ...":
//     (A2,b2) (x) (A1,b1) = (A2A1, A2b1+b2)) applied chunk to chunk: the
//     prefix of chunks < c, applied to h0, is exactly the state the next
//     chunk starts from.  With fewer CTAs than rows, a chunk's predecessor
//     is finished before the chunk is claimed, so the wait is normally free;
//     it is bounded by a timer in any case.
//   * Tiles of x / delta / z ([Tt, DT]) and B / C ([Tt, N]) are streamed by
//     TMA (cp.async.bulk.tensor, no multicast) through a STAGES-deep ring of
//     shared-memory slots; y is staged in shared memory and written by a TMA
//     store.  Out-of-range rows/columns of a ragged tail are zero-filled by
//     the TMA unit, and tokens past the end are made identity updates
//     (Delta = 0 => Abar = 1, Bbar*x = 0), so the carried state is exact.
#include "device_common.cuh"
#include "scan_params.h"

namespace ssm {

constexpr int align_up(int v, int a) { return (v + a - 1) / a * a; }

template <typename InT, typename OutT, int NS, int LPC, int WARPS, int TT, int STAGES>
struct FwdCfg {
  static constexpr int NPL = NS / LPC;    // states per lane
  static constexpr int DTW = 32 / LPC;    // channels per warp
  static constexpr int DT = WARPS * DTW;  // channels per CTA
  static constexpr int THREADS = WARPS * 32;
  static constexpr bool BF16_IN = sizeof(InT) == 2;
  static constexpr int XTILE = align_up(TT * DT * (int)sizeof(InT), 128);
  static constexpr int BCTILE = align_up(TT * NS * (int)sizeof(InT), 128);
  static constexpr int SLOT = 3 * XTILE + 2 * BCTILE;
  static constexpr int BCF_BYTES = BF16_IN ? 2 * 2 * TT * NS * 4 : 0;
  static constexpr int YTILE = align_up(TT * DT * (int)sizeof(OutT), 128);
  static constexpr int OFF_BCF = STAGES * SLOT;
  static constexpr int OFF_Y = OFF_BCF + BCF_BYTES;
  static constexpr int OFF_BAR = OFF_Y + 2 * YTILE;
  static constexpr int OFF_META = OFF_BAR + STAGES * 8;
  static constexpr int SMEM = OFF_META + STAGES * 8;
  static_assert(NS % LPC == 0, "LPC must divide N");
  static_assert(TT % LPC == 0, "LPC must divide the stage length");
  static_assert(DT * (int)sizeof(InT) % 16 == 0, "TMA rows need 16-byte multiples");
  static_assert(DT * (int)sizeof(OutT) % 16 == 0, "TMA rows need 16-byte multiples");
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

template <typename InT, typename OutT, int NS, int LPC, int WARPS, int TT, int STAGES>
__global__ void __launch_bounds__(WARPS * 32)
    fwd_tma_kernel(const __grid_constant__ TmaMaps maps, const FwdParams p) {
  using Cfg = FwdCfg<InT, OutT, NS, LPC, WARPS, TT, STAGES>;
  constexpr int NPL = Cfg::NPL, DTW = Cfg::DTW, DT = Cfg::DT;
  extern __shared__ __align__(1024) unsigned char smem[];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c_loc = lane / LPC;            // channel within the warp
  const int q = lane % LPC;                // state group of this lane
  const int ch = warp * DTW + c_loc;       // channel within the CTA tile
  const int lane_base = c_loc * LPC;

  float *bcf = reinterpret_cast<float *>(smem + Cfg::OFF_BCF);
  OutT *ytile = reinterpret_cast<OutT *>(smem + Cfg::OFF_Y);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::OFF_BAR);
  int *meta = reinterpret_cast<int *>(smem + Cfg::OFF_META);

  const unsigned int epoch = *reinterpret_cast<volatile unsigned int *>(&p.ctl->epoch);
  const uint32_t tx_bytes = (p.has_z ? 3 : 2) * TT * DT * sizeof(InT) + 2 * TT * NS * sizeof(InT);

  // ---- issuer state (thread 0 only) ----
  long long iss_item = 0;
  int iss_st = 0, iss_nst = 0;
  bool iss_done = false;
  long long iss_g = 0;  // next global stage to issue

  auto stages_of = [&](long long item) -> int {
    const int seg = (int)(item / p.rows);
    const int len = min(p.Tseg, p.L - seg * p.Tseg);
    return (len + TT - 1) / TT;
  };
  auto claim = [&]() {
    const unsigned long long it = atomicAdd(&p.ctl->tile, 1ULL);
    if (it >= (unsigned long long)p.total_items) {
      iss_done = true;
      return;
    }
    iss_item = (long long)it;
    iss_st = 0;
    iss_nst = stages_of(iss_item);
  };
  auto issue = [&]() {  // issue global stage iss_g into slot iss_g % STAGES
    const int s = (int)(iss_g % STAGES);
    ++iss_g;
    if (iss_done) {
      meta[2 * s] = -1;
      meta[2 * s + 1] = 0;
      mbar_arrive(&bars[s]);
      return;
    }
    const int row = (int)(iss_item % p.rows), seg = (int)(iss_item / p.rows);
    const int b = row / p.nDT, d0 = (row % p.nDT) * DT;
    const int t0 = seg * p.Tseg + iss_st * TT;
    meta[2 * s] = (int)iss_item;
    meta[2 * s + 1] = iss_st;
    unsigned char *sb = smem + s * Cfg::SLOT;
    mbar_arrive_expect_tx(&bars[s], tx_bytes);
    tma_load_3d(sb, &maps.x, &bars[s], d0, t0, b);
    tma_load_3d(sb + Cfg::XTILE, &maps.dt, &bars[s], d0, t0, b);
    if (p.has_z) tma_load_3d(sb + 2 * Cfg::XTILE, &maps.z, &bars[s], d0, t0, b);
    tma_load_3d(sb + 3 * Cfg::XTILE, &maps.B, &bars[s], 0, t0, b);
    tma_load_3d(sb + 3 * Cfg::XTILE + Cfg::BCTILE, &maps.C, &bars[s], 0, t0, b);
    if (++iss_st == iss_nst) claim();
  };

  if (tid == 0) {
#pragma unroll
    for (int i = 0; i < STAGES; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (tid == 0) {
    claim();
    for (int i = 0; i < STAGES - 1; ++i) issue();
  }

  // ---- per-row registers ----
  float h[NPL], A2[NPL];
#pragma unroll
  for (int n = 0; n < NPL; ++n) { h[n] = 0.f; A2[n] = 0.f; }
  float Dd = 0.f, bias = 0.f;
  // coordinates of the previous stage's y tile (thread 0 stores it)
  int prev_d0 = 0, prev_t0 = 0, prev_b = 0;
  bool have_prev = false, aborted = false;

  long long g = 0;
  for (;; ++g) {
    const int s = (int)(g % STAGES);
    const uint32_t par = (uint32_t)((g / STAGES) & 1);
    const bool ok = mbar_wait_bounded(&bars[s], par, p.timeout_ns);
    const int item = meta[2 * s], st = meta[2 * s + 1];
    if constexpr (Cfg::BF16_IN) {
      if (ok && item >= 0) {  // B/C of this stage -> fp32, shared by all channels
        const __nv_bfloat162 *src =
            reinterpret_cast<const __nv_bfloat162 *>(smem + s * Cfg::SLOT + 3 * Cfg::XTILE);
        float2 *dst = reinterpret_cast<float2 *>(bcf + (g & 1) * 2 * TT * NS);
        static_assert(Cfg::BCTILE == TT * NS * 2, "B and C tiles must be contiguous");
        for (int i = tid; i < TT * NS; i += Cfg::THREADS) dst[i] = __bfloat1622float2(src[i]);
      }
    }
    // One barrier per stage: (a) converted B/C visible, (b) every warp has
    // finished stage g-1, so its slot and y tile may be reused.
    if (__syncthreads_or(!ok)) {
      aborted = true;
      break;
    }
    if (item < 0) break;

    const int row = item % p.rows, seg = item / p.rows;
    const int b = row / p.nDT, d0 = (row % p.nDT) * DT;
    const int t0 = seg * p.Tseg + st * TT;
    const int nst = stages_of(item);

    if (tid == 0) {
      if (have_prev) {
        tma_store_3d(&maps.y, ytile + ((g - 1) & 1) * (Cfg::YTILE / sizeof(OutT)), prev_d0,
                     prev_t0, prev_b);
        bulk_commit();
      }
      issue();  // global stage g + STAGES - 1 into the slot stage g-1 used
      prev_d0 = d0; prev_t0 = t0; prev_b = b;
      have_prev = true;
    }

    const int d = d0 + ch;
    const bool valid_ch = d < p.D;
    if (st == 0) {  // first stage of a work item: parameters and carried state
#pragma unroll
      for (int n = 0; n < NPL; ++n)
        A2[n] = valid_ch ? __ldg(p.A + (size_t)d * NS + q * NPL + n) * kLog2e : 0.f;
      Dd = (p.has_D && valid_ch) ? __ldg(p.Dv + d) : 0.f;
      bias = (p.has_bias && valid_ch) ? __ldg(p.bias + d) : 0.f;
      if (seg == 0) {
#pragma unroll
        for (int n = 0; n < NPL; ++n)
          h[n] = (p.has_h0 && valid_ch) ? __ldg(p.h0 + ((size_t)b * p.D + d) * NS + q * NPL + n)
                                        : 0.f;
      } else {
        const unsigned long long want = ((unsigned long long)epoch << 32) | (unsigned)seg;
        unsigned long long *flag = p.ws_flags + (size_t)row * WARPS + warp;
        bool got = ld_acquire_u64(flag) == want;
        if (!got) {
          const uint64_t tstart = globaltimer_ns();
          while (true) {
            __nanosleep(100);
            if (ld_acquire_u64(flag) == want) { got = true; break; }
            if (globaltimer_ns() - tstart > p.timeout_ns) break;
          }
        }
        if (!__all_sync(FULL_MASK, got) && lane == 0) atomicCAS(&p.ctl->status, 0, kStatusTimeout);
        const float *src = p.ws_state + ((size_t)row * DT + ch) * NS + q * NPL;
#pragma unroll
        for (int n = 0; n < NPL; ++n) h[n] = __ldcg(src + n);
      }
    }

    // ---- the stage: TT tokens of DT channels ----
    const unsigned char *sb = smem + s * Cfg::SLOT;
    const InT *xs = reinterpret_cast<const InT *>(sb);
    const InT *ds = reinterpret_cast<const InT *>(sb + Cfg::XTILE);
    const InT *zs = reinterpret_cast<const InT *>(sb + 2 * Cfg::XTILE);
    const float *Bf, *Cf;
    if constexpr (Cfg::BF16_IN) {
      Bf = bcf + (g & 1) * 2 * TT * NS;
      Cf = Bf + TT * NS;
    } else {
      Bf = reinterpret_cast<const float *>(sb + 3 * Cfg::XTILE);
      Cf = reinterpret_cast<const float *>(sb + 3 * Cfg::XTILE + Cfg::BCTILE);
    }
    OutT *yt = ytile + (g & 1) * (Cfg::YTILE / sizeof(OutT));
    const int nvalid = min(TT, p.L - t0);

#pragma unroll 2
    for (int tt = 0; tt < TT; tt += LPC) {
      const int to = tt + q;  // this lane's own token
      const float xo = to_f32(xs[to * DT + ch]);
      const float v = to_f32(ds[to * DT + ch]) + bias;
      float dlt = p.softplus ? softplus_f(v) : v;
      dlt = (to < nvalid) ? dlt : 0.f;  // past the end: identity update
      const float dtx = dlt * xo;
      float yp[LPC];
#pragma unroll
      for (int j = 0; j < LPC; ++j) {
        const float dj = (LPC == 1) ? dlt : __shfl_sync(FULL_MASK, dlt, lane_base + j);
        const float dxj = (LPC == 1) ? dtx : __shfl_sync(FULL_MASK, dtx, lane_base + j);
        float bv[NPL], cv[NPL];
        load_vec<NPL>(Bf + (tt + j) * NS + q * NPL, bv);
        load_vec<NPL>(Cf + (tt + j) * NS + q * NPL, cv);
        float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
        for (int n = 0; n < NPL; ++n) {
          const float a = ex2_approx(dj * A2[n]);
          h[n] = fmaf(a, h[n], dxj * bv[n]);
          if (n & 1) acc1 = fmaf(cv[n], h[n], acc1);
          else acc0 = fmaf(cv[n], h[n], acc0);
        }
        yp[j] = acc0 + acc1;
      }
      const float ys = reduce_scatter<LPC>(yp, q);
      float yv = fmaf(Dd, xo, ys);
      if (p.has_z) yv *= silu_f(to_f32(zs[to * DT + ch]));
      yt[to * DT + ch] = from_f32<OutT>(yv);
    }
    fence_proxy_async_smem();  // y tile -> visible to the TMA store
    if (tid == 0) bulk_wait_read<0>();  // the store issued this stage has read its tile

    if (st == nst - 1) {  // last stage of the work item: hand the state on
      if (seg == p.nseg - 1) {
        if (p.want_hlast && valid_ch) {
          float *dst = p.h_last + ((size_t)b * p.D + d) * NS + q * NPL;
#pragma unroll
          for (int n = 0; n < NPL; ++n) dst[n] = h[n];
        }
      } else if (item != p.drop_item) {
        float *dst = p.ws_state + ((size_t)row * DT + ch) * NS + q * NPL;
#pragma unroll
        for (int n = 0; n < NPL; ++n) __stcg(dst + n, h[n]);
        __threadfence();
        __syncwarp();
        if (lane == 0)
          st_release_u64(p.ws_flags + (size_t)row * WARPS + warp,
                         ((unsigned long long)epoch << 32) | (unsigned)(seg + 1));
      }
    }
  }

  __syncthreads();
  if (tid == 0) {
    if (aborted) {
      atomicCAS(&p.ctl->status, 0, kStatusTimeout);
      // wait (bounded) for loads still in flight into this CTA's slots
      for (long long k = g; k < iss_g; ++k)
        (void)mbar_wait_bounded(&bars[k % STAGES], (uint32_t)((k / STAGES) & 1), p.timeout_ns);
    } else if (have_prev) {
      tma_store_3d(&maps.y, ytile + ((g - 1) & 1) * (Cfg::YTILE / sizeof(OutT)), prev_d0,
                   prev_t0, prev_b);
      bulk_commit();
    }
    bulk_wait<0>();
    __threadfence();
    const unsigned int prev = atomicAdd(&p.ctl->done, 1u);
    if (prev == gridDim.x - 1) {  // last CTA of this launch: reset for the next call
      p.ctl->tile = 0ULL;
      p.ctl->done = 0u;
      p.ctl->epoch = epoch + 1u;
      __threadfence();
    }
  }
}

// ---------------------------------------------------------------------------
// host-side variant table
// ---------------------------------------------------------------------------

constexpr int kTT = 64;
constexpr int kStages = 3;

template <typename InT, typename OutT, int NS, int LPC, int WARPS>
static cudaError_t run_variant(const LaunchShape *ls, const TmaMaps *maps, const FwdParams *p,
                               cudaStream_t stream, size_t *smem_out, int *occ_out) {
  using Cfg = FwdCfg<InT, OutT, NS, LPC, WARPS, kTT, kStages>;
  auto kern = fwd_tma_kernel<InT, OutT, NS, LPC, WARPS, kTT, kStages>;
  if (Cfg::SMEM > 227 * 1024) return cudaErrorInvalidValue;  // does not fit one SM
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
  if (e != cudaSuccess) {
    cudaGetLastError();  // clear, so a later launch check does not see it
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

template <typename InT, typename OutT, int NS, int LPC>
static cudaError_t by_warps(const LaunchShape *ls, const TmaMaps *maps, const FwdParams *p,
                            cudaStream_t st, size_t *sm, int *oc) {
  switch (ls->warps) {
    case 2: return run_variant<InT, OutT, NS, LPC, 2>(ls, maps, p, st, sm, oc);
    case 4: return run_variant<InT, OutT, NS, LPC, 4>(ls, maps, p, st, sm, oc);
    case 8: return run_variant<InT, OutT, NS, LPC, 8>(ls, maps, p, st, sm, oc);
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
  switch (ls->ns) {
    case 4:
      if constexpr (sizeof(InT) == 4) return by_lpc<InT, OutT, 4>(ls, maps, p, st, sm, oc);
      return cudaErrorInvalidValue;
    case 8: return by_lpc<InT, OutT, 8>(ls, maps, p, st, sm, oc);
    case 16: return by_lpc<InT, OutT, 16>(ls, maps, p, st, sm, oc);
    default: return cudaErrorInvalidValue;
  }
}

static cudaError_t dispatch(int in_dtype, int out_dtype, const LaunchShape *ls,
                            const TmaMaps *maps, const FwdParams *p, cudaStream_t st,
                            size_t *sm, int *oc) {
  if (ls->tt != kTT || ls->stages != kStages) return cudaErrorInvalidValue;
  if (in_dtype == 0 && out_dtype == 0) return by_ns<float, float>(ls, maps, p, st, sm, oc);
  if (in_dtype == 1 && out_dtype == 1)
    return by_ns<__nv_bfloat16, __nv_bfloat16>(ls, maps, p, st, sm, oc);
  if (in_dtype == 1 && out_dtype == 0) return by_ns<__nv_bfloat16, float>(ls, maps, p, st, sm, oc);
  return cudaErrorInvalidValue;
}

cudaError_t launch_fwd_tma(int in_dtype, int out_dtype, const LaunchShape &ls,
                           const TmaMaps &maps, const FwdParams &p, cudaStream_t stream) {
  return dispatch(in_dtype, out_dtype, &ls, &maps, &p, stream, nullptr, nullptr);
}

cudaError_t fwd_tma_smem_and_occupancy(int in_dtype, int out_dtype, const LaunchShape &ls,
                                       size_t *smem, int *blocks_per_sm) {
  return dispatch(in_dtype, out_dtype, &ls, nullptr, nullptr, nullptr, smem, blocks_per_sm);
}

}  // namespace ssm
