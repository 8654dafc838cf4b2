// scan_fwd_dispatch.cu -- dtype dispatch of the fused forward kernel and the
// choice of its launch shape.
#include <algorithm>

#include "scan_fwd_kernel.cuh"

namespace ssm {

static cudaError_t dispatch(int in_dtype, int out_dtype, const LaunchShape *ls,
                            const TmaMaps *maps, const FwdParams *p, cudaStream_t st,
                            VariantInfo *vi) {
  if (in_dtype == 0 && out_dtype == 0) return fwd_dispatch_f32(ls, maps, p, st, vi);
  if (in_dtype == 1 && out_dtype == 1) return fwd_dispatch_bf16(ls, maps, p, st, vi);
  if (in_dtype == 1 && out_dtype == 0) return fwd_dispatch_bf16_f32(ls, maps, p, st, vi);
  return cudaErrorInvalidValue;
}

cudaError_t launch_fwd_tma(int in_dtype, int out_dtype, const LaunchShape &ls,
                           const TmaMaps &maps, const FwdParams &p, cudaStream_t stream) {
  return dispatch(in_dtype, out_dtype, &ls, &maps, &p, stream, nullptr);
}

cudaError_t fwd_variant_info(int in_dtype, int out_dtype, const LaunchShape &ls,
                             VariantInfo *vi) {
  return dispatch(in_dtype, out_dtype, &ls, nullptr, nullptr, nullptr, vi);
}

namespace {

// Relative throughput of the variants at equal busy warps per SM, measured on
// B200 (bf16 layer workloads).  Splitting a channel over 4 lanes balances the
// per-lane B / C loads against the shuffle readout best; longer stages
// amortise the per-stage waits but raise register pressure when a lane
// prepares many tokens (TT / LPC); 2-warp CTAs pay the load warp and barrier
// traffic of twice as many CTAs.
double shape_weight(int lpc, int tt) {
  const int i = tt == 16 ? 0 : tt == 32 ? 1 : 2;
  static const double w1[3] = {0.45, 0.45, 0.42}, w2[3] = {0.68, 0.75, 0.7},
                      w4[3] = {0.9, 1.0, 0.92}, w8[3] = {0.8, 0.9, 0.97},
                      w16[3] = {0.5, 0.6, 0.68};
  switch (lpc) {
    case 1: return w1[i];
    case 2: return w2[i];
    case 4: return w4[i];
    case 8: return w8[i];
    default: return w16[i];
  }
}
double warps_weight(int warps) { return warps == 2 ? 0.8 : 1.0; }

// Parts per row for P CTAs over R rows of S stages: the fewest parts that
// keep every CTA within ~5% of the mean item count (P <= R).
int parts_per_row(int64_t R, int64_t P, int64_t S) {
  if (P >= R) return 1;
  int best_m = 1;
  double best_bal = 0.0;
  for (int m = 1; m <= 64 && m <= S; ++m) {
    const int64_t items = R * m;
    const double bal = ((double)items / P) / (double)((items + P - 1) / P);
    if (bal > best_bal + 1e-9) { best_bal = bal; best_m = m; }
    if (bal >= 0.95) return m;
  }
  return best_m;
}

}  // namespace

// Rows (batch x channel tiles) are the only independent chains, so at most
// `rows` CTAs can be busy: grid P <= min(rows, CTAs resident on the device),
// taken as a multiple of the SM count when that scores better (every SM then
// gets the same work).  Score = busy scan warps per SM (saturating at 12) x
// balance of CTAs over SMs x the measured weights above.  Ties go to fewer
// warps per CTA (more, smaller CTAs measured faster at equal warps per SM).
cudaError_t choose_fwd_shape(int in_dtype, int out_dtype, int64_t batch, int64_t seqlen,
                             int64_t dim, int ns, bool zoh, int sms, const FwdOverrides &o,
                             FwdShape *out) {
  const int ei = in_dtype == 1 ? 2 : 4, eo = out_dtype == 1 ? 2 : 4;
  bool found = false;
  double best_score = -1.0;
  FwdShape best{};
  for (int lpc : {1, 2, 4, 8, 16}) {
    if (lpc > ns || (o.lpc && lpc != o.lpc)) continue;
    for (int warps : {2, 4, 8}) {
      if (o.warps && warps != o.warps) continue;
      for (int tt : {32, 64, 16}) {
        if ((o.tt && tt != o.tt) || (zoh && tt == 16)) continue;
        const int DT = warps * 32 / lpc;
        if ((DT * ei) % 16 || (DT * eo) % 16) continue;
        LaunchShape ls{lpc, warps, tt, kStages, ns, 0, 0, zoh};
        VariantInfo vi{};
        if (fwd_variant_info(in_dtype, out_dtype, ls, &vi) != cudaSuccess || vi.occ < 1) {
          cudaGetLastError();
          continue;
        }
        const int64_t rows = batch * ((dim + DT - 1) / DT);
        const int64_t cap = std::min<int64_t>(rows, (int64_t)vi.occ * sms);
        const int64_t balanced = cap >= sms ? cap / sms * sms : cap;
        const double w = shape_weight(lpc, tt) * warps_weight(warps);
        auto score_of = [&](int64_t g) {
          const int64_t per_sm = (g + sms - 1) / sms;  // CTAs on the busiest SM
          const double busy = (double)g * warps / sms;
          const double balance = (double)g / (double)(per_sm * sms);
          return std::min(busy, 12.0) / 12.0 * balance * w - 1e-3 * warps;
        };
        int64_t grid = score_of(balanced) >= score_of(cap) ? balanced : cap;
        if (o.grid > 0) grid = std::min<int64_t>(o.grid, (int64_t)vi.occ * sms);
        const double score = score_of(grid);
        if (!found || score > best_score) {
          found = true;
          best_score = score;
          best = FwdShape{ls, DT, rows, 0, 0, 0, 0};
          best.ls.grid = (int)grid;
          best.ls.smem = vi.smem;
          best.ring = vi.ring;
        }
      }
    }
  }
  if (!found) return cudaErrorInvalidValue;
  const int64_t S = (seqlen + best.ls.tt - 1) / best.ls.tt;
  const int m0 = parts_per_row(best.rows, best.ls.grid, S);
  const int64_t PL = (S + m0 - 1) / m0;
  const int64_t m = (S + PL - 1) / PL;
  if (best.rows * S > INT32_MAX || best.rows * m > INT32_MAX) return cudaErrorInvalidValue;
  best.S = (int)S;
  best.PL = (int)PL;
  best.parts = (int)m;
  best.ls.grid = (int)std::max<int64_t>(1, std::min<int64_t>(best.ls.grid, best.rows * m));
  *out = best;
  return cudaSuccess;
}

}  // namespace ssm
