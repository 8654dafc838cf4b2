// scan_fwd_dispatch.cu -- dtype dispatch of the fused forward kernel and the
// choice of its launch shape (lanes per channel, channels per lane, warps,
// stage length, segments, grid).
#include <algorithm>
#include <cmath>

#include "scan_fwd_kernel.cuh"

namespace ssm {

// variant tables (scan_fwd_<dtypes>_<part>.cu)
#define SSM_TABLE(tag)                                                                 \
  cudaError_t fwd_table_##tag(const LaunchShape *, const TmaMaps *, const FwdParams *, \
                              cudaStream_t, VariantInfo *);                            \
  int fwd_list_##tag(VariantDesc *, int);
SSM_TABLE(bf16_a)
SSM_TABLE(bf16_b)
SSM_TABLE(bf16_c)
SSM_TABLE(bf16_conv)
SSM_TABLE(bf16_f32)
SSM_TABLE(f32_a)
SSM_TABLE(f32_b)
SSM_TABLE(f32_conv)
#undef SSM_TABLE

namespace {

using TableFn = cudaError_t (*)(const LaunchShape *, const TmaMaps *, const FwdParams *,
                                cudaStream_t, VariantInfo *);
using ListFn = int (*)(VariantDesc *, int);

struct Tables {
  const TableFn *run;
  const ListFn *list;
  int n;
};

Tables tables_for(int in_dtype, int out_dtype) {
  static const TableFn bf16_run[] = {fwd_table_bf16_a, fwd_table_bf16_b, fwd_table_bf16_c,
                                     fwd_table_bf16_conv};
  static const ListFn bf16_list[] = {fwd_list_bf16_a, fwd_list_bf16_b, fwd_list_bf16_c,
                                     fwd_list_bf16_conv};
  static const TableFn bf16f_run[] = {fwd_table_bf16_f32};
  static const ListFn bf16f_list[] = {fwd_list_bf16_f32};
  static const TableFn f32_run[] = {fwd_table_f32_a, fwd_table_f32_b, fwd_table_f32_conv};
  static const ListFn f32_list[] = {fwd_list_f32_a, fwd_list_f32_b, fwd_list_f32_conv};
  if (in_dtype == 1 && out_dtype == 1) return {bf16_run, bf16_list, 4};
  if (in_dtype == 1 && out_dtype == 0) return {bf16f_run, bf16f_list, 1};
  if (in_dtype == 0 && out_dtype == 0) return {f32_run, f32_list, 3};
  return {nullptr, nullptr, 0};
}

cudaError_t dispatch(int in_dtype, int out_dtype, const LaunchShape *ls, const TmaMaps *maps,
                     const FwdParams *p, cudaStream_t st, VariantInfo *vi) {
  if (ls->stages != kStages) return cudaErrorInvalidValue;
  if (p && (p->zoh != ls->zoh)) return cudaErrorInvalidValue;
  const Tables t = tables_for(in_dtype, out_dtype);
  for (int i = 0; i < t.n; ++i) {
    const cudaError_t e = t.run[i](ls, maps, p, st, vi);
    if (e != cudaErrorNotSupported) return e;
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_fwd_tma(int in_dtype, int out_dtype, const LaunchShape &ls,
                           const TmaMaps &maps, const FwdParams &p, cudaStream_t stream) {
  return dispatch(in_dtype, out_dtype, &ls, &maps, &p, stream, nullptr);
}

cudaError_t fwd_variant_info(int in_dtype, int out_dtype, const LaunchShape &ls,
                             VariantInfo *vi) {
  return dispatch(in_dtype, out_dtype, &ls, nullptr, nullptr, nullptr, vi);
}

int fwd_variants(int in_dtype, int out_dtype, VariantDesc *out, int max) {
  const Tables t = tables_for(in_dtype, out_dtype);
  int n = 0;
  for (int i = 0; i < t.n; ++i) {
    const int room = std::max(0, max - n);
    n += t.list[i](out ? out + std::min(n, max) : nullptr, out ? room : 0);
  }
  return n;
}

namespace {

// Relative throughput of the variants at equal busy warps per SM on B200
// (bf16 layer workloads).  One channel per lane: splitting a channel over 4
// lanes balances the per-lane B / C loads against the shuffle readout best;
// longer stages amortise the per-stage waits but raise register pressure.
// Two channels per lane load and widen each B / C value once for both
// (fewer instructions per update) but halve the lanes; measured on B200 they
// run at about the speed of one channel per lane with the same warps busy.
double shape_weight(int lpc, int kc, int tt) {
  const int i = tt == 16 ? 0 : tt == 32 ? 1 : 2;
  if (kc == 2) {
    static const double v2[3] = {0.6, 0.65, 0.6}, v4[3] = {0.8, 0.85, 0.8},
                        v8[3] = {0.9, 0.95, 0.95};
    return lpc == 2 ? v2[i] : lpc == 4 ? v4[i] : v8[i];
  }
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

// The software-pipelined loop (bit 0) and the five-CTA register cap (bit 1)
// relative to the plain variant, measured on B200: with 8 lanes per channel
// and 64-token stages the pipelined loop gains 3-5 % on the layer shapes;
// elsewhere, and with segments, the plain loop was as fast or faster.  B and
// C widened by the load warp (bit 2) took 2-10 % longer on every workload
// (wider slots cost a CTA per SM at 64-token stages; at equal occupancy the
// removed widening did not shorten the latency-bound loop).  A quarter of
// the exponentials on the FMA pipe (bit 3) took 4-27 % longer, in the carry
// pass too although its special-function pipe is the busiest (82 %): the
// polynomial's eight instructions per exponential cost more issue than the
// relief is worth.  Preparing two tokens ahead in the pipelined loop (bit 4)
// gained a further 3.7 % on the 130M layer and 1.4 % on the 1.4B layer
// (three or four tokens ahead under a four-CTA register cap gained less:
// 2.6 / 1.4 % and 0.6 / -0.6 %); on the long sequence's segmented 4-lane,
// 32-token scan every pipelined form was slower than the plain loop.
double opt_weight(int opt, int lpc, int tt, int segments) {
  if (opt == 0) return 1.0;
  if (opt & 4) return 0.9;
  if (opt & 8) return 0.9;
  if (segments > 1 || lpc != 8 || tt != 64) return 0.97;
  return opt == 17 ? 1.08 : opt == 1 ? 1.05 : opt == 2 ? 1.04 : 1.03;
}
// With segments, the 131k-token rows favoured 4 lanes x 32-token stages over
// 8 lanes x 64-token stages by about 10 % more than the layer shapes do.
double segmented_weight(int lpc, int tt, int segments) {
  return segments > 1 && lpc == 8 && tt == 64 ? 0.93 : 1.0;
}

// Cost of the carry pass per state update it covers, relative to the fused
// scan's (one exponential and the state update, no readout or gate).
constexpr double kCarryCost = 0.6;
// Busy scan warps per SM beyond which more do not help.
constexpr double kWarpsSaturate = 12.0;

// Parts per segment for P CTAs over R independent chains of S stages: the
// fewest parts that keep every CTA within ~5% of the mean item count.
int parts_per_chain(int64_t R, int64_t P, int64_t S) {
  // more CTAs than chains (an explicit grid): enough parts for every CTA
  if (P >= R) return (int)std::max<int64_t>(1, std::min<int64_t>(S, (P + R - 1) / R));
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

// The carry pass for a main variant: same dstate, stage length, zero-order
// hold and conv flags.  Measured on B200 (131k-token rows, 8 segments): the
// carry pass in the main variant's own lane split ran its exponentials at
// ~76 % of the special-function rate, while one lane per channel (few warps
// per SM) took 45 % longer.  So: the main variant's split and its B/C
// widening option first, then 4 lanes per channel.  o_lpc / o_opt (1 + the
// OPT bits) / o_kc restrict the choice when non-zero.
bool pick_carry(int in_dtype, int out_dtype, const VariantDesc &main, int sms,
                const VariantDesc *all, int nall, int o_lpc, int o_opt, int o_kc,
                LaunchShape *cls, int *cDT, int *cocc) {
  int best = -1;
  double best_score = -1.0;
  for (int i = 0; i < nall; ++i) {
    const VariantDesc &v = all[i];
    if (!v.carry || v.ns != main.ns || v.zoh != main.zoh || v.tt != main.tt ||
        v.conv != main.conv || (o_lpc && v.lpc != o_lpc) || (o_opt && v.opt != o_opt - 1) ||
        (o_kc && v.kc != o_kc))
      continue;
    const double score = (v.lpc == main.lpc && v.kc == main.kc ? 2.0 : 0.0) +
                         ((v.opt & 4) == (main.opt & 4) ? 1.0 : 0.0) +
                         (v.kc == 2 ? 0.5 : 0.0) + (v.lpc == 4 ? 0.25 : 0.0);
    if (score > best_score) { best_score = score; best = i; }
  }
  if (best < 0) return false;
  const VariantDesc &v = all[best];
  LaunchShape ls{v.lpc, v.warps, v.tt, kStages, v.ns, 0, 0, v.zoh};
  ls.kc = v.kc;
  ls.carry = true;
  ls.conv = v.conv;
  ls.opt = v.opt;
  VariantInfo vi{};
  if (fwd_variant_info(in_dtype, out_dtype, ls, &vi) != cudaSuccess || vi.occ < 1) {
    cudaGetLastError();
    return false;
  }
  ls.smem = vi.smem;
  ls.grid = vi.occ * sms;
  *cls = ls;
  *cDT = v.warps * (32 / v.lpc) * v.kc;
  *cocc = vi.occ;
  return true;
}

}  // namespace

// Score = busy scan warps per SM (saturating) x balance of work over the
// SMs x the measured variant weight / (1 + carry-pass cost).  Segments
// multiply the independent chains of a row (and so the busy warps) at the
// price of the carry pass over the earlier segments' tokens.  Ties go to
// fewer warps per CTA.
cudaError_t choose_fwd_shape(int in_dtype, int out_dtype, int64_t batch, int64_t seqlen,
                             int64_t dim, int ns, bool zoh, bool conv, int sms,
                             const FwdOverrides &o, FwdShape *out) {
  const int ei = in_dtype == 1 ? 2 : 4, eo = out_dtype == 1 ? 2 : 4;
  constexpr int kMaxVariants = 256;
  VariantDesc all[kMaxVariants];
  const int nall = std::min(kMaxVariants, fwd_variants(in_dtype, out_dtype, all, kMaxVariants));
  bool found = false;
  double best_score = -1.0;
  FwdShape best{};
  for (int vi_ = 0; vi_ < nall; ++vi_) {
    const VariantDesc &v = all[vi_];
    if (v.carry || v.ns != ns || v.zoh != zoh || v.conv != conv) continue;
    if ((o.lpc && v.lpc != o.lpc) || (o.warps && v.warps != o.warps) ||
        (o.tt && v.tt != o.tt) || (o.kc && v.kc != o.kc) || (o.opt && v.opt != o.opt - 1))
      continue;
    const int DT = v.warps * (32 / v.lpc) * v.kc;
    if ((DT * ei) % 16 || (DT * eo) % 16) continue;
    if (v.kc == 2 && dim % 2) continue;
    LaunchShape ls{v.lpc, v.warps, v.tt, kStages, ns, 0, 0, zoh};
    ls.kc = v.kc;
    ls.conv = conv;
    ls.opt = v.opt;
    VariantInfo info{};
    if (fwd_variant_info(in_dtype, out_dtype, ls, &info) != cudaSuccess || info.occ < 1) {
      cudaGetLastError();
      continue;
    }
    const int64_t rows = batch * ((dim + DT - 1) / DT);
    const int64_t S = std::max<int64_t>(1, (seqlen + v.tt - 1) / v.tt);
    for (int M : {1, 2, 4, 8, 16}) {
      if (o.segments && M != o.segments) continue;
      const double w = shape_weight(v.lpc, v.kc, v.tt) * warps_weight(v.warps) *
                       opt_weight(v.opt, v.lpc, v.tt, M) * segmented_weight(v.lpc, v.tt, M);
      if (M > 1 && S < 4 * M) continue;  // each segment keeps a few stages
      LaunchShape cls{};
      int cDT = 0, cocc = 0;
      if (M > 1 && !pick_carry(in_dtype, out_dtype, v, sms, all, nall, o.carry_lpc, o.carry_opt,
                               o.carry_kc, &cls, &cDT, &cocc))
        continue;
      const int64_t vrows = rows * M;
      const int64_t cap = std::min(vrows, (int64_t)info.occ * sms);
      const int64_t balanced = cap >= sms ? cap / sms * sms : cap;
      auto score_of = [&](int64_t g) {
        const int64_t per_sm = (g + sms - 1) / sms;  // CTAs on the busiest SM
        const double busy = (double)g * v.warps / sms;
        const double balance = (double)g / (double)(per_sm * sms);
        const double carry = M > 1 ? kCarryCost * (double)(M - 1) / M : 0.0;
        return std::min(busy, kWarpsSaturate) / kWarpsSaturate * balance * w / (1.0 + carry) -
               1e-3 * v.warps - 1e-4 * M;
      };
      int64_t grid = score_of(balanced) >= score_of(cap) ? balanced : cap;
      // an explicit grid is taken as is (the ticket schedule needs no
      // co-residency); it is capped by the number of items below
      if (o.grid > 0) grid = o.grid;
      const double score = score_of(grid);
      if (!found || score > best_score) {
        found = true;
        best_score = score;
        best = FwdShape{};
        best.ls = ls;
        best.ls.grid = (int)grid;
        best.ls.smem = info.smem;
        best.DT = DT;
        best.rows = rows;
        best.S = (int)S;
        best.M = M;
        best.ring = info.ring;
        best.cls = cls;
        best.cDT = cDT;
      }
    }
  }
  if (!found) return cudaErrorInvalidValue;
  const int64_t S = best.S;
  int M = best.M;
  int64_t SPS = S;
  if (M > 1) {
    // carry sub-chunks of Q stages; segments are whole numbers of sub-chunks
    // and every segment but the last is full
    const int64_t Q = std::max<int64_t>(1, std::min<int64_t>(2048 / best.ls.tt, S / (4 * M)));
    SPS = (S + M - 1) / M;
    SPS = (SPS + Q - 1) / Q * Q;
    M = (int)((S + SPS - 1) / SPS);
    best.Q = (int)Q;
    best.nq = (int)(SPS / Q);
    best.crows = batch * ((dim + best.cDT - 1) / best.cDT);
    const int64_t citems = best.crows * (int64_t)(M - 1) * best.nq;
    if (citems > INT32_MAX) return cudaErrorInvalidValue;
    best.cls.grid = (int)std::max<int64_t>(1, std::min<int64_t>(best.cls.grid, citems));
  }
  if (M <= 1) {
    M = 1;
    SPS = S;
    best.Q = 0;
    best.nq = 0;
    best.crows = 0;
  }
  best.M = M;
  best.SPS = (int)SPS;
  const int64_t vrows = best.rows * M;
  const int m0 = parts_per_chain(vrows, best.ls.grid, SPS);
  const int64_t PL = (SPS + m0 - 1) / m0;
  const int64_t m = (SPS + PL - 1) / PL;
  if (vrows * S > INT32_MAX || vrows * m > INT32_MAX) return cudaErrorInvalidValue;
  best.PL = (int)PL;
  best.parts = (int)m;
  best.ls.grid = (int)std::max<int64_t>(1, std::min<int64_t>(best.ls.grid, vrows * m));
  *out = best;
  return cudaSuccess;
}

cudaError_t choose_map_shape(int in_dtype, int out_dtype, int64_t batch, int64_t dim,
                             const FwdShape &fs, int sms, MapShape *out) {
  constexpr int kMaxVariants = 256;
  VariantDesc all[kMaxVariants];
  const int nall = std::min(kMaxVariants, fwd_variants(in_dtype, out_dtype, all, kMaxVariants));
  const VariantDesc main{fs.ls.ns, fs.ls.lpc, fs.ls.kc, fs.ls.warps, fs.ls.tt, fs.ls.zoh, false,
                         fs.ls.conv, fs.ls.opt};
  LaunchShape cls{};
  int cDT = 0, cocc = 0;
  if (!pick_carry(in_dtype, out_dtype, main, sms, all, nall, 0, 0, 0, &cls, &cDT, &cocc))
    return cudaErrorInvalidValue;
  const int64_t rows = batch * ((dim + cDT - 1) / cDT);
  const int64_t S = fs.S;
  // enough independent sub-chunks for two waves of resident CTAs
  const int64_t want = std::max<int64_t>(1, (2LL * cocc * sms + rows - 1) / rows);
  const int64_t Q = (S + std::min(S, want) - 1) / std::min(S, want);
  const int64_t nsub = (S + Q - 1) / Q;
  if (rows * nsub > INT32_MAX) return cudaErrorInvalidValue;
  cls.grid = (int)std::max<int64_t>(1, std::min<int64_t>(cls.grid, rows * nsub));
  *out = MapShape{cls, cDT, rows, (int)Q, (int)nsub};
  return cudaSuccess;
}

}  // namespace ssm
