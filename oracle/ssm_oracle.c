/*
 * ssm_oracle.c -- plain, sequential, double-precision CPU restatement of the
 * selective state-space scan.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call this code:
 * only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline / reference
 * leg may load, call or link it.  It shares no code, header, table or helper
 * with the CUDA library; the two only ever see the same seeded inputs.
 *
 * Sources (page title, then section):
 *  [P1] "Selective Scan trong Mamba toi uu chuoi dai the nao?" (thecsnote.cc)
 *       - "Tai sao Mamba can Selective Scan?": h_t = Abar h_{t-1} + Bbar x_t,
 *         y_t = C h_t.
 *       - "Selection pha vo convolution kernel co dinh": B_t, C_t and
 *         Delta_t = softplus(theta + s(x_t)) vary per token, giving the
 *         time-varying recurrence h_t = Abar_t h_{t-1} + Bbar_t x_t.
 *       - "Vi du Python": diagonal A, Abar = exp(Delta*A); its zero-order-hold
 *         input matrix Bbar = expm1(Delta*A)/A * B (kept here as an option).
 *       - "Selective Scan thay doi inference chuoi dai nhu the nao?": decoding
 *         updates a fixed-size state one token at a time.
 *  [P3] "Selective (Data-Dependent) SSM Scan" (cartesia-pytorch, problem 15)
 *       - "Step-by-Step Approach" 3-4: elementwise update h = A_t*h + B_t*x_t,
 *         readout y_t = C_t*h taken from the UPDATED state.
 *  The default input coefficient is Bbar_t = Delta_t * B_t (the simplified
 *  discretisation the library targets: "(Delta_t*B_t)*x_t"); the output is
 *  y_t = C_t . h_t + D*x_t, optionally multiplied by silu(z_t), with
 *  silu(z) = z * sigmoid(z).  Every floating-point step is done in double.
 *
 * Layouts (row-major, contiguous): x, delta, z, y: (B, L, D); Bm, Cm:
 * (B, L, N); A: (D, N); D, bias: (D); h0, h_last, state: (B, D, N).
 * In the elementwise variant x, A, B, C, y are (B, L, D) and h0, h_last are
 * (B, D).
 *
 * ssm_oracle_bwd is the reverse-mode gradient of the forward pass (the
 * chain rule applied to the same steps), pinned by central finite
 * differences of ssm_oracle_fwd.
 *
 * ORACLE_MUTANT (compile-time, tests only) plants one deliberate mistake so a
 * test can show that the pins catch it.  The default build has none.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>

#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0
#endif

/* Arithmetic type of the forward recurrence.  The parity oracle is the
 * default double build.  ORACLE_FP32 (set only by the CPU-baseline timing
 * build) compiles the same forward loop with a single-precision state and
 * accumulator, the "fp32-accumulate" CPU baseline; the other entry points
 * are left out of that build. */
#ifdef ORACLE_FP32
#include <tgmath.h>
typedef float orc_real;
#else
typedef double orc_real;
#endif

/* Option bits understood by the oracle.  They are the oracle's own
 * definitions; the Python wrapper maps keyword arguments onto them. */
#define ORC_HAS_Z 1u
#define ORC_HAS_D 2u
#define ORC_SOFTPLUS 4u
#define ORC_HAS_BIAS 8u
#define ORC_HAS_H0 16u
#define ORC_ZOH 128u

/* softplus(v) = log(1 + e^v), written in the overflow-free form
 * max(v, 0) + log1p(e^{-|v|}).  [P1] "Selection ...": Delta = softplus(.). */
double ssm_oracle_softplus(double v) {
#if ORACLE_MUTANT == 5
  return log(1.0 + exp(v)) + 1e-3; /* biased softplus */
#else
  return (v > 0.0 ? v : 0.0) + log1p(exp(-fabs(v)));
#endif
}

/* silu(z) = z * sigmoid(z) = z / (1 + e^{-z}). */
double ssm_oracle_silu(double z) {
#if ORACLE_MUTANT == 6
  return 1.0 / (1.0 + exp(-z)); /* sigmoid instead of silu */
#else
  return z / (1.0 + exp(-z));
#endif
}

/* One token of the Mamba-form recurrence for one channel (b, d).
 * h[0..N) is updated in place; returns y for this token.  [P1] "Selection
 * ...": Abar_t = exp(Delta_t*A), Bbar_t = Delta_t*B_t (or ZOH), h updated
 * first, readout from the updated state ([P3] step 4). */
static double token_update(int64_t N, uint32_t flags, double xv_in, double dv,
                           double bias, const double *Arow, const double *Bt,
                           const double *Ct, double Dd, double zv, orc_real *h) {
  const orc_real xv = (orc_real)xv_in;
  orc_real v = (orc_real)(dv + bias);
  orc_real dt = (flags & ORC_SOFTPLUS) ? (orc_real)ssm_oracle_softplus(v) : v;
#if ORACLE_MUTANT == 7
  dt = (flags & ORC_SOFTPLUS) ? ssm_oracle_softplus(dv) : dv; /* bias dropped */
#endif
  orc_real acc = 0.0;
  for (int64_t n = 0; n < N; ++n) {
    orc_real a = (orc_real)Arow[n];
    orc_real abar = exp(dt * a);
#if ORACLE_MUTANT == 1
    abar = exp(-dt * a); /* sign flip */
#endif
    orc_real bbar;
    if (flags & ORC_ZOH)
#if ORACLE_MUTANT == 16
      bbar = (a != 0.0 ? expm1(dt * a) / a : 0.0) * (orc_real)Bt[n]; /* A = 0 limit lost */
#else
      bbar = (a != 0.0 ? expm1(dt * a) / a : dt) * (orc_real)Bt[n];
#endif
    else
      bbar = dt * (orc_real)Bt[n];
#if ORACLE_MUTANT == 2
    acc += Ct[n] * h[n]; /* readout from the state before the update */
#endif
    h[n] = abar * h[n] + bbar * xv;
#if ORACLE_MUTANT == 8
    h[n] = abar * h[n] + bbar; /* input x dropped */
#endif
#if ORACLE_MUTANT != 2
#if ORACLE_MUTANT == 9
    acc += Bt[n] * h[n]; /* B used as readout instead of C */
#else
    acc += (orc_real)Ct[n] * h[n];
#endif
#endif
  }
  if (flags & ORC_HAS_D) {
#if ORACLE_MUTANT != 3
    acc += (orc_real)Dd * xv;
#endif
  }
  if (flags & ORC_HAS_Z) {
#if ORACLE_MUTANT == 4
    acc = (acc - Dd * xv) * ssm_oracle_silu(zv) + ((flags & ORC_HAS_D) ? Dd * xv : 0.0);
#else
    acc *= ssm_oracle_silu(zv);
#endif
  }
  return acc;
}

/* Full-sequence forward pass: for every channel (b, d) run t = 0..L-1 in
 * order.  Returns 0, or -1 on a bad argument / allocation failure.  h_last
 * may be NULL. */
int ssm_oracle_fwd(int64_t Bsz, int64_t L, int64_t D, int64_t N, uint32_t flags,
                   const double *x, const double *delta, const double *bias,
                   const double *A, const double *Bm, const double *Cm,
                   const double *Dv, const double *z, const double *h0,
                   double *y, double *h_last) {
  if (Bsz < 0 || L < 0 || D < 0 || N < 1) return -1;
  if (!x || !delta || !A || !Bm || !Cm || !y) return -1;
  if ((flags & ORC_HAS_Z) && !z) return -1;
  if ((flags & ORC_HAS_D) && !Dv) return -1;
  if ((flags & ORC_HAS_BIAS) && !bias) return -1;
  if ((flags & ORC_HAS_H0) && !h0) return -1;
  orc_real *h = (orc_real *)malloc((size_t)N * sizeof(orc_real));
  if (!h) return -1;
  for (int64_t b = 0; b < Bsz; ++b) {
    for (int64_t d = 0; d < D; ++d) {
      for (int64_t n = 0; n < N; ++n) {
        h[n] = (flags & ORC_HAS_H0) ? (orc_real)h0[(b * D + d) * N + n] : 0.0;
#if ORACLE_MUTANT == 10
        h[n] = 0.0; /* h0 ignored */
#endif
      }
      for (int64_t t = 0; t < L; ++t) {
        size_t i = (size_t)((b * L + t) * D + d);
        size_t j = (size_t)((b * L + t) * N);
#if ORACLE_MUTANT == 11
        /* B and C taken from the previous token */
        if (t > 0) j -= (size_t)N;
#endif
        y[i] = token_update(N, flags, x[i], delta[i],
                            (flags & ORC_HAS_BIAS) ? bias[d] : 0.0, A + d * N,
                            Bm + j, Cm + j, (flags & ORC_HAS_D) ? Dv[d] : 0.0,
                            (flags & ORC_HAS_Z) ? z[i] : 0.0, h);
      }
      if (h_last)
        for (int64_t n = 0; n < N; ++n) h_last[(b * D + d) * N + n] = h[n];
    }
  }
  free(h);
  return 0;
}

#ifndef ORACLE_FP32
/* Causal depthwise convolution of the x branch followed by silu, the
 * front-end that feeds the scan's x ([P5] section 5.3 names the fused
 * causal_conv1d + selective_scan_fn kernels; the operation is read as the
 * standard one of that name): per channel d, with x_in = 0 before t = 0,
 *   u[b,t,d] = bias[d] + sum_{k=0}^{K-1} w[d,k] * x_in[b, t-(K-1)+k, d],
 *   out[b,t,d] = silu(u[b,t,d]).
 * w[d, K-1] multiplies the current token.  x_in, out: (B, L, D); w: (D, K);
 * bias: (D) or NULL.  Returns 0, or -1 on a bad argument. */
int ssm_oracle_causal_conv_silu(int64_t Bsz, int64_t L, int64_t D, int64_t K,
                                const double *x_in, const double *w, const double *bias,
                                double *out) {
  if (Bsz < 0 || L < 0 || D < 0 || K < 1 || !x_in || !w || !out) return -1;
  for (int64_t b = 0; b < Bsz; ++b)
    for (int64_t t = 0; t < L; ++t)
      for (int64_t d = 0; d < D; ++d) {
        double u = bias ? bias[d] : 0.0;
#if ORACLE_MUTANT == 18
        u = 0.0; /* bias dropped */
#endif
        for (int64_t k = 0; k < K; ++k) {
          int64_t src = t - (K - 1) + k;
#if ORACLE_MUTANT == 19
          src += 1; /* window shifted one token into the future */
#endif
          if (src < 0 || src >= L) continue;
#if ORACLE_MUTANT == 17
          u += w[d * K + (K - 1 - k)] * x_in[(b * L + src) * D + d]; /* taps reversed */
#else
          u += w[d * K + k] * x_in[(b * L + src) * D + d];
#endif
        }
        out[(b * L + t) * D + d] = ssm_oracle_silu(u);
      }
  return 0;
}

/* One decode step ([P1] inference section): state (B, D, N) is read, updated
 * with one token and written back; y is (B, D).  x, delta, z: (B, D);
 * Bm, Cm: (B, N). */
int ssm_oracle_step(int64_t Bsz, int64_t D, int64_t N, uint32_t flags,
                    const double *x, const double *delta, const double *bias,
                    const double *A, const double *Bm, const double *Cm,
                    const double *Dv, const double *z, double *state, double *y) {
  if (Bsz < 0 || D < 0 || N < 1) return -1;
  if (!x || !delta || !A || !Bm || !Cm || !state || !y) return -1;
  if ((flags & ORC_HAS_Z) && !z) return -1;
  if ((flags & ORC_HAS_D) && !Dv) return -1;
  if ((flags & ORC_HAS_BIAS) && !bias) return -1;
  for (int64_t b = 0; b < Bsz; ++b) {
    for (int64_t d = 0; d < D; ++d) {
      size_t i = (size_t)(b * D + d);
      y[i] = token_update(N, flags, x[i], delta[i],
                          (flags & ORC_HAS_BIAS) ? bias[d] : 0.0, A + d * N,
                          Bm + b * N, Cm + b * N,
                          (flags & ORC_HAS_D) ? Dv[d] : 0.0,
                          (flags & ORC_HAS_Z) ? z[i] : 0.0, state + i * N);
    }
  }
  return 0;
}

/* Elementwise variant ([P3] steps 2-5): A_t is the transition itself,
 * h = A_t*h + B_t*x_t, y_t = C_t*h (after the update).  All of x, A, B, C, y
 * are (B, L, D); h0 and h_last are (B, D) and may be NULL (h0 = 0). */
int ssm_oracle_direct(int64_t Bsz, int64_t L, int64_t D, const double *x,
                      const double *A, const double *Bm, const double *Cm,
                      const double *h0, double *y, double *h_last) {
  if (Bsz < 0 || L < 0 || D < 0) return -1;
  if (!x || !A || !Bm || !Cm || !y) return -1;
  for (int64_t b = 0; b < Bsz; ++b) {
    for (int64_t d = 0; d < D; ++d) {
      double h = h0 ? h0[b * D + d] : 0.0;
      for (int64_t t = 0; t < L; ++t) {
        size_t i = (size_t)((b * L + t) * D + d);
#if ORACLE_MUTANT == 12
        h = Bm[i] * x[i] + (t > 0 ? A[i - D] : A[i]) * h; /* A from previous token */
#else
        h = A[i] * h + Bm[i] * x[i];
#endif
        y[i] = Cm[i] * h;
      }
      if (h_last) h_last[b * D + d] = h;
    }
  }
  return 0;
}

/* Reverse-mode gradient of ssm_oracle_fwd (Delta*B input coefficient; the
 * zero-order-hold option is not covered and returns -1) for a loss whose
 * derivatives are dy = dL/dy (B, L, D) and dh_last = dL/dh_last (B, D, N,
 * NULL for 0).  For each channel the states h_0 .. h_L are recomputed and
 * kept, then t runs L-1 .. 0 applying the chain rule to the forward steps of
 * [P1] "Selection pha vo convolution kernel co dinh" / "Vi du Python":
 *   v = delta + bias, Delta = softplus(v), abar_n = exp(Delta A_n),
 *   h_t = abar h_{t-1} + Delta B_t x_t,  s_t = C_t . h_t + D x_t,
 *   y_t = s_t silu(z_t),
 * with g = dL/dh_t carried backwards (g <- g * abar after each token).
 * dx, ddelta, dz: (B, L, D); dB, dC: (B, L, N); dA: (D, N); dD, dbias: (D);
 * dh0: (B, D, N).  Outputs for absent inputs may be NULL.  Returns 0, or -1
 * on a bad argument / allocation failure. */
int ssm_oracle_bwd(int64_t Bsz, int64_t L, int64_t D, int64_t N, uint32_t flags,
                   const double *x, const double *delta, const double *bias,
                   const double *A, const double *Bm, const double *Cm,
                   const double *Dv, const double *z, const double *h0,
                   const double *dy, const double *dh_last, double *dx, double *ddelta,
                   double *dbias, double *dA, double *dB, double *dC, double *dD,
                   double *dz, double *dh0) {
  if (Bsz < 0 || L < 0 || D < 0 || N < 1) return -1;
  if (flags & ORC_ZOH) return -1;
  if (!x || !delta || !A || !Bm || !Cm || !dy || !dx || !ddelta || !dA || !dB || !dC)
    return -1;
  if ((flags & ORC_HAS_Z) && (!z || !dz)) return -1;
  if ((flags & ORC_HAS_D) && (!Dv || !dD)) return -1;
  if ((flags & ORC_HAS_BIAS) && (!bias || !dbias)) return -1;
  if ((flags & ORC_HAS_H0) && !h0) return -1;
  for (int64_t k = 0; k < D * N; ++k) dA[k] = 0.0;
  for (int64_t k = 0; k < Bsz * L * N; ++k) dB[k] = dC[k] = 0.0;
  for (int64_t k = 0; k < D; ++k) {
    if (dD) dD[k] = 0.0;
    if (dbias) dbias[k] = 0.0;
  }
  double *hs = (double *)malloc((size_t)(L + 1) * (size_t)N * sizeof(double));
  double *g = (double *)malloc((size_t)N * sizeof(double));
  if (!hs || !g) {
    free(hs);
    free(g);
    return -1;
  }
  for (int64_t b = 0; b < Bsz; ++b) {
    for (int64_t d = 0; d < D; ++d) {
      const double *Arow = A + d * N;
      const double bv = (flags & ORC_HAS_BIAS) ? bias[d] : 0.0;
      const double Dd = (flags & ORC_HAS_D) ? Dv[d] : 0.0;
      /* forward, keeping every state: hs[t*N ..] = h_t (h_0 = h0) */
      for (int64_t n = 0; n < N; ++n)
        hs[n] = (flags & ORC_HAS_H0) ? h0[(b * D + d) * N + n] : 0.0;
      for (int64_t t = 0; t < L; ++t) {
        size_t i = (size_t)((b * L + t) * D + d), j = (size_t)((b * L + t) * N);
        double v = delta[i] + bv;
        double dt = (flags & ORC_SOFTPLUS) ? ssm_oracle_softplus(v) : v;
        for (int64_t n = 0; n < N; ++n)
          hs[(t + 1) * N + n] = exp(dt * Arow[n]) * hs[t * N + n] + dt * Bm[j + n] * x[i];
      }
      /* backward */
      for (int64_t n = 0; n < N; ++n) g[n] = dh_last ? dh_last[(b * D + d) * N + n] : 0.0;
      for (int64_t t = L - 1; t >= 0; --t) {
        size_t i = (size_t)((b * L + t) * D + d), j = (size_t)((b * L + t) * N);
        const double xv = x[i];
        const double v = delta[i] + bv;
        const double dt = (flags & ORC_SOFTPLUS) ? ssm_oracle_softplus(v) : v;
        const double *ht = hs + (t + 1) * N, *hp = hs + t * N;
        double s = Dd * xv;
        for (int64_t n = 0; n < N; ++n) s += Cm[j + n] * ht[n];
        double ds = dy[i];
        if (flags & ORC_HAS_Z) {
          const double zv = z[i], sig = 1.0 / (1.0 + exp(-zv));
          ds = dy[i] * zv * sig;                          /* dy * silu(z) */
          dz[i] = dy[i] * s * sig * (1.0 + zv * (1.0 - sig)); /* silu'(z) */
#if ORACLE_MUTANT == 15
          dz[i] = dy[i] * s * sig; /* sigmoid in place of silu' */
#endif
        }
        double dxi = ds * Dd;
        if (flags & ORC_HAS_D) dD[d] += ds * xv;
        double ddt = 0.0;
        for (int64_t n = 0; n < N; ++n) {
          const double abar = exp(dt * Arow[n]);
          dC[j + n] += ds * ht[n];
          g[n] += ds * Cm[j + n];
          const double dabar = g[n] * hp[n];
          ddt += dabar * abar * Arow[n] + g[n] * Bm[j + n] * xv;
#if ORACLE_MUTANT == 14
          ddt -= g[n] * Bm[j + n] * xv; /* Delta's input term dropped */
#endif
          dA[d * N + n] += dabar * abar * dt;
          dB[j + n] += g[n] * dt * xv;
          dxi += g[n] * dt * Bm[j + n];
          g[n] *= abar;
#if ORACLE_MUTANT == 13
          g[n] /= abar; /* state gradient not carried through Abar */
#endif
        }
        dx[i] = dxi;
        const double dv = (flags & ORC_SOFTPLUS) ? ddt / (1.0 + exp(-v)) : ddt;
        ddelta[i] = dv;
        if (flags & ORC_HAS_BIAS) dbias[d] += dv;
      }
      if (dh0)
        for (int64_t n = 0; n < N; ++n) dh0[(b * D + d) * N + n] = g[n];
    }
  }
  free(hs);
  free(g);
  return 0;
}
#endif /* ORACLE_FP32 */
