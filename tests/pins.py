"""Pins for the CPU oracle: checks against facts the pages and the mathematics
fix, each computed by a route other than the oracle's own loop.

Every pin takes an ``oracle.Oracle`` and raises AssertionError on mismatch,
so ``test_oracle_mutants.py`` can run the same pins against builds of the
oracle with one planted mistake and show that some pin catches each.

Page references (title, section):
  [P1] "Selective Scan trong Mamba toi uu chuoi dai the nao?" (thecsnote.cc)
  [P3] "Selective (Data-Dependent) SSM Scan" (cartesia-pytorch, problem 15)
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _close(got, want, rtol, atol=0.0, what=""):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape, f"{what}: shape {got.shape} != {want.shape}"
    err = np.abs(got - want)
    lim = atol + rtol * np.abs(want)
    bad = np.argwhere(err > lim)
    assert bad.size == 0, (f"{what}: {len(bad)} mismatches, first at {tuple(bad[0])}: "
                           f"got {got[tuple(bad[0])]!r} want {want[tuple(bad[0])]!r}")


def _normwise(got, want, tol, what=""):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    scale = max(np.max(np.abs(want)), 1e-300)
    e = np.max(np.abs(got - want)) / scale
    assert e <= tol, f"{what}: normwise error {e:.3e} > {tol:.1e}"


def _softplus_ref(v):
    # numpy's logaddexp(0, v) = log(e^0 + e^v): a library routine, not the oracle's code
    return np.logaddexp(0.0, v)


def _silu_ref(z):
    return z * (0.5 * (1.0 + np.tanh(0.5 * z)))   # sigmoid via tanh: another route


# --------------------------------------------------------------------------
# Hand-computed worked cases (exact dyadic arithmetic)
# --------------------------------------------------------------------------

def pin_hand_direct(orc):
    """[P3] steps 3-4: h = A_t*h + B_t*x_t, y_t = C_t*h after the update.
    Dyadic values, so every product is exact:
      h1 = 1/2*1 + 1*2 = 5/2,        y1 = 1*5/2 = 5/2
      h2 = 1/4*5/2 + 2*1 = 21/8,     y2 = 1/2*21/8 = 21/16
      h3 = 2*21/8 + (-1)*4 = 5/4,    y3 = 3*5/4 = 15/4"""
    x = np.array([2.0, 1.0, 4.0]).reshape(1, 3, 1)
    A = np.array([0.5, 0.25, 2.0]).reshape(1, 3, 1)
    B = np.array([1.0, 2.0, -1.0]).reshape(1, 3, 1)
    C = np.array([1.0, 0.5, 3.0]).reshape(1, 3, 1)
    y, hl = orc.direct(x, A, B, C, h0=np.array([[1.0]]))
    _close(y.ravel(), [2.5, 21 / 16, 3.75], 0, 0, "hand direct y")
    _close(hl.ravel(), [1.25], 0, 0, "hand direct h_last")


def pin_hand_mamba(orc):
    """[P1] time-varying recurrence with Abar = exp(Delta*A), Bbar = Delta*B,
    plus the D skip.  A = (-ln2, -2 ln2) makes Abar = 2^(-Delta(n+1)), so with
    integer Delta every value is dyadic (only ln2's rounding enters, ~1e-16):
      t1: Delta=1, Abar=(1/2,1/4), b=1*(1,2)*1=(1,2):    h=(3,4),        y=3+4+0.5*1=7.5
      t2: Delta=1, Abar=(1/2,1/4), b=1*(-1,1)*2=(-2,2):  h=(-1/2,3),     y=-1-3+0.5*2=-3
      t3: Delta=2, Abar=(1/4,1/16), b=2*(2,0)*(-1)=(-4,0): h=(-33/8,3/16), y=-33/8+3/4-1/2=-31/8"""
    A = np.array([[-math.log(2.0), -2.0 * math.log(2.0)]])
    x = np.array([1.0, 2.0, -1.0]).reshape(1, 3, 1)
    dlt = np.array([1.0, 1.0, 2.0]).reshape(1, 3, 1)
    B = np.array([[1.0, 2.0], [-1.0, 1.0], [2.0, 0.0]]).reshape(1, 3, 2)
    C = np.array([[1.0, 1.0], [2.0, -1.0], [1.0, 4.0]]).reshape(1, 3, 2)
    h0 = np.array([4.0, 8.0]).reshape(1, 1, 2)
    y, hl = orc.fwd(x, dlt, A, B, C, D=np.array([0.5]), h0=h0, delta_softplus=False)
    _close(y.ravel(), [7.5, -3.0, -3.875], 1e-13, 1e-13, "hand mamba y")
    _close(hl.ravel(), [-4.125, 0.1875], 1e-13, 1e-13, "hand mamba h_last")
    # gate: silu(0) = 0 exactly; silu(40) = 40/(1+e^-40) = 40 to 1e-15; silu(-40) ~ -1.7e-16
    z = np.array([0.0, 40.0, -40.0]).reshape(1, 3, 1)
    y, _ = orc.fwd(x, dlt, A, B, C, D=np.array([0.5]), z=z, h0=h0, delta_softplus=False)
    _close(y.ravel(), [0.0, -120.0, 0.0], 1e-13, 1e-13, "hand mamba gated y")


def pin_softplus_values(orc):
    """[P1] Delta = softplus(theta + s(x)): with A=0 (Abar=1), h0=0, B=C=x=1 and
    no skip, y equals Delta itself, so the scan exposes softplus(raw + bias).
    softplus(0) = ln 2 exactly; large |v| checked against the library's
    log1p/exp."""
    raws = np.array([0.0, -1.0, 30.0, -30.0, 3.5, -7.25])
    bias = np.array([0.0, 1.0, 0.0, 0.0, -0.5, 0.25])
    for r, b in zip(raws, bias):
        one = np.ones((1, 1, 1))
        y, _ = orc.fwd(one, np.full((1, 1, 1), r), np.zeros((1, 1)), one.reshape(1, 1, 1),
                       one.reshape(1, 1, 1), delta_bias=np.array([b]), delta_softplus=True)
        v = r + b
        want = math.log(2.0) if v == 0.0 else (v + math.log1p(math.exp(-v)) if v > 0
                                                  else math.log1p(math.exp(v)))
        _close(y.ravel(), [want], 1e-14, 0, f"softplus({v})")


# --------------------------------------------------------------------------
# Closed forms
# --------------------------------------------------------------------------

def pin_lti_convolution(orc, seed=11):
    """[P1] "Tai sao Mamba can Selective Scan?": with Delta, B, C constant over
    t and h0 = 0 the recurrence is a causal convolution y = x * K with
    K_k = C Abar^k Bbar.  Computed here as a direct O(L^2) sum with Abar^k by
    np.power, per channel d."""
    rng = np.random.default_rng(seed)
    Bsz, L, D, N = 2, 24, 3, 4
    A = -rng.uniform(0.2, 2.0, size=(D, N))
    dlt_d = rng.uniform(0.05, 0.6, size=D)               # constant over t, per channel
    Bv = rng.standard_normal((Bsz, N))                   # constant over t, per batch
    Cv = rng.standard_normal((Bsz, N))
    x = rng.standard_normal((Bsz, L, D))
    dlt = np.broadcast_to(dlt_d, (Bsz, L, D)).copy()
    Bm = np.broadcast_to(Bv[:, None, :], (Bsz, L, N)).copy()
    Cm = np.broadcast_to(Cv[:, None, :], (Bsz, L, N)).copy()
    y, hl = orc.fwd(x, dlt, A, Bm, Cm, delta_softplus=False)
    want = np.zeros((Bsz, L, D))
    for b in range(Bsz):
        for d in range(D):
            abar = np.exp(dlt_d[d] * A[d])
            K = np.array([np.sum(Cv[b] * np.power(abar, k) * dlt_d[d] * Bv[b]) for k in range(L)])
            for t in range(L):
                want[b, t, d] = sum(K[k] * x[b, t - k, d] for k in range(t + 1))
    _close(y, want, 1e-11, 1e-12, "LTI convolution")
    # state after L steps: sum_j Abar^(L-1-j) Bbar x_j
    for b in range(Bsz):
        for d in range(D):
            abar = np.exp(dlt_d[d] * A[d])
            hs = sum(np.power(abar, L - 1 - j) * dlt_d[d] * Bv[b] * x[b, j, d] for j in range(L))
            _close(hl[b, d], hs, 1e-11, 1e-12, "LTI final state")


def brute_force_fwd(x, dlt_raw, A, Bm, Cm, D=None, z=None, bias=None, h0=None, softplus=True,
                    zoh=False):
    """[P1] "Selection pha vo ...": the contribution of x_j to y_t is
    C_t (Abar_t ... Abar_{j+1}) Bbar_j x_j.  Sum those terms explicitly
    (explicit products, no recurrence), add h0's term C_t (Abar_t..Abar_1) h0,
    the skip D x_t, then the gate.  The state after token t is
    sum_{j<=t} (prod_{i=j+1..t} Abar_i) Bbar_j x_j + (prod_{i<=t} Abar_i) h0."""
    Bsz, L, Dm = x.shape
    N = A.shape[1]
    v = dlt_raw + (0.0 if bias is None else bias[None, None, :])
    dt = _softplus_ref(v) if softplus else v
    y = np.zeros((Bsz, L, Dm))
    hl = np.zeros((Bsz, Dm, N))
    for b in range(Bsz):
        for d in range(Dm):
            abar = np.exp(dt[b, :, d, None] * A[d][None, :])          # (L, N)
            if zoh:
                safe = np.where(A[d] != 0, A[d], 1.0)
                coef = np.where(A[d] != 0, np.expm1(dt[b, :, d, None] * A[d]) / safe,
                                dt[b, :, d, None])
            else:
                coef = dt[b, :, d, None] * np.ones(N)
            bbar = coef * Bm[b]                                       # (L, N)

            def state_after(t):
                s = np.zeros(N)
                for j in range(t + 1):
                    prod = np.ones(N)
                    for i in range(j + 1, t + 1):
                        prod = prod * abar[i]
                    s = s + prod * bbar[j] * x[b, j, d]
                if h0 is not None:
                    prod = np.ones(N)
                    for i in range(t + 1):
                        prod = prod * abar[i]
                    s = s + prod * h0[b, d]
                return s

            for t in range(L):
                st = state_after(t)
                yv = np.sum(Cm[b, t] * st)
                if D is not None:
                    yv += D[d] * x[b, t, d]
                if z is not None:
                    yv *= _silu_ref(z[b, t, d])
                y[b, t, d] = yv
            hl[b, d] = state_after(L - 1) if L > 0 else (h0[b, d] if h0 is not None else 0.0)
    return y, hl


def pin_brute_force(orc, seed=12):
    """Time-varying coefficients, every option on (bias, softplus, D, gate, h0)."""
    rng = np.random.default_rng(seed)
    Bsz, L, D, N = 2, 13, 3, 4
    x = rng.standard_normal((Bsz, L, D))
    dr = rng.standard_normal((Bsz, L, D)) - 0.5
    z = rng.standard_normal((Bsz, L, D))
    A = -rng.uniform(0.1, 3.0, size=(D, N))
    Bm = rng.standard_normal((Bsz, L, N))
    Cm = rng.standard_normal((Bsz, L, N))
    Dv = rng.standard_normal(D)
    bias = rng.uniform(-2, 1, size=D)
    h0 = rng.standard_normal((Bsz, D, N))
    y, hl = orc.fwd(x, dr, A, Bm, Cm, D=Dv, z=z, delta_bias=bias, h0=h0)
    wy, wh = brute_force_fwd(x, dr, A, Bm, Cm, D=Dv, z=z, bias=bias, h0=h0)
    _close(y, wy, 1e-10, 1e-12, "brute force y")
    _close(hl, wh, 1e-10, 1e-12, "brute force h_last")
    # softplus off, no optional inputs
    y, hl = orc.fwd(x, np.abs(dr), A, Bm, Cm, delta_softplus=False)
    wy, wh = brute_force_fwd(x, np.abs(dr), A, Bm, Cm, softplus=False)
    _close(y, wy, 1e-10, 1e-12, "brute force y (plain)")
    _close(hl, wh, 1e-10, 1e-12, "brute force h_last (plain)")


def pin_zoh_limits(orc, seed=19):
    """[P1] "Vi du Python" discretises with zero-order hold,
    Bbar = expm1(Delta A) / A * B.  Its value where A = 0 is the limit
    Delta * B (expm1(u) / u -> 1), and near A = 0 it is continuous.  Checked
    with every option on against the brute-force products (whose ZOH
    coefficient takes numpy's expm1 and the limit by an explicit select):
    some A entries exactly 0, some at +-1e-8, the rest ordinary negative
    values; then the exact-zero and the 1e-8 runs must agree to ~1e-8
    relative (continuity of the coefficient at 0)."""
    rng = np.random.default_rng(seed)
    Bsz, L, D, N = 2, 11, 3, 4
    x = rng.standard_normal((Bsz, L, D))
    dr = rng.standard_normal((Bsz, L, D)) - 0.5
    z = rng.standard_normal((Bsz, L, D))
    Bm = rng.standard_normal((Bsz, L, N))
    Cm = rng.standard_normal((Bsz, L, N))
    Dv = rng.standard_normal(D)
    bias = rng.uniform(-2, 1, size=D)
    h0 = rng.standard_normal((Bsz, D, N))
    A = -rng.uniform(0.1, 3.0, size=(D, N))
    A[0, :] = 0.0                    # a whole channel at the limit
    A[1, 1] = 0.0
    A[2, 0], A[2, 3] = 1e-8, -1e-8   # next to it, on both sides
    y, hl = orc.fwd(x, dr, A, Bm, Cm, D=Dv, z=z, delta_bias=bias, h0=h0, zoh=True)
    wy, wh = brute_force_fwd(x, dr, A, Bm, Cm, D=Dv, z=z, bias=bias, h0=h0, zoh=True)
    _close(y, wy, 1e-10, 1e-12, "ZOH brute force y (A = 0 and near 0)")
    _close(hl, wh, 1e-10, 1e-12, "ZOH brute force h_last (A = 0 and near 0)")
    # A = 0 on every state: Abar = 1, Bbar = Delta * B, so the ZOH scan equals
    # the Delta*B scan exactly (same prefix sum)
    A0 = np.zeros((D, N))
    yz, hz = orc.fwd(x, dr, A0, Bm, Cm, D=Dv, z=z, delta_bias=bias, h0=h0, zoh=True)
    yd, hd = orc.fwd(x, dr, A0, Bm, Cm, D=Dv, z=z, delta_bias=bias, h0=h0, zoh=False)
    _close(yz, yd, 1e-15, 1e-15, "ZOH at A = 0 equals Delta*B")
    _close(hz, hd, 1e-15, 1e-15, "ZOH h_last at A = 0 equals Delta*B")
    # continuity: A = +-1e-8 moves the result by O(1e-8) relative only
    ye, he = orc.fwd(x, dr, np.full((D, N), 1e-8), Bm, Cm, D=Dv, z=z, delta_bias=bias, h0=h0,
                     zoh=True)
    _normwise(ye, yz, 1e-6, "ZOH continuity at A = 0 (y)")
    _normwise(he, hz, 1e-6, "ZOH continuity at A = 0 (h_last)")


def compose(prefix, cur):
    """[P1] "Scan bien recurrence ...": T2(T1(h)) = A2 A1 h + A2 b1 + b2, i.e.
    (A2, b2) (x) (A1, b1) = (A2*A1, A2*b1 + b2); ``cur`` is applied after
    ``prefix``."""
    a1, b1 = prefix
    a2, b2 = cur
    return a2 * a1, a2 * b1 + b2


def tree_scan_states(abar, bx, h0):
    """Inclusive prefix of the affine maps by Hillis-Steele doubling (log2 L
    rounds of pairwise composition: a grouping entirely unlike the sequential
    loop), then applied to h0."""
    L = abar.shape[0]
    a, b = abar.copy(), bx.copy()
    s = 1
    while s < L:
        na, nb = a.copy(), b.copy()
        for t in range(s, L):
            na[t], nb[t] = compose((a[t - s], b[t - s]), (a[t], b[t]))
        a, b, s = na, nb, 2 * s
    return a * h0[None, :] + b


def pin_tree_scan(orc, seed=13):
    """Associativity: the tree-grouped composition of the per-token affine
    maps gives the same states, hence the same y, as the sequential loop."""
    rng = np.random.default_rng(seed)
    Bsz, L, D, N = 1, 37, 2, 8
    x = rng.standard_normal((Bsz, L, D))
    dr = rng.standard_normal((Bsz, L, D))
    A = -rng.uniform(0.1, 4.0, size=(D, N))
    Bm = rng.standard_normal((Bsz, L, N))
    Cm = rng.standard_normal((Bsz, L, N))
    h0 = rng.standard_normal((Bsz, D, N))
    y, hl = orc.fwd(x, dr, A, Bm, Cm, h0=h0)
    dt = _softplus_ref(dr)
    for d in range(D):
        abar = np.exp(dt[0, :, d, None] * A[d][None, :])
        bx = dt[0, :, d, None] * Bm[0] * x[0, :, d, None]
        hs = tree_scan_states(abar, bx, h0[0, d])
        _close(y[0, :, d], np.sum(Cm[0] * hs, axis=1), 1e-11, 1e-12, "tree-scan y")
        _close(hl[0, d], hs[-1], 1e-11, 1e-12, "tree-scan h_last")


def pin_degenerate(orc, seed=14):
    """The A=0 family.  (i) [P3] step 6, elementwise form with A=0: the state
    holds only the current token, so y_t = C_t B_t x_t.  (ii) Mamba form with
    Abar = 0 (A = -1e30 makes exp underflow to exactly 0): memoryless,
    y_t = sum_n C_t Delta_t B_t x_t + D x_t.  (iii) Mamba form with A = 0
    (Abar = 1): the state is the running sum h0 + sum_{j<=t} Delta_j B_j x_j."""
    rng = np.random.default_rng(seed)
    Bsz, L, D, N = 2, 9, 3, 4
    x = rng.standard_normal((Bsz, L, D))
    Bd = rng.standard_normal((Bsz, L, D))
    Cd = rng.standard_normal((Bsz, L, D))
    y, hl = orc.direct(x, np.zeros_like(x), Bd, Cd, h0=rng.standard_normal((Bsz, D)))
    _close(y, Cd * Bd * x, 1e-15, 0, "direct A=0")
    _close(hl, Bd[:, -1] * x[:, -1], 1e-15, 0, "direct A=0 h_last")
    dr = rng.standard_normal((Bsz, L, D))
    Bm = rng.standard_normal((Bsz, L, N))
    Cm = rng.standard_normal((Bsz, L, N))
    Dv = rng.standard_normal(D)
    h0 = rng.standard_normal((Bsz, D, N))
    dt = _softplus_ref(dr)
    y, hl = orc.fwd(x, dr, np.full((D, N), -1e30), Bm, Cm, D=Dv, h0=h0)
    want = np.einsum("bln,bld->bld", Cm * Bm, dt * x) + Dv[None, None, :] * x
    _close(y, want, 1e-12, 1e-13, "mamba Abar=0")
    y, hl = orc.fwd(x, dr, np.zeros((D, N)), Bm, Cm, h0=h0)
    incr = dt[..., None] * Bm[:, :, None, :] * x[..., None]     # (B, L, D, N)
    states = h0[:, None] + np.cumsum(incr, axis=1)
    _close(y, np.einsum("bln,bldn->bld", Cm, states), 1e-12, 1e-12, "mamba A=0 prefix sum")
    _close(hl, states[:, -1], 1e-12, 1e-12, "mamba A=0 h_last")


def pin_skip_and_gate(orc, seed=15):
    """With B = 0 the state never moves from h0 = 0, so y_t = D x_t silu(z_t):
    isolates the skip term and the gate's placement around it."""
    rng = np.random.default_rng(seed)
    Bsz, L, D, N = 1, 7, 5, 2
    x = rng.standard_normal((Bsz, L, D))
    z = rng.standard_normal((Bsz, L, D)) * 3
    Dv = rng.standard_normal(D)
    y, _ = orc.fwd(x, rng.standard_normal((Bsz, L, D)), -np.ones((D, N)),
                   np.zeros((Bsz, L, N)), rng.standard_normal((Bsz, L, N)), D=Dv, z=z)
    _close(y, Dv[None, None, :] * x * _silu_ref(z), 1e-14, 1e-15, "skip and gate")


def pin_h0_split(orc, seed=16):
    """The state is the scan's checkpoint ([P1] inference section): running
    [0,k) then [k,L) from h0 = h_last of the first part equals the full run."""
    rng = np.random.default_rng(seed)
    Bsz, L, D, N = 2, 20, 3, 4
    x = rng.standard_normal((Bsz, L, D))
    dr = rng.standard_normal((Bsz, L, D))
    z = rng.standard_normal((Bsz, L, D))
    A = -rng.uniform(0.1, 2.0, size=(D, N))
    Bm = rng.standard_normal((Bsz, L, N))
    Cm = rng.standard_normal((Bsz, L, N))
    Dv = rng.standard_normal(D)
    h0 = rng.standard_normal((Bsz, D, N))
    yf, hf = orc.fwd(x, dr, A, Bm, Cm, D=Dv, z=z, h0=h0)
    for k in (1, 7, 19):
        y1, h1 = orc.fwd(x[:, :k], dr[:, :k], A, Bm[:, :k], Cm[:, :k], D=Dv, z=z[:, :k], h0=h0)
        y2, h2 = orc.fwd(x[:, k:], dr[:, k:], A, Bm[:, k:], Cm[:, k:], D=Dv, z=z[:, k:], h0=h1)
        _close(np.concatenate([y1, y2], axis=1), yf, 1e-13, 1e-14, f"split at {k}")
        _close(h2, hf, 1e-13, 1e-14, f"split at {k} h_last")


def pin_decode(orc, seed=17):
    """[P1] inference section: decoding applies one update per token to a
    fixed-size state.  Stepping L tokens must reproduce the brute-force
    unrolled outputs and final state."""
    rng = np.random.default_rng(seed)
    Bsz, L, D, N = 2, 8, 3, 4
    x = rng.standard_normal((Bsz, L, D))
    dr = rng.standard_normal((Bsz, L, D))
    z = rng.standard_normal((Bsz, L, D))
    A = -rng.uniform(0.1, 2.0, size=(D, N))
    Bm = rng.standard_normal((Bsz, L, N))
    Cm = rng.standard_normal((Bsz, L, N))
    Dv = rng.standard_normal(D)
    bias = rng.uniform(-1, 1, size=D)
    h0 = rng.standard_normal((Bsz, D, N))
    state = h0.copy()
    ys = []
    for t in range(L):
        yt, state = orc.step(state, x[:, t], dr[:, t], A, Bm[:, t], Cm[:, t], D=Dv, z=z[:, t],
                             delta_bias=bias)
        ys.append(yt)
    wy, wh = brute_force_fwd(x, dr, A, Bm, Cm, D=Dv, z=z, bias=bias, h0=h0)
    _close(np.stack(ys, axis=1), wy, 1e-10, 1e-12, "decode y")
    _close(state, wh, 1e-10, 1e-12, "decode state")
    yf, hf = orc.fwd(x, dr, A, Bm, Cm, D=Dv, z=z, delta_bias=bias, h0=h0)
    _close(np.stack(ys, axis=1), yf, 1e-13, 1e-14, "decode vs fwd")


def pin_p1_numpy_example(orc):
    """[P1] "Vi du Python": the page's worked example (L=8, N=4, seed 0,
    A = -exp(linspace(-1, 0.5, N)), Delta = log1p(exp(normal)), zero-order
    hold) evaluates the states twice, sequentially and by composing affine
    maps, and states that the two differ by floating-point error only.  The
    draws are regenerated from the recipe in tests/golden/p1_numpy_example.json;
    the oracle's ZOH option, read out one state component at a time
    (C_t = e_n), must give those states."""
    with open(os.path.join(GOLDEN, "p1_numpy_example.json")) as f:
        g = json.load(f)
    L, N = g["L"], g["N"]
    rng = np.random.default_rng(g["seed"])
    draws = {}
    for name, shape in g["draw_order"]:
        draws[name] = rng.normal(size=tuple(shape))
    x = draws["x"]
    Bt = draws["B_t"]
    raw = draws["delta_raw"][:, 0]
    A = -np.exp(np.linspace(g["A_linspace"][0], g["A_linspace"][1], N))
    dt = np.log1p(np.exp(raw))
    abar = np.exp(dt[:, None] * A[None, :])
    bbar = np.expm1(dt[:, None] * A[None, :]) / A[None, :] * Bt
    bx = bbar * x[:, None]
    seq = np.zeros((L, N))
    h = np.zeros(N)
    for t in range(L):
        h = abar[t] * h + bx[t]
        seq[t] = h
    tree = tree_scan_states(abar, bx, np.zeros(N))
    assert np.max(np.abs(seq - tree)) <= g["max_error_bound"], "page's own claim"
    for n in range(N):
        Cm = np.zeros((1, L, N))
        Cm[0, :, n] = 1.0
        y, hl = orc.fwd(x.reshape(1, L, 1), raw.reshape(1, L, 1), A.reshape(1, N),
                        Bt.reshape(1, L, N), Cm, delta_softplus=True, zoh=True)
        _close(y[0, :, 0], seq[:, n], 1e-12, 1e-14, f"P1 example state n={n}")
        _close(hl[0, 0, n], seq[-1, n], 1e-12, 1e-14, "P1 example final state")


def pin_p3_shape_example(orc):
    """[P3] worked example: batch=2, seq_len=6, d=4, A = sigmoid(randn),
    h0 = zeros(batch, d) gives an output of shape (2, 6, 4).  Values checked
    against the unrolled products (x_j's weight in y_t is C_t A_t..A_{j+1} B_j)."""
    with open(os.path.join(GOLDEN, "p3_shape_example.json")) as f:
        g = json.load(f)
    bsz, sl, d = g["batch"], g["seq_len"], g["d"]
    rng = np.random.default_rng(g["seed"])
    x, B, C = (rng.standard_normal((bsz, sl, d)) for _ in range(3))
    A = 1.0 / (1.0 + np.exp(-rng.standard_normal((bsz, sl, d))))
    y, hl = orc.direct(x, A, B, C, h0=np.zeros((bsz, d)))
    assert list(y.shape) == g["output_shape"]
    want = np.zeros_like(y)
    for t in range(sl):
        acc = np.zeros((bsz, d))
        for j in range(t + 1):
            w = np.ones((bsz, d))
            for i in range(j + 1, t + 1):
                w = w * A[:, i]
            acc += w * B[:, j] * x[:, j]
        want[:, t] = C[:, t] * acc
    _close(y, want, 1e-12, 1e-14, "P3 example values")


def _fd_case(orc, rng, options):
    """Analytic gradients of L = sum(w*y) + sum(u*h_last) from orc.bwd against
    central finite differences of orc.fwd, element by element."""
    bsz, sl, d, n = 2, 5, 3, 4
    inp = {"x": rng.standard_normal((bsz, sl, d)), "delta": rng.standard_normal((bsz, sl, d)),
           "A": -np.exp(rng.standard_normal((d, n)) * 0.5),
           "B": rng.standard_normal((bsz, sl, n)), "C": rng.standard_normal((bsz, sl, n))}
    if options:
        inp.update(z=rng.standard_normal((bsz, sl, d)), D=rng.standard_normal(d),
                   delta_bias=rng.standard_normal(d) * 0.3,
                   h0=rng.standard_normal((bsz, d, n)) * 0.5)
    else:
        inp["delta"] = np.abs(inp["delta"]) * 0.3 + 0.05   # Delta itself, softplus off
    w = rng.standard_normal((bsz, sl, d))
    u = rng.standard_normal((bsz, d, n))

    def loss(vals):
        y, hl = orc.fwd(vals["x"], vals["delta"], vals["A"], vals["B"], vals["C"],
                        D=vals.get("D"), z=vals.get("z"), delta_bias=vals.get("delta_bias"),
                        h0=vals.get("h0"), delta_softplus=options)
        return float(np.sum(w * y) + np.sum(u * hl))

    grads = orc.bwd(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], w, D=inp.get("D"),
                    z=inp.get("z"), delta_bias=inp.get("delta_bias"), h0=inp.get("h0"),
                    dh_last=u, delta_softplus=options)
    for name, arr in inp.items():
        fd = np.zeros_like(arr)
        for k in np.ndindex(arr.shape):
            eps = 1e-6 * max(1.0, abs(arr[k]))
            plus = {kk: vv.copy() for kk, vv in inp.items()}
            minus = {kk: vv.copy() for kk, vv in inp.items()}
            plus[name][k] += eps
            minus[name][k] -= eps
            fd[k] = (loss(plus) - loss(minus)) / (2 * eps)
        _close(grads[name], fd, 1e-6, 1e-7 * max(1.0, float(np.max(np.abs(fd)))),
               f"d loss / d {name} ({'all options' if options else 'plain'})")


def pin_backward_finite_differences(orc, seed=18):
    """The backward oracle (reverse-mode chain rule through softplus, the
    exp(Delta A) transition, the Delta B x input, the C readout, the D skip
    and the silu gate) against central finite differences of the forward
    oracle, for every element of every input, with all options on and with
    none."""
    rng = np.random.default_rng(seed)
    _fd_case(orc, rng, True)
    _fd_case(orc, rng, False)


def pin_causal_conv(orc, seed=20):
    """The conv front-end of the x branch ([P5] section 5.3 names the fused
    causal_conv1d): per channel u_t = bias + sum_k w[k] x_{t-(K-1)+k} with
    x = 0 before the sequence, then silu.
    (i) identity taps (0, 0, 0, 1), no bias: the output is silu(x) itself;
    (ii) a hand-computed dyadic case (K = 4, one channel):
         x = (1, 2, -1, 4, 0.5), w = (0.5, -1, 0.25, 2), bias = 0.5:
         u_0 = 0.5 + 2*1                              = 2.5
         u_1 = 0.5 + 0.25*1 + 2*2                     = 4.75
         u_2 = 0.5 - 1*1 + 0.25*2 + 2*(-1)            = -2
         u_3 = 0.5 + 0.5*1 - 1*2 + 0.25*(-1) + 2*4    = 6.75
         u_4 = 0.5 + 0.5*2 - 1*(-1) + 0.25*4 + 2*0.5  = 4.5
    (iii) random taps against numpy's full convolution with the taps
    reversed (a library routine), truncated to the first L outputs;
    (iv) causality: changing x at t0 leaves every output before t0 alone."""
    silu = _silu_ref
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((2, 9, 3))
    w = np.zeros((3, 4))
    w[:, 3] = 1.0
    _close(orc.causal_conv_silu(x, w), silu(x), 1e-15, 1e-15, "identity taps")
    xh = np.array([1.0, 2.0, -1.0, 4.0, 0.5]).reshape(1, 5, 1)
    wh = np.array([[0.5, -1.0, 0.25, 2.0]])
    u = np.array([2.5, 4.75, -2.0, 6.75, 4.5])
    _close(orc.causal_conv_silu(xh, wh, np.array([0.5])).ravel(), silu(u), 1e-15, 1e-15,
           "hand conv")
    Bsz, L, D, K = 2, 17, 5, 4
    x = rng.standard_normal((Bsz, L, D))
    w = rng.standard_normal((D, K))
    bias = rng.standard_normal(D)
    got = orc.causal_conv_silu(x, w, bias)
    want = np.zeros_like(x)
    for b in range(Bsz):
        for d in range(D):
            want[b, :, d] = silu(bias[d] + np.convolve(x[b, :, d], w[d, ::-1])[:L])
    _close(got, want, 1e-13, 1e-14, "conv vs numpy.convolve")
    x2 = x.copy()
    x2[:, 9] += 3.0
    got2 = orc.causal_conv_silu(x2, w, bias)
    _close(got2[:, :9], got[:, :9], 0, 0, "causality")
    assert np.all(np.abs(got2[:, 9] - got[:, 9]) > 0), "the changed token itself moves"


ALL_PINS = [pin_hand_direct, pin_hand_mamba, pin_softplus_values, pin_lti_convolution,
            pin_brute_force, pin_tree_scan, pin_degenerate, pin_skip_and_gate, pin_h0_split,
            pin_decode, pin_p1_numpy_example, pin_p3_shape_example,
            pin_backward_finite_differences, pin_zoh_limits, pin_causal_conv]
