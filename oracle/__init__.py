"""CPU oracle for the selective scan: TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference leg may import this package.  The library under
``selective_state_space_31_b200`` never imports it, and it imports nothing
from that library.

The arithmetic lives in ``ssm_oracle.c`` (plain C, every step in double);
this module only compiles it with gcc and marshals numpy arrays through
ctypes.  See that file's header for the passages each function restates.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssm_oracle.c")

HAS_Z = 1
HAS_D = 2
SOFTPLUS = 4
HAS_BIAS = 8
HAS_H0 = 16
ZOH = 128

_dp = ctypes.POINTER(ctypes.c_double)
_build_lock = threading.Lock()


def lib_path(mutant: int = 0, fp32: bool = False) -> str:
    if fp32:
        return os.path.join(_HERE, "libssm_oracle_fp32.so")
    name = "libssm_oracle.so" if mutant == 0 else f"libssm_oracle_mutant{mutant}.so"
    return os.path.join(_HERE, name)


def build(mutant: int = 0, force: bool = False, fp32: bool = False) -> str:
    """Compile the oracle (optionally with one planted mistake) with gcc.
    ``fp32`` builds the single-precision-accumulate forward loop used only as
    a timed CPU baseline (never for parity)."""
    out = lib_path(mutant, fp32)
    with _build_lock:
        if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(_SRC):
            cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", f"-DORACLE_MUTANT={mutant}"]
            if fp32:
                cmd.append("-DORACLE_FP32")
            cmd += ["-o", out + ".tmp", _SRC, "-lm"]
            subprocess.check_call(cmd)
            os.replace(out + ".tmp", out)
    return out


def _arr(a, shape=None):
    if a is None:
        return None
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float64))
    if shape is not None and a.shape != tuple(shape):
        a = a.reshape(shape)
    return a


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_dp)


class Oracle:
    """ctypes front end of one compiled oracle build."""

    def __init__(self, mutant: int = 0, fp32: bool = False):
        self.mutant, self.fp32 = mutant, fp32
        self._lib = ctypes.CDLL(build(mutant, fp32=fp32))
        i64, u32 = ctypes.c_int64, ctypes.c_uint32
        self._lib.ssm_oracle_fwd.argtypes = [i64, i64, i64, i64, u32] + [_dp] * 11
        self._lib.ssm_oracle_fwd.restype = ctypes.c_int
        self._lib.ssm_oracle_softplus.argtypes = [ctypes.c_double]
        self._lib.ssm_oracle_softplus.restype = ctypes.c_double
        self._lib.ssm_oracle_silu.argtypes = [ctypes.c_double]
        self._lib.ssm_oracle_silu.restype = ctypes.c_double
        if fp32:   # the timing build has the forward loop only
            return
        self._lib.ssm_oracle_step.argtypes = [i64, i64, i64, u32] + [_dp] * 10
        self._lib.ssm_oracle_step.restype = ctypes.c_int
        self._lib.ssm_oracle_direct.argtypes = [i64, i64, i64] + [_dp] * 7
        self._lib.ssm_oracle_direct.restype = ctypes.c_int
        self._lib.ssm_oracle_bwd.argtypes = [i64, i64, i64, i64, u32] + [_dp] * 20
        self._lib.ssm_oracle_bwd.restype = ctypes.c_int
        self._lib.ssm_oracle_causal_conv_silu.argtypes = [i64, i64, i64, i64] + [_dp] * 4
        self._lib.ssm_oracle_causal_conv_silu.restype = ctypes.c_int

    def softplus(self, v: float) -> float:
        return self._lib.ssm_oracle_softplus(float(v))

    def silu(self, z: float) -> float:
        return self._lib.ssm_oracle_silu(float(z))

    def fwd(self, x, delta, A, B, C, D=None, z=None, delta_bias=None, h0=None,
            delta_softplus=True, zoh=False):
        """Mamba-form scan.  x, delta, z: (Bsz, L, Dm); B, C: (Bsz, L, N);
        A: (Dm, N); D, delta_bias: (Dm,); h0: (Bsz, Dm, N).
        Returns (y (Bsz, L, Dm), h_last (Bsz, Dm, N)) as float64 arrays."""
        x = _arr(x)
        Bsz, L, Dm = x.shape
        A = _arr(A)
        N = A.shape[1]
        delta = _arr(delta, x.shape)
        Bm = _arr(B, (Bsz, L, N))
        Cm = _arr(C, (Bsz, L, N))
        z = _arr(z, x.shape)
        Dv = _arr(D, (Dm,))
        bias = _arr(delta_bias, (Dm,))
        h0 = _arr(h0, (Bsz, Dm, N))
        flags = ((HAS_Z if z is not None else 0) | (HAS_D if Dv is not None else 0)
                 | (SOFTPLUS if delta_softplus else 0) | (HAS_BIAS if bias is not None else 0)
                 | (HAS_H0 if h0 is not None else 0) | (ZOH if zoh else 0))
        y = np.empty((Bsz, L, Dm), np.float64)
        hl = np.empty((Bsz, Dm, N), np.float64)
        rc = self._lib.ssm_oracle_fwd(Bsz, L, Dm, N, flags, _ptr(x), _ptr(delta), _ptr(bias),
                                      _ptr(A), _ptr(Bm), _ptr(Cm), _ptr(Dv), _ptr(z), _ptr(h0),
                                      _ptr(y), _ptr(hl))
        if rc != 0:
            raise ValueError("oracle fwd rejected its arguments")
        return y, hl

    def causal_conv_silu(self, x_in, w, bias=None):
        """silu(causal depthwise conv of x_in (Bsz, L, D) with w (D, K) and
        bias (D,)), float64 (Bsz, L, D)."""
        x_in = _arr(x_in)
        Bsz, L, Dm = x_in.shape
        w = _arr(w)
        K = w.shape[1]
        bias = _arr(bias, (Dm,))
        out = np.empty_like(x_in)
        rc = self._lib.ssm_oracle_causal_conv_silu(Bsz, L, Dm, K, _ptr(x_in), _ptr(w), _ptr(bias),
                                                   _ptr(out))
        if rc != 0:
            raise ValueError("oracle conv rejected its arguments")
        return out

    def fwd_conv(self, x_in, conv_w, conv_b, delta, A, B, C, **kw):
        """The scan fed by the conv front-end: x = silu(causal_conv(x_in));
        returns (y, h_last, x)."""
        x = self.causal_conv_silu(x_in, conv_w, conv_b)
        y, hl = self.fwd(x, delta, A, B, C, **kw)
        return y, hl, x

    def bwd(self, x, delta, A, B, C, dy, D=None, z=None, delta_bias=None, h0=None,
            dh_last=None, delta_softplus=True):
        """Gradients of the Mamba-form scan (Delta*B coefficient) for
        dL/dy = dy (Bsz, L, Dm) and dL/dh_last = dh_last (Bsz, Dm, N) or None.
        Returns a dict with x, delta, A, B, C and, where given, D, z,
        delta_bias, h0 (float64 arrays shaped like the inputs)."""
        x = _arr(x)
        Bsz, L, Dm = x.shape
        A = _arr(A)
        N = A.shape[1]
        delta = _arr(delta, x.shape)
        Bm = _arr(B, (Bsz, L, N))
        Cm = _arr(C, (Bsz, L, N))
        z = _arr(z, x.shape)
        Dv = _arr(D, (Dm,))
        bias = _arr(delta_bias, (Dm,))
        h0 = _arr(h0, (Bsz, Dm, N))
        dy = _arr(dy, x.shape)
        dhl = _arr(dh_last, (Bsz, Dm, N))
        flags = ((HAS_Z if z is not None else 0) | (HAS_D if Dv is not None else 0)
                 | (SOFTPLUS if delta_softplus else 0) | (HAS_BIAS if bias is not None else 0)
                 | (HAS_H0 if h0 is not None else 0))
        out = {"x": np.empty_like(x), "delta": np.empty_like(x), "A": np.empty_like(A),
               "B": np.empty_like(Bm), "C": np.empty_like(Cm)}
        if Dv is not None:
            out["D"] = np.empty_like(Dv)
        if z is not None:
            out["z"] = np.empty_like(z)
        if bias is not None:
            out["delta_bias"] = np.empty_like(bias)
        out["h0"] = np.empty((Bsz, Dm, N), np.float64)
        g = lambda k: _ptr(out.get(k))
        rc = self._lib.ssm_oracle_bwd(Bsz, L, Dm, N, flags, _ptr(x), _ptr(delta), _ptr(bias),
                                      _ptr(A), _ptr(Bm), _ptr(Cm), _ptr(Dv), _ptr(z), _ptr(h0),
                                      _ptr(dy), _ptr(dhl), g("x"), g("delta"), g("delta_bias"),
                                      g("A"), g("B"), g("C"), g("D"), g("z"), g("h0"))
        if rc != 0:
            raise ValueError("oracle bwd rejected its arguments")
        return out

    def step(self, state, x, delta, A, B, C, D=None, z=None, delta_bias=None,
             delta_softplus=True):
        """One decode step.  state: (Bsz, Dm, N) (not modified; a new array is
        returned); x, delta, z: (Bsz, Dm); B, C: (Bsz, N).
        Returns (y (Bsz, Dm), new_state)."""
        st = np.array(state, dtype=np.float64, copy=True, order="C")
        Bsz, Dm, N = st.shape
        x = _arr(x, (Bsz, Dm))
        delta = _arr(delta, (Bsz, Dm))
        A = _arr(A, (Dm, N))
        Bm = _arr(B, (Bsz, N))
        Cm = _arr(C, (Bsz, N))
        z = _arr(z, (Bsz, Dm))
        Dv = _arr(D, (Dm,))
        bias = _arr(delta_bias, (Dm,))
        flags = ((HAS_Z if z is not None else 0) | (HAS_D if Dv is not None else 0)
                 | (SOFTPLUS if delta_softplus else 0) | (HAS_BIAS if bias is not None else 0))
        y = np.empty((Bsz, Dm), np.float64)
        rc = self._lib.ssm_oracle_step(Bsz, Dm, N, flags, _ptr(x), _ptr(delta), _ptr(bias),
                                       _ptr(A), _ptr(Bm), _ptr(Cm), _ptr(Dv), _ptr(z),
                                       _ptr(st), _ptr(y))
        if rc != 0:
            raise ValueError("oracle step rejected its arguments")
        return y, st

    def direct(self, x, A, B, C, h0=None):
        """Elementwise variant: all of x, A, B, C are (Bsz, L, Dm); h0 (Bsz, Dm).
        Returns (y (Bsz, L, Dm), h_last (Bsz, Dm))."""
        x = _arr(x)
        Bsz, L, Dm = x.shape
        A = _arr(A, x.shape)
        Bm = _arr(B, x.shape)
        Cm = _arr(C, x.shape)
        h0 = _arr(h0, (Bsz, Dm))
        y = np.empty((Bsz, L, Dm), np.float64)
        hl = np.empty((Bsz, Dm), np.float64)
        rc = self._lib.ssm_oracle_direct(Bsz, L, Dm, _ptr(x), _ptr(A), _ptr(Bm), _ptr(Cm),
                                         _ptr(h0), _ptr(y), _ptr(hl))
        if rc != 0:
            raise ValueError("oracle direct rejected its arguments")
        return y, hl


_default = None
_fp32 = None


def get() -> Oracle:
    """The unmutated oracle (built on first use)."""
    global _default
    if _default is None:
        _default = Oracle(0)
    return _default


def get_fp32() -> Oracle:
    """The fp32-accumulate timing build (forward loop only)."""
    global _fp32
    if _fp32 is None:
        _fp32 = Oracle(0, fp32=True)
    return _fp32


def channel_blocks(Bsz: int, D: int, width: int = 64):
    """Every channel of a (Bsz, ., D) problem as blocks (b, d0, d1) of at
    most ``width`` channels, batch-major."""
    return [(b, d0, min(D, d0 + width)) for b in range(Bsz) for d0 in range(0, D, width)]


def fwd_blocks(x, delta, A, B, C, blocks, consume, D=None, z=None, delta_bias=None, h0=None,
               delta_softplus=True, zoh=False, threads=None, oracle: Oracle | None = None):
    """Run the oracle over channel blocks (b, d0, d1) on a pool of host
    threads (the C loop runs without the GIL).  Each block is an independent
    sub-problem (batch 1, channels d0..d1) cut out of the full arrays;
    ``consume((b, d0, d1), y, h_last)`` receives its float64 results
    (y: (L, d1-d0), h_last: (d1-d0, N)) on a worker thread.  B and C are
    converted to float64 once per batch element.  Returns the thread count."""
    import concurrent.futures as cf

    orc = oracle or get()
    threads = threads or os.cpu_count() or 1
    bc = {}
    for b in sorted({blk[0] for blk in blocks}):
        bc[b] = (np.ascontiguousarray(np.asarray(B)[b:b + 1], dtype=np.float64),
                 np.ascontiguousarray(np.asarray(C)[b:b + 1], dtype=np.float64))
    A = np.asarray(A)

    def one(blk):
        b, d0, d1 = blk
        sl = lambda a: None if a is None else np.asarray(a)[b:b + 1, :, d0:d1]
        Bb, Cb = bc[b]
        y, hl = orc.fwd(sl(x), sl(delta), A[d0:d1], Bb, Cb,
                        None if D is None else np.asarray(D)[d0:d1], sl(z),
                        None if delta_bias is None else np.asarray(delta_bias)[d0:d1],
                        None if h0 is None else np.asarray(h0)[b:b + 1, d0:d1],
                        delta_softplus=delta_softplus, zoh=zoh)
        consume(blk, y[0], hl[0])

    with cf.ThreadPoolExecutor(max_workers=threads) as ex:
        for f in [ex.submit(one, blk) for blk in blocks]:
            f.result()
    return threads


def fwd_rows(x, delta, A, B, C, rows, D=None, z=None, delta_bias=None, h0=None,
             delta_softplus=True, oracle: Oracle | None = None, zoh=False):
    """Run the oracle on selected channels only.  ``rows`` is a list of (b, d)
    pairs; every array keeps its full layout and only the needed slices are
    copied.  Returns (y[len(rows), L], h_last[len(rows), N])."""
    orc = oracle or get()
    ys, hs = [], []
    for (b, d) in rows:
        sl = lambda a: None if a is None else np.asarray(a)[b:b + 1, :, d:d + 1]
        yb, hb = orc.fwd(sl(x), sl(delta), np.asarray(A)[d:d + 1], np.asarray(B)[b:b + 1],
                         np.asarray(C)[b:b + 1],
                         None if D is None else np.asarray(D)[d:d + 1], sl(z),
                         None if delta_bias is None else np.asarray(delta_bias)[d:d + 1],
                         None if h0 is None else np.asarray(h0)[b:b + 1, d:d + 1],
                         delta_softplus=delta_softplus, zoh=zoh)
        ys.append(yb[0, :, 0])
        hs.append(hb[0, 0])
    return np.stack(ys), np.stack(hs)
