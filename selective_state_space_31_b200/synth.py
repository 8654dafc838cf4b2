"""Seeded synthetic inputs for the selective scan.

This module holds no part of the scan's arithmetic: it only draws random
numbers, rounds them to the storage dtype and lays them out.  Both the CUDA
path (through the tests and the benchmark) and the CPU oracle are fed from
here.

Every field is drawn from its own numpy ``default_rng([seed, field])`` stream
in float32 and, for bf16 workloads, rounded to bf16 with round-to-nearest-even.
The arrays handed out are float32 arrays whose values are exactly
representable in the storage dtype, so uploading them as bf16 is lossless and
the oracle sees exactly the stored values.

Workloads (shapes and value distributions of the five standard cases):

* ``tiny_fp32``      B=1, L=512, D=64, N=16, fp32; x, B, C ~ N(0,1);
  delta_raw = N(0,1) - 1 (softplus applied in the scan); A[d,n] = -(n+1);
  D ~ N(0,1); h0 = 0; no gate; seed 0.
* ``mamba130m_layer`` B=8, L=2048, D=1536, N=16, bf16 in/out; x, delta_raw, z,
  B, C ~ N(0,1); bias[d] = log(expm1(u)), u ~ U[1e-3, 0.1]; A = -(n+1) fp32;
  D ~ N(0,1) fp32; silu(z) gate on.
* ``mamba1p4b_layer`` B=4, L=8192, D=4096, N=16, same distributions, plus
  h0 ~ N(0, 0.1^2) fp32 (0.1 read as the standard deviation).
* ``long_seq``       B=1, L=131072, D=2560, N=16, same distributions.
* ``decode``         B=256, D=5120, N=16, 1024 single-token steps; per step
  x, delta_raw, z (B, D) and B, C (B, N) bf16 ~ N(0,1); bias, A, D as above;
  h0 ~ N(0, 0.1^2) fp32.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

# field ids: one independent random stream per field
_F_X, _F_DELTA, _F_Z, _F_B, _F_C, _F_BIAS, _F_D, _F_H0, _F_A, _F_CONV_W, _F_CONV_B = range(11)


def round_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); return them as
    float32.  NaN/Inf are not produced by the generators and not handled."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return (u.astype(np.uint32) << 16).view(np.float32)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """uint16 bit patterns of float32 values that are exactly bf16."""
    return (np.ascontiguousarray(a, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _rng(seed, fid, *extra):
    return np.random.default_rng([int(seed), int(fid), *[int(e) for e in extra]])


def _normal(seed, fid, shape, dtype, *extra, scale=1.0, shift=0.0):
    a = _rng(seed, fid, *extra).standard_normal(size=shape, dtype=np.float32)
    if scale != 1.0:
        a *= np.float32(scale)
    if shift != 0.0:
        a += np.float32(shift)
    return round_bf16(a) if dtype == "bf16" else a


def s4d_real_A(D: int, N: int) -> np.ndarray:
    """A[d, n] = -(n + 1) (S4D-real initialisation), fp32 (D, N)."""
    return np.ascontiguousarray(np.broadcast_to(-(np.arange(N, dtype=np.float32) + 1.0), (D, N)))


def dt_bias(seed: int, D: int) -> np.ndarray:
    """bias[d] = log(expm1(u)), u ~ U[1e-3, 0.1] (inverse-softplus init), fp32."""
    u = _rng(seed, _F_BIAS).uniform(1e-3, 0.1, size=D)
    return np.log(np.expm1(u)).astype(np.float32)


@dataclass
class ScanInputs:
    """One forward-pass workload.  Float32 arrays hold values exact in
    ``in_dtype``; optional fields are None when the workload has none."""
    name: str
    Bsz: int
    L: int
    D: int
    N: int
    in_dtype: str          # "f32" or "bf16"
    out_dtype: str
    x: np.ndarray
    delta: np.ndarray
    A: np.ndarray
    B: np.ndarray
    C: np.ndarray
    Dskip: np.ndarray | None = None
    z: np.ndarray | None = None
    delta_bias: np.ndarray | None = None
    h0: np.ndarray | None = None
    delta_softplus: bool = True
    want_h_last: bool = True
    zoh: bool = False          # zero-order-hold input matrix instead of Delta * B
    meta: dict = field(default_factory=dict)

    @property
    def updates(self) -> int:
        return self.Bsz * self.L * self.D * self.N


def make_fwd(Bsz, L, D, N, *, in_dtype="bf16", out_dtype=None, seed=0, has_z=True,
             has_D=True, has_bias=True, has_h0=False, delta_softplus=True,
             delta_shift=0.0, A=None, name="custom", zoh=False) -> ScanInputs:
    """Generic seeded forward workload with the standard distributions."""
    out_dtype = out_dtype or in_dtype
    x = _normal(seed, _F_X, (Bsz, L, D), in_dtype)
    delta = _normal(seed, _F_DELTA, (Bsz, L, D), in_dtype, shift=delta_shift)
    Bm = _normal(seed, _F_B, (Bsz, L, N), in_dtype)
    Cm = _normal(seed, _F_C, (Bsz, L, N), in_dtype)
    z = _normal(seed, _F_Z, (Bsz, L, D), in_dtype) if has_z else None
    Dv = _rng(seed, _F_D).standard_normal(D, dtype=np.float32) if has_D else None
    bias = dt_bias(seed, D) if has_bias else None
    h0 = (_rng(seed, _F_H0).standard_normal((Bsz, D, N), dtype=np.float32) * np.float32(0.1)
          if has_h0 else None)
    A = s4d_real_A(D, N) if A is None else np.ascontiguousarray(A, dtype=np.float32)
    return ScanInputs(name, Bsz, L, D, N, in_dtype, out_dtype, x, delta, A, Bm, Cm, Dv, z,
                      bias, h0, delta_softplus, True, zoh)


def tiny_fp32(seed=0, shape=None):
    """B=1, L=512, D=64, N=16 fp32; delta_raw = N(0,1) - 1; no gate, no bias.
    ``shape`` = (B, L, D) resizes any workload with its distributions kept
    (for profiling on smaller copies)."""
    B, L, D = shape or (1, 512, 64)
    return make_fwd(B, L, D, 16, in_dtype="f32", seed=seed, has_z=False, has_bias=False,
                    has_h0=False, delta_shift=-1.0, name="tiny_fp32")


def mamba130m_layer(seed=1, shape=None):
    B, L, D = shape or (8, 2048, 1536)
    return make_fwd(B, L, D, 16, seed=seed, name="mamba130m_layer")


def mamba1p4b_layer(seed=2, shape=None):
    B, L, D = shape or (4, 8192, 4096)
    return make_fwd(B, L, D, 16, seed=seed, has_h0=True, name="mamba1p4b_layer")


def long_seq(seed=3, shape=None):
    B, L, D = shape or (1, 131072, 2560)
    return make_fwd(B, L, D, 16, seed=seed, name="long_seq")


FWD_WORKLOADS = {
    "tiny_fp32": tiny_fp32,
    "mamba130m_layer": mamba130m_layer,
    "mamba1p4b_layer": mamba1p4b_layer,
    "long_seq": long_seq,
}


@dataclass
class DecodeInputs:
    """Decode workload: constant parameters plus per-step token generators."""
    name: str
    Bsz: int
    D: int
    N: int
    steps: int
    seed: int
    A: np.ndarray
    Dskip: np.ndarray
    delta_bias: np.ndarray
    h0: np.ndarray
    in_dtype: str = "bf16"

    def token(self, t: int):
        """Inputs of step t: dict of x, delta, z (B, D) and B, C (B, N)."""
        s, fid = self.seed, 100
        return {
            "x": _normal(s, fid + _F_X, (self.Bsz, self.D), self.in_dtype, t),
            "delta": _normal(s, fid + _F_DELTA, (self.Bsz, self.D), self.in_dtype, t),
            "z": _normal(s, fid + _F_Z, (self.Bsz, self.D), self.in_dtype, t),
            "B": _normal(s, fid + _F_B, (self.Bsz, self.N), self.in_dtype, t),
            "C": _normal(s, fid + _F_C, (self.Bsz, self.N), self.in_dtype, t),
        }

    @property
    def updates_per_step(self) -> int:
        return self.Bsz * self.D * self.N


def make_decode(Bsz=256, D=5120, N=16, steps=1024, seed=4, name="decode") -> DecodeInputs:
    h0 = _rng(seed, _F_H0).standard_normal((Bsz, D, N), dtype=np.float32) * np.float32(0.1)
    return DecodeInputs(name, Bsz, D, N, steps, seed, s4d_real_A(D, N),
                        _rng(seed, _F_D).standard_normal(D, dtype=np.float32),
                        dt_bias(seed, D), h0)


def make_direct(Bsz, L, D, *, seed=0, in_dtype="f32", has_h0=True, a_zero=False):
    """Elementwise-variant workload: x, B, C ~ N(0,1); A = sigmoid(N(0,1))
    (values in (0,1)), or exactly 0; h0 ~ N(0,1) or None."""
    x = _normal(seed, _F_X, (Bsz, L, D), in_dtype)
    Bm = _normal(seed, _F_B, (Bsz, L, D), in_dtype)
    Cm = _normal(seed, _F_C, (Bsz, L, D), in_dtype)
    if a_zero:
        A = np.zeros((Bsz, L, D), np.float32)
    else:
        g = _rng(seed, _F_A).standard_normal((Bsz, L, D), dtype=np.float32)
        A = (1.0 / (1.0 + np.exp(-g.astype(np.float64)))).astype(np.float32)
        A = round_bf16(A) if in_dtype == "bf16" else A
    h0 = _rng(seed, _F_H0).standard_normal((Bsz, D), dtype=np.float32) if has_h0 else None
    return {"x": x, "A": A, "B": Bm, "C": Cm, "h0": h0, "in_dtype": in_dtype}


def make_conv(D: int, width: int = 4, seed: int = 0):
    """Taps and bias of the causal conv front-end of the x branch, fp32:
    w (D, width) and b (D,) ~ U(-1/sqrt(width), 1/sqrt(width)) (the uniform
    fan-in initialisation of a depthwise convolution with `width` taps)."""
    bound = 1.0 / np.sqrt(width)
    w = _rng(seed, _F_CONV_W).uniform(-bound, bound, size=(D, width)).astype(np.float32)
    b = _rng(seed, _F_CONV_B).uniform(-bound, bound, size=D).astype(np.float32)
    return w, b
