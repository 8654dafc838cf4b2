"""The fitted polynomials in the device code match the scripts that derive
them (csrc/fit_log1p.py, csrc/fit_exp2.py), and their float32 error bounds
hold.  No GPU needed."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "selective_state_space_31_b200", "csrc")


def _load(name):
    spec = importlib.util.spec_from_file_location(name, os.path.join(CSRC, name + ".py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _device_constants(func):
    src = open(os.path.join(CSRC, "device_common.cuh")).read()
    body = src[src.index(func):]
    body = body[:body.index("\n}\n")]
    return {float(v) for v in re.findall(r"(-?\d+\.\d+(?:e-?\d+)?)f", body)}


def test_log1p_coefficients_match_the_fit():
    fit = _load("fit_log1p")
    coef = fit.fit(8)
    consts = _device_constants("float log1p_unit(float u)")
    for c in coef[1:]:          # (the constant term is written as 1.0f)
        assert any(abs(float(c) - k) <= 1e-9 * max(1.0, abs(k)) for k in consts), float(c)
    assert fit.max_rel_error(coef) < 2.5e-7


def test_exp2_coefficients_match_the_fit():
    fit = _load("fit_exp2")
    coef = fit.fit(4)
    consts = _device_constants("float2 exp2_fma2(float2 x)")
    for c in coef:
        assert any(abs(float(c) - k) <= 1e-9 * max(1.0, abs(k)) for k in consts), float(c)
    assert fit.max_rel_error(coef) < 2.0e-7


def test_exp2_reduction_emulated_in_float32():
    """The device function's steps in numpy float32 (round to an integer by
    the 1.5 * 2^23 addition, polynomial, exponent add) against float64 2^x,
    including the clamp ends and exact powers of two at integers."""
    fit = _load("fit_exp2")
    coef = fit.fit(4)
    x = np.concatenate([np.linspace(-124.9, 126.9, 200001), np.arange(-125, 128)]).astype(np.float32)
    xc = np.clip(x, np.float32(-125), np.float32(127))
    magic = np.float32(12582912.0)
    t = (xc + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    f = (xc - n).astype(np.float32)
    p = fit.evaluate(coef, f)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    y = bits.view(np.float32).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(y - ref) / ref) < 2.5e-7
    ints = np.arange(-125, 128)
    yi = y[-len(ints):]
    assert np.array_equal(yi, np.exp2(ints.astype(np.float64)))
