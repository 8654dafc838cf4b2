"""ssm_scan_fwd_noalloc, the allocation-free forward entry point, for callers
that cannot call cudaMalloc (an allocator that owns the device up front, a
plugin that must not bypass its host's allocator).  Called through the C ABI
and checked against the plan-based ssm_scan_fwd on the same inputs, twice in
a row (the entry point reuses its fixed scratch between calls).

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

import gpu_util as gu
from selective_state_space_31_b200 import binding as bnd
from selective_state_space_31_b200 import synth

pytestmark = pytest.mark.gpu


def _noalloc_fn():
    lib = bnd.load_library()
    fn = lib.ssm_scan_fwd_noalloc
    fn.argtypes = [ctypes.POINTER(bnd.Desc)] + [ctypes.c_void_p] * 12
    fn.restype = ctypes.c_int
    return fn


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


@pytest.mark.parametrize("shape,dt,zoh", [((4, 1000, 256, 16), "bf16", False),
                                          ((2, 333, 64, 8), "f32", False),
                                          ((2, 333, 64, 16), "bf16", True)])
def test_noalloc_matches_plan_entry_point(shape, dt, zoh):
    Bz, L, D, N = shape
    inp = synth.make_fwd(Bz, L, D, N, in_dtype=dt, seed=41, has_h0=True, zoh=zoh)
    dev = gu.upload(inp)
    plan = gu.make_plan(inp)
    y_ref, h_ref = gu.run_gpu(inp, plan, dev)
    fn = _noalloc_fn()
    desc = plan.desc
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        y = torch.full((Bz, L, D), float("nan"), dtype=gu.TDT[dt], device="cuda")
        hl = torch.full((Bz, D, N), float("nan"), dtype=torch.float32, device="cuda")
        rc = fn(ctypes.byref(desc), _ptr(dev["x"]), _ptr(dev["delta"]), _ptr(dev["delta_bias"]),
                _ptr(dev["A"]), _ptr(dev["B"]), _ptr(dev["C"]), _ptr(dev["D"]), _ptr(dev["z"]),
                _ptr(dev["h0"]), _ptr(y), _ptr(hl), ctypes.c_void_p(stream))
        assert rc == bnd.OK, bnd.status_string(rc)
        torch.cuda.synchronize()
        gy = y.float().cpu().numpy().astype(np.float64)
        gh = hl.cpu().numpy().astype(np.float64)
        gu.assert_parity(gy, y_ref, gh, h_ref, gu.TOL[dt], f"noalloc call {call}")


def test_noalloc_rejects_problems_beyond_its_scratch():
    fn = _noalloc_fn()
    # 64 x 8192 channels x 16 states of fp32 carry need 32 MiB > the fixed 4 MiB
    desc = bnd.Desc(64, 4096, 8192, 16, bnd.BF16, bnd.BF16,
                    bnd.DELTA_SOFTPLUS | bnd.WANT_HLAST)
    dummy = torch.empty(16, dtype=torch.float32, device="cuda")
    p = _ptr(dummy)
    rc = fn(ctypes.byref(desc), p, p, None, p, p, p, None, None, None, p, p, None)
    assert rc == bnd.ERR_UNSUPPORTED
