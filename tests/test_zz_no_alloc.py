"""ssm_scan_fwd_noalloc, the allocation-free forward entry point, for callers
that cannot call cudaMalloc (an allocator that owns the device up front, a
plugin that must not bypass its host's allocator).  Called through the C ABI
and checked against the plan-based ssm_scan_fwd on the same inputs, twice in
a row (the entry point reuses its fixed scratch between calls): both run the
same kernel in the same launch shape, so the results must be bit-identical;
one call is also compared with the CPU oracle directly.

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


def _lib():
    lib = bnd.load_library()
    lib.ssm_scan_fwd_noalloc.argtypes = [ctypes.POINTER(bnd.Desc)] + [ctypes.c_void_p] * 12
    lib.ssm_scan_fwd_noalloc.restype = ctypes.c_int
    lib.ssm_scan_noalloc_status.argtypes = []
    lib.ssm_scan_noalloc_status.restype = ctypes.c_int
    lib.ssm_scan_noalloc_set_debug.argtypes = [ctypes.c_uint64, ctypes.c_int64]
    lib.ssm_scan_noalloc_set_debug.restype = ctypes.c_int
    return lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _call(lib, desc, dev, y, hl):
    stream = torch.cuda.current_stream().cuda_stream
    return lib.ssm_scan_fwd_noalloc(
        ctypes.byref(desc), _ptr(dev["x"]), _ptr(dev["delta"]), _ptr(dev["delta_bias"]),
        _ptr(dev["A"]), _ptr(dev["B"]), _ptr(dev["C"]), _ptr(dev["D"]), _ptr(dev["z"]),
        _ptr(dev["h0"]), _ptr(y), _ptr(hl), ctypes.c_void_p(stream))


@pytest.mark.parametrize("shape,dt,zoh", [((4, 1000, 256, 16), "bf16", False),
                                          ((2, 333, 64, 8), "f32", False),
                                          ((2, 333, 64, 16), "bf16", True),
                                          ((8, 512, 1536, 16), "bf16", False)])
def test_noalloc_matches_plan_entry_point(shape, dt, zoh):
    Bz, L, D, N = shape
    inp = synth.make_fwd(Bz, L, D, N, in_dtype=dt, seed=41, has_h0=True, zoh=zoh)
    dev = gu.upload(inp)
    plan = gu.make_plan(inp)
    plan.set_config(segments=1)   # the launch shape the allocation-free entry point takes
    y_ref, h_ref = gu.run_gpu(inp, plan, dev)
    lib = _lib()
    for call in range(2):
        y = torch.full((Bz, L, D), float("nan"), dtype=gu.TDT[dt], device="cuda")
        hl = torch.full((Bz, D, N), float("nan"), dtype=torch.float32, device="cuda")
        rc = _call(lib, plan.desc, dev, y, hl)
        assert rc == bnd.OK, bnd.status_string(rc)
        assert lib.ssm_scan_noalloc_status() == bnd.OK
        gy = y.float().cpu().numpy().astype(np.float64)
        gh = hl.cpu().numpy().astype(np.float64)
        assert np.array_equal(gy, y_ref), f"call {call}: y differs from the plan entry point"
        assert np.array_equal(gh, h_ref), f"call {call}: h_last differs from the plan entry point"
        if call == 0:
            ry, rh = gu.run_oracle(inp)
            gu.assert_parity(gy, ry, gh, rh, gu.TOL[dt], "noalloc against the oracle")


def test_noalloc_rejects_problems_beyond_its_scratch():
    lib = _lib()
    # 64 x 8192 channels x 16 states of fp32 carry need 32 MiB > the fixed 4 MiB
    desc = bnd.Desc(64, 4096, 8192, 16, bnd.BF16, bnd.BF16,
                    bnd.DELTA_SOFTPLUS | bnd.WANT_HLAST)
    dummy = torch.empty(16, dtype=torch.float32, device="cuda")
    p = _ptr(dummy)
    fn = lib.ssm_scan_fwd_noalloc
    rc = fn(ctypes.byref(desc), p, p, None, p, p, p, None, None, None, p, p, None)
    assert rc == bnd.ERR_UNSUPPORTED
    # dstate outside what the fast path takes: rejected before anything runs
    bad = bnd.Desc(1, 64, 64, (1 << 32) + 16, bnd.BF16, bnd.BF16, bnd.DELTA_SOFTPLUS)
    assert fn(ctypes.byref(bad), p, p, None, p, p, p, None, None, None, p, None, None) \
        == bnd.ERR_UNSUPPORTED


def test_noalloc_timeout_is_reported():
    """A part that never hands its state on makes the CTA running the next
    part of that row wait until the bound expires: the call's status query
    reports SSM_ERR_TIMEOUT, and the next call is exact again."""
    inp = synth.make_fwd(8, 512, 1536, 16, seed=43)
    dev = gu.upload(inp)
    plan = gu.make_plan(inp)
    plan.set_config(segments=1)   # the launch shape the allocation-free entry point takes
    info = plan.info()
    assert info["parts_per_row"] >= 2, info
    y_ref, h_ref = gu.run_gpu(inp, plan, dev)
    lib = _lib()
    y = torch.empty((8, 512, 1536), dtype=torch.bfloat16, device="cuda")
    hl = torch.empty((8, 1536, 16), dtype=torch.float32, device="cuda")
    # the first part of row 0 ends at stage PL - 1; the CTA running part 2 of row 0 waits for it
    lib.ssm_scan_noalloc_set_debug(50_000_000, info["stages_per_part"] - 1)
    try:
        assert _call(lib, plan.desc, dev, y, hl) == bnd.OK
        assert lib.ssm_scan_noalloc_status() == bnd.ERR_TIMEOUT
    finally:
        lib.ssm_scan_noalloc_set_debug(0, -1)
    assert lib.ssm_scan_noalloc_status() == bnd.OK
    assert _call(lib, plan.desc, dev, y, hl) == bnd.OK
    assert lib.ssm_scan_noalloc_status() == bnd.OK
    assert np.array_equal(y.float().cpu().numpy().astype(np.float64), y_ref)
    assert np.array_equal(hl.cpu().numpy().astype(np.float64), h_ref)
