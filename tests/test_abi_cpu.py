"""The C-ABI library loads and exports every entry point declared in
include/*.h, and rejects bad arguments synchronously (no GPU needed)."""
import ctypes
import glob
import os
import re

import pytest
import torch

from selective_state_space_31_b200 import binding as bnd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        names += re.findall(r"SSM_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    from selective_state_space_31_b200 import build
    build.build()
    return bnd.load_library()


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 10
    raw = ctypes.CDLL(bnd.LIB_PATH)
    missing = [n for n in names if not hasattr(raw, n)]
    assert not missing, missing


def test_flag_and_status_values_match_the_header():
    """The binding's flag, dtype and status constants are the values the C
    header defines."""
    src = open(os.path.join(ROOT, "include", "ssm_scan.h")).read()
    defined = {name: int(val) for name, val in re.findall(r"\b(SSM_[A-Z0-9_]+)\s*=\s*(\d+)", src)}
    expect = {"SSM_HAS_Z": bnd.HAS_Z, "SSM_HAS_D": bnd.HAS_D,
              "SSM_DELTA_SOFTPLUS": bnd.DELTA_SOFTPLUS, "SSM_HAS_DELTA_BIAS": bnd.HAS_DELTA_BIAS,
              "SSM_HAS_H0": bnd.HAS_H0, "SSM_WANT_HLAST": bnd.WANT_HLAST,
              "SSM_A_DIRECT": bnd.A_DIRECT, "SSM_ZOH": bnd.ZOH, "SSM_F32": bnd.F32,
              "SSM_BF16": bnd.BF16, "SSM_OK": bnd.OK, "SSM_ERR_INVALID_ARG": bnd.ERR_INVALID_ARG}
    for name, val in expect.items():
        assert defined.get(name) == val, (name, defined.get(name), val)


def test_status_strings(lib):
    for s in range(7):
        assert bnd.status_string(s)
    assert lib.ssm_scan_version() >= 100


def _create(lib, **kw):
    d = dict(batch=1, seqlen=8, dim=16, dstate=16, in_dtype=bnd.BF16, out_dtype=bnd.BF16,
             flags=bnd.WANT_HLAST | bnd.DELTA_SOFTPLUS)
    d.update(kw)
    desc = bnd.Desc(d["batch"], d["seqlen"], d["dim"], d["dstate"], d["in_dtype"],
                    d["out_dtype"], d["flags"])
    h = ctypes.c_void_p()
    rc = lib.ssm_scan_create(ctypes.byref(h), ctypes.byref(desc), 0)
    if rc == bnd.OK:
        lib.ssm_scan_destroy(h)
    return rc


@pytest.mark.parametrize("kw,want", [
    (dict(batch=-1), bnd.ERR_INVALID_ARG),
    (dict(dstate=0), bnd.ERR_INVALID_ARG),
    (dict(dstate=65), bnd.ERR_UNSUPPORTED),
    (dict(in_dtype=7), bnd.ERR_INVALID_ARG),
    (dict(flags=1 << 20), bnd.ERR_INVALID_ARG),
    (dict(flags=bnd.A_DIRECT, dstate=4), bnd.ERR_INVALID_ARG),
    (dict(flags=bnd.A_DIRECT | bnd.HAS_Z, dstate=1), bnd.ERR_INVALID_ARG),
    (dict(seqlen=1 << 40), bnd.ERR_UNSUPPORTED),
])
def test_create_validates_before_touching_cuda(lib, kw, want):
    assert _create(lib, **kw) == want


def test_null_arguments(lib):
    assert lib.ssm_scan_create(None, None, 0) == bnd.ERR_INVALID_ARG
    assert lib.ssm_scan_fwd(*([None] * 13)) == bnd.ERR_INVALID_ARG
    assert lib.ssm_scan_fwd_host(*([None] * 12), 0, None) == bnd.ERR_INVALID_ARG
    assert lib.ssm_scan_step_host(*([None] * 11), 0, None) == bnd.ERR_INVALID_ARG
    assert lib.ssm_scan_step(*([None] * 12)) == bnd.ERR_INVALID_ARG
    assert lib.ssm_scan_get_status(None) == bnd.ERR_INVALID_ARG
    assert lib.ssm_scan_destroy(None) == bnd.ERR_INVALID_ARG


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device error path")
def test_valid_desc_without_device_is_a_cuda_error(lib):
    assert _create(lib) == bnd.ERR_CUDA


def test_binding_refuses_missing_library(tmp_path):
    with pytest.raises(RuntimeError):
        # a fresh loader pointed at a path that does not exist
        saved = bnd._lib
        bnd._lib = None
        try:
            bnd.load_library(str(tmp_path / "nope.so"))
        finally:
            bnd._lib = saved


def test_probe_exp2_validates_before_touching_cuda(lib):
    assert lib.ssm_probe_exp2(None, None, None, -1, None) == bnd.ERR_INVALID_ARG
    assert lib.ssm_probe_exp2(None, None, None, 4, None) == bnd.ERR_INVALID_ARG
    assert lib.ssm_probe_exp2(None, None, None, 0, None) == bnd.OK
