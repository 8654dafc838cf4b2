"""The causal conv front-end of the x branch fused into the scan
(ssm_scan_fwd_conv) against the oracle's conv + scan: every compiled conv
variant, segments, the general kernel, the optional conv output, and the
refusals of the entry points that do not take it."""
import numpy as np
import pytest
import torch

import gpu_util as gu
import oracle
from selective_state_space_31_b200 import binding as bnd
from selective_state_space_31_b200 import synth

pytestmark = pytest.mark.gpu


def _conv_case(Bz, L, Dm, N, dt="bf16", seed=71, cfg=None, want_xconv=True, expect_path=None):
    inp = synth.make_fwd(Bz, L, Dm, N, in_dtype=dt, seed=seed, has_h0=True)
    w, cb = synth.make_conv(Dm, seed=seed)
    dev = gu.upload(inp)
    flags = bnd.flags_for(z=inp.z, D=inp.Dskip, delta_bias=inp.delta_bias, h0=inp.h0,
                          conv=True)
    plan = bnd.Plan(Bz, L, Dm, N, gu.TDT[dt], gu.TDT[dt], flags, "cuda")
    if cfg:
        plan.set_config(**cfg)
    info = plan.info()
    if expect_path is not None:
        assert info["path"] == expect_path, info
    xc = torch.full((Bz, L, Dm), float("nan"), dtype=gu.TDT[dt], device="cuda") \
        if want_xconv else None
    y, hl = plan.fwd_conv(dev["x"], gu.dev_tensor(w), dev["delta"], dev["A"], dev["B"], dev["C"],
                          conv_b=gu.dev_tensor(cb), D=dev["D"], z=dev["z"],
                          delta_bias=dev["delta_bias"], h0=dev["h0"], x_conv=xc)
    torch.cuda.synchronize()
    assert plan.status() == 0
    ry, rh, rx = oracle.get().fwd_conv(inp.x, w, cb, inp.delta, inp.A, inp.B, inp.C, D=inp.Dskip,
                                       z=inp.z, delta_bias=inp.delta_bias, h0=inp.h0)
    tol = gu.TOL[dt]
    gy = y.float().cpu().numpy().astype(np.float64)
    gh = hl.cpu().numpy().astype(np.float64)
    gu.assert_parity(gy, ry, gh, rh, tol, f"conv {cfg} {info}")
    if want_xconv:
        gx = xc.float().cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(gx))
        assert gu.normwise(gx, rx) <= tol, gu.normwise(gx, rx)
    plan.close()
    return info


def test_conv_default_bf16():
    info = _conv_case(2, 1000, 256, 16, expect_path=0)
    assert info["path"] == 0


@pytest.mark.parametrize("dt", ["bf16", "f32"])
def test_conv_every_variant(dt):
    vs = [v for v in bnd.list_variants(gu.TDT[dt]) if v["conv"] and not v["carry"]]
    assert vs
    for v in vs:
        for M in (1, 4):
            cfg = dict(lanes_per_chan=v["lanes_per_chan"], warps_per_cta=v["warps_per_cta"],
                       tile_t=v["tile_t"], chans_per_lane=v["chans_per_lane"], segments=M)
            info = _conv_case(2, 1500, 128, v["dstate"], dt=dt, cfg=cfg, want_xconv=M == 1,
                              seed=72)
            assert info["segments"] == M and info["chans_per_lane"] == v["chans_per_lane"]


def test_conv_parts_chained_across_ctas():
    _conv_case(3, 389, 64, 16, cfg=dict(grid=3, segments=1), seed=73)


@pytest.mark.parametrize("shape,dt", [((2, 77, 37, 16), "bf16"), ((1, 130, 24, 12), "f32")])
def test_conv_general_path(shape, dt):
    _conv_case(*shape, dt=dt, seed=74, expect_path=1)


def test_conv_refusals():
    inp = synth.make_fwd(1, 64, 64, 16, seed=75)
    dev = gu.upload(inp)
    flags = bnd.flags_for(z=inp.z, D=inp.Dskip, delta_bias=inp.delta_bias, conv=True)
    plan = bnd.Plan(1, 64, 64, 16, torch.bfloat16, torch.bfloat16, flags, "cuda")
    with pytest.raises(bnd.SsmError) as e:
        plan.fwd(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"], D=dev["D"], z=dev["z"],
                 delta_bias=dev["delta_bias"])
    assert e.value.status == bnd.ERR_INVALID_ARG
    state = torch.zeros((1, 64, 16), device="cuda")
    with pytest.raises(bnd.SsmError) as e:
        plan.step(state, dev["x"][:, 0], dev["delta"][:, 0], dev["A"], dev["B"][:, 0],
                  dev["C"][:, 0], D=dev["D"], z=dev["z"][:, 0], delta_bias=dev["delta_bias"])
    assert e.value.status == bnd.ERR_UNSUPPORTED
    with pytest.raises(bnd.SsmError) as e:
        bnd.Plan(1, 64, 64, 16, torch.bfloat16, torch.bfloat16, flags | bnd.ZOH, "cuda")
    assert e.value.status == bnd.ERR_UNSUPPORTED
