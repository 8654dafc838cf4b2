"""GPU parity of the backward pass (ssm_scan_bwd) against the fp64 backward
oracle, itself pinned by finite differences of the forward oracle.

Tolerance: normwise error (max |gpu - oracle| / max |oracle|) <= 1e-4 for
every gradient.  The kernel accumulates in fp32 (relative rounding 6e-8 per
operation, ex2.approx 2.4e-7) along chains of up to L*N terms (the carried
state gradient over L tokens; dA, dB, dC, dD and the bias gradient sum over
tokens, batch or channels): at L <= 100 and N <= 16 that is about 1.6e3
terms, a worst-case linear growth near 1e-4 and a typical square-root growth
near 3e-6."""
import numpy as np
import pytest
import torch

import gpu_util as gu
import oracle
from selective_state_space_31_b200 import binding as bnd
from selective_state_space_31_b200 import synth

pytestmark = pytest.mark.gpu

TOL_BWD = 1e-4


def _round_bf16(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).float().numpy()


def _check(inp, dh_last=True, want_dh0=True, seed=0, cfg=None):
    rng = np.random.default_rng(seed)
    dy = rng.standard_normal((inp.Bsz, inp.L, inp.D)).astype(np.float32)
    if inp.out_dtype == "bf16":
        dy = _round_bf16(dy)
    dhl = rng.standard_normal((inp.Bsz, inp.D, inp.N)).astype(np.float32) if dh_last else None
    plan = gu.make_plan(inp)
    if cfg:
        plan.set_config(**cfg)
    dev = gu.upload(inp)
    g = plan.bwd(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"],
                 gu.dev_tensor(dy, inp.out_dtype), D=dev["D"], z=dev["z"],
                 delta_bias=dev["delta_bias"], h0=dev["h0"],
                 dh_last=gu.dev_tensor(dhl) if dhl is not None else None, want_dh0=want_dh0)
    torch.cuda.synchronize()
    ref = oracle.get().bwd(inp.x, inp.delta, inp.A, inp.B, inp.C, dy, D=inp.Dskip, z=inp.z,
                           delta_bias=inp.delta_bias, h0=inp.h0, dh_last=dhl,
                           delta_softplus=inp.delta_softplus)
    for name, got in g.items():
        err = gu.normwise(got.cpu().numpy(), ref[name])
        assert err <= TOL_BWD, f"d/d{name}: normwise {err:.2e}"
    if not want_dh0:
        assert "h0" not in g


def test_bwd_fp32_all_options():
    """Gate, skip, bias, softplus, h0 and dh_last; L = 100 is not a multiple
    of the 16-token recomputation chunk."""
    _check(synth.make_fwd(2, 100, 40, 16, in_dtype="f32", seed=51, has_h0=True), seed=1)


def test_bwd_fp32_plain():
    """No gate, skip, bias, softplus or h0 (Delta given directly, positive)."""
    inp = synth.make_fwd(3, 37, 24, 4, in_dtype="f32", seed=52, has_z=False, has_D=False,
                         has_bias=False, delta_softplus=False)
    inp.delta = np.abs(inp.delta) * np.float32(0.3) + np.float32(0.05)
    _check(inp, dh_last=False, want_dh0=False, seed=2)


def test_bwd_bf16_inputs_and_dy():
    _check(synth.make_fwd(2, 64, 32, 16, seed=53, has_h0=True), seed=3)


def test_bwd_dstate_not_a_power_of_two():
    _check(synth.make_fwd(2, 50, 16, 12, in_dtype="f32", seed=54, has_h0=True), seed=4)


def test_bwd_refuses_zero_order_hold():
    inp = synth.make_fwd(1, 8, 16, 16, in_dtype="f32", seed=55, zoh=True)
    plan = gu.make_plan(inp)
    dev = gu.upload(inp)
    dy = torch.zeros((1, 8, 16), dtype=torch.float32, device="cuda")
    with pytest.raises(bnd.SsmError) as e:
        plan.bwd(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"], dy, D=dev["D"],
                 z=dev["z"], delta_bias=dev["delta_bias"])
    assert e.value.status == bnd.ERR_UNSUPPORTED


def test_bwd_channels_not_a_multiple_of_the_warp_group():
    """dim % 8 != 0: a warp's channels span two batch elements, so dB and dC
    take one atomic per lane instead of the warp's reduce-scatter."""
    _check(synth.make_fwd(2, 70, 37, 16, in_dtype="f32", seed=56, has_h0=True), seed=5)


def test_bwd_large_dstate():
    """dstate 32: sixteen states per lane (no warp reduction of dB / dC)."""
    _check(synth.make_fwd(1, 40, 16, 32, in_dtype="f32", seed=57, has_h0=True), seed=6)


def test_bwd_130m_layer_sampled():
    """The 130M-layer shape at full size in bf16: finite gradients, and the
    per-channel ones (dA, dD, delta bias) and dh0 on sampled channels
    against the oracle run over those channels only.  (dB / dC sum over
    every channel, so they are checked on the small shapes above.)"""
    inp = synth.make_fwd(8, 2048, 1536, 16, seed=58)
    rng = np.random.default_rng(7)
    dy = _round_bf16(rng.standard_normal((inp.Bsz, inp.L, inp.D)).astype(np.float32))
    plan = gu.make_plan(inp)
    dev = gu.upload(inp)
    g = plan.bwd(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"],
                 gu.dev_tensor(dy, "bf16"), D=dev["D"], z=dev["z"],
                 delta_bias=dev["delta_bias"])
    torch.cuda.synchronize()
    for name, t in g.items():
        assert bool(torch.isfinite(t).all()), name
    chans = [0, 7, 8, 777, 1535]
    sub = lambda a: np.ascontiguousarray(a[:, :, chans])
    ref = oracle.get().bwd(sub(inp.x), sub(inp.delta), inp.A[chans], inp.B, inp.C, sub(dy),
                           D=inp.Dskip[chans], z=sub(inp.z), delta_bias=inp.delta_bias[chans])
    got_x = g["x"].cpu().numpy()[:, :, chans]
    assert gu.normwise(got_x, ref["x"]) <= 2e-2
    assert gu.normwise(g["delta"].cpu().numpy()[:, :, chans], ref["delta"]) <= 2e-2
    assert gu.normwise(g["A"].cpu().numpy()[chans], ref["A"]) <= 2e-2
    assert gu.normwise(g["D"].cpu().numpy()[chans], ref["D"]) <= 2e-2


# ---------------------------------------------------------------------------
# the fused backward kernel (TMA-fed row tiles; two or four scan warps)
# ---------------------------------------------------------------------------

def _check_fused(inp, warps, dh_last=True, want_dh0=True, seed=0):
    """_check with the fused kernel's scan warps forced, after checking that
    the plan takes the fused kernel with that shape."""
    plan = gu.make_plan(inp)
    plan.set_config(bwd_warps_per_cta=warps)
    assert plan.info()["bwd_warps_per_cta"] == warps
    plan.close()
    _check(inp, dh_last=dh_last, want_dh0=want_dh0, seed=seed,
           cfg=dict(bwd_warps_per_cta=warps))


@pytest.mark.parametrize("warps", [2, 4])
@pytest.mark.parametrize("ns", [16, 8])
def test_bwd_fused_fp32_ragged(warps, ns):
    """fp32, every option, L = 77 (the last 8-token stage holds 5 tokens)
    and D = 72 (the last row tile is partly past the channels)."""
    _check_fused(synth.make_fwd(2, 77, 72, ns, in_dtype="f32", seed=59 + ns, has_h0=True),
                 warps, seed=8)


@pytest.mark.parametrize("warps", [2, 4])
def test_bwd_fused_bf16_in_bf16_and_f32_dy(warps):
    _check_fused(synth.make_fwd(3, 150, 64, 16, seed=61, has_h0=True), warps, seed=9)
    _check_fused(synth.make_fwd(2, 96, 48, 16, out_dtype="f32", seed=62, has_h0=True), warps,
                 seed=10)


def test_bwd_fused_no_gate_no_softplus():
    inp = synth.make_fwd(2, 45, 32, 16, in_dtype="f32", seed=63, has_z=False, has_D=False,
                         has_bias=False, delta_softplus=False)
    inp.delta = np.abs(inp.delta) * np.float32(0.3) + np.float32(0.05)
    _check_fused(inp, 2, dh_last=False, want_dh0=False, seed=11)


def test_bwd_fused_single_token_and_one_stage():
    _check_fused(synth.make_fwd(1, 1, 32, 16, in_dtype="f32", seed=64, has_h0=True), 2, seed=12)
    _check_fused(synth.make_fwd(2, 8, 32, 16, in_dtype="f32", seed=65, has_h0=True), 4, seed=13)


def test_bwd_fused_deterministic():
    """Every gradient but the batch sums (dA, dD, delta bias: atomics over
    the batch) is bitwise reproducible: dB and dC add the row tiles' sums
    in a fixed order."""
    inp = synth.make_fwd(2, 300, 128, 16, seed=66, has_h0=True)
    rng = np.random.default_rng(14)
    dy = gu.dev_tensor(_round_bf16(rng.standard_normal((2, 300, 128)).astype(np.float32)), "bf16")
    plan = gu.make_plan(inp)
    assert plan.info()["bwd_warps_per_cta"] in (2, 4)
    dev = gu.upload(inp)
    run = lambda: plan.bwd(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"], dy, D=dev["D"],
                           z=dev["z"], delta_bias=dev["delta_bias"], h0=dev["h0"])
    g1, g2 = run(), run()
    torch.cuda.synchronize()
    for name in ("x", "delta", "B", "C", "z", "h0"):
        assert torch.equal(g1[name], g2[name]), name
    assert plan.status() == 0


def test_bwd_130m_layer_every_channel():
    """The 130M-layer shape at full size (8 x 2048 x 1536, N = 16, bf16,
    every option, dh_last given) against the fp64 oracle on every channel:
    the oracle runs per block of 64 channels of one batch element on all
    host threads; per-channel gradients (x, delta, z, h0) are compared
    block by block, A, D and the bias gradient after summing the batch,
    and dB, dC (sums over channels) after adding every block's share.
    Tolerance 1e-3 normwise: fp32 sums over up to 2048 tokens x 8 batch
    elements (or 1536 channels for dB, dC) from the same bf16-valued
    inputs as the oracle's."""
    import concurrent.futures as cf
    import os
    import threading

    inp = synth.make_fwd(8, 2048, 1536, 16, seed=58)
    rng = np.random.default_rng(15)
    dy = _round_bf16(rng.standard_normal((inp.Bsz, inp.L, inp.D)).astype(np.float32))
    dhl = rng.standard_normal((inp.Bsz, inp.D, inp.N)).astype(np.float32)
    plan = gu.make_plan(inp)
    assert plan.info()["bwd_warps_per_cta"] in (2, 4)
    dev = gu.upload(inp)
    g = plan.bwd(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"], gu.dev_tensor(dy, "bf16"),
                 D=dev["D"], z=dev["z"], delta_bias=dev["delta_bias"],
                 dh_last=gu.dev_tensor(dhl))
    torch.cuda.synchronize()
    assert plan.status() == 0
    got = {k: v.cpu().numpy() for k, v in g.items()}
    orc = oracle.get()
    lock = threading.Lock()
    err = {k: [0.0, 0.0] for k in ("x", "delta", "z", "h0")}
    acc = {"A": np.zeros((inp.D, inp.N)), "D": np.zeros(inp.D), "delta_bias": np.zeros(inp.D),
           "B": np.zeros((inp.Bsz, inp.L, inp.N)), "C": np.zeros((inp.Bsz, inp.L, inp.N))}

    def one(blk):
        b, d0, d1 = blk
        sl = lambda a: np.ascontiguousarray(a[b:b + 1, :, d0:d1])
        r = orc.bwd(sl(inp.x), sl(inp.delta), inp.A[d0:d1], inp.B[b:b + 1], inp.C[b:b + 1],
                    sl(dy), D=inp.Dskip[d0:d1], z=sl(inp.z), delta_bias=inp.delta_bias[d0:d1],
                    dh_last=np.ascontiguousarray(dhl[b:b + 1, d0:d1]))
        part = {k: (np.abs(got[k][b:b + 1, :, d0:d1] - r[k]).max(), np.abs(r[k]).max())
                for k in ("x", "delta", "z")}
        part["h0"] = (np.abs(got["h0"][b:b + 1, d0:d1] - r["h0"]).max(), np.abs(r["h0"]).max())
        with lock:
            for k, (e, m) in part.items():
                err[k][0] = max(err[k][0], e)
                err[k][1] = max(err[k][1], m)
            acc["A"][d0:d1] += r["A"]
            acc["D"][d0:d1] += r["D"]
            acc["delta_bias"][d0:d1] += r["delta_bias"]
            acc["B"][b] += r["B"][0]
            acc["C"][b] += r["C"][0]

    with cf.ThreadPoolExecutor(max_workers=os.cpu_count() or 1) as ex:
        for f in [ex.submit(one, blk) for blk in oracle.channel_blocks(inp.Bsz, inp.D, 64)]:
            f.result()
    for k, (e, m) in err.items():
        assert e <= 1e-3 * m, f"d/d{k}: normwise {e / m:.2e}"
    for k, ref in acc.items():
        e = gu.normwise(got[k], ref)
        assert e <= 1e-3, f"d/d{k}: normwise {e:.2e}"


@pytest.mark.parametrize("segments", [2, 4, 16])
@pytest.mark.parametrize("in_dt", ["f32", "bf16"])
def test_bwd_fused_segments(segments, in_dt):
    """Segments of a row tile walked at the same time: the map pass's
    forward maps give each segment its start state, its adjoint maps the
    gradient flowing in from the later segments; ragged L (the last 8-token
    stage holds 3 tokens, the last segment is short), every option."""
    inp = synth.make_fwd(2, 603, 64, 16, in_dtype=in_dt, seed=67 + segments, has_h0=True)
    plan = gu.make_plan(inp)
    plan.set_config(bwd_segments=segments)
    info = plan.info()
    assert info["bwd_segments"] >= 2, info
    plan.close()
    _check(inp, seed=16 + segments, cfg=dict(bwd_segments=segments))


def test_bwd_long_row_picks_segments():
    """One long row (few row tiles): the planner splits it into segments."""
    inp = synth.make_fwd(1, 4000, 64, 16, in_dtype="f32", seed=69, has_h0=True)
    plan = gu.make_plan(inp)
    assert plan.info()["bwd_segments"] > 1, plan.info()
    plan.close()
    _check(inp, seed=17)
