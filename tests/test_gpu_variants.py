"""Every compiled variant of the fused forward kernel against the oracle:
lanes per channel, channels per lane, scan warps, stage length, the
zero-order-hold flag, and segments (the carry pass plus the fold of its maps
at each segment's start), on ragged lengths with h0 and every option on.

Each test walks the variant table the library reports, so a variant that
exists is a variant that is tested; the failures of one table are collected
and reported together."""
import numpy as np
import pytest

import gpu_util as gu
from selective_state_space_31_b200 import binding as bnd
from selective_state_space_31_b200 import synth

pytestmark = pytest.mark.gpu


def _variants(in_dt, out_dt, ns, zoh, carry=False):
    return [v for v in bnd.list_variants(gu.TDT[in_dt], gu.TDT[out_dt])
            if v["dstate"] == ns and bool(v["zoh"]) == zoh and bool(v["carry"]) == carry
            and not v["conv"]]


def _run(inp, dev, cfg):
    plan = gu.make_plan(inp)
    plan.set_config(**cfg)
    info = plan.info()
    gy, gh = gu.run_gpu(inp, plan, dev)
    st = plan.status()
    plan.close()
    return info, gy, gh, st


def _sweep(inp, in_dt, out_dt, segments_list, grids=(0,)):
    tol = gu.TOL["f32" if in_dt == "f32" and out_dt == "f32" else "bf16"]
    dev = gu.upload(inp)
    ry, rh = gu.run_oracle(inp)
    mains = _variants(in_dt, out_dt, inp.N, inp.zoh)
    assert mains, "no compiled variant"
    failures, ran, carries = [], 0, set()
    for v in mains:
        for M in segments_list:
            for grid in grids:
                cfg = dict(lanes_per_chan=v["lanes_per_chan"], warps_per_cta=v["warps_per_cta"],
                           tile_t=v["tile_t"], chans_per_lane=v["chans_per_lane"],
                           segments=M, grid=grid, scan_loop=1 + v["opt"])
                try:
                    info, gy, gh, st = _run(inp, dev, cfg)
                except bnd.SsmError as e:
                    failures.append(f"{cfg}: refused ({e})")
                    continue
                ran += 1
                key = (info["lanes_per_chan"], info["chans_per_lane"], info["warps_per_cta"],
                       info["tile_t"])
                if key != (v["lanes_per_chan"], v["chans_per_lane"], v["warps_per_cta"],
                           v["tile_t"]) or info["segments"] != M or \
                        info["scan_loop"] != 1 + v["opt"]:
                    failures.append(f"{cfg}: plan chose {info}")
                if M > 1:
                    carries.add((v["lanes_per_chan"], v["chans_per_lane"], v["tile_t"]))
                    if info["launches_per_call"] != 2:
                        failures.append(f"{cfg}: {info['launches_per_call']} launches")
                try:
                    assert st == 0, f"device status {st}"
                    gu.assert_parity(gy, ry, gh, rh, tol, str(cfg))
                except AssertionError as e:
                    failures.append(str(e))
    assert not failures, f"{len(failures)} of {ran} runs failed:\n" + "\n".join(failures)
    return ran, carries


@pytest.mark.parametrize("ns", [16, 8])
def test_bf16_every_variant_and_segments(ns):
    """bf16 in/out, all options, h0, a ragged L: every variant alone, with
    4 segments, and with a grid of 3 CTAs (parts chained across CTAs)."""
    inp = synth.make_fwd(2, 2100, 128, ns, seed=61, has_h0=True)
    ran, carries = _sweep(inp, "bf16", "bf16", (1, 4))
    assert ran >= 8
    _sweep(synth.make_fwd(3, 389, 64, ns, seed=62, has_h0=True), "bf16", "bf16", (1,),
           grids=(3,))


@pytest.mark.parametrize("ns", [16, 8])
def test_bf16_zoh_every_variant_and_segments(ns):
    inp = synth.make_fwd(2, 2100, 128, ns, seed=63, has_h0=True, zoh=True)
    _sweep(inp, "bf16", "bf16", (1, 2))


@pytest.mark.parametrize("ns", [16, 8])
def test_bf16_in_f32_out_every_variant(ns):
    inp = synth.make_fwd(2, 1500, 64, ns, out_dtype="f32", seed=64, has_h0=True)
    _sweep(inp, "bf16", "f32", (1, 2))


@pytest.mark.parametrize("ns", [16, 8, 4])
@pytest.mark.parametrize("zoh", [False, True])
def test_f32_every_variant_and_segments(ns, zoh):
    """fp32 in/out at the fp32 tolerance (1e-5), segments included: the fold
    of the carry maps keeps fp32 accuracy."""
    inp = synth.make_fwd(2, 1200, 32, ns, in_dtype="f32", seed=65, has_h0=True, zoh=zoh)
    _sweep(inp, "f32", "f32", (1, 4))


@pytest.mark.parametrize("in_dt,out_dt,zoh", [("bf16", "bf16", False), ("bf16", "bf16", True),
                                               ("bf16", "f32", False), ("f32", "f32", False)])
def test_every_carry_variant(in_dt, out_dt, zoh):
    """Each compiled carry-pass variant (lanes per channel and options forced),
    behind a main variant of the same stage length (and lane split where one
    exists), with 4 segments on a ragged length: the maps it leaves, folded
    at each segment's start, give the oracle's result."""
    for ns in (16, 8):
        carries = _variants(in_dt, out_dt, ns, zoh, carry=True)
        if not carries:
            continue
        inp = synth.make_fwd(2, 1800, 64, ns, in_dtype=in_dt, out_dtype=out_dt, seed=69,
                             has_h0=True, zoh=zoh)
        tol = gu.TOL["f32" if in_dt == "f32" and out_dt == "f32" else "bf16"]
        dev = gu.upload(inp)
        ry, rh = gu.run_oracle(inp)
        mains = _variants(in_dt, out_dt, ns, zoh)
        failures = []
        for c in carries:
            same = [v for v in mains if (v["lanes_per_chan"], v["chans_per_lane"], v["tile_t"]) ==
                    (c["lanes_per_chan"], c["chans_per_lane"], c["tile_t"])]
            cands = same or [v for v in mains if v["tile_t"] == c["tile_t"]]
            if not cands:
                failures.append(f"carry {c}: no main variant with its stage length")
                continue
            v = cands[0]
            cfg = dict(lanes_per_chan=v["lanes_per_chan"], warps_per_cta=v["warps_per_cta"],
                       tile_t=v["tile_t"], chans_per_lane=v["chans_per_lane"], segments=4,
                       scan_loop=1 + v["opt"], carry_lanes_per_chan=c["lanes_per_chan"],
                       carry_loop=1 + c["opt"], carry_chans_per_lane=c["chans_per_lane"])
            try:
                info, gy, gh, st = _run(inp, dev, cfg)
            except bnd.SsmError as e:
                failures.append(f"{cfg}: refused ({e})")
                continue
            if (info["carry_lanes_per_chan"], info["carry_loop"], info["carry_chans_per_lane"]) != \
                    (c["lanes_per_chan"], 1 + c["opt"], c["chans_per_lane"]) or info["segments"] != 4:
                failures.append(f"{cfg}: plan chose {info}")
            try:
                assert st == 0, f"device status {st}"
                gu.assert_parity(gy, ry, gh, rh, tol, f"carry {c} main {v}")
            except AssertionError as e:
                failures.append(str(e))
        assert not failures, "\n".join(failures)


@pytest.mark.parametrize("M", [2, 4, 8])
@pytest.mark.parametrize("h0", [False, True])
def test_segments_ragged_lengths(M, h0):
    """Segment boundaries, carry sub-chunks and the last short segment at
    several ragged lengths, long enough for eight segments."""
    for L in (2049, 4000, 5555):
        inp = synth.make_fwd(1, L, 256, 16, seed=66 + L, has_h0=h0)
        plan = gu.make_plan(inp)
        plan.set_config(segments=M)
        info = plan.info()
        assert info["segments"] >= 2, info
        gy, gh = gu.run_gpu(inp, plan)
        ry, rh = gu.run_oracle(inp)
        gu.assert_parity(gy, ry, gh, rh, gu.TOL["bf16"], f"L={L} {info}")
        assert plan.status() == 0


def test_segments_deterministic_and_replayable():
    """A segmented call (two launches) is bitwise reproducible, and replays
    from a CUDA graph to the same bits."""
    import torch
    inp = synth.make_fwd(1, 8192, 512, 16, seed=67, has_h0=True)
    plan = gu.make_plan(inp)
    plan.set_config(segments=4)
    assert plan.info()["segments"] == 4
    dev = gu.upload(inp)
    y1, h1 = gu.run_gpu(inp, plan, dev)
    y2, h2 = gu.run_gpu(inp, plan, dev)
    assert np.array_equal(y1, y2) and np.array_equal(h1, h2)
    y = torch.empty((1, 8192, 512), dtype=torch.bfloat16, device="cuda")
    hl = torch.empty((1, 512, 16), dtype=torch.float32, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        plan.fwd(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"], D=dev["D"], z=dev["z"],
                 delta_bias=dev["delta_bias"], h0=dev["h0"], y=y, h_last=hl)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        plan.fwd(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"], D=dev["D"], z=dev["z"],
                 delta_bias=dev["delta_bias"], h0=dev["h0"], y=y, h_last=hl)
    for _ in range(3):
        y.zero_()
        g.replay()
    torch.cuda.synchronize()
    assert np.array_equal(y.float().cpu().numpy().astype(np.float64), y1)
    assert np.array_equal(hl.cpu().numpy().astype(np.float64), h1)
    assert plan.status() == 0


def test_progress_without_co_residency():
    """Items go out in ticket order, so a grid far larger than what fits on
    the device at once (CTAs that start only after others have left) still
    ends every carried-state wait: with a 50 ms bound, status stays 0 and the
    result is exact."""
    inp = synth.make_fwd(8, 1024, 1536, 16, seed=68)
    plan = gu.make_plan(inp)
    plan.set_config(lanes_per_chan=4, warps_per_cta=4, tile_t=32, chans_per_lane=1, segments=1,
                    grid=20000)
    info = plan.info()
    assert info["parts_per_row"] >= 2 and info["grid"] > 148 * 8, info
    plan.set_debug(wait_timeout_ns=50_000_000)
    gy, gh = gu.run_gpu(inp, plan)
    assert plan.status() == 0
    ry, rh = gu.run_oracle(inp)
    gu.assert_parity(gy, ry, gh, rh, gu.TOL["bf16"], str(info))


def test_sixteen_segments():
    """Sixteen segments: the last segments fold sixty-odd sub-chunk maps
    before their first token; ragged length, h0 on."""
    inp = synth.make_fwd(1, 8190, 256, 16, seed=70, has_h0=True)
    plan = gu.make_plan(inp)
    plan.set_config(segments=16, tile_t=32)
    info = plan.info()
    assert info["segments"] == 16, info
    gy, gh = gu.run_gpu(inp, plan)
    assert plan.status() == 0
    ry, rh = gu.run_oracle(inp)
    gu.assert_parity(gy, ry, gh, rh, gu.TOL["bf16"], str(info))


@pytest.mark.parametrize("shape,segments", [((3, 2100, 512), 0), ((1, 4100, 128), 16),
                                            ((2, 1100, 256), 4)])
def test_parts_past_a_short_last_segment(shape, segments):
    """Plans whose last segment is shorter than the others, so that some of
    its parts begin past its end (14 segments of 5 one-stage parts over 66
    stages: the last segment holds one stage): those parts are empty and
    every stage is scanned once."""
    inp = synth.make_fwd(*shape, 16, seed=76, has_h0=True)
    plan = gu.make_plan(inp)
    if segments:
        plan.set_config(segments=segments, tile_t=32)
    info = plan.info()
    M, SPS, S = info["segments"], info["stages_per_segment"], info["stages_per_row"]
    assert M >= 2 and S - (M - 1) * SPS < SPS, info
    plan.set_debug(wait_timeout_ns=200_000_000)
    gy, gh = gu.run_gpu(inp, plan)
    assert plan.status() == 0
    ry, rh = gu.run_oracle(inp)
    gu.assert_parity(gy, ry, gh, rh, gu.TOL["bf16"], str(info))


def test_segment_layouts_sweep():
    """Many (length, segments, stage, grid) layouts on a small row set: every
    stage scanned once whatever the segments' and parts' lengths (short last
    segments, parts past a segment's end, more CTAs than items), parity and
    status 0 with a 200 ms wait bound."""
    failures, ran = [], 0
    for L in (130, 257, 700, 1031, 2500, 4099):
        inp = synth.make_fwd(1, L, 64, 16, seed=80 + L % 97, has_h0=True)
        ry, rh = gu.run_oracle(inp)
        dev = gu.upload(inp)
        for M in (2, 4, 8, 16):
            for tt in (32, 64):
                for grid in (0, 37):
                    plan = gu.make_plan(inp)
                    try:
                        plan.set_config(segments=M, tile_t=tt, grid=grid)
                    except bnd.SsmError:
                        plan.close()
                        continue
                    info = plan.info()
                    plan.set_debug(wait_timeout_ns=200_000_000)
                    gy, gh = gu.run_gpu(inp, plan, dev)
                    st = plan.status()
                    plan.close()
                    ran += 1
                    try:
                        assert st == 0, f"status {st}"
                        gu.assert_parity(gy, ry, gh, rh, gu.TOL["bf16"], f"L={L} {info}")
                    except AssertionError as e:
                        failures.append(str(e))
    assert ran >= 24, ran
    assert not failures, "\n".join(failures[:10])
