"""ssm_scan_fwd_host: the forward pass on host buffers, streamed through the
device in chunks of tokens with the state carried from chunk to chunk,
against the oracle on the same inputs (ragged last chunks, a single chunk,
pageable memory, every option, fp32 with zero-order hold), and the device
path's result for the same plan."""
import numpy as np
import pytest
import torch

import gpu_util as gu
from selective_state_space_31_b200 import binding as bnd
from selective_state_space_31_b200 import synth

pytestmark = pytest.mark.gpu


def _host(inp, pin=True):
    def t(a, dt):
        if a is None:
            return None
        v = torch.from_numpy(np.ascontiguousarray(a)).to(dt)
        return v.pin_memory() if pin else v
    idt = gu.TDT[inp.in_dtype]
    return dict(x=t(inp.x, idt), delta=t(inp.delta, idt), z=t(inp.z, idt), B=t(inp.B, idt),
                C=t(inp.C, idt), A=t(inp.A, torch.float32), D=t(inp.Dskip, torch.float32),
                delta_bias=t(inp.delta_bias, torch.float32), h0=t(inp.h0, torch.float32))


def _run_host(inp, chunk_tokens=0, pin=True, plan=None):
    plan = plan or gu.make_plan(inp)
    h = _host(inp, pin)
    y, hl = plan.fwd_host(h["x"], h["delta"], h["A"], h["B"], h["C"], D=h["D"], z=h["z"],
                          delta_bias=h["delta_bias"], h0=h["h0"], chunk_tokens=chunk_tokens)
    torch.cuda.synchronize()
    return y.float().numpy().astype(np.float64), hl.numpy().astype(np.float64)


@pytest.mark.parametrize("chunk", [0, 192, 1000, 5000])
def test_host_bf16_chunks_against_oracle(chunk):
    """bf16 with every option and h0; 1000 tokens in chunks of 192 (the last
    holds 40), the library's choice, exactly one chunk, and a chunk longer
    than the sequence."""
    inp = synth.make_fwd(2, 1000, 256, 16, seed=71, has_h0=True)
    gy, gh = _run_host(inp, chunk)
    ry, rh = gu.run_oracle(inp)
    gu.assert_parity(gy, ry, gh, rh, gu.TOL["bf16"], f"chunk {chunk}")


def test_host_fp32_zoh_and_pageable_memory():
    inp = synth.make_fwd(2, 700, 64, 16, in_dtype="f32", seed=72, has_h0=True, zoh=True)
    ry, rh = gu.run_oracle(inp)
    for pin in (True, False):
        gy, gh = _run_host(inp, 128, pin=pin)
        gu.assert_parity(gy, ry, gh, rh, gu.TOL["f32"], f"pinned {pin}")


def test_host_matches_device_path_and_reuses_its_staging():
    """The same plan on device buffers and on host buffers (twice, then with
    another chunk length): every result within the bf16 tolerance of the
    device path, and the repeated host call bitwise equal to the first."""
    inp = synth.make_fwd(3, 2100, 512, 16, seed=73, has_h0=True)
    plan = gu.make_plan(inp)
    dy, dh = gu.run_gpu(inp, plan)
    y1, h1 = _run_host(inp, 300, plan=plan)
    y2, h2 = _run_host(inp, 300, plan=plan)
    y3, h3 = _run_host(inp, 512, plan=plan)
    assert np.array_equal(y1, y2) and np.array_equal(h1, h2)
    for gy, gh in ((y1, h1), (y3, h3)):
        gu.assert_parity(gy, dy, gh, dh, gu.TOL["bf16"], "host vs device")
    assert plan.status() == 0


def test_host_long_rows_segmented_chunks():
    """Chunks long enough for the planner's segments (the carry pass runs
    inside every chunk)."""
    inp = synth.make_fwd(1, 20000, 256, 16, seed=74, has_h0=True)
    gy, gh = _run_host(inp, 8192)
    ry, rh = gu.run_oracle(inp)
    gu.assert_parity(gy, ry, gh, rh, gu.TOL["bf16"], "segmented chunks")


def test_host_refuses_conv_plans():
    inp = synth.make_fwd(1, 64, 32, 16, seed=75)
    flags = bnd.flags_for(z=inp.z, D=inp.Dskip, delta_bias=inp.delta_bias, conv=True)
    plan = bnd.Plan(1, 64, 32, 16, torch.bfloat16, torch.bfloat16, flags)
    lib = bnd.load_library()
    rc = lib.ssm_scan_fwd_host(plan._h, None, None, None, None, None, None, None, None, None,
                               None, None, 0, None)
    assert rc == bnd.ERR_UNSUPPORTED


@pytest.mark.parametrize("chunk_rows", [0, 3, 64])
def test_host_decode_steps_against_oracle(chunk_rows):
    """ssm_scan_step_host: 20 decode steps with the token's inputs and y on
    the host and the state resident on the device, batch in chunks of 3 rows
    (the last holds 1), the library's choice, and one chunk; y at every step
    and the final state against the oracle stepping the same tokens."""
    import oracle
    dec = synth.make_decode(Bsz=10, D=96, N=16, steps=20, seed=77)
    bf, f32 = torch.bfloat16, torch.float32
    up = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a)).to("cuda", dt)
    pin = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a)).to(dt).pin_memory()
    flags = bnd.flags_for(z=1, D=1, delta_bias=1)
    plan = bnd.Plan(dec.Bsz, 1, dec.D, dec.N, bf, bf, flags)
    A, Dv, bias = up(dec.A, f32), up(dec.Dskip, f32), up(dec.delta_bias, f32)
    state = up(dec.h0, f32)
    ostate = dec.h0.astype(np.float64)
    orc = oracle.get()
    for t in range(dec.steps):
        tok = dec.token(t)
        y = plan.step_host(state, pin(tok["x"], bf), pin(tok["delta"], bf), A, pin(tok["B"], bf),
                           pin(tok["C"], bf), D=Dv, z=pin(tok["z"], bf), delta_bias=bias,
                           chunk_rows=chunk_rows)
        torch.cuda.synchronize()
        ry, ostate = orc.step(ostate, tok["x"], tok["delta"], dec.A, tok["B"], tok["C"],
                              D=dec.Dskip, z=tok["z"], delta_bias=dec.delta_bias)
        assert gu.normwise(y.float().numpy(), ry) <= gu.TOL["bf16"], t
    assert gu.normwise(state.cpu().numpy(), ostate) <= 1e-5
    assert plan.status() == 0
