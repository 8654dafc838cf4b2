"""GPU parity at the full sizes of the five standard workloads, in the launch
shape the benchmark uses (the plan's default), against the oracle on EVERY
channel row: the oracle runs over all (b, d) rows in channel blocks on all
host threads, and the comparison is element by element.

Criteria (the scan's error metric): per output tensor max|g - r| / max|r|,
and for y the same ratio per channel row (b, d) over time, maxed over rows.
Decode: every channel of y at every one of the 1024 steps (per step and
batch row) and every channel of the final state."""
import concurrent.futures as cf
import os
import threading

import numpy as np
import pytest
import torch

import gpu_util as gu
import oracle
from selective_state_space_31_b200 import binding as bnd
from selective_state_space_31_b200 import synth

pytestmark = pytest.mark.gpu


class ErrAccumulator:
    """Running normwise errors over blocks of a (Bsz, L, D) output and its
    (Bsz, D, N) final state, plus the worst per-row error of y."""

    def __init__(self, gy, gh):
        self.gy, self.gh = gy, gh
        self.lock = threading.Lock()
        self.dy = self.ry = self.dh = self.rh = 0.0
        self.row = 0.0
        self.row_at = None
        self.blocks = 0
        self.finite = True

    def __call__(self, blk, y, h):
        b, d0, d1 = blk
        g = self.gy[b, :, d0:d1].astype(np.float64)
        gh = self.gh[b, d0:d1].astype(np.float64)
        finite = bool(np.all(np.isfinite(g)) and np.all(np.isfinite(gh)))
        diff = np.abs(g - y)
        ref = np.abs(y)
        row = np.max(diff, axis=0) / np.maximum(np.max(ref, axis=0), 1e-30)
        k = int(np.argmax(row))
        with self.lock:
            self.finite &= finite
            self.dy = max(self.dy, float(diff.max()))
            self.ry = max(self.ry, float(ref.max()))
            self.dh = max(self.dh, float(np.max(np.abs(gh - h))))
            self.rh = max(self.rh, float(np.max(np.abs(h))))
            if row[k] > self.row:
                self.row, self.row_at = float(row[k]), (b, d0 + k)
            self.blocks += 1

    def check(self, tol, what):
        assert self.finite, f"{what}: non-finite output"
        ey, eh = self.dy / max(self.ry, 1e-30), self.dh / max(self.rh, 1e-30)
        assert ey <= tol and self.row <= tol and eh <= tol, (
            f"{what}: y {ey:.2e}, worst row {self.row:.2e} at {self.row_at}, "
            f"h_last {eh:.2e} (tol {tol:.0e})")
        return ey, self.row, eh


def run_full(inp):
    plan = gu.make_plan(inp)
    info = plan.info()
    dev = gu.upload(inp)
    y, hl = plan.fwd(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"], D=dev["D"],
                     z=dev["z"], delta_bias=dev["delta_bias"], h0=dev["h0"])
    torch.cuda.synchronize()
    assert plan.status() == 0
    gy, gh = y.float().cpu().numpy(), hl.cpu().numpy()
    del dev, y, hl
    plan.close()
    return info, gy, gh


def check_every_row(inp, gy, gh, tol, what):
    # blocks of about 2M tokens x channels keep each worker's fp64 copies small
    width = max(1, min(inp.D, (1 << 21) // max(inp.L, 1)))
    acc = ErrAccumulator(gy, gh)
    blocks = oracle.channel_blocks(inp.Bsz, inp.D, width)
    oracle.fwd_blocks(inp.x, inp.delta, inp.A, inp.B, inp.C, blocks, acc, D=inp.Dskip, z=inp.z,
                      delta_bias=inp.delta_bias, h0=inp.h0, delta_softplus=inp.delta_softplus,
                      zoh=inp.zoh)
    assert acc.blocks == len(blocks)
    return acc.check(tol, what)


def test_tiny_fp32_full_oracle():
    inp = synth.tiny_fp32()
    info, gy, gh = run_full(inp)
    check_every_row(inp, gy, gh, gu.TOL["f32"], f"tiny {info}")


@pytest.mark.parametrize("name", ["mamba130m_layer", "mamba1p4b_layer", "long_seq"])
def test_bf16_layer_workloads_every_row(name):
    inp = synth.FWD_WORKLOADS[name]()
    info, gy, gh = run_full(inp)
    check_every_row(inp, gy, gh, gu.TOL["bf16"], f"{name} {info}")


def test_decode_1024_steps_every_channel():
    """1024 consecutive decode steps on the (256, 5120, 16) state from
    h0 ~ N(0, 0.1^2), against the oracle stepping the same tokens on every
    channel: y of every channel at every step (normwise per step and batch
    row) and the whole final state."""
    dec = synth.make_decode()
    bf, f32 = torch.bfloat16, torch.float32
    up = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a)).to("cuda", dt)
    A, Dv, bias = up(dec.A, f32), up(dec.Dskip, f32), up(dec.delta_bias, f32)
    state = up(dec.h0, f32)
    threads = os.cpu_count() or 1
    slices = [(b0, min(dec.Bsz, b0 + max(1, dec.Bsz // threads)))
              for b0 in range(0, dec.Bsz, max(1, dec.Bsz // threads))]
    ostate = dec.h0.astype(np.float64)
    orc = oracle.get()
    worst_y = 0.0
    with cf.ThreadPoolExecutor(max_workers=threads) as ex:
        for t in range(dec.steps):
            tok = dec.token(t)
            y = bnd.step(state, up(tok["x"], bf), up(tok["delta"], bf), A, up(tok["B"], bf),
                         up(tok["C"], bf), D=Dv, z=up(tok["z"], bf), delta_bias=bias)

            def one(sl):
                b0, b1 = sl
                return orc.step(ostate[b0:b1], tok["x"][b0:b1], tok["delta"][b0:b1], dec.A,
                                tok["B"][b0:b1], tok["C"][b0:b1], D=dec.Dskip,
                                z=tok["z"][b0:b1], delta_bias=dec.delta_bias)

            res = list(ex.map(one, slices))
            ry = np.concatenate([r[0] for r in res])
            ostate = np.concatenate([r[1] for r in res])
            gy = y.float().cpu().numpy()
            assert np.all(np.isfinite(gy)), f"step {t}: non-finite y"
            e = np.max(np.abs(gy - ry), axis=1) / np.maximum(np.max(np.abs(ry), axis=1), 1e-30)
            worst_y = max(worst_y, float(e.max()))
    assert worst_y <= gu.TOL["bf16"], worst_y
    gs = state.cpu().numpy()
    assert np.all(np.isfinite(gs))
    assert gu.normwise(gs, ostate) <= 1e-5, gu.normwise(gs, ostate)


@pytest.mark.parametrize("name", ["mamba130m_layer", "long_seq"])
def test_host_buffer_path_every_row(name):
    """The workload through ssm_scan_fwd_host (pinned host buffers, the
    library's chunking) at full size, every (b, d) row against the oracle."""
    inp = synth.FWD_WORKLOADS[name]()
    plan = gu.make_plan(inp)
    idt = gu.TDT[inp.in_dtype]
    pin = lambda a, dt: None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(dt).pin_memory()
    y, hl = plan.fwd_host(pin(inp.x, idt), pin(inp.delta, idt), pin(inp.A, torch.float32),
                          pin(inp.B, idt), pin(inp.C, idt), D=pin(inp.Dskip, torch.float32),
                          z=pin(inp.z, idt), delta_bias=pin(inp.delta_bias, torch.float32),
                          h0=pin(inp.h0, torch.float32))
    torch.cuda.synchronize()
    assert plan.status() == 0
    plan.close()
    check_every_row(inp, y.float().numpy(), hl.numpy(), gu.TOL["bf16"], f"{name} host path")
