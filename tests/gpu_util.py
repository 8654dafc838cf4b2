"""Shared helpers of the GPU parity tests: upload seeded inputs, run the CUDA
library through its binding, and compare with the CPU oracle.

Pass criterion (the scan's error metric): for each output tensor,
max_i |gpu_i - oracle_i| / max_i |oracle_i| (normwise); for y additionally the
same ratio per channel row (b, d) over time, maxed over rows.  Tolerances:
1e-5 for fp32 inputs/outputs, 2e-2 for bf16 inputs with fp32 state (the
bf16 rounding of y alone is up to 2^-9 relative)."""
from __future__ import annotations

import numpy as np
import torch

TOL = {"f32": 1e-5, "bf16": 2e-2}
TDT = {"f32": torch.float32, "bf16": torch.bfloat16}


def dev_tensor(a, dtype="f32", device="cuda"):
    if a is None:
        return None
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(
        device=device, dtype=TDT[dtype])


def upload(inp, device="cuda"):
    """ScanInputs -> dict of device tensors in their storage dtypes."""
    return {
        "x": dev_tensor(inp.x, inp.in_dtype, device),
        "delta": dev_tensor(inp.delta, inp.in_dtype, device),
        "A": dev_tensor(inp.A, "f32", device),
        "B": dev_tensor(inp.B, inp.in_dtype, device),
        "C": dev_tensor(inp.C, inp.in_dtype, device),
        "D": dev_tensor(inp.Dskip, "f32", device),
        "z": dev_tensor(inp.z, inp.in_dtype, device),
        "delta_bias": dev_tensor(inp.delta_bias, "f32", device),
        "h0": dev_tensor(inp.h0, "f32", device),
    }


def make_plan(inp, device="cuda"):
    from selective_state_space_31_b200 import binding as bnd
    flags = bnd.flags_for(z=inp.z, D=inp.Dskip, delta_bias=inp.delta_bias, h0=inp.h0,
                          delta_softplus=inp.delta_softplus, want_h_last=inp.want_h_last,
                          zoh=inp.zoh)
    return bnd.Plan(inp.Bsz, inp.L, inp.D, inp.N, TDT[inp.in_dtype], TDT[inp.out_dtype], flags,
                    device)


def run_gpu(inp, plan=None, dev=None):
    plan = plan or make_plan(inp)
    dev = dev or upload(inp)
    y, hl = plan.fwd(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"], D=dev["D"],
                     z=dev["z"], delta_bias=dev["delta_bias"], h0=dev["h0"])
    torch.cuda.synchronize()
    return y.float().cpu().numpy().astype(np.float64), hl.cpu().numpy().astype(np.float64)


def run_oracle(inp):
    import oracle
    return oracle.get().fwd(inp.x, inp.delta, inp.A, inp.B, inp.C, D=inp.Dskip, z=inp.z,
                            delta_bias=inp.delta_bias, h0=inp.h0,
                            delta_softplus=inp.delta_softplus, zoh=inp.zoh)


def normwise(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    if ref.size == 0:
        return 0.0
    return float(np.max(np.abs(got - ref)) / max(np.max(np.abs(ref)), 1e-30))


def rowwise(got_y, ref_y):
    """max over (b, d) rows of the normwise error over time (y is (B, L, D))."""
    if ref_y.size == 0:
        return 0.0
    num = np.max(np.abs(got_y - ref_y), axis=1)
    den = np.maximum(np.max(np.abs(ref_y), axis=1), 1e-30)
    return float(np.max(num / den))


def assert_parity(got_y, ref_y, got_h, ref_h, tol, what=""):
    assert np.all(np.isfinite(got_y)) and np.all(np.isfinite(got_h)), f"{what}: non-finite output"
    ey, er, eh = normwise(got_y, ref_y), rowwise(got_y, ref_y), normwise(got_h, ref_h)
    assert ey <= tol and er <= tol and eh <= tol, (
        f"{what}: y {ey:.2e}, y per-row {er:.2e}, h_last {eh:.2e} (tol {tol:.0e})")
    return ey, er, eh
