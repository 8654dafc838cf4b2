"""bench.py pieces that run without a GPU: the algorithmic counts behind the
roofline, and the reference arm (the CPU oracle on a bounded sample)."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_algorithmic_counts_130m_layer():
    sys.path.insert(0, ROOT)
    import bench
    from selective_state_space_31_b200 import synth
    inp = synth.make_fwd(8, 2048, 1536, 16, seed=1)   # shape of the 130M layer, no draws needed
    c = bench.algorithmic_counts(inp)
    B, L, D, N = 8, 2048, 1536, 16
    assert c["updates"] == B * L * D * N
    assert c["mufu"] == B * L * D * N + 4 * B * L * D           # exp per update + softplus + gate
    # x, delta, z, y in bf16 + B, C in bf16 + fp32 A, D, bias + fp32 h_last
    assert c["bytes"] == 2 * 4 * B * L * D + 2 * 2 * B * L * N + 4 * D * N + 8 * D + 4 * B * D * N


def test_reference_arm_prints_one_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny_fp32", "--steps", "2", "--warmup", "1",
                        "--cpu-budget-s", "0.3"], capture_output=True, text=True, timeout=600,
                       cwd=ROOT)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    out = json.loads(lines[0])
    assert out["impl"] == "reference" and out["value"] > 0
    assert out["cpu_baseline"]["kind"] == "oracle" and out["cpu_baseline"]["cores"] >= 1
    assert out["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_with_zero_order_hold():
    """--zoh reaches the oracle: its rate is measured on the zero-order-hold
    recurrence (a different program than the default's)."""
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny_fp32", "--steps", "1", "--warmup", "0", "--zoh",
                        "--cpu-budget-s", "0.3"], capture_output=True, text=True, timeout=600,
                       cwd=ROOT)
    assert r.returncode == 0, r.stderr
    out = json.loads([l for l in r.stdout.splitlines() if l.strip()][0])
    assert out["impl"] == "reference" and out["value"] > 0


def test_cli_flags():
    sys.path.insert(0, ROOT)
    import bench
    argv = sys.argv
    try:
        sys.argv = ["bench.py", "--bwd", "--zoh", "--workload", "mamba1p4b_layer"]
        a = bench.parse_args()
    finally:
        sys.argv = argv
    assert a.bwd and a.zoh and a.workload == "mamba1p4b_layer" and a.gpus == 1
    assert a.warmup >= 3
