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


def test_default_headline_is_the_largest_workload():
    """With no flags the headline is the long sequence, the largest
    single-GPU workload (B*L*D*N of every forward workload compared)."""
    sys.path.insert(0, ROOT)
    import bench
    a = bench.parse_args([])
    assert a.workload == "long_seq" and a.steps >= 1 and a.warmup >= 3
    sizes = {"tiny_fp32": 1 * 512 * 64, "mamba130m_layer": 8 * 2048 * 1536,
             "mamba1p4b_layer": 4 * 8192 * 4096, "long_seq": 1 * 131072 * 2560}
    assert max(sizes, key=sizes.get) == a.workload


def test_both_arms_name_the_same_config():
    """The reference arm's config is exactly our arm's for the same workload."""
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny_fp32", "--steps", "1", "--warmup", "0",
                        "--cpu-budget-s", "0.1"], capture_output=True, text=True, timeout=600,
                       cwd=ROOT)
    assert r.returncode == 0, r.stderr
    ref = json.loads([l for l in r.stdout.splitlines() if l.strip()][0])
    sys.path.insert(0, ROOT)
    import bench
    from selective_state_space_31_b200 import synth
    assert ref["config"] == bench.arm_config(synth.tiny_fp32(), 1, False)


def test_backward_counts():
    sys.path.insert(0, ROOT)
    import bench
    from selective_state_space_31_b200 import synth
    inp = synth.make_fwd(2, 64, 32, 16, seed=1)
    f, b = bench.algorithmic_counts(inp), bench.algorithmic_counts(inp, backward=True)
    B, L, D, N = 2, 64, 32, 16
    assert b["mufu"] == 3 * B * L * D * N + 2 * 4 * B * L * D
    # gradients are fp32: the backward moves well over twice the forward's bytes
    assert b["bytes"] > 2 * f["bytes"]
    assert b["bytes"] >= 4 * 3 * B * L * D + 4 * 2 * B * L * N + 8 * B * D * (L // 16) * N
