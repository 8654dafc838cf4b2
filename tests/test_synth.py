"""Seeded input generator: determinism, shapes, and bf16 rounding against
torch's own float32 -> bfloat16 conversion (round to nearest even)."""
import numpy as np
import torch

from selective_state_space_31_b200 import synth


def test_round_bf16_matches_torch():
    rng = np.random.default_rng(0)
    a = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10,
                        np.array([1.0, -0.0, 65504.0, 1e-38, 3.0e38], np.float32)])
    # include exact ties: 1 + 2^-8 (tie, even -> down) and 1 + 3*2^-8 (tie, odd -> up)
    a = np.concatenate([a, np.array([1 + 2**-8, 1 + 3 * 2**-8, -(1 + 2**-8)], np.float32)])
    ours = synth.round_bf16(a)
    ref = torch.from_numpy(a).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(ours.view(np.uint32), ref.view(np.uint32))
    assert np.array_equal(synth.bf16_bits(ours), torch.from_numpy(a).to(torch.bfloat16)
                          .view(torch.int16).numpy().view(np.uint16))


def test_deterministic_and_shapes():
    a = synth.make_fwd(2, 33, 24, 16, seed=5, has_h0=True)
    b = synth.make_fwd(2, 33, 24, 16, seed=5, has_h0=True)
    for f in ("x", "delta", "z", "B", "C", "Dskip", "delta_bias", "h0", "A"):
        assert np.array_equal(getattr(a, f), getattr(b, f)), f
    assert a.x.shape == (2, 33, 24) and a.B.shape == (2, 33, 16) and a.h0.shape == (2, 24, 16)
    assert np.array_equal(synth.round_bf16(a.x), a.x)  # already bf16-exact
    c = synth.make_fwd(2, 33, 24, 16, seed=6)
    assert not np.array_equal(a.x, c.x)


def test_workload_recipes():
    t = synth.tiny_fp32()
    assert (t.Bsz, t.L, t.D, t.N, t.in_dtype) == (1, 512, 64, 16, "f32")
    assert t.z is None and t.delta_bias is None and t.h0 is None
    assert np.allclose(t.A[3], -(np.arange(16) + 1))
    # delta_raw = N(0,1) - 1
    assert -1.2 < float(t.delta.mean()) < -0.8
    bias = synth.dt_bias(1, 4096)
    u = np.log1p(np.exp(bias.astype(np.float64)))     # softplus(bias) recovers u
    assert u.min() >= 1e-3 * 0.999 and u.max() <= 0.1 * 1.001


def test_decode_tokens():
    dec = synth.make_decode(Bsz=4, D=8, N=16, steps=3, seed=4)
    t0, t0b, t1 = dec.token(0), dec.token(0), dec.token(1)
    assert np.array_equal(t0["x"], t0b["x"]) and not np.array_equal(t0["x"], t1["x"])
    assert t0["B"].shape == (4, 16) and t0["z"].shape == (4, 8)
