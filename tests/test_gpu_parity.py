"""GPU parity of the CUDA library against the CPU oracle on seeded inputs of
sizes the oracle finishes in seconds: several chunks and pipeline stages, a
ragged tail, every kernel variant and option, edge cases."""
import numpy as np
import pytest
import torch

import gpu_util as gu
from selective_state_space_31_b200 import synth

pytestmark = pytest.mark.gpu


def _case(inp, cfg=None, expect_path=None):
    plan = gu.make_plan(inp)
    if cfg:
        plan.set_config(**cfg)
    info = plan.info()
    if expect_path is not None:
        assert info["path"] == expect_path, info
    gy, gh = gu.run_gpu(inp, plan)
    ry, rh = gu.run_oracle(inp)
    gu.assert_parity(gy, ry, gh, rh, gu.TOL[inp.in_dtype if inp.out_dtype == inp.in_dtype
                                             else "bf16"], f"{inp.name} {cfg} {info}")
    assert plan.status() == 0
    return plan


def test_tiny_fp32_workload():
    """The tiny fp32 case (B=1, L=512, D=64, N=16), fp32 tolerance 1e-5."""
    _case(synth.tiny_fp32(), expect_path=0)


@pytest.mark.parametrize("lpc,warps", [(4, 4), (8, 2), (16, 4)])
@pytest.mark.parametrize("grid", [5, 40])
def test_parts_chained_across_ctas(lpc, warps, grid):
    """grid=5 splits rows between CTAs; grid=40 gives CTAs less than a row
    each, so a row passes through a chain of CTAs."""
    inp = synth.make_fwd(3, 389, 64, 16, seed=21, has_h0=True)
    _case(inp, dict(lanes_per_chan=lpc, warps_per_cta=warps, grid=grid, tile_t=32,
                    chans_per_lane=1, segments=1), expect_path=0)


@pytest.mark.parametrize("grid", [1, 2, 7, 0, 64, 5000])
def test_schedule_grid_sizes(grid):
    """One CTA walking every unit, small grids, the default, and grids
    larger than the work (capped by the number of items)."""
    inp = synth.make_fwd(2, 1000, 128, 16, seed=22, has_h0=True)
    _case(inp, dict(grid=grid, segments=1), expect_path=0)


@pytest.mark.parametrize("N", [4, 8, 16])
def test_fp32_fast_path_dstate(N):
    inp = synth.make_fwd(2, 200, 32, N, in_dtype="f32", seed=23, has_h0=True)
    _case(inp, expect_path=0)


@pytest.mark.parametrize("N", [8, 16])
def test_bf16_in_fp32_out(N):
    inp = synth.make_fwd(2, 257, 48, N, in_dtype="bf16", out_dtype="f32", seed=24)
    _case(inp, expect_path=0)


@pytest.mark.parametrize("shape,dt", [((2, 77, 37, 16), "bf16"), ((1, 130, 24, 1), "f32"),
                                      ((2, 64, 16, 2), "f32"), ((1, 65, 40, 12), "bf16"),
                                      ((1, 33, 8, 32), "f32"), ((1, 20, 8, 64), "bf16"),
                                      ((2, 50, 16, 4), "bf16")])
def test_general_path(shape, dt):
    """Shapes the fast path does not take run on the general kernel."""
    Bz, L, D, N = shape
    inp = synth.make_fwd(Bz, L, D, N, in_dtype=dt, seed=25, has_h0=True)
    _case(inp, expect_path=1)


@pytest.mark.parametrize("softplus,z,bias,D,h0", [(False, False, False, False, False),
                                                  (True, False, True, False, True),
                                                  (False, True, False, True, False)])
def test_option_combinations(softplus, z, bias, D, h0):
    inp = synth.make_fwd(2, 150, 64, 16, seed=26, has_z=z, has_bias=bias, has_D=D, has_h0=h0,
                         delta_softplus=softplus)
    if not softplus:
        inp.delta = np.abs(inp.delta) * np.float32(0.1)   # keep Delta positive and small
        inp.delta = synth.round_bf16(inp.delta)
    _case(inp, expect_path=0)


def test_misaligned_pointers_take_general_kernel():
    inp = synth.make_fwd(1, 100, 64, 16, seed=27)
    plan = gu.make_plan(inp)
    dev = gu.upload(inp)
    # views that start 2 bytes into a buffer: valid, but not 16-byte aligned
    for k in ("x", "delta", "z"):
        buf = torch.empty(dev[k].numel() + 1, dtype=dev[k].dtype, device="cuda")
        buf[1:].copy_(dev[k].reshape(-1))
        dev[k] = buf[1:].view(dev[k].shape)
        assert dev[k].data_ptr() % 16 != 0
    gy, gh = gu.run_gpu(inp, plan, dev)
    ry, rh = gu.run_oracle(inp)
    gu.assert_parity(gy, ry, gh, rh, gu.TOL["bf16"], "misaligned")


def test_zero_length_and_empty():
    inp = synth.make_fwd(2, 0, 16, 16, in_dtype="f32", seed=28, has_h0=True)
    gy, gh = gu.run_gpu(inp)
    assert gy.shape == (2, 0, 16)
    np.testing.assert_array_equal(gh, inp.h0.astype(np.float64))
    inp = synth.make_fwd(0, 10, 16, 16, in_dtype="f32", seed=28)
    gy, gh = gu.run_gpu(inp)
    assert gy.shape == (0, 10, 16)


def test_deterministic():
    inp = synth.make_fwd(2, 700, 128, 16, seed=29, has_h0=True)
    plan = gu.make_plan(inp)
    plan.set_config(grid=7)
    dev = gu.upload(inp)
    a = gu.run_gpu(inp, plan, dev)
    b = gu.run_gpu(inp, plan, dev)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_h0_split_matches_full_run():
    """Resuming from h_last of [0, k) reproduces the full run on [k, L)."""
    inp = synth.make_fwd(2, 512, 64, 16, in_dtype="f32", seed=30, has_h0=True)
    full_y, full_h = gu.run_gpu(inp)
    k = 200
    first = synth.make_fwd(2, k, 64, 16, in_dtype="f32", seed=30, has_h0=True)
    for f in ("x", "delta", "z", "B", "C"):
        setattr(first, f, getattr(inp, f)[:, :k].copy())
    y1, h1 = gu.run_gpu(first)
    second = synth.make_fwd(2, 512 - k, 64, 16, in_dtype="f32", seed=30, has_h0=True)
    for f in ("x", "delta", "z", "B", "C"):
        setattr(second, f, getattr(inp, f)[:, k:].copy())
    second.h0 = h1.astype(np.float32)
    y2, h2 = gu.run_gpu(second)
    assert gu.normwise(np.concatenate([y1, y2], axis=1), full_y) < 1e-5
    assert gu.normwise(h2, full_h) < 1e-5


def test_elementwise_variant_page_example():
    """The elementwise example's shapes (batch=2, seq_len=6, d=4, A in (0,1),
    h0 = 0): output (2, 6, 4), values against the oracle."""
    import oracle
    from selective_state_space_31_b200 import binding as bnd
    d = synth.make_direct(2, 6, 4, seed=31, has_h0=False)
    dev = {k: gu.dev_tensor(d[k]) for k in ("x", "A", "B", "C")}
    y, hl = bnd.direct(dev["x"], dev["A"], dev["B"], dev["C"])
    assert tuple(y.shape) == (2, 6, 4)
    ry, rh = oracle.get().direct(d["x"], d["A"], d["B"], d["C"])
    gu.assert_parity(y.cpu().numpy(), ry, hl.cpu().numpy(), rh, 1e-5, "direct")


@pytest.mark.parametrize("dt,a_zero", [("bf16", False), ("f32", True), ("f32", False)])
def test_elementwise_variant(dt, a_zero):
    import oracle
    from selective_state_space_31_b200 import binding as bnd
    d = synth.make_direct(3, 777, 96, seed=32, in_dtype=dt, a_zero=a_zero)
    dev = {k: gu.dev_tensor(d[k], dt) for k in ("x", "A", "B", "C")}
    h0 = gu.dev_tensor(d["h0"])
    y, hl = bnd.direct(dev["x"], dev["A"], dev["B"], dev["C"], h0=h0)
    ry, rh = oracle.get().direct(d["x"], d["A"], d["B"], d["C"], h0=d["h0"])
    gu.assert_parity(y.float().cpu().numpy(), ry, hl.cpu().numpy(), rh, gu.TOL[dt], "direct")
    if a_zero:   # memoryless: y_t = C_t B_t x_t
        np.testing.assert_allclose(y.cpu().numpy(), d["C"] * d["B"] * d["x"], rtol=1e-6, atol=1e-6)


@pytest.mark.parametrize("N,dt", [(16, "bf16"), (16, "f32"), (8, "bf16"), (4, "f32"),
                                  (32, "f32"), (12, "f32")])
def test_decode_steps_match_full_sequence(N, dt):
    """L decode steps reproduce the oracle's full-sequence outputs and state."""
    import oracle
    from selective_state_space_31_b200 import binding as bnd
    inp = synth.make_fwd(4, 40, 96, N, in_dtype=dt, seed=33, has_h0=True)
    dev = gu.upload(inp)
    state = dev["h0"].clone()
    ys = []
    for t in range(inp.L):
        ys.append(bnd.step(state, dev["x"][:, t].contiguous(), dev["delta"][:, t].contiguous(),
                           dev["A"], dev["B"][:, t].contiguous(), dev["C"][:, t].contiguous(),
                           D=dev["D"], z=dev["z"][:, t].contiguous(),
                           delta_bias=dev["delta_bias"]))
    y = torch.stack(ys, dim=1).float().cpu().numpy()
    ry, rh = oracle.get().fwd(inp.x, inp.delta, inp.A, inp.B, inp.C, D=inp.Dskip, z=inp.z,
                              delta_bias=inp.delta_bias, h0=inp.h0)
    gu.assert_parity(y, ry, state.cpu().numpy(), rh, gu.TOL[dt], f"decode N={N}")


def test_decode_streaming_many_tiles_per_cta():
    """Enough channels that the streaming step kernel's CTAs each run several
    state tiles through their ring, with a ragged last tile (16 x 4004
    channels = 1001 tiles of 64): three steps against the oracle on every
    channel."""
    import oracle
    from selective_state_space_31_b200 import binding as bnd
    inp = synth.make_fwd(16, 3, 4004, 16, in_dtype="bf16", seed=35, has_h0=True)
    dev = gu.upload(inp)
    state = dev["h0"].clone()
    ys = []
    for t in range(inp.L):
        ys.append(bnd.step(state, dev["x"][:, t].contiguous(), dev["delta"][:, t].contiguous(),
                           dev["A"], dev["B"][:, t].contiguous(), dev["C"][:, t].contiguous(),
                           D=dev["D"], z=dev["z"][:, t].contiguous(),
                           delta_bias=dev["delta_bias"]))
    y = torch.stack(ys, dim=1).float().cpu().numpy()
    ry, rh = oracle.get().fwd(inp.x, inp.delta, inp.A, inp.B, inp.C, D=inp.Dskip, z=inp.z,
                              delta_bias=inp.delta_bias, h0=inp.h0)
    gu.assert_parity(y, ry, state.cpu().numpy(), rh, gu.TOL["bf16"], "decode, many tiles")


@pytest.mark.parametrize("cfg", [None, dict(lanes_per_chan=4, warps_per_cta=4, tile_t=32),
                                 dict(lanes_per_chan=8, warps_per_cta=4, tile_t=64, grid=2),
                                 dict(lanes_per_chan=16, warps_per_cta=4, tile_t=64),
                                 dict(lanes_per_chan=4, warps_per_cta=4, tile_t=32,
                                      chans_per_lane=2),
                                 dict(lanes_per_chan=8, warps_per_cta=4, tile_t=32,
                                      chans_per_lane=2, segments=2)])
@pytest.mark.parametrize("shift", [0.0, 3.0])
def test_zoh_fused(cfg, shift):
    """Zero-order hold ([P1] "Vi du Python": Bbar = (exp(Delta A) - 1)/A * B)
    on the fused kernel: bf16, gate, skip, bias, h0, ragged L.  shift=3 moves
    Delta up so most |Delta A| take the e - 1 branch; shift=0 keeps most in
    the Taylor branch."""
    inp = synth.make_fwd(3, 389, 64, 16, seed=41, has_h0=True, delta_shift=shift, zoh=True)
    _case(inp, cfg, expect_path=0)


@pytest.mark.parametrize("N", [4, 16])
def test_zoh_fp32_and_zero_A(N):
    """fp32 zero-order hold at the fp32 tolerance, with some A entries 0 (the
    limit Bbar = Delta * B) and some tiny."""
    A = -np.tile(np.arange(1, N + 1, dtype=np.float32), (32, 1))
    A[::3, 0] = 0.0
    A[1::3, 1] = -1e-6
    inp = synth.make_fwd(2, 200, 32, N, in_dtype="f32", seed=42, has_h0=True, A=A, zoh=True)
    _case(inp, expect_path=0)


def test_zoh_general_path():
    """Zero-order hold on the general kernel (odd dim and dstate)."""
    inp = synth.make_fwd(2, 77, 37, 12, in_dtype="f32", seed=43, has_h0=True, zoh=True)
    _case(inp, expect_path=1)


@pytest.mark.parametrize("N,dt", [(16, "bf16"), (4, "f32"), (12, "f32")])
def test_zoh_decode_steps(N, dt):
    """Zero-order-hold decode steps reproduce the oracle's full sequence."""
    import oracle
    from selective_state_space_31_b200 import binding as bnd
    inp = synth.make_fwd(4, 24, 96, N, in_dtype=dt, seed=44, has_h0=True, delta_shift=1.0,
                         zoh=True)
    dev = gu.upload(inp)
    state = dev["h0"].clone()
    ys = []
    for t in range(inp.L):
        ys.append(bnd.step(state, dev["x"][:, t].contiguous(), dev["delta"][:, t].contiguous(),
                           dev["A"], dev["B"][:, t].contiguous(), dev["C"][:, t].contiguous(),
                           D=dev["D"], z=dev["z"][:, t].contiguous(),
                           delta_bias=dev["delta_bias"], zoh=True))
    y = torch.stack(ys, dim=1).float().cpu().numpy()
    ry, rh = gu.run_oracle(inp)
    gu.assert_parity(y, ry, state.cpu().numpy(), rh, gu.TOL[dt], f"zoh decode N={N}")


def test_zoh_refused_with_elementwise_variant():
    from selective_state_space_31_b200 import binding as bnd
    with pytest.raises(bnd.SsmError):
        bnd.Plan(1, 4, 8, 1, torch.float32, torch.float32, bnd.A_DIRECT | bnd.ZOH,
                 torch.device("cuda", 0))


@pytest.mark.parametrize("case", ["abar_zero", "a_zero"])
@pytest.mark.parametrize("dim,path", [(64, 0), (37, 1)])
def test_degenerate_A(case, dim, path):
    """The Mamba form's degenerate transitions on the fused (dim 64) and the
    general (dim 37) kernel: A = -1e30 makes Abar exactly 0 (memoryless,
    y_t = (sum_n C_t Delta_t B_t x_t + D x_t) silu(z_t), checked against that
    closed form too); A = 0 makes Abar = 1 and the state a prefix sum of
    Delta B x from h0."""
    A = np.full((dim, 16), -1e30 if case == "abar_zero" else 0.0, np.float32)
    inp = synth.make_fwd(2, 389, dim, 16, in_dtype="f32", seed=45, has_h0=True, A=A)
    plan = _case(inp, expect_path=path)
    if case == "abar_zero":
        gy, _ = gu.run_gpu(inp, plan)
        v = inp.delta.astype(np.float64) + inp.delta_bias[None, None, :]
        dlt = np.maximum(v, 0) + np.log1p(np.exp(-np.abs(v)))
        cb = np.einsum("bln,bln->bl", inp.C.astype(np.float64), inp.B.astype(np.float64))
        s = cb[:, :, None] * dlt * inp.x + inp.Dskip[None, None, :] * inp.x
        zz = inp.z.astype(np.float64)
        ref = s * zz / (1.0 + np.exp(-zz))
        assert gu.normwise(gy, ref) <= gu.TOL["f32"]


def test_fwd_replayed_from_a_cuda_graph():
    """Two forward calls captured in one CUDA graph and replayed four times:
    the launch epoch and finished-CTA counter live on the device (no memset,
    no host round trip), so every replay hands carried states between CTAs
    correctly and reproduces the eager result bit for bit."""
    inp = synth.make_fwd(3, 389, 64, 16, seed=46, has_h0=True)
    plan = gu.make_plan(inp)
    plan.set_config(lanes_per_chan=4, warps_per_cta=4, grid=4, tile_t=32, chans_per_lane=1,
                    segments=1)  # 6 rows on 4 CTAs
    assert plan.info()["parts_per_row"] >= 2
    dev = gu.upload(inp)
    y = torch.empty((inp.Bsz, inp.L, inp.D), dtype=torch.bfloat16, device="cuda")
    hl = torch.empty((inp.Bsz, inp.D, inp.N), dtype=torch.float32, device="cuda")

    def call():
        plan.fwd(dev["x"], dev["delta"], dev["A"], dev["B"], dev["C"], D=dev["D"], z=dev["z"],
                 delta_bias=dev["delta_bias"], h0=dev["h0"], y=y, h_last=hl)

    call()
    torch.cuda.synchronize()
    y_ref, hl_ref = y.clone(), hl.clone()
    ry, rh = gu.run_oracle(inp)
    gu.assert_parity(y_ref.float().cpu().numpy(), ry, hl_ref.cpu().numpy(), rh, gu.TOL["bf16"],
                     "eager")
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        call()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        call()
        call()
    for _ in range(4):
        y.zero_()
        hl.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(y, y_ref) and torch.equal(hl, hl_ref)
    assert plan.status() == 0
    del graph


def test_timeout_is_reported_without_hanging():
    """A work item that never hands its state on makes the CTA running the
    next part of that row wait until the bound expires: the kernel records
    SSM_ERR_TIMEOUT and returns; the plan stays usable and the next call is
    exact again."""
    inp = synth.make_fwd(4, 512, 32, 16, seed=34)
    plan = gu.make_plan(inp)
    plan.set_config(lanes_per_chan=4, warps_per_cta=4, grid=3, chans_per_lane=1, segments=1)
    info = plan.info()
    S, PL = info["stages_per_row"], info["stages_per_part"]
    assert info["rows"] == 4 and info["grid"] == 3 and info["parts_per_row"] >= 2, info
    # the first part of row 2 ends at stage PL - 1; the CTA running part 2 of row 2 waits for it
    plan.set_debug(wait_timeout_ns=50_000_000, drop_unit=2 * S + PL - 1)
    dev = gu.upload(inp)
    gu.run_gpu(inp, plan, dev)
    assert plan.status() == 5  # SSM_ERR_TIMEOUT
    plan.set_debug(0, -1)
    gy, gh = gu.run_gpu(inp, plan, dev)
    ry, rh = gu.run_oracle(inp)
    gu.assert_parity(gy, ry, gh, rh, gu.TOL["bf16"], "after timeout")
    assert plan.status() == 0
