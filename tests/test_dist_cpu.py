"""Multi-process (gloo, world_size 2, CPU) checks of the replica logic that
bench.py uses on N GPUs: the slowest rank's time decides and the work of all
ranks adds up.  No GPU needed."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys
    import torch.distributed as dist
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        got = bench.max_over_ranks([10.0 + rank, 5.0 - rank, 0.5 * rank])
        value = bench.replica_throughput(1000, world, got[0])
        q.put((rank, got, value))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, value in results:
        assert got == [11.0, 5.0, 0.5]          # max over ranks, same on every rank
        assert value == pytest.approx(1000 * 2 / 11.0e-3)


def test_single_process_is_identity():
    import bench
    assert bench.max_over_ranks([3.0, 4.0]) == [3.0, 4.0]
    assert bench.replica_throughput(10, 1, 2.0) == pytest.approx(5000.0)


# ---------------------------------------------------------------------------
# the sequence split over ranks (lshard): exchange and composition of maps
# ---------------------------------------------------------------------------

class _OracleOps:
    """The three steps of lshard.fwd computed by the CPU oracle, on CPU
    tensors, so the exchange between gloo ranks is checked without a GPU:
    the map of a piece is (state from 0, sum of Delta), composition is
    h <- exp(A s) h + e, and fwd is the oracle's scan from the given state."""

    def __init__(self):
        import oracle
        self.orc = oracle.get()

    def seq_map(self, x, delta, A, B, delta_bias=None):
        import numpy as np
        import torch
        Bz, L, Dm = x.shape
        N = A.shape[1]
        _, hl = self.orc.fwd(x.numpy(), delta.numpy(), A.numpy(), B.numpy(),
                             np.zeros((Bz, L, N)),
                             delta_bias=None if delta_bias is None else delta_bias.numpy())
        v = delta.numpy().astype(np.float64) + (0.0 if delta_bias is None
                                                else delta_bias.numpy()[None, None, :])
        sp = np.vectorize(self.orc.softplus)(v)
        return torch.from_numpy(hl), torch.from_numpy(sp.sum(axis=1))

    def fold_maps(self, count, maps_h, maps_s, A, h0=None):
        import numpy as np
        import torch
        h = np.zeros(maps_h.shape[1:]) if h0 is None else h0.numpy().astype(np.float64)
        for j in range(count):
            h = np.exp(A.numpy()[None] * maps_s[j].numpy()[..., None]) * h + maps_h[j].numpy()
        return torch.from_numpy(h)

    def fwd(self, x, delta, A, B, C, D=None, z=None, delta_bias=None, h0=None, y=None,
            h_last=None):
        import torch
        np_ = lambda t: None if t is None else t.numpy()
        yy, hl = self.orc.fwd(np_(x), np_(delta), np_(A), np_(B), np_(C), D=np_(D), z=np_(z),
                              delta_bias=np_(delta_bias), h0=np_(h0))
        return torch.from_numpy(yy), torch.from_numpy(hl)


def _lshard_worker(rank, world, port, q):
    import sys

    import numpy as np
    import torch
    import torch.distributed as dist
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    sys.path.insert(0, os.path.join(root, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from selective_state_space_31_b200 import lshard, synth
        inp = synth.make_fwd(2, 12 * world, 5, 4, in_dtype="f32", seed=81, has_h0=True)
        P = inp.L // world
        sl = lambda a: torch.from_numpy(np.ascontiguousarray(a[:, rank * P:(rank + 1) * P]))
        t = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a))
        y, hl = lshard.fwd(_OracleOps(), sl(inp.x), sl(inp.delta), t(inp.A), sl(inp.B),
                           sl(inp.C), D=t(inp.Dskip), z=sl(inp.z), delta_bias=t(inp.delta_bias),
                           h0=t(inp.h0))
        q.put((rank, y.numpy(), hl.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_lshard_exchange_gloo(world):
    """Each gloo rank scans its piece of the sequence from the state that the
    all-gathered maps of the earlier pieces give; the pieces joined equal the
    oracle's scan of the whole sequence, and the last rank's state is its
    h_last."""
    import numpy as np

    import oracle
    from selective_state_space_31_b200 import synth
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_lshard_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=180) for _ in procs), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    inp = synth.make_fwd(2, 12 * world, 5, 4, in_dtype="f32", seed=81, has_h0=True)
    ry, rh = oracle.get().fwd(inp.x, inp.delta, inp.A, inp.B, inp.C, D=inp.Dskip, z=inp.z,
                              delta_bias=inp.delta_bias, h0=inp.h0)
    gy = np.concatenate([r[1] for r in res], axis=1)
    np.testing.assert_allclose(gy, ry, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(res[-1][2], rh, rtol=1e-10, atol=1e-12)
