"""Maps of whole sequences (ssm_scan_seq_map) and their composition
(ssm_scan_fold_maps), the pieces of a scan whose sequence is split over
devices: each map against the oracle, and a sequence cut into W pieces run
piece by piece (the exchange of maps that lshard.fwd does over ranks is
replaced by keeping them in one process) against the oracle's scan of the
whole sequence."""
import numpy as np
import pytest
import torch

import gpu_util as gu
import oracle
from selective_state_space_31_b200 import binding as bnd
from selective_state_space_31_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shape,dt,zoh", [((2, 3000, 256, 16), "bf16", False),
                                          ((1, 700, 64, 8), "f32", False),
                                          ((2, 1000, 128, 16), "bf16", True),
                                          ((2, 333, 37, 12), "f32", False)])
def test_seq_map_matches_oracle(shape, dt, zoh):
    """map_h = the state the sequence reaches from 0, map_s = sum of Delta;
    the last shape takes the general kernel."""
    Bz, L, Dm, N = shape
    inp = synth.make_fwd(Bz, L, Dm, N, in_dtype=dt, seed=91, zoh=zoh)
    dev = gu.upload(inp)
    plan = gu.make_plan(inp)
    mh, ms = plan.seq_map(dev["x"], dev["delta"], dev["A"], dev["B"],
                          delta_bias=dev["delta_bias"])
    torch.cuda.synchronize()
    assert plan.status() == 0
    orc = oracle.get()
    _, rh = orc.fwd(inp.x, inp.delta, inp.A, inp.B, np.zeros_like(inp.C),
                    delta_bias=inp.delta_bias, zoh=zoh)
    v = inp.delta.astype(np.float64) + inp.delta_bias[None, None, :]
    rs = np.vectorize(orc.softplus)(v).sum(axis=1)
    tol = gu.TOL[dt]
    assert gu.normwise(mh.cpu().numpy(), rh) <= tol
    assert gu.normwise(ms.cpu().numpy(), rs) <= max(tol, 1e-5)


@pytest.mark.parametrize("W", [2, 4])
@pytest.mark.parametrize("dt", ["bf16", "f32"])
def test_pieces_compose_to_the_whole_sequence(W, dt):
    Bz, L, Dm, N = 2, 4096, 256, 16
    inp = synth.make_fwd(Bz, L, Dm, N, in_dtype=dt, seed=92, has_h0=True)
    dev = gu.upload(inp)
    P = L // W
    flags = bnd.flags_for(z=inp.z, D=inp.Dskip, delta_bias=inp.delta_bias, h0=inp.h0)
    plan = bnd.Plan(Bz, P, Dm, N, gu.TDT[dt], gu.TDT[dt], flags, "cuda")
    piece = lambda t, r: t[:, r * P:(r + 1) * P].contiguous()
    maps = [plan.seq_map(piece(dev["x"], r), piece(dev["delta"], r), dev["A"],
                         piece(dev["B"], r), delta_bias=dev["delta_bias"]) for r in range(W)]
    maps_h = torch.stack([m[0] for m in maps])
    maps_s = torch.stack([m[1] for m in maps])
    ys, hl = [], None
    for r in range(W):
        hs = plan.fold_maps(r, maps_h, maps_s, dev["A"], h0=dev["h0"])
        y, hl = plan.fwd(piece(dev["x"], r), piece(dev["delta"], r), dev["A"], piece(dev["B"], r),
                         piece(dev["C"], r), D=dev["D"], z=piece(dev["z"], r),
                         delta_bias=dev["delta_bias"], h0=hs)
        ys.append(y)
    torch.cuda.synchronize()
    assert plan.status() == 0
    gy = torch.cat(ys, dim=1).float().cpu().numpy().astype(np.float64)
    ry, rh = gu.run_oracle(inp)
    gu.assert_parity(gy, ry, hl.cpu().numpy().astype(np.float64), rh, gu.TOL[dt],
                     f"{W} pieces")
