"""The scan with its sequence split over ranks (one process per GPU,
torch.distributed): rank r holds tokens [r*L/W, (r+1)*L/W) of every input.

Each rank computes the map of its own piece (ssm_scan_seq_map: the sum of
Delta and the state reached from 0), the maps are all-gathered (one record
of batch*dim*(dstate+1) fp32 per rank, into local memory), and rank r
composes the maps of ranks 0..r-1 onto h0 (ssm_scan_fold_maps): that is the
exact state at its first token ("Scan bien recurrence thanh phep toan co the
song song hoa ra sao?": per-token maps compose associatively).  It then
scans its piece from that state.  The exchange is one all-gather of small
records; no device reads another's memory.

``ops`` is anything with the Plan methods seq_map, fold_maps and fwd (the
CUDA plan in use; tests may pass another implementation of the same three
steps to check the exchange on CPU ranks)."""
from __future__ import annotations

import torch
import torch.distributed as dist


def start_state(ops, x, delta, A, B, delta_bias=None, h0=None, group=None):
    """The exact state at this rank's first token: the maps of all earlier
    ranks composed onto h0 (h0, when given, is the whole sequence's start
    state and the same on every rank)."""
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    # every rank computes its map (the last one's is used by no one, but all
    # ranks then take the same steps and the wall time is unchanged)
    map_h, map_s = ops.seq_map(x, delta, A, B, delta_bias=delta_bias)
    rec = torch.cat([map_h.reshape(-1), map_s.reshape(-1)])
    recs = [torch.empty_like(rec) for _ in range(world)]
    dist.all_gather(recs, rec, group=group)
    nh = map_h.numel()
    maps_h = torch.stack([r[:nh] for r in recs[:max(rank, 1)]]).reshape(-1, *map_h.shape)
    maps_s = torch.stack([r[nh:] for r in recs[:max(rank, 1)]]).reshape(-1, *map_s.shape)
    return ops.fold_maps(rank, maps_h.contiguous(), maps_s.contiguous(), A, h0=h0)


def fwd(ops, x, delta, A, B, C, D=None, z=None, delta_bias=None, h0=None, group=None,
        y=None, h_last=None):
    """This rank's piece of the scan of a sequence split over the group.
    ``ops`` must be created for this piece's length with HAS_H0 set.  Returns
    (y of the piece, state after the piece); the last rank's state is the
    whole sequence's h_last."""
    hs = start_state(ops, x, delta, A, B, delta_bias=delta_bias, h0=h0, group=group)
    return ops.fwd(x, delta, A, B, C, D=D, z=z, delta_bias=delta_bias, h0=hs, y=y,
                   h_last=h_last)
