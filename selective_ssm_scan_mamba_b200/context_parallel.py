"""Context-parallel prefill: one long context split over the ranks of a
process group, each rank holding a consecutive chunk of whole blocks.

The forward recurrence is affine in its state, so each chunk acts on its start
state as h -> P h + H (P: product of the chunk's decays, H: the state it
reaches from zero). Each rank computes its chunk's (H, P) with
``bdscan.chunk_summary``; one all-gather gives every rank all summaries;
``bdscan.carry_fold`` composes those of the ranks before it into its start
state; a local ``bdscan.prefill`` from that state writes the chunk's y, its
block-boundary states (the cache) and its final state. The last rank's final
state is the whole context's.

The exchange is one all-gather of 2 x batch x D x N fp32 values per rank
(torch.distributed, NCCL on GPUs). Every compute step runs in the library's
kernels.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import bdscan


def prefill_context_parallel(x, dt, A, B, C, Dskip, block, group=None, z=None, h0=None, dt_softplus=True,
                             want_y=True, want_boundary=True):
    """Prefill of this rank's chunk of a context split over ``group`` in rank order.

    x, dt, z: [batch, L_r, D]; B, C: [batch, L_r, N]; L_r a multiple of ``block``
    (chunks may differ in length). h0: the context's initial state
    [batch, D, N] (the same on every rank; None = zero). Returns
    (y or None, h_out, boundary or None) for this chunk, as ``bdscan.prefill``.
    """
    rank = dist.get_rank(group)
    world = dist.get_world_size(group)
    H, P = bdscan.chunk_summary(x, dt, A, B, C, Dskip, block, dt_softplus=dt_softplus)
    mine = torch.stack([H, P])                            # [2, batch, D, N]
    parts = [torch.empty_like(mine) for _ in range(world)]
    dist.all_gather(parts, mine, group=group)
    gathered = torch.stack(parts)                         # [world, 2, batch, D, N], rank order
    H_all = gathered[:, 0].contiguous()
    P_all = gathered[:, 1].contiguous()
    h_in = bdscan.carry_fold(H_all, P_all, rank, h0=h0)
    return bdscan.prefill(x, dt, A, B, C, Dskip, block, z=z, h0=h_in, dt_softplus=dt_softplus, want_y=want_y,
                          want_boundary=want_boundary)
