"""Request sharding across ranks (one process per GPU).

Drafting, confidence and verification are independent per request, so each rank owns
a contiguous block of B_local requests (weak scaling).  The prefix scheduler is the
one global step: it allocates verify slots over the whole batch against one
steps-per-second curve, so the fp32 survival scores of every rank are all-gathered
before it, every rank runs the same deterministic scheduler on the global batch, and
each keeps the lengths of its own requests.  Noise keys use the global request index
(``b_offset``), so results do not depend on how the batch is sharded.
"""
from __future__ import annotations


def request_offset(rank: int, B_local: int) -> int:
    """Global index of this rank's first request."""
    return rank * B_local


def gather_scores(P_local, out=None, group=None):
    """All-gather [B_local, gamma] fp32 scores into the global [world * B_local, gamma].

    Rank r's block lands at rows r * B_local .. (r + 1) * B_local - 1 (NCCL on GPUs,
    gloo on CPU tensors).
    """
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    if out is None:
        out = torch.empty((world * P_local.shape[0],) + tuple(P_local.shape[1:]),
                          dtype=P_local.dtype, device=P_local.device)
    dist.all_gather_into_tensor(out, P_local.contiguous(), group=group)
    return out


def local_lengths(L_global, rank: int, B_local: int):
    """This rank's slice of the global verify lengths."""
    start = request_offset(rank, B_local)
    return L_global[start:start + B_local]
