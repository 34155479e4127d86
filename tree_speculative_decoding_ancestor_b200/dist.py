"""Multi-GPU helper of the batch-sharded path.

Sequences are independent through every step (mask, attention, verification,
commit), so with several GPUs each rank verifies its own batch and the data
path has no collective.  The one optional exchange is a global view of the
verification results: all_gather_accepted gives every rank the accepted
tokens, paths and counts of every rank's batch, in rank order -- one
all-gather per tensor over the process group (NCCL over NVLink/NVSwitch for
device tensors; gloo for host tensors).  Ranks may hold batches of different
sizes: the sizes are gathered first and the tensors padded to the largest.
"""

from __future__ import annotations

import torch

from .binding import VerifyResult


def all_gather_accepted(result: VerifyResult, group=None) -> VerifyResult:
    """The verification results of every rank's batch, concatenated along the
    batch in rank order (entries beyond a sequence's n_accepted are as the
    verifier left them).  Every rank must call it, with results of the same
    Tmax."""
    import torch.distributed as dist

    world = dist.get_world_size(group)
    dev = result.n_accepted.device
    B = result.n_accepted.shape[0]
    sizes = [torch.zeros(1, dtype=torch.int64, device=dev) for _ in range(world)]
    dist.all_gather(sizes, torch.tensor([B], dtype=torch.int64, device=dev), group=group)
    sizes = [int(s.item()) for s in sizes]
    bmax = max(sizes)
    out = []
    for t in result:
        padded = torch.zeros((bmax,) + tuple(t.shape[1:]), dtype=t.dtype, device=dev)
        padded[:B] = t
        parts = [torch.empty_like(padded) for _ in range(world)]
        dist.all_gather(parts, padded, group=group)
        out.append(torch.cat([p[:n] for p, n in zip(parts, sizes)], dim=0))
    return VerifyResult(*out)
