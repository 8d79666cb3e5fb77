"""Host-side helpers for running the forward on several GPUs, one process each.

Every (batch, head, query block) tile of the forward is independent: a multi-GPU
run splits batch elements (or heads) across ranks and needs no exchange on the
data path.  Only timings are reduced across ranks, with a max, so that a job is
as fast as its slowest rank.
"""

from __future__ import annotations

from typing import Tuple


def batch_shard(B: int, rank: int, world: int) -> Tuple[int, int]:
    """Contiguous [start, stop) slice of B batch elements owned by ``rank``.

    The first ``B % world`` ranks own one extra element; a rank may own none.
    """
    if world < 1 or not 0 <= rank < world or B < 0:
        raise ValueError("bad shard request")
    base, extra = divmod(B, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def max_over_ranks(value: float, world: int) -> float:
    """Maximum of ``value`` over all ranks of the default process group.

    Uses a CUDA tensor when the group's backend is NCCL and a CPU tensor
    otherwise (gloo).  With ``world == 1`` it returns ``value`` unchanged.
    """
    if world == 1:
        return float(value)
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(value)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
