"""Host-side helpers for running the kernels on several GPUs, one process each.

Every (batch, head, query block) tile of the forward -- and every (batch, head)
slice of the gradients -- is independent: a multi-GPU run splits batch elements,
or for a long sequence with few batch elements its heads, across ranks and
needs no exchange on the data path.  Only timings are reduced across ranks,
with a max, so that a job is as fast as its slowest rank.
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


def head_shard(H: int, rank: int, world: int) -> Tuple[int, int]:
    """Contiguous [start, stop) slice of H heads owned by ``rank`` (as batch_shard).

    Head sharding serves long sequences with a batch too small to split
    (one genomic sequence of 131072 tokens): each rank runs its heads of the
    same sequence, whose layout rows depend on the head alone.
    """
    return batch_shard(H, rank, world)


def head_rows(row_ptr, col_idx, nb: int, h0: int, h1: int):
    """The block-CSR rows of heads [h0, h1) of a head-major layout, as a CSR of
    h1 - h0 heads (row_ptr rebased to 0): the layout a rank owning those heads
    builds with bsa_layout_from_csr."""
    import numpy as np
    rp = np.asarray(row_ptr, dtype=np.int64)
    lo, hi = int(rp[h0 * nb]), int(rp[h1 * nb])
    return (rp[h0 * nb:h1 * nb + 1] - lo).astype(np.int32), np.asarray(col_idx[lo:hi], dtype=np.int32)


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
