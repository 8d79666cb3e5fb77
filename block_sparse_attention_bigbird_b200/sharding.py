"""Host-side helpers for running the kernels on several GPUs, one process each.

Every (batch, head, query block) tile of the forward -- and every (batch, head)
slice of the gradients -- is independent: a multi-GPU run splits batch elements,
or for a long sequence with few batch elements its heads, across ranks and
needs no exchange on the data path.  Only timings are reduced across ranks,
with a max, so that a job is as fast as its slowest rank.

A long sequence can also be split by ranges of query blocks, every rank reading
the whole K and V of each head (replicated by a plain read): the forward then
needs no exchange either (each rank owns its rows of O and lse), while in the
backward each rank's dK and dV are partial sums over its query rows and are
added across ranks (``sum_over_ranks``), the one data-path collective.
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


def query_block_shard(row_ptr, nb: int, H: int, rank: int, world: int) -> Tuple[int, int]:
    """Contiguous [start, stop) range of query blocks owned by ``rank``.

    The cut points balance the non-zero blocks summed over heads (a global row
    holds every key block, so equal block counts would not give equal work):
    rank r's range ends at the first block where the running total reaches
    (r + 1) / world of the whole.  A rank may own an empty range.
    """
    import numpy as np
    if world < 1 or not 0 <= rank < world or nb < 0 or H < 1:
        raise ValueError("bad shard request")
    rp = np.asarray(row_ptr, dtype=np.int64)
    if rp.shape[0] != H * nb + 1:
        raise ValueError("row_ptr must have H * nb + 1 entries")
    per_block = (rp[1:] - rp[:-1]).reshape(H, nb).sum(axis=0)  # work of query block i over heads
    cum = np.concatenate([[0], np.cumsum(per_block)])
    total = int(cum[-1])

    def cut(r: int) -> int:  # first block boundary whose running total reaches r / world of the whole
        if r <= 0:
            return 0
        if r >= world:
            return nb
        return int(np.searchsorted(cum, (total * r + world - 1) // world, side="left"))

    return cut(rank), cut(rank + 1)


def query_rows(row_ptr, col_idx, nb: int, H: int, q0: int, q1: int):
    """The layout's block-CSR with only query blocks [q0, q1) of every head kept
    (the other rows empty): the layout of a rank owning those query blocks,
    built with bsa_layout_from_csr over the full sequence length."""
    import numpy as np
    rp = np.asarray(row_ptr, dtype=np.int64)
    ci = np.asarray(col_idx, dtype=np.int32)
    counts = (rp[1:] - rp[:-1]).reshape(H, nb).copy()
    keep = np.zeros(nb, dtype=bool)
    keep[q0:q1] = True
    counts[:, ~keep] = 0
    out_rp = np.concatenate([[0], np.cumsum(counts.reshape(-1))]).astype(np.int32)
    pieces = [ci[rp[h * nb + i]:rp[h * nb + i + 1]] for h in range(H) for i in range(q0, q1)]
    out_ci = np.concatenate(pieces).astype(np.int32) if pieces else np.zeros(0, dtype=np.int32)
    return out_rp, out_ci


def sum_over_ranks(t, world: int):
    """In-place sum of tensor ``t`` over all ranks of the default process group
    (NCCL for CUDA tensors, gloo for CPU ones); returns ``t``."""
    if world == 1:
        return t
    import torch.distributed as dist
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return t


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
