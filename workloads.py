"""Synthetic workloads for the BigBird block-sparse attention forward pass.

This module only describes the five benchmark shapes and draws their seeded
inputs.  It holds none of the attention or layout arithmetic, so that both the
CUDA path (through its binding) and the CPU oracle can be fed the very same
tensors without sharing any code of the method itself.

Input recipe (the same for every shape):
  * ``torch.Generator().manual_seed(seed)`` on the CPU;
  * draw ``q``, ``k``, ``v`` in that order as fp32 ``randn(B, H, L, d)``;
  * multiply by the per-shape factors below (all exact powers of two);
  * round to bf16 (round-to-nearest-even, torch's ``.to(torch.bfloat16)``).
The key-padding mask, when a shape has one, is 1 (keep) for the first
``L - key_pad_tail`` positions of every sequence and 0 after that.
"""

from __future__ import annotations

import dataclasses
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    description: str
    B: int
    H: int
    L: int
    d: int
    block: int
    window: int        # window radius, in blocks
    n_global: int      # number of global blocks (linspace rule)
    n_random: int      # random blocks per (head, query block)
    seed: int = 0      # layout seed (Philox key word 0)
    q_mul: float = 1.0
    k_mul: float = 1.0
    v_mul: float = 1.0
    key_pad_tail: int = 0   # number of trailing key positions masked out

    @property
    def nb(self) -> int:
        return self.L // self.block

    def as_dict(self) -> dict:
        return dataclasses.asdict(self)


WORKLOADS = {
    "tiny_b1h2l512": Workload(
        "tiny_b1h2l512", "B=1 H=2 L=512: 8 blocks, window +-1, global {0}, 1 random",
        B=1, H=2, L=512, d=64, block=64, window=1, n_global=1, n_random=1),
    "bert_b8h12l4096": Workload(
        "bert_b8h12l4096", "BERT-base shape B=8 H=12 L=4096: window +-1, 2 global, 3 random",
        B=8, H=12, L=4096, d=64, block=64, window=1, n_global=2, n_random=3),
    "long_b4h12l16384": Workload(
        "long_b4h12l16384", "B=4 H=12 L=16384: window +-2, 2 global, 3 random, k x2",
        B=4, H=12, L=16384, d=64, block=64, window=2, n_global=2, n_random=3, k_mul=2.0),
    "dense_globals_b1h16l8192": Workload(
        "dense_globals_b1h16l8192", "B=1 H=16 L=8192: window +-2, 13 global, 8 random",
        B=1, H=16, L=8192, d=64, block=64, window=2, n_global=13, n_random=8),
    "genomic_b1h8l131072": Workload(
        "genomic_b1h8l131072",
        "B=1 H=8 L=131072: window +-4, 2 global, 3 random, N(0,0.5^2), last 3072 keys padded",
        B=1, H=8, L=131072, d=64, block=64, window=4, n_global=2, n_random=3,
        q_mul=0.5, k_mul=0.5, v_mul=0.5, key_pad_tail=3072),
}

# Short aliases c1..c5 in the order the shapes are listed above.
ALIASES = {f"c{i + 1}": name for i, name in enumerate(WORKLOADS)}


def get(name: str) -> Workload:
    return WORKLOADS[ALIASES.get(name, name)]


def custom(B: int, H: int, L: int, window: int, n_global: int, n_random: int,
           seed: int = 0, key_pad_tail: int = 0, q_mul: float = 1.0,
           k_mul: float = 1.0, v_mul: float = 1.0, d: int = 64,
           block: int = 64) -> Workload:
    """A workload of arbitrary shape, drawn with the same recipe."""
    return Workload(f"custom_b{B}h{H}l{L}", "custom", B=B, H=H, L=L, d=d, block=block,
                    window=window, n_global=n_global, n_random=n_random, seed=seed,
                    q_mul=q_mul, k_mul=k_mul, v_mul=v_mul, key_pad_tail=key_pad_tail)


def make_qkv(w: Workload, data_seed: int = 0):
    """q, k, v as contiguous bf16 CPU tensors of shape [B, H, L, d]."""
    g = torch.Generator().manual_seed(data_seed)
    shape = (w.B, w.H, w.L, w.d)
    q = torch.randn(shape, generator=g, dtype=torch.float32)
    k = torch.randn(shape, generator=g, dtype=torch.float32)
    v = torch.randn(shape, generator=g, dtype=torch.float32)
    if w.q_mul != 1.0:
        q.mul_(w.q_mul)
    if w.k_mul != 1.0:
        k.mul_(w.k_mul)
    if w.v_mul != 1.0:
        v.mul_(w.v_mul)
    return (q.to(torch.bfloat16).contiguous(), k.to(torch.bfloat16).contiguous(),
            v.to(torch.bfloat16).contiguous())


def make_grad(w: Workload, seed: int = 1) -> torch.Tensor:
    """A loss gradient dL/dO for the backward: fp32 randn(B, H, L, d) from
    ``torch.Generator().manual_seed(seed)``, rounded to bf16."""
    g = torch.Generator().manual_seed(seed)
    return torch.randn((w.B, w.H, w.L, w.d), generator=g, dtype=torch.float32).to(torch.bfloat16).contiguous()


def make_key_mask(w: Workload) -> Optional[torch.Tensor]:
    """uint8 [B, L] key-padding mask (1 = keep), or None when the shape has none."""
    if w.key_pad_tail <= 0:
        return None
    m = torch.ones((w.B, w.L), dtype=torch.uint8)
    m[:, w.L - w.key_pad_tail:] = 0
    return m


def make_block_csr(H: int, nb: int, seed: int, p_empty: float = 0.1, p_full: float = 0.05,
                   max_len: Optional[int] = None, full_blocks=()):
    """A caller's block mask in CSR form (rows head-major), seeded.

    Each row (h, i) is empty with probability ``p_empty``, lists every key block
    with probability ``p_full`` and otherwise holds 1..max_len blocks drawn with
    replacement, in the drawn order (so rows come unsorted and may repeat a
    block).  Query blocks in ``full_blocks`` list every key block in every head.
    Returns (row_ptr int32 [H*nb+1], col_idx int32 [nnz]).
    """
    import numpy as np
    rng = np.random.default_rng(seed)
    max_len = max_len or max(1, nb // 3)
    full = set(int(x) for x in full_blocks)
    row_ptr, cols = [0], []
    for _h in range(H):
        for i in range(nb):
            u = rng.random()
            if i in full or (u >= p_empty and u < p_empty + p_full):
                row = list(rng.permutation(nb))
            elif u < p_empty:
                row = []
            else:
                row = list(rng.integers(0, nb, size=int(rng.integers(1, max_len + 1))))
            cols.extend(int(c) for c in row)
            row_ptr.append(len(cols))
    return np.asarray(row_ptr, dtype=np.int32), np.asarray(cols, dtype=np.int32)


def make_router_csr(H: int, nb: int, k_global: int, window: int, seed: int):
    """Block CSR of a router-style layout, seeded: in each head ``k_global`` query
    blocks drawn at random list every key block; every other query block i
    lists the blocks j with |i - j| <= window.  Rows head-major, ascending."""
    import numpy as np
    rng = np.random.default_rng(seed)
    row_ptr, cols = [0], []
    for _h in range(H):
        chosen = set(int(x) for x in rng.choice(nb, size=min(k_global, nb), replace=False))
        for i in range(nb):
            row = range(nb) if i in chosen else range(max(0, i - window), min(nb, i + window + 1))
            cols.extend(row)
            row_ptr.append(len(cols))
    return np.asarray(row_ptr, dtype=np.int32), np.asarray(cols, dtype=np.int32)
