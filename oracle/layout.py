"""Oracle BigBird block layout (plain Python + numpy).  TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import this module.  It shares no code with the CUDA library.

Sources (page titles and sections):
  [BigBird] "BigBird 稀疏注意力机制解析：如何突破 Transformer 的序列长度限制"
            (qqiyuan.cn), section 核心实现 -- global attention, sliding window,
            random attention; section 代码实现 -- ``_select_global_tokens``.
  [Primer]  "BERT 稀疏注意力机制入门指南" (qqiyuan.cn), section "PyTorch 实现基础
            稀疏注意力" -- window clipped at the sequence ends.
  [SQA]     "Transformer计算效率优化：SQA稀疏注意力机制详解", section 3.1 --
            the attention mask is stored at block granularity.

Readings taken where the pages are silent or garbled (all at BLOCK granularity):
  * globals: n_g == 1 -> {0}; n_g >= 2 -> floor(k (nb-1) / (n_g-1)), k = 0..n_g-1,
    in exact integers, deduplicated.  This is the page's
    ``linspace(0, n-1, n_g).long()`` evaluated without float rounding.
  * a global query block attends to every key block; every row contains every
    global key block.
  * window: |i - j| <= w, clipped to [0, nb-1] with no wrap-around (the page's
    ``triu(w).tril(-w)`` is empty as printed; the primer's clipping is used).
  * random: r distinct blocks drawn without replacement from the blocks outside
    window and globals, by a partial Fisher-Yates shuffle driven by the raw
    64-bit stream of numpy's Philox4x64-10 with key = [seed, 0] and initial
    counter = [0, i, h, 0]; fewer than r candidates -> take them all.
  * the layout depends on (h, i) only and is shared by every batch element.
"""

from __future__ import annotations

import numpy as np


def global_blocks(nb: int, n_global: int, explicit=None) -> list[int]:
    """Sorted distinct global block indices ([BigBird] 代码实现, linspace rule)."""
    if explicit is not None:
        g = sorted({int(x) for x in explicit})
        if g and (g[0] < 0 or g[-1] >= nb):
            raise ValueError("explicit global block out of range")
        return g
    if n_global <= 0:
        return []
    if n_global == 1:
        return [0]
    return sorted({(k * (nb - 1)) // (n_global - 1) for k in range(n_global)})


def window_blocks(i: int, nb: int, w: int) -> list[int]:
    """Blocks j with |i - j| <= w, clipped at both ends ([Primer], [BigBird])."""
    return list(range(max(0, i - w), min(nb - 1, i + w) + 1))


def philox_stream(seed: int, i: int, h: int, count: int) -> list[int]:
    """First ``count`` raw 64-bit words of Philox4x64-10 for query block i, head h."""
    if count <= 0:
        return []
    key = np.array([seed & 0xFFFFFFFFFFFFFFFF, 0], dtype=np.uint64)  # no float round trip
    bg = np.random.Philox(key=key, counter=np.array([0, i, h, 0], dtype=np.uint64))
    return [int(x) for x in bg.random_raw(count)]


def random_blocks(candidates: list[int], r: int, stream: list[int]) -> list[int]:
    """Partial Fisher-Yates: the first min(r, m) entries of a shuffled copy."""
    c = list(candidates)
    m = len(c)
    take = min(r, m)
    for t in range(take):
        j = t + stream[t] % (m - t)
        c[t], c[j] = c[j], c[t]
    return c[:take]


def row_blocks(h: int, i: int, nb: int, window: int, globals_: list[int],
               n_random: int, seed: int) -> list[int]:
    """Sorted key-block list of query block i of head h."""
    gset = set(globals_)
    if i in gset:
        return list(range(nb))
    wset = set(window_blocks(i, nb, window))
    cand = [j for j in range(nb) if j not in wset and j not in gset]
    take = min(n_random, len(cand))
    rnd = random_blocks(cand, n_random, philox_stream(seed, i, h, take))
    return sorted(wset | gset | set(rnd))


def build_layout(H: int, L: int, block: int, window: int, n_global: int,
                 n_random: int, seed: int, explicit_globals=None) -> dict:
    """CSR layout: rows ordered head-major then query block, int32 columns."""
    if L % block:
        raise ValueError("L must be a multiple of block")
    nb = L // block
    g = global_blocks(nb, n_global, explicit_globals)
    row_ptr = [0]
    cols: list[int] = []
    for h in range(H):
        for i in range(nb):
            r = row_blocks(h, i, nb, window, g, n_random, seed)
            cols.extend(r)
            row_ptr.append(len(cols))
    return {
        "H": H, "L": L, "block": block, "nb": nb, "globals": g,
        "row_ptr": np.asarray(row_ptr, dtype=np.int64),
        "col_idx": np.asarray(cols, dtype=np.int32),
    }


def row(layout: dict, h: int, i: int) -> np.ndarray:
    nb = layout["nb"]
    rp = layout["row_ptr"]
    return layout["col_idx"][rp[h * nb + i]:rp[h * nb + i + 1]]


def block_mask(layout: dict) -> np.ndarray:
    """Dense boolean [H, nb, nb] block mask M ([SQA] 3.1: mask kept per block)."""
    H, nb = layout["H"], layout["nb"]
    m = np.zeros((H, nb, nb), dtype=bool)
    for h in range(H):
        for i in range(nb):
            m[h, i, row(layout, h, i)] = True
    return m
