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


# ----------------------------------------------------------------------------- token level
# Readings for the token-level layout (window and global set in tokens, not whole
# blocks; [BigBird] 核心实现 gives its window in tokens, w = 64 in its example):
#   * G: global tokens; explicit, or the linspace rule over tokens:
#     n_g == 1 -> {0}, n_g >= 2 -> floor(k (L-1) / (n_g-1)).
#   * allowed(h, i, j) = i in G  or  j in G  or  |i - j| <= w  or
#     (block(i) holds no global token and block(j) is a random block of block(i)).
#   * random blocks stay at block granularity (the pages draw blocks): for a query
#     block I without a global token, n_random blocks drawn as at block level from
#     the blocks outside the band's blocks {J : |I - J| <= floor((w + 63) / 64)} and
#     outside the blocks holding a global token, with the same Philox stream.
#   * blocks are 64 tokens (the kernels' key blocks); L is a multiple of 64.


def global_tokens(L: int, n_global: int, explicit=None) -> list[int]:
    """Sorted distinct global token indices (the linspace rule, over tokens)."""
    if explicit is not None:
        g = sorted({int(x) for x in explicit})
        if g and (g[0] < 0 or g[-1] >= L):
            raise ValueError("explicit global token out of range")
        return g
    if n_global <= 0:
        return []
    if n_global == 1:
        return [0]
    return sorted({(k * (L - 1)) // (n_global - 1) for k in range(n_global)})


def token_random_blocks(h: int, I: int, nb: int, window: int, gblocks: set, n_random: int, seed: int) -> list[int]:
    """Random key blocks of query block I (none when I holds a global token)."""
    if I in gblocks:
        return []
    wb = (window + 63) // 64
    band = set(window_blocks(I, nb, wb))
    cand = [j for j in range(nb) if j not in band and j not in gblocks]
    take = min(n_random, len(cand))
    return random_blocks(cand, n_random, philox_stream(seed, I, h, take))


def build_token_layout(H: int, L: int, window: int, n_global: int, n_random: int, seed: int,
                       explicit_globals=None) -> dict:
    """Token-level layout: the allowed-pair rule above, plus its block CSR (the key
    blocks holding at least one allowed key of some query token of the block)."""
    if L % 64:
        raise ValueError("L must be a multiple of 64")
    nb = L // 64
    g = global_tokens(L, n_global, explicit_globals)
    gblocks = {t // 64 for t in g}
    rand = [[token_random_blocks(h, I, nb, window, gblocks, n_random, seed) for I in range(nb)] for h in range(H)]
    gt = np.zeros(L, dtype=bool)
    gt[g] = True
    row_ptr = [0]
    cols: list[int] = []
    for h in range(H):
        for I in range(nb):
            keys = np.zeros(nb, dtype=bool)
            for i in range(64 * I, 64 * I + 64):
                keys |= token_allowed(None, h, i, L, _parts=(window, gt, rand)).reshape(nb, 64).any(axis=1)
            cols.extend(int(j) for j in np.nonzero(keys)[0])
            row_ptr.append(len(cols))
    return {"H": H, "L": L, "block": 64, "nb": nb, "globals": sorted(gblocks),
            "row_ptr": np.asarray(row_ptr, dtype=np.int64), "col_idx": np.asarray(cols, dtype=np.int32),
            "token": {"window": window, "globals": g, "random": rand}}


def token_allowed(layout: dict, h: int, i: int, L: int, _parts=None) -> np.ndarray:
    """Boolean [L]: the keys query token i of head h attends (the rule above)."""
    if _parts is None:
        tk = layout["token"]
        gt = np.zeros(L, dtype=bool)
        gt[tk["globals"]] = True
        window, rand = tk["window"], tk["random"]
    else:
        window, gt, rand = _parts
    if gt[i]:
        return np.ones(L, dtype=bool)
    j = np.arange(L)
    m = gt | (np.abs(j - i) <= window)
    for J in rand[h][i // 64]:
        m[64 * J:64 * J + 64] = True
    return m
