"""Oracle masked-dense attention in fp64 (numpy).  TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import this module.  It shares no code with the CUDA library.

Definition followed:
  [ASTformula] "Adapt or Perish: 新手入门指南 – Adaptive Sparse Transformer 核心原理与实战",
      the sparse-attention formula  SparseAttention(Q,K,V) = Softmax(Q K^T / sqrt(d_k) (.) M) V,
      M in {0,1}^{n x n}.
  [Primer] "BERT 稀疏注意力机制入门指南", PyTorch 实现 -- entries outside the mask are
      filled with -1e9 before the softmax.
  [MHA]   "BERT多头注意力机制深度解析", BlockSparseAttention -- fill -1e10, blocks of 64.

Reading: "(.) M" restricts the softmax to the entries where M = 1 (the pages'
own code fills the others with a huge negative number, which in fp64 gives
exactly zero weight); here they are set to -inf.  d_k is the head dimension.
A key-padding mask removes keys (mask 0) from every row.  A row whose attended
set is empty gets O = 0 and lse = -inf.  lse is the natural log of the sum of
exp over the attended keys of the SCALED scores.

The computation is deliberately masked-dense: for each query block the scores
against ALL L keys are formed, the entries outside M set to -inf, then
softmax and the product with V, exactly as the formula reads.
"""

from __future__ import annotations

import math

import numpy as np

from . import layout as _layout


def _as_f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # torch tensor: any float dtype -> fp64 is exact
        x = x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def token_mask_row(layout: dict, h: int, i: int, L: int) -> np.ndarray:
    """Boolean mask of the keys attended by query block i of head h: [L] for a
    block layout (every token of the block alike), [block, L] for a token-level
    one (one row per query token, oracle.layout.token_allowed)."""
    block = layout["block"]
    if "token" in layout:
        return np.stack([_layout.token_allowed(layout, h, t, L) for t in range(i * block, (i + 1) * block)])
    m = np.zeros(L, dtype=bool)
    for j in _layout.row(layout, h, i):
        m[j * block:(j + 1) * block] = True
    return m


def masked_softmax_av(s: np.ndarray, allowed: np.ndarray, v: np.ndarray):
    """Softmax of s restricted to ``allowed`` (broadcast over rows), then times v.

    Returns (O, lse).  Rows with nothing allowed give O = 0, lse = -inf.
    """
    s = np.where(allowed, s, -np.inf)
    mx = s.max(axis=-1, keepdims=True)
    empty = ~np.isfinite(mx)
    mx_safe = np.where(empty, 0.0, mx)
    e = np.exp(s - mx_safe)
    l = e.sum(axis=-1, keepdims=True)
    with np.errstate(divide="ignore", invalid="ignore"):
        o = np.where(empty, 0.0, (e @ v) / np.where(empty, 1.0, l))
        lse = np.where(empty[..., 0], -np.inf, (mx_safe + np.log(np.where(empty, 1.0, l)))[..., 0])
    return o, lse


def attention(q, k, v, layout: dict, key_mask=None, scale=None, query_blocks=None, pairs=None):
    """O [B,H,L,d] and lse [B,H,L] in fp64 for the block layout (masked-dense).

    ``query_blocks`` optionally restricts the computation to those query blocks
    and ``pairs`` to those (batch element, head) pairs (the other rows of the
    result stay zero); the arithmetic is unchanged.
    """
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    B, H, L, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    km = None if key_mask is None else _as_f64(key_mask) != 0
    block, nb = layout["block"], layout["nb"]
    assert layout["H"] == H and layout["L"] == L
    out = np.zeros((B, H, L, d))
    lse = np.zeros((B, H, L))
    for b, h in ([(b, h) for b in range(B) for h in range(H)] if pairs is None else pairs):
        kt = k[b, h].T
        for i in (range(nb) if query_blocks is None else query_blocks):
            allowed = token_mask_row(layout, h, i, L)
            if km is not None:
                allowed = allowed & km[b]
            rows = slice(i * block, (i + 1) * block)
            s = (q[b, h, rows] @ kt) * scale
            out[b, h, rows], lse[b, h, rows] = masked_softmax_av(s, allowed, v[b, h])
    return out, lse


def attention_rows(q, k, v, layout: dict, b: int, h: int, tokens, key_mask=None,
                   scale=None):
    """O [n, d] and lse [n] for selected query tokens of (b, h) only."""
    qb, kb, vb = _as_f64(q[b, h]), _as_f64(k[b, h]), _as_f64(v[b, h])
    L, d = kb.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    tokens = np.asarray(tokens, dtype=np.int64)
    block = layout["block"]
    km = None if key_mask is None else _as_f64(key_mask[b]) != 0
    o = np.zeros((len(tokens), d))
    lse = np.zeros(len(tokens))
    for n, t in enumerate(tokens):
        if "token" in layout:
            allowed = _layout.token_allowed(layout, h, int(t), L)
        else:
            allowed = token_mask_row(layout, h, int(t) // block, L)
        if km is not None:
            allowed = allowed & km
        s = (qb[t] @ kb.T) * scale
        o_n, lse_n = masked_softmax_av(s[None, :], allowed[None, :], vb)
        o[n], lse[n] = o_n[0], lse_n[0]
    return o, lse


def attention_bruteforce(q, k, v, layout: dict, key_mask=None, scale=None):
    """Scalar loops with math.exp over explicit attended-key sets.  Tiny shapes only."""
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    B, H, L, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    block = layout["block"]
    out = np.zeros((B, H, L, d))
    lse = np.zeros((B, H, L))
    for b in range(B):
        for h in range(H):
            for t in range(L):
                if "token" in layout:
                    cand = [int(p) for p in np.nonzero(_layout.token_allowed(layout, h, t, L))[0]]
                else:
                    cand = [p for j in _layout.row(layout, h, t // block) for p in range(j * block, (j + 1) * block)]
                keys = [p for p in cand if key_mask is None or int(key_mask[b][p]) != 0]
                if not keys:
                    lse[b, h, t] = -math.inf
                    continue
                s = {p: sum(q[b, h, t, c] * k[b, h, p, c] for c in range(d)) * scale
                     for p in keys}
                mx = max(s.values())
                den = sum(math.exp(s[p] - mx) for p in keys)
                lse[b, h, t] = mx + math.log(den)
                for c in range(d):
                    out[b, h, t, c] = sum(math.exp(s[p] - lse[b, h, t]) * v[b, h, p, c]
                                          for p in keys)
    return out, lse
