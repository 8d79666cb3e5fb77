"""Oracle gradients of the block-sparse attention in fp64 (numpy).  TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import this module.  It shares no code with the CUDA library.

What is differentiated: the forward of ``oracle.attention``, i.e. the masked
attention Softmax(Q K^T / sqrt(d_k) (.) M) V of "Adapt or Perish: 新手入门指南 –
Adaptive Sparse Transformer 核心原理与实战" (sparse-attention formula), with
(.) M read as restricting the softmax to M and a key-padding mask removing keys.
The pages train these models ("BERT 稀疏注意力机制入门指南", 生产环境部署建议:
mixed-precision training, gradient checkpointing; "BigBird 稀疏注意力机制解析",
避坑指南: mixed precision, gradient checkpointing) but print no gradient
formula, so the gradient is the plain derivative of that forward.

For a loss whose gradient with respect to O is dO, with S = Q K^T * scale
restricted to the attended keys and P = softmax(S) row by row:
    dV  = P^T dO
    dP  = dO V^T
    dS  = P (.) (dP - D),   D = rowsum(P (.) dP)        (the softmax Jacobian)
    dQ  = dS K * scale,     dK = dS^T Q * scale
Entries outside the attended set have P = 0 and hence dS = 0; a row with no
attended key has P = 0 and contributes nothing.

The computation is masked-dense like the forward: for each query block the
scores against all L keys are formed, the excluded entries get P = 0, and the
four products above are taken over the full key range.
"""

from __future__ import annotations

import math

import numpy as np

from .attention import _as_f64, token_mask_row


def attention_backward(q, k, v, dout, layout: dict, key_mask=None, scale=None,
                       with_magnitude: bool = False, query_blocks=None):
    """dq, dk, dv [B,H,L,d] in fp64 for the loss gradient ``dout`` = dL/dO.

    ``query_blocks`` optionally restricts the sums to those query blocks (dq of
    the other rows stays zero, dk and dv hold only their contributions); the
    arithmetic is unchanged.

    With ``with_magnitude`` also returns, per output element, a sum of absolute
    values that bounds the terms it is summed from (same shapes):
      |dq|-terms  scale * (P (.) (|dP| + Dabs)) |K|
      |dk|-terms  scale * (P (.) (|dP| + Dabs))^T |Q|
      |dv|-terms  P^T |dO|
    with Dabs = rowsum(|dO| (.) |O|) >= |D|.  A relative error e in P, in dS or in
    the factors of D moves the result by at most e times this sum, which is what
    a tolerance needs.
    """
    q, k, v, do = _as_f64(q), _as_f64(k), _as_f64(v), _as_f64(dout)
    B, H, L, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    km = None if key_mask is None else _as_f64(key_mask) != 0
    block, nb = layout["block"], layout["nb"]
    assert layout["H"] == H and layout["L"] == L
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    if with_magnitude:
        mq, mk, mv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for b in range(B):
        for h in range(H):
            kb, vb = k[b, h], v[b, h]
            for i in (range(nb) if query_blocks is None else query_blocks):
                rows = slice(i * block, (i + 1) * block)
                allowed = token_mask_row(layout, h, i, L)
                if km is not None:
                    allowed = allowed & km[b]
                s = np.where(allowed, (q[b, h, rows] @ kb.T) * scale, -np.inf)
                mx = s.max(axis=-1, keepdims=True)
                empty = ~np.isfinite(mx)
                e = np.exp(s - np.where(empty, 0.0, mx))          # 0 where excluded
                den = e.sum(axis=-1, keepdims=True)
                p = np.where(empty, 0.0, e / np.where(empty, 1.0, den))
                dp = do[b, h, rows] @ vb.T
                D = (p * dp).sum(axis=-1, keepdims=True)
                ds = p * (dp - D)
                dq[b, h, rows] = (ds @ kb) * scale
                dk[b, h] += (ds.T @ q[b, h, rows]) * scale
                dv[b, h] += p.T @ do[b, h, rows]
                if with_magnitude:
                    dabs = (np.abs(do[b, h, rows]) * np.abs(p @ vb)).sum(axis=-1, keepdims=True)
                    w = p * (np.abs(dp) + dabs)
                    mq[b, h, rows] = (w @ np.abs(kb)) * scale
                    mk[b, h] += (w.T @ np.abs(q[b, h, rows])) * scale
                    mv[b, h] += p.T @ np.abs(do[b, h, rows])
    if with_magnitude:
        return dq, dk, dv, (mq, mk, mv)
    return dq, dk, dv


def attention_backward_rows(q, k, v, dout, layout: dict, b: int, h: int, query_tokens=(), key_tokens=(),
                            key_mask=None, scale=None):
    """Selected rows of the gradients of one (b, h), in fp64, with their magnitudes.

    Returns (dq [nq, d], dk [nk, d], dv [nk, d], (mq, mk, mv)) for the query
    tokens ``query_tokens`` and the key tokens ``key_tokens``: the same
    definition as ``attention_backward``, evaluated only on the query rows that
    the requested outputs depend on (for a key p, every query row whose block
    attends p's block), block by block over all L keys as in the masked-dense
    form.
    """
    qb, kb, vb, dob = (_as_f64(x[b, h]) for x in (q, k, v, dout))
    L, d = kb.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    block, nb = layout["block"], layout["nb"]
    km = None if key_mask is None else _as_f64(key_mask[b]) != 0
    key_tokens = np.asarray([int(p) for p in key_tokens], dtype=np.int64)
    query_tokens = [int(t) for t in query_tokens]
    kblocks = sorted({int(p) // block for p in key_tokens})
    dq = np.zeros((len(query_tokens), d))
    dk = np.zeros((len(key_tokens), d))
    dv = np.zeros((len(key_tokens), d))
    mq, mk, mv = np.zeros_like(dq), np.zeros_like(dk), np.zeros_like(dv)
    for i in range(nb):
        allowed = token_mask_row(layout, h, i, L)
        whole = any(allowed[j * block] for j in kblocks)  # the block's rows reach a requested key
        mine = [(n, t) for n, t in enumerate(query_tokens) if t // block == i]
        if not whole and not mine:
            continue
        if km is not None:
            allowed = allowed & km
        rows = np.arange(i * block, (i + 1) * block) if whole else np.asarray([t for _, t in mine])
        s = np.where(allowed, (qb[rows] @ kb.T) * scale, -np.inf)
        mx = s.max(axis=-1, keepdims=True)
        empty = ~np.isfinite(mx)
        e = np.exp(s - np.where(empty, 0.0, mx))
        p = np.where(empty, 0.0, e / np.where(empty, 1.0, e.sum(axis=-1, keepdims=True)))
        dp = dob[rows] @ vb.T
        D = (p * dp).sum(axis=-1, keepdims=True)
        ds = p * (dp - D)
        dabs = (np.abs(dob[rows]) * np.abs(p @ vb)).sum(axis=-1, keepdims=True)
        w = p * (np.abs(dp) + dabs)
        for n, t in mine:
            r = int(np.nonzero(rows == t)[0][0])
            dq[n] = (ds[r] @ kb) * scale
            mq[n] = (w[r] @ np.abs(kb)) * scale
        if whole and len(key_tokens):
            dk += (ds[:, key_tokens].T @ qb[rows]) * scale
            mk += (w[:, key_tokens].T @ np.abs(qb[rows])) * scale
            dv += p[:, key_tokens].T @ dob[rows]
            mv += p[:, key_tokens].T @ np.abs(dob[rows])
    return dq, dk, dv, (mq, mk, mv)
