"""Pins for the oracle gradients (CPU only).

- Central finite differences of the (separately pinned) oracle forward, on tiny
  shapes with key padding and empty rows: the gradient formula is checked
  against the function it differentiates, not against itself.
- torch autograd through fp64 scaled_dot_product_attention on an all-ones
  layout (a library routine).
- Closed forms: the columns of dV sum to the sum of dO over non-empty rows;
  constant keys give dQ = 0; excluded keys get dK = dV = 0; dO = 0 gives zeros.
- The magnitude sums that set the GPU tolerances, against per-token, per-key
  scalar loops with math.exp (to 1e-12 relative).
"""

import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import attention as OA
from oracle import backward as OB
from oracle import layout as OL


def _rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g, dtype=torch.float64).numpy()


def _loss(q, k, v, do, lay, km, scale):
    o, _ = OA.attention(q, k, v, lay, key_mask=km, scale=scale)
    return float((o * do).sum())


def _fd_grad(x, f, eps=1e-6):
    g = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        idx = it.multi_index
        old = x[idx]
        x[idx] = old + eps
        fp = f()
        x[idx] = old - eps
        fm = f()
        x[idx] = old
        g[idx] = (fp - fm) / (2 * eps)
    return g


def _empty_row_layout(H, L, block):
    """Rows with a gap: query block 1 of head 0 attends nothing."""
    nb = L // block
    rp, cols = [0], []
    for h in range(H):
        for i in range(nb):
            row = [] if (h == 0 and i == 1) else sorted({i, (i + 2) % nb, 0})
            cols.extend(row)
            rp.append(len(cols))
    return {"H": H, "L": L, "block": block, "nb": nb,
            "row_ptr": np.asarray(rp, dtype=np.int64), "col_idx": np.asarray(cols, dtype=np.int32)}


@pytest.mark.parametrize("case", ["bigbird", "padded", "empty_row", "scaled"])
def test_matches_finite_differences(case):
    B, H, L, d = 2, 2, 8, 3
    block = 2
    lay = OL.build_layout(H, L, block, 1, 1, 1, 5) if case != "empty_row" else _empty_row_layout(H, L, block)
    km = None
    if case == "padded":
        km = np.ones((B, L), dtype=np.uint8)
        km[1, -3:] = 0
        km[0, 2] = 0
    scale = 0.7 if case == "scaled" else None
    q, k, v, do = (_rand((B, H, L, d), s) for s in (1, 2, 3, 4))
    dq, dk, dv = OB.attention_backward(q, k, v, do, lay, key_mask=km, scale=scale)
    f = lambda: _loss(q, k, v, do, lay, km, scale)  # noqa: E731
    for x, g in ((q, dq), (k, dk), (v, dv)):
        g_fd = _fd_grad(x, f)
        assert np.abs(g - g_fd).max() < 1e-7 * max(1.0, np.abs(g_fd).max())


@pytest.mark.parametrize("kind", ["wide_window", "all_global"])
def test_all_ones_layout_equals_autograd(kind):
    B, H, L, d = 1, 2, 192, 8
    nb = L // 64
    lay = OL.build_layout(H, L, 64, nb - 1, 0, 0, 0) if kind == "wide_window" else \
        OL.build_layout(H, L, 64, 0, nb, 0, 0)
    q, k, v, do = (torch.from_numpy(_rand((B, H, L, d), s)) for s in (7, 8, 9, 10))
    qt, kt, vt = (x.clone().requires_grad_(True) for x in (q, k, v))
    F.scaled_dot_product_attention(qt, kt, vt).backward(do)
    dq, dk, dv = OB.attention_backward(q, k, v, do, lay)
    for a, t in ((dq, qt), (dk, kt), (dv, vt)):
        assert np.abs(a - t.grad.numpy()).max() < 1e-11


def test_closed_forms():
    B, H, L, d = 2, 2, 64 * 6, 4
    lay = OL.build_layout(H, L, 64, 1, 1, 1, 3)
    q, k, v, do = (_rand((B, H, L, d), s) for s in (11, 12, 13, 14))
    km = np.ones((B, L), dtype=np.uint8)
    km[0, 100:140] = 0
    dq, dk, dv = OB.attention_backward(q, k, v, do, lay, key_mask=km)
    # every row attends some key, so each row of P sums to one
    assert np.abs(dv.sum(axis=2) - do.sum(axis=2)).max() < 1e-11
    # keys the mask drops get no gradient
    assert np.all(dk[0, :, 100:140] == 0) and np.all(dv[0, :, 100:140] == 0)
    # constant keys: every score of a row is equal, so dQ = 0
    kc = np.broadcast_to(_rand((B, H, 1, d), 15), k.shape).copy()
    dq_c, _, _ = OB.attention_backward(q, kc, v, do, lay)
    assert np.abs(dq_c).max() < 1e-12
    # dO = 0: all gradients vanish
    z = OB.attention_backward(q, k, v, np.zeros_like(do), lay)
    assert all(np.all(x == 0) for x in z)


def test_unattended_keys_and_empty_rows():
    B, H, L, d = 1, 2, 64 * 5, 4
    nb = L // 64
    # head 0: every query block attends only block 0 (blocks 1.. get nothing);
    # head 1: query block 2 attends nothing
    rp, cols = [0], []
    for h in range(H):
        for i in range(nb):
            row = [0] if h == 0 else ([] if i == 2 else [i, (i + 1) % nb])
            cols.extend(row)
            rp.append(len(cols))
    lay = {"H": H, "L": L, "block": 64, "nb": nb,
           "row_ptr": np.asarray(rp, dtype=np.int64), "col_idx": np.asarray(cols, dtype=np.int32)}
    q, k, v, do = (_rand((B, H, L, d), s) for s in (21, 22, 23, 24))
    dq, dk, dv = OB.attention_backward(q, k, v, do, lay)
    assert np.all(dk[0, 0, 64:] == 0) and np.all(dv[0, 0, 64:] == 0)
    assert np.all(dq[0, 1, 128:192] == 0)
    # head 0: P puts all weight on block 0 row by row, so dV of block 0 = sum of dO
    assert np.abs(dv[0, 0, :64].sum(axis=0) - do[0, 0].sum(axis=0)).max() < 1e-11


def test_magnitudes_bound_the_results():
    B, H, L, d = 1, 2, 64 * 4, 8
    lay = OL.build_layout(H, L, 64, 1, 1, 1, 9)
    q, k, v, do = (_rand((B, H, L, d), s) for s in (31, 32, 33, 34))
    dq, dk, dv, (mq, mk, mv) = OB.attention_backward(q, k, v, do, lay, with_magnitude=True)
    for g, m in ((dq, mq), (dk, mk), (dv, mv)):
        assert np.all(np.abs(g) <= m * (1 + 1e-12) + 1e-15)
    _, _, dv2 = OB.attention_backward(q, k, v, do, lay)
    assert np.array_equal(dv, dv2)
    assert math.isfinite(float(mq.max()))


def test_rows_api_matches_full():
    B, H, L, d = 2, 2, 64 * 7, 8
    lay = OL.build_layout(H, L, 64, 1, 1, 2, 4)
    q, k, v, do = (_rand((B, H, L, d), s) for s in (41, 42, 43, 44))
    km = np.ones((B, L), dtype=np.uint8)
    km[1, -50:] = 0
    dq, dk, dv, (mq, mk, mv) = OB.attention_backward(q, k, v, do, lay, key_mask=km, with_magnitude=True)
    qt, kt = [0, 5, 63, 64, 200, 447], [1, 64, 130, 300, 420, 446]
    for b in range(B):
        for h in range(H):
            rq, rk, rv, (sq, sk, sv) = OB.attention_backward_rows(q, k, v, do, lay, b, h, qt, kt, key_mask=km)
            assert np.abs(rq - dq[b, h, qt]).max() < 1e-12
            assert np.abs(rk - dk[b, h, kt]).max() < 1e-12
            assert np.abs(rv - dv[b, h, kt]).max() < 1e-12
            for a, m in ((sq, mq[b, h, qt]), (sk, mk[b, h, kt]), (sv, mv[b, h, kt])):
                assert np.abs(a - m).max() < 1e-12


def _magnitudes_by_scalar_loops(q, k, v, do, lay, km, scale):
    """The magnitude sums of the docstring, written out term by term: for each
    (b, h, query token t) the attended key set is listed from the layout's block
    row and the key mask, P comes from math.exp, and every sum is a Python loop.
    Nothing here is masked-dense and nothing is shared with the oracle's numpy form."""
    B, H, L, d = q.shape
    block = lay["block"]
    mq, mk, mv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for b in range(B):
        for h in range(H):
            for t in range(L):
                blocks = [int(j) for j in OL.row(lay, h, t // block)]
                keys = [p for j in blocks for p in range(j * block, (j + 1) * block)
                        if km is None or int(km[b][p]) != 0]
                if not keys:
                    continue
                s = {p: scale * sum(q[b, h, t, c] * k[b, h, p, c] for c in range(d)) for p in keys}
                mx = max(s.values())
                den = sum(math.exp(s[p] - mx) for p in keys)
                P = {p: math.exp(s[p] - mx) / den for p in keys}
                o = [sum(P[p] * v[b, h, p, c] for p in keys) for c in range(d)]
                dabs = sum(abs(do[b, h, t, c]) * abs(o[c]) for c in range(d))
                for p in keys:
                    dp = sum(do[b, h, t, c] * v[b, h, p, c] for c in range(d))
                    w = P[p] * (abs(dp) + dabs)
                    for c in range(d):
                        mq[b, h, t, c] += scale * w * abs(k[b, h, p, c])
                        mk[b, h, p, c] += scale * w * abs(q[b, h, t, c])
                        mv[b, h, p, c] += P[p] * abs(do[b, h, t, c])
    return mq, mk, mv


def test_magnitudes_match_scalar_loops():
    # Pins the with_magnitude sums (their Dabs, |dP| and |K| / |Q| / |dO| factors)
    # against an explicit per-token, per-key evaluation, with a padded key tail and
    # a non-default scale so that a dropped factor or a transposed operand shows.
    B, H, L, d = 1, 2, 64 * 3, 3
    lay = OL.build_layout(H, L, 64, 0, 1, 1, 11)
    q, k, v, do = (_rand((B, H, L, d), s) for s in (51, 52, 53, 54))
    km = np.ones((B, L), dtype=np.uint8)
    km[0, -20:] = 0
    _, _, _, (mq, mk, mv) = OB.attention_backward(q, k, v, do, lay, key_mask=km, scale=0.7,
                                                  with_magnitude=True)
    rq, rk, rv = _magnitudes_by_scalar_loops(q, k, v, do, lay, km, 0.7)
    for got, ref in ((mq, rq), (mk, rk), (mv, rv)):
        assert np.abs(got - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max())
    assert np.all(mk[0, :, -20:] == 0) and np.all(mv[0, :, -20:] == 0)
