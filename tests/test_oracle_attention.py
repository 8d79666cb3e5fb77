"""Pins for the oracle attention (CPU only).

Library routines (torch's fp64 scaled_dot_product_attention and logsumexp),
closed forms (q = 0, constant v, one-hot v), the pages' own -1e10 fill
convention, and scalar brute force on tiny shapes.
"""

import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import attention as OA
from oracle import layout as OL


def _rand(B, H, L, d, seed=0):
    g = torch.Generator().manual_seed(seed)
    return [torch.randn((B, H, L, d), generator=g, dtype=torch.float64) for _ in range(3)]


def _dense_ref(q, k, v, scale=None):
    o = F.scaled_dot_product_attention(q, k, v, scale=scale)
    s = (q @ k.transpose(-1, -2)) * (scale if scale is not None else 1 / math.sqrt(q.shape[-1]))
    return o.numpy(), torch.logsumexp(s, dim=-1).numpy()


@pytest.mark.parametrize("kind", ["wide_window", "all_global"])
def test_all_ones_layout_equals_dense(kind):
    B, H, L, d = 2, 2, 256, 16
    q, k, v = _rand(B, H, L, d)
    nb = L // 64
    if kind == "wide_window":
        lay = OL.build_layout(H, L, 64, nb - 1, 0, 0, 0)
    else:
        lay = OL.build_layout(H, L, 64, 0, nb, 0, 0)
    assert int(lay["row_ptr"][-1]) == H * nb * nb
    o, lse = OA.attention(q, k, v, lay)
    o_ref, lse_ref = _dense_ref(q, k, v)
    assert np.abs(o - o_ref).max() < 1e-12
    assert np.abs(lse - lse_ref).max() < 1e-12


def test_explicit_scale_matches_library():
    q, k, v = _rand(1, 1, 128, 8, seed=3)
    lay = OL.build_layout(1, 128, 64, 1, 0, 0, 0)
    o, lse = OA.attention(q, k, v, lay, scale=0.3)
    o_ref, lse_ref = _dense_ref(q, k, v, scale=0.3)
    assert np.abs(o - o_ref).max() < 1e-12 and np.abs(lse - lse_ref).max() < 1e-12


def test_page_fill_convention_equals_restriction():
    # The pages fill excluded scores with -1e10 and take a plain softmax.
    B, H, L, d = 1, 2, 512, 16
    q, k, v = _rand(B, H, L, d, seed=1)
    lay = OL.build_layout(H, L, 64, 1, 1, 1, 0)
    o, _ = OA.attention(q, k, v, lay)
    mask = torch.from_numpy(np.repeat(np.repeat(OL.block_mask(lay), 64, axis=1), 64, axis=2))
    s = (q @ k.transpose(-1, -2)) / math.sqrt(d)
    s = s.masked_fill(~mask[None], -1e10)
    o_page = (torch.softmax(s, dim=-1) @ v).numpy()
    assert np.abs(o - o_page).max() < 1e-12


def test_zero_queries_give_mean_and_log_count():
    B, H, L, d = 1, 2, 512, 8
    _, k, v = _rand(B, H, L, d, seed=2)
    q = torch.zeros_like(k)
    lay = OL.build_layout(H, L, 64, 1, 1, 1, 0)
    km = torch.ones((B, L), dtype=torch.uint8)
    km[:, 500:] = 0
    o, lse = OA.attention(q, k, v, lay, key_mask=km)
    for h in range(H):
        for t in range(0, L, 37):
            keys = [p for j in OL.row(lay, h, t // 64) for p in range(64 * j, 64 * j + 64) if p < 500]
            assert abs(lse[0, h, t] - math.log(len(keys))) < 1e-12
            assert np.abs(o[0, h, t] - v[0, h, keys].mean(0).numpy()).max() < 1e-12
    # global query block 0 attends every unpadded key: lse = ln(L_valid)
    assert np.abs(lse[0, :, :64] - math.log(500)).max() < 1e-12


def test_constant_values_give_constant_output():
    q, k, _ = _rand(2, 2, 256, 8, seed=4)
    v = torch.full_like(q, -1.75)
    lay = OL.build_layout(2, 256, 64, 0, 1, 1, 5)
    o, _ = OA.attention(q, k, v, lay)
    assert np.abs(o + 1.75).max() < 1e-12


def test_one_hot_values_reveal_weights():
    # v[p] = e_p, so O[t] is the attention-weight row of token t.
    L, block = 16, 4
    q, k, _ = _rand(1, 1, L, L, seed=5)
    v = torch.eye(L, dtype=torch.float64)[None, None]
    lay = OL.build_layout(1, L, block, 0, 1, 1, 9)
    o, lse = OA.attention(q, k, v, lay)
    w = o[0, 0]
    assert np.abs(w.sum(1) - 1).max() < 1e-12
    allowed = np.repeat(np.repeat(OL.block_mask(lay)[0], block, 0), block, 1)
    assert np.all(w[~allowed] == 0) and np.all(w[allowed] > 0)
    s = (q[0, 0] @ k[0, 0].T).numpy() / math.sqrt(L)
    assert np.abs(np.log(w[allowed]) - (s - lse[0, 0][:, None])[allowed]).max() < 1e-12


@pytest.mark.parametrize("case", [
    dict(L=8, block=2, w=1, g=1, r=1, d=3),
    dict(L=12, block=3, w=0, g=2, r=2, d=4),
    dict(L=10, block=2, w=1, g=0, r=1, d=2),
])
def test_bruteforce_tiny(case):
    B, H = 2, 2
    q, k, v = _rand(B, H, case["L"], case["d"], seed=6)
    lay = OL.build_layout(H, case["L"], case["block"], case["w"], case["g"], case["r"], 11)
    km = torch.ones((B, case["L"]), dtype=torch.uint8)
    km[1, -3:] = 0
    for mask in (None, km):
        o, lse = OA.attention(q, k, v, lay, key_mask=mask)
        ob, lseb = OA.attention_bruteforce(q, k, v, lay, key_mask=mask)
        assert np.abs(o - ob).max() < 1e-12
        assert np.abs(lse - lseb).max() < 1e-12


def test_key_mask_outside_row_changes_nothing_and_block_mask_removes_block():
    B, H, L, d = 1, 1, 512, 8
    q, k, v = _rand(B, H, L, d, seed=7)
    lay = OL.build_layout(H, L, 64, 1, 0, 0, 0)   # rows: window only
    o0, l0 = OA.attention(q, k, v, lay)
    km = torch.ones((B, L), dtype=torch.uint8)
    km[0, 7 * 64:] = 0                           # block 7: outside rows 0..5
    o1, l1 = OA.attention(q, k, v, lay, key_mask=km)
    assert np.abs(o1[0, 0, :6 * 64] - o0[0, 0, :6 * 64]).max() == 0
    # block 7 masked == block 7 removed from rows 6 and 7
    cols = []
    rp = [0]
    for i in range(8):
        r = [j for j in OL.row(lay, 0, i) if j != 7]
        cols += r
        rp.append(len(cols))
    lay2 = dict(lay, row_ptr=np.array(rp), col_idx=np.array(cols, dtype=np.int32))
    o2, l2 = OA.attention(q, k, v, lay2)
    assert np.abs(o1[0, 0, 6 * 64:7 * 64] - o2[0, 0, 6 * 64:7 * 64]).max() < 1e-15
    assert np.abs(l1[0, 0, 6 * 64:7 * 64] - l2[0, 0, 6 * 64:7 * 64]).max() < 1e-15


def test_fully_masked_row_gives_zero_and_neg_inf():
    q, k, v = _rand(1, 1, 256, 8, seed=8)
    lay = OL.build_layout(1, 256, 64, 0, 0, 0, 0)   # each block attends itself only
    km = torch.ones((1, 256), dtype=torch.uint8)
    km[0, 64:128] = 0
    o, lse = OA.attention(q, k, v, lay, key_mask=km)
    assert np.all(o[0, 0, 64:128] == 0) and np.all(np.isneginf(lse[0, 0, 64:128]))
    assert np.all(np.isfinite(lse[0, 0, :64]))


def test_rows_api_matches_full():
    q, k, v = _rand(2, 2, 512, 16, seed=9)
    lay = OL.build_layout(2, 512, 64, 1, 1, 1, 0)
    km = torch.ones((2, 512), dtype=torch.uint8)
    km[1, 400:] = 0
    o, lse = OA.attention(q, k, v, lay, key_mask=km)
    toks = [0, 5, 63, 64, 200, 511]
    for b in range(2):
        for h in range(2):
            orr, lr = OA.attention_rows(q, k, v, lay, b, h, toks, key_mask=km)
            assert np.abs(orr - o[b, h, toks]).max() < 1e-13
            assert np.abs(lr - lse[b, h, toks]).max() < 1e-13
