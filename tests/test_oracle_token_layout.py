"""Pins of the oracle's token-level layout (window and global set in tokens).

The rule (oracle.layout, token level): allowed(h, i, j) = i in G or j in G or
|i - j| <= w or block(j) is a random block of block(i) (random blocks only for
query blocks without a global token, drawn as at block level outside the band's
blocks and the global-token blocks).  Checked against computations that do not
use it: torch's scaled_dot_product_attention with masks built here from the
plain conditions (band only; band and global tokens; a band as wide as the
sequence), the block-level builder (the block CSR must be the block layout with
window floor((w + 63) / 64) and the global-token blocks as globals), and scalar
loops on a tiny case with key padding.
"""

import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import attention as OA
from oracle import layout as OL


def _qkv(B, H, L, d, seed):
    g = torch.Generator().manual_seed(seed)
    return [torch.randn(B, H, L, d, generator=g, dtype=torch.float64) for _ in range(3)]


def _sdpa(q, k, v, allowed):
    o = F.scaled_dot_product_attention(q, k, v, attn_mask=torch.as_tensor(allowed))
    return o.numpy()


@pytest.mark.parametrize("w", [0, 17, 64, 100, 200])
def test_band_only_equals_sdpa_with_a_band_mask(w):
    B, H, L, d = 1, 2, 64 * 6, 16
    q, k, v = _qkv(B, H, L, d, seed=w)
    lay = OL.build_token_layout(H, L, w, 0, 0, 1)
    o, _ = OA.attention(q, k, v, lay)
    i = torch.arange(L)
    band = (i[:, None] - i[None, :]).abs() <= w
    assert np.abs(o - _sdpa(q, k, v, band)).max() < 1e-12


@pytest.mark.parametrize("w,globals_", [(0, [5, 70, 200]), (33, [0, 1, 63, 64, 300]), (90, [383])])
def test_band_and_global_tokens_equal_sdpa(w, globals_):
    B, H, L, d = 2, 1, 64 * 6, 8
    q, k, v = _qkv(B, H, L, d, seed=len(globals_) + w)
    lay = OL.build_token_layout(H, L, w, len(globals_), 0, 3, explicit_globals=globals_)
    o, lse = OA.attention(q, k, v, lay)
    i = torch.arange(L)
    gt = torch.zeros(L, dtype=torch.bool)
    gt[globals_] = True
    allowed = ((i[:, None] - i[None, :]).abs() <= w) | gt[:, None] | gt[None, :]
    assert np.abs(o - _sdpa(q, k, v, allowed)).max() < 1e-12
    s = (q @ k.transpose(-1, -2)) / math.sqrt(d)
    lse_ref = torch.logsumexp(s.masked_fill(~allowed, -math.inf), dim=-1).numpy()
    assert np.abs(lse - lse_ref).max() < 1e-12


def test_window_as_wide_as_the_sequence_is_dense():
    B, H, L, d = 1, 2, 64 * 3, 8
    q, k, v = _qkv(B, H, L, d, seed=9)
    lay = OL.build_token_layout(H, L, L, 2, 3, 4)
    o, _ = OA.attention(q, k, v, lay)
    assert np.abs(o - F.scaled_dot_product_attention(q, k, v).numpy()).max() < 1e-12


@pytest.mark.parametrize("w,n_global,n_random,seed", [(10, 3, 2, 1), (64, 0, 3, 2), (100, 5, 1, 3), (0, 2, 4, 4)])
def test_block_csr_is_the_block_layout_of_the_band_and_global_blocks(w, n_global, n_random, seed):
    H, L = 3, 64 * 16
    lay = OL.build_token_layout(H, L, w, n_global, n_random, seed)
    g_tok = OL.global_tokens(L, n_global)
    g_blocks = sorted({t // 64 for t in g_tok})
    ref = OL.build_layout(H, L, 64, (w + 63) // 64, len(g_blocks), n_random, seed, explicit_globals=g_blocks)
    assert np.array_equal(lay["row_ptr"], ref["row_ptr"]) and np.array_equal(lay["col_idx"], ref["col_idx"])
    # a random block is wholly allowed to every token of its query block
    for h in range(H):
        for I in range(lay["nb"]):
            for J in lay["token"]["random"][h][I]:
                for i in (64 * I, 64 * I + 37, 64 * I + 63):
                    assert OL.token_allowed(lay, h, i, L)[64 * J:64 * J + 64].all()


def test_masked_dense_equals_scalar_loops_with_key_padding():
    B, H, L, d = 1, 2, 64 * 3, 4
    q, k, v = _qkv(B, H, L, d, seed=5)
    lay = OL.build_token_layout(H, L, 21, 2, 1, 6, explicit_globals=[7, 130])
    km = np.ones((B, L), dtype=np.uint8)
    km[0, 150:] = 0
    o, lse = OA.attention(q, k, v, lay, key_mask=km)
    o2, lse2 = OA.attention_bruteforce(q, k, v, lay, key_mask=km)
    assert np.abs(o - o2).max() < 1e-12
    fin = np.isfinite(lse2)
    assert np.array_equal(fin, np.isfinite(lse)) and np.abs(lse[fin] - lse2[fin]).max() < 1e-12


def test_backward_oracle_on_a_token_layout_equals_autograd():
    """oracle.backward with a token-level layout against torch autograd through a
    dense softmax masked by the token rule written out here per pair."""
    from oracle import backward as OB
    B, H, L, d = 1, 2, 64 * 4, 8
    q, k, v = _qkv(B, H, L, d, seed=11)
    do = _qkv(B, H, L, d, seed=12)[0]
    lay = OL.build_token_layout(H, L, 21, 2, 1, 3)
    g = OL.global_tokens(L, 2)
    i = torch.arange(L)
    allowed = torch.zeros(H, L, L, dtype=torch.bool)
    for h in range(H):
        gt = torch.zeros(L, dtype=torch.bool)
        gt[g] = True
        base = ((i[:, None] - i[None, :]).abs() <= 21) | gt[:, None] | gt[None, :]
        for I in range(L // 64):
            for J in lay["token"]["random"][h][I]:
                base[64 * I:64 * I + 64, 64 * J:64 * J + 64] = True
        allowed[h] = base
    qq, kk, vv = (t.clone().requires_grad_() for t in (q, k, v))
    s = (qq @ kk.transpose(-1, -2)) / math.sqrt(d)
    o = torch.softmax(s.masked_fill(~allowed[None], -math.inf), -1) @ vv
    o.backward(do)
    got = OB.attention_backward(q, k, v, do, lay)
    for a, b in zip(got, (qq.grad, kk.grad, vv.grad)):
        assert np.abs(a - b.numpy()).max() < 1e-12
