"""Token-level layouts (bsa_layout_build_tokens): the library's tables against the
oracle's rule (CPU), and the forward against the fp64 oracle (GPU).

CPU: the block CSR and the global-token bits equal the oracle's; every tile entry
the library leaves without its per-row-mask flag for a half joins two blocks whose
every token pair the oracle's rule allows (the kernels apply no mask there);
entries with the flag lie in the rows of that half.
GPU: windows below, at and above one block and not multiples of 64, global tokens
not aligned to blocks (explicit and by the linspace rule, some in one block
together), random blocks, a partially padded key tail, ragged tiles and split
global rows, L = 16384 on sampled rows, and d = 128; O max-abs 2e-2, lse max-abs
1e-3, the parity tolerances.  The backward over token layouts against the oracle's
gradients at the backward suite's bounds (2^-6 of each element's sum of absolute
terms plus 2^-8 of its value).
"""

import numpy as np
import pytest
import torch

import workloads
from block_sparse_attention_bigbird_b200 import bsa
from oracle import attention as OA
from oracle import layout as OL

SHIFT_MEMBER, SHIFT_MASK = 24, 26

CPU_CASES = [  # H, L, window, n_global, n_random, seed, explicit global tokens
    (2, 64 * 12, 17, 0, 2, 1, None),
    (3, 64 * 16, 100, 3, 3, 2, None),
    (2, 64 * 10, 64, 0, 0, 3, [5, 6, 70, 383, 600]),
    (1, 64 * 20, 0, 2, 4, 4, None),
    (2, 64 * 9, 300, 1, 1, 5, None),
]


@pytest.mark.parametrize("H,L,w,ng,nr,seed,gt", CPU_CASES)
def test_tables_match_the_oracle_rule(H, L, w, ng, nr, seed, gt):
    lay = bsa.bsa_layout_build_tokens(H, L, w, ng, nr, seed, global_tokens=gt)
    ref = OL.build_token_layout(H, L, w, ng, nr, seed, explicit_globals=gt)
    rp, ci = bsa.bsa_layout_csr(lay)
    assert np.array_equal(rp, ref["row_ptr"]) and np.array_equal(ci, ref["col_idx"])
    win, bits = bsa.bsa_layout_token_masks(lay)
    assert win == w
    want = np.zeros(L // 64, dtype=np.uint64)
    for t in ref["token"]["globals"]:
        want[t // 64] |= np.uint64(1) << np.uint64(t % 64)
    assert np.array_equal(bits, want)
    # entries without the mask flag: every pair of the two blocks allowed by the rule
    pair_q, pair_ptr, pair_ent = bsa.bsa_layout_tiles(lay)
    P = len(pair_q)
    allowed_cache = {}

    def allowed_rows(h, I):
        if (h, I) not in allowed_cache:
            allowed_cache[(h, I)] = np.stack([OL.token_allowed(ref, h, i, L) for i in range(64 * I, 64 * I + 64)])
        return allowed_cache[(h, I)]

    for h in range(H):
        for p in range(P):
            for x in range(pair_ptr[h * P + p], pair_ptr[h * P + p + 1]):
                e = int(pair_ent[x])
                J = e & 0xFFFFFF
                for half in (0, 1):
                    I = int(pair_q[p][half])
                    member = (e >> (SHIFT_MEMBER + half)) & 1
                    masked = (e >> (SHIFT_MASK + half)) & 1
                    if not member:
                        assert not masked
                        continue
                    block = allowed_rows(h, I)[:, 64 * J:64 * J + 64]
                    assert block.any()  # a listed block holds an allowed pair of the half
                    if not masked:
                        assert block.all(), (h, I, J)


def test_block_layouts_report_no_token_part_and_bad_arguments_are_refused():
    blk = bsa.bsa_layout_build(1, 64 * 4, 64, 1, 1, 1, 0)
    with pytest.raises(bsa.BsaError):
        bsa.bsa_layout_token_masks(blk)
    lay = bsa.bsa_layout_build_tokens(1, 64 * 4, 10, 1, 1, 0)
    fake = 1 << 20
    # the backward takes token layouts: argument checks pass, the layout is not uploaded
    code = bsa.lib.bsa_backward(fake, fake, fake, fake, fake, fake, 1, 1, 64 * 4, 64, lay.handle, None, 0.0,
                                fake, fake, fake, fake, 1 << 20, None)
    assert code == bsa.BSA_ERR_LAYOUT_MISMATCH
    for bad in ((0, 64, 1, 0, 0), (1, 100, 1, 0, 0), (1, 64, -1, 0, 0), (1, 64, 1, -1, 0), (1, 64, 1, 0, -1)):
        with pytest.raises(bsa.BsaError):
            bsa.bsa_layout_build_tokens(*bad)
    with pytest.raises(bsa.BsaError):
        bsa.bsa_layout_build_tokens(1, 128, 1, global_tokens=[128])


GPU_CASES = [  # name, B, H, L, window, n_global, n_random, seed, global tokens, key pad, d
    ("band17_random", 2, 2, 64 * 13, 17, 0, 2, 1, None, 0, 64),
    ("band100_globals_linspace", 1, 3, 64 * 16, 100, 3, 3, 2, None, 0, 64),
    ("window64_unaligned_globals", 2, 2, 64 * 10, 64, 0, 0, 3, [5, 6, 70, 383, 600], 0, 64),
    ("diagonal_only_globals_random", 1, 2, 64 * 20, 0, 2, 4, 4, None, 0, 64),
    ("wide_window_padding", 2, 2, 64 * 9, 300, 1, 1, 5, None, 100, 64),
    ("globals_split_rows", 1, 2, 64 * 64, 40, 2, 3, 6, [10, 4000], 0, 64),
    ("band50_head_dim_128", 1, 2, 64 * 18, 50, 2, 2, 7, None, 30, 128),
]


@pytest.mark.parametrize("name,B,H,L,w,ng,nr,seed,gt,pad,d", GPU_CASES, ids=[c[0] for c in GPU_CASES])
@pytest.mark.gpu
@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
def test_token_layout_forward_matches_oracle(name, B, H, L, w, ng, nr, seed, gt, pad, d):
    wl = workloads.custom(B, H, L, 1, 0, 0, seed=seed, key_pad_tail=pad, d=d)
    q, k, v = workloads.make_qkv(wl, data_seed=seed)
    km = workloads.make_key_mask(wl) if pad else None
    lay = bsa.bsa_layout_build_tokens(H, L, w, ng, nr, seed, global_tokens=gt)
    bsa.bsa_layout_upload(lay)
    dev = torch.device("cuda")
    out, lse = bsa.bsa_forward(q.to(dev), k.to(dev), v.to(dev), lay, key_mask=km.to(dev) if km is not None else None)
    assert bsa.bsa_sync_status() == 0
    ref = OL.build_token_layout(H, L, w, ng, nr, seed, explicit_globals=gt)
    o_ref, l_ref = OA.attention(q, k, v, ref, key_mask=km)
    o, l = out.float().cpu().numpy(), lse.cpu().numpy()
    assert np.all(np.isfinite(o))
    fin = np.isfinite(l_ref)
    assert np.array_equal(np.isneginf(l), ~fin)
    assert np.abs(o - o_ref).max() <= 2e-2
    assert np.abs(l[fin] - l_ref[fin]).max() <= 1e-3


@pytest.mark.gpu
@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
def test_token_layout_long_sequence_sampled_rows():
    """L = 16384, window 200 tokens, 5 global tokens by the linspace rule, 3 random
    blocks: the rows of the global tokens' blocks and of sampled other blocks of two
    (batch, head) pairs against the oracle, each row from its own token mask."""
    B, H, L = 2, 3, 16384
    wl = workloads.custom(B, H, L, 1, 0, 0, seed=8)
    q, k, v = workloads.make_qkv(wl, data_seed=8)
    lay = bsa.bsa_layout_build_tokens(H, L, 200, 5, 3, 8)
    bsa.bsa_layout_upload(lay)
    dev = torch.device("cuda")
    out, lse = bsa.bsa_forward(q.to(dev), k.to(dev), v.to(dev), lay)
    assert bsa.bsa_sync_status() == 0
    g = OL.global_tokens(L, 5)
    gb = {t // 64 for t in g}
    rand = [[OL.token_random_blocks(h, I, L // 64, 200, gb, 3, 8) for I in range(L // 64)] for h in range(H)]
    gt = np.zeros(L, dtype=bool)
    gt[g] = True
    ref = {"H": H, "L": L, "block": 64, "nb": L // 64, "token": {"window": 200, "globals": g, "random": rand}}
    rng = np.random.default_rng(0)
    tokens = sorted(set([t for b_ in gb for t in range(64 * b_, 64 * b_ + 64, 7)] +
                        list(rng.integers(0, L, 60)) + [0, L - 1]))
    for b, h in ((0, 0), (1, 2)):
        o_ref, l_ref = OA.attention_rows(q, k, v, ref, b, h, tokens)
        o = out[b, h].float().cpu().numpy()[tokens]
        l = lse[b, h].cpu().numpy()[tokens]
        assert np.abs(o - o_ref).max() <= 2e-2
        assert np.abs(l - l_ref).max() <= 1e-3


BWD_CASES = [  # name, B, H, L, window, n_global, n_random, seed, global tokens, key pad
    ("band17_random", 2, 2, 64 * 13, 17, 0, 2, 1, None, 0),
    ("band100_globals", 1, 3, 64 * 16, 100, 3, 3, 2, None, 0),
    ("unaligned_globals_padding", 2, 2, 64 * 10, 64, 0, 1, 3, [5, 6, 70, 383, 600], 100),
    ("globals_split_rows", 1, 2, 64 * 64, 40, 2, 3, 6, [10, 4000], 0),
]


@pytest.mark.parametrize("name,B,H,L,w,ng,nr,seed,gt,pad", BWD_CASES, ids=[c[0] for c in BWD_CASES])
@pytest.mark.gpu
@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
def test_token_layout_backward_matches_oracle(name, B, H, L, w, ng, nr, seed, gt, pad):
    from oracle import backward as OB
    from test_backward import _check_grads
    wl = workloads.custom(B, H, L, 1, 0, 0, seed=seed, key_pad_tail=pad)
    q, k, v = workloads.make_qkv(wl, data_seed=seed)
    do = workloads.make_grad(wl, seed=100 + seed)
    km = workloads.make_key_mask(wl) if pad else None
    lay = bsa.bsa_layout_build_tokens(H, L, w, ng, nr, seed, global_tokens=gt)
    bsa.bsa_layout_upload(lay)
    dev = torch.device("cuda")
    qd, kd, vd, dod = q.to(dev), k.to(dev), v.to(dev), do.to(dev)
    kmd = km.to(dev) if km is not None else None
    out, lse = bsa.bsa_forward(qd, kd, vd, lay, key_mask=kmd)
    dq, dk, dv = bsa.bsa_backward(qd, kd, vd, out, dod, lse, lay, key_mask=kmd)
    assert bsa.bsa_sync_status() == 0
    ref = OL.build_token_layout(H, L, w, ng, nr, seed, explicit_globals=gt)
    dq_r, dk_r, dv_r, mags = OB.attention_backward(q, k, v, do, ref, key_mask=km, with_magnitude=True)
    _check_grads([t.float().cpu().numpy() for t in (dq, dk, dv)], (dq_r, dk_r, dv_r), mags)


def test_random_token_layouts_equal_the_oracle():
    """A seeded sweep of token-level layouts: the library's block CSR and global bits
    equal the oracle's, bit for bit, for windows from 0 to past the sequence, global
    tokens by rule and explicit (duplicates, neighbours, both ends), and random
    block counts from 0 to more than there are candidates."""
    rng = np.random.default_rng(123)
    for _ in range(40):
        H = int(rng.integers(1, 4))
        nb = int(rng.integers(1, 14))
        L = 64 * nb
        w = int(rng.choice([0, 1, 31, 63, 64, 65, 127, 200, L + 5]))
        nr = int(rng.integers(0, 6))
        seed = int(rng.integers(0, 2 ** 40))
        if rng.random() < 0.5:
            gt = None
            ng = int(rng.integers(0, 5))
        else:
            gt = [int(x) for x in rng.integers(0, L, int(rng.integers(0, 6)))]
            if gt and rng.random() < 0.5:
                gt += [gt[0], L - 1, 0]
            ng = len(gt)
        lay = bsa.bsa_layout_build_tokens(H, L, w, ng, nr, seed, global_tokens=gt)
        ref = OL.build_token_layout(H, L, w, ng, nr, seed, explicit_globals=gt)
        rp, ci = bsa.bsa_layout_csr(lay)
        assert np.array_equal(rp, ref["row_ptr"]) and np.array_equal(ci, ref["col_idx"]), (H, L, w, ng, nr, seed, gt)
        _, bits = bsa.bsa_layout_token_masks(lay)
        want = np.zeros(nb, dtype=np.uint64)
        for t in ref["token"]["globals"]:
            want[t // 64] |= np.uint64(1) << np.uint64(t % 64)
        assert np.array_equal(bits, want)
