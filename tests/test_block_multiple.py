"""Layouts at a block size that is a multiple of 64 (128, 256, ...).

The kernels run 64-key blocks.  A layout at block 64 m is expanded exactly:
query block I's row becomes the rows of its m 64-blocks, each listing the m
64-blocks of every key block in it -- attention restricted to (64 m)-blocks is
attention restricted to those 64-blocks.
CPU: the caller's view (bsa_layout_csr) is the BigBird layout at that block size,
bit-exact against the oracle's builder; the tiles the kernels run reproduce the
oracle's token-level mask exactly; caller CSRs at block 128 likewise.
GPU: forward and gradients on block-128 layouts against the fp64 oracle, which
works on the 128-token blocks directly.
"""

import numpy as np
import pytest
import torch

import workloads
from block_sparse_attention_bigbird_b200 import bsa
from oracle import attention as OA
from oracle import backward as OB
from oracle import layout as OL


def _token_mask_from_tiles(lay, H, L):
    """[H, L/64, L/64] 64-block mask the kernels run, from the query tiles."""
    nb = L // 64
    pair_q, pair_ptr, pair_ent = bsa.bsa_layout_tiles(lay)
    P = len(pair_q)
    m = np.zeros((H, nb, nb), dtype=bool)
    for h in range(H):
        for p, (a, b) in enumerate(pair_q):
            for e in pair_ent[pair_ptr[h * P + p]:pair_ptr[h * P + p + 1]]:
                col, bits = int(e & 0xFFFFFF), int(e >> 24)
                if bits & 1:
                    m[h, a, col] = True
                if bits & 2:
                    m[h, b, col] = True
    return m


def _oracle_mask64(ref, H, L):
    """The oracle's token mask of a layout at any block size, at 64-block granularity."""
    blk = ref["block"]
    bm = OL.block_mask(ref)  # [H, L/blk, L/blk]
    tok = np.repeat(np.repeat(bm, blk, axis=1), blk, axis=2)
    return tok[:, ::64, ::64]


@pytest.mark.parametrize("block,H,L,window,n_global,n_random,seed", [
    (128, 2, 128 * 10, 1, 1, 2, 3),
    (128, 3, 128 * 17, 2, 2, 3, 0),
    (256, 2, 256 * 7, 1, 1, 1, 9),
    (128, 1, 128, 0, 1, 0, 0),
])
def test_build_at_larger_blocks(block, H, L, window, n_global, n_random, seed):
    lay = bsa.bsa_layout_build(H, L, block, window, n_global, n_random, seed)
    rp, ci = bsa.bsa_layout_csr(lay)
    ref = OL.build_layout(H, L, block, window, n_global, n_random, seed)
    assert np.array_equal(rp, ref["row_ptr"].astype(np.int32)) and np.array_equal(ci, ref["col_idx"])
    assert list(bsa.bsa_layout_globals(lay)) == ref["globals"]
    assert np.array_equal(_token_mask_from_tiles(lay, H, L), _oracle_mask64(ref, H, L))


def test_caller_csr_at_block_128():
    H, nbu = 2, 11
    rp, ci = workloads.make_block_csr(H, nbu, seed=17, p_empty=0.2, p_full=0.1)
    lay = bsa.bsa_layout_from_csr(H, 128 * nbu, rp, ci, block=128)
    r2, c2 = bsa.bsa_layout_csr(lay)
    assert len(r2) == H * nbu + 1
    ref = {"H": H, "L": 128 * nbu, "block": 128, "nb": nbu, "row_ptr": r2.astype(np.int64), "col_idx": c2}
    for x in range(H * nbu):
        assert list(c2[r2[x]:r2[x + 1]]) == sorted(set(ci[rp[x]:rp[x + 1]].tolist()))
    assert np.array_equal(_token_mask_from_tiles(lay, H, 128 * nbu), _oracle_mask64(ref, H, 128 * nbu))


def test_blocks_not_a_multiple_of_64_are_unsupported():
    with pytest.raises(bsa.BsaError) as e:
        bsa.bsa_layout_build(1, 960, 96, 1, 1, 1, 0)
    assert e.value.code == bsa.BSA_ERR_UNSUPPORTED
    with pytest.raises(bsa.BsaError):
        bsa.bsa_layout_build(1, 1000, 128, 1, 1, 1, 0)  # L not a multiple of the block


@pytest.mark.gpu
@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
@pytest.mark.parametrize("block,B,H,L,window,n_global,n_random,pad", [
    (128, 2, 2, 128 * 12, 1, 2, 2, 90),
    (256, 1, 2, 256 * 6, 1, 1, 1, 0),
])
def test_parity_at_larger_blocks(block, B, H, L, window, n_global, n_random, pad):
    w = workloads.custom(B, H, L, window, n_global, n_random, seed=5, key_pad_tail=pad)
    lay = bsa.bsa_layout_build(H, L, block, window, n_global, n_random, 5)
    bsa.bsa_layout_upload(lay)
    ref = OL.build_layout(H, L, block, window, n_global, n_random, 5)
    q, k, v = workloads.make_qkv(w, 0)
    do = workloads.make_grad(w, seed=100)
    km = workloads.make_key_mask(w)
    dev = torch.device("cuda")
    kmd = km.to(dev) if km is not None else None
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    out, lse = bsa.bsa_forward(qd, kd, vd, lay, key_mask=kmd)
    dq, dk, dv = bsa.bsa_backward(qd, kd, vd, out, do.to(dev), lse, lay, key_mask=kmd)
    assert bsa.bsa_sync_status() == 0
    o_ref, lse_ref = OA.attention(q, k, v, ref, key_mask=km)
    assert np.abs(out.float().cpu().numpy() - o_ref).max() <= 2e-2
    fin = np.isfinite(lse_ref)
    assert np.abs(lse.cpu().numpy()[fin] - lse_ref[fin]).max() <= 1e-3
    g_ref = OB.attention_backward(q, k, v, do, ref, key_mask=km, with_magnitude=True)
    for got, r, mg in zip((dq, dk, dv), g_ref[:3], g_ref[3]):
        err = np.abs(got.float().cpu().numpy() - r)
        assert np.all(err <= 2.0 ** -6 * mg + 2.0 ** -8 * np.abs(r) + 1e-6)
