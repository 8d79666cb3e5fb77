"""Layouts from a caller's block CSR (bsa_layout_from_csr).

CPU: argument checks, row normalisation, the pairing of dense query blocks and
the tile decomposition of arbitrary rows (empty ones included); a BigBird CSR
fed back in gives the BigBird layout's tiles entry for entry.
GPU: the forward on such layouts against the fp64 oracle, which takes the same
rows (sorted and deduplicated in numpy, not by the library).
"""

import numpy as np
import pytest
import torch

import workloads
from block_sparse_attention_bigbird_b200 import bsa
from oracle import attention as OA
from oracle import layout as OL


def _oracle_layout(H, L, row_ptr, col_idx):
    """The oracle's layout dict for the same rows (sorted, deduplicated in numpy)."""
    nb = L // 64
    rp, cols = [0], []
    for x in range(H * nb):
        cols.extend(sorted(set(int(c) for c in col_idx[row_ptr[x]:row_ptr[x + 1]])))
        rp.append(len(cols))
    return {"H": H, "L": L, "block": 64, "nb": nb,
            "row_ptr": np.asarray(rp, dtype=np.int64), "col_idx": np.asarray(cols, dtype=np.int32)}


def _check_tiles(lay, ref):
    """Every tile's entries are its two rows' union with the right membership bits,
    ordered both-first; an all-empty tile holds one entry without bits."""
    H, nb = ref["H"], ref["nb"]
    pair_q, pair_ptr, pair_ent = bsa.bsa_layout_tiles(lay)
    seen = sorted(int(x) for x in pair_q.ravel() if x >= 0)
    assert seen == list(range(nb))
    P = len(pair_q)
    for h in range(H):
        for p, (a, b) in enumerate(pair_q):
            ent = pair_ent[pair_ptr[h * P + p]:pair_ptr[h * P + p + 1]]
            ra = set(OL.row(ref, h, int(a)).tolist())
            rb = set(OL.row(ref, h, int(b)).tolist()) if b >= 0 else set()
            if not ra and not rb:
                assert list(ent) == [0]
                continue
            cols, bits = ent & 0xFFFFFF, ent >> 24
            assert sorted(cols.tolist()) == sorted(ra | rb)
            for c, m in zip(cols.tolist(), bits.tolist()):
                assert m == (1 if c in ra else 0) | (2 if c in rb else 0)
            nboth = int(np.sum(bits == 3))
            assert np.all(bits[:nboth] == 3) and not np.any(bits[nboth:] == 3)


@pytest.mark.parametrize("name", ["c2", "c4"])
def test_bigbird_csr_round_trip(name):
    """A BigBird CSR given back as a caller's CSR yields the same rows, the same
    dense blocks (the globals) and the very same tiles."""
    w = workloads.get(name)
    lay = bsa.bsa_layout_build(w.H, w.L, 64, w.window, w.n_global, w.n_random, w.seed)
    rp, ci = bsa.bsa_layout_csr(lay)
    lay2 = bsa.bsa_layout_from_csr(w.H, w.L, rp, ci)
    rp2, ci2 = bsa.bsa_layout_csr(lay2)
    assert np.array_equal(rp, rp2) and np.array_equal(ci, ci2)
    assert np.array_equal(bsa.bsa_layout_globals(lay), bsa.bsa_layout_globals(lay2))
    for x, y in zip(bsa.bsa_layout_tiles(lay), bsa.bsa_layout_tiles(lay2)):
        assert np.array_equal(x, y)


def test_rows_sorted_and_deduplicated():
    H, nb = 3, 23
    rp, ci = workloads.make_block_csr(H, nb, seed=4)
    lay = bsa.bsa_layout_from_csr(H, 64 * nb, rp, ci)
    rp2, ci2 = bsa.bsa_layout_csr(lay)
    ref = _oracle_layout(H, 64 * nb, rp, ci)
    assert np.array_equal(rp2, ref["row_ptr"].astype(np.int32))
    assert np.array_equal(ci2, ref["col_idx"])


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
def test_tiles_of_arbitrary_rows(seed):
    H, nb = 2, [1, 7, 30, 61][seed]
    rp, ci = workloads.make_block_csr(H, nb, seed=seed, p_empty=0.3, p_full=0.1)
    lay = bsa.bsa_layout_from_csr(H, 64 * nb, rp, ci)
    _check_tiles(lay, _oracle_layout(H, 64 * nb, rp, ci))


def test_dense_blocks_pair_together():
    H, nb = 2, 20
    rp, ci = workloads.make_block_csr(H, nb, seed=9, p_full=0.0, full_blocks=[3, 11, 12])
    lay = bsa.bsa_layout_from_csr(H, 64 * nb, rp, ci)
    assert bsa.bsa_layout_globals(lay).tolist() == [3, 11, 12]
    pair_q, _, _ = bsa.bsa_layout_tiles(lay)
    dense = {3, 11, 12}
    for a, b in pair_q:
        if b >= 0:
            assert (a in dense) == (b in dense)


def test_block_full_in_one_head_only_is_not_dense():
    H, nb = 2, 4
    rows = [[0, 1, 2, 3], [1], [2], [3],      # head 0: block 0 full
            [0], [1], [2], [3]]               # head 1: block 0 not
    rp = np.cumsum([0] + [len(r) for r in rows]).astype(np.int32)
    ci = np.asarray([c for r in rows for c in r], dtype=np.int32)
    lay = bsa.bsa_layout_from_csr(H, 64 * nb, rp, ci)
    assert bsa.bsa_layout_globals(lay).size == 0


def test_all_rows_empty():
    H, nb = 2, 5
    rp = np.zeros(H * nb + 1, dtype=np.int32)
    lay = bsa.bsa_layout_from_csr(H, 64 * nb, rp, np.zeros(0, np.int32))
    _, _, pair_ent = bsa.bsa_layout_tiles(lay)
    assert np.all(pair_ent == 0)
    _check_tiles(lay, _oracle_layout(H, 64 * nb, rp, np.zeros(0, np.int32)))


def _raw_from_csr(H, L, block, rp, ci):
    out = bsa.ctypes.c_void_p()
    P = bsa.ctypes.POINTER(bsa.ctypes.c_int32)
    rpp = None if rp is None else np.ascontiguousarray(rp, dtype=np.int32).ctypes.data_as(P)
    cip = None if ci is None else np.ascontiguousarray(ci, dtype=np.int32).ctypes.data_as(P)
    code = bsa.lib.bsa_layout_from_csr(H, L, block, rpp, cip, bsa.ctypes.byref(out))
    if code == 0:
        bsa.lib.bsa_layout_free(out)
    else:
        assert not out.value
    return code


def test_rejects_bad_csr():
    nb = 4
    good_rp = np.array([0, 1, 2, 3, 4], dtype=np.int32)
    good_ci = np.array([0, 1, 2, 3], dtype=np.int32)
    assert _raw_from_csr(1, 64 * nb, 64, good_rp, good_ci) == bsa.BSA_OK
    assert _raw_from_csr(1, 64 * nb, 96, good_rp, good_ci) == bsa.BSA_ERR_UNSUPPORTED
    assert _raw_from_csr(1, 64 * nb, 32, good_rp, good_ci) == bsa.BSA_ERR_UNSUPPORTED
    assert _raw_from_csr(0, 64 * nb, 64, good_rp, good_ci) == bsa.BSA_ERR_INVALID_ARG
    assert _raw_from_csr(1, 64 * nb + 3, 64, good_rp, good_ci) == bsa.BSA_ERR_INVALID_ARG
    assert _raw_from_csr(1, 64 * nb, 64, None, good_ci) == bsa.BSA_ERR_INVALID_ARG
    assert _raw_from_csr(1, 64 * nb, 64, good_rp, None) == bsa.BSA_ERR_INVALID_ARG
    assert _raw_from_csr(1, 64 * nb, 64, np.array([1, 1, 2, 3, 4]), good_ci) == bsa.BSA_ERR_INVALID_ARG
    assert _raw_from_csr(1, 64 * nb, 64, np.array([0, 2, 1, 3, 4]), good_ci) == bsa.BSA_ERR_INVALID_ARG
    assert _raw_from_csr(1, 64 * nb, 64, good_rp, np.array([0, 1, 4, 3])) == bsa.BSA_ERR_INVALID_ARG
    assert _raw_from_csr(1, 64 * nb, 64, good_rp, np.array([0, -1, 2, 3])) == bsa.BSA_ERR_INVALID_ARG
    # an empty layout needs no col_idx
    assert _raw_from_csr(1, 64 * nb, 64, np.zeros(nb + 1), None) == bsa.BSA_OK
    with pytest.raises(bsa.BsaError):
        bsa.bsa_layout_from_csr(1, 64 * nb, good_rp[:-1], good_ci)


# ------------------------------------------------------------------ GPU parity

O_TOL = 2e-2
LSE_TOL = 1e-3

CASES = [
    # name, B, H, nb, (row_ptr, col_idx), key padding tail
    ("random_rows", 2, 3, 40, workloads.make_block_csr(3, 40, seed=11, p_empty=0.15, p_full=0.05), 0),
    ("random_rows_padded", 2, 2, 33, workloads.make_block_csr(2, 33, seed=12, p_empty=0.1), 150),
    ("router_globals_split", 1, 4, 64, workloads.make_router_csr(4, 64, k_global=3, window=2, seed=13), 0),
    ("dense_blocks", 1, 2, 50, workloads.make_block_csr(2, 50, seed=14, p_full=0.0, full_blocks=[0, 7, 49]), 0),
    ("all_empty", 1, 2, 6, (np.zeros(2 * 6 + 1, np.int32), np.zeros(0, np.int32)), 0),
]


@pytest.mark.gpu
@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
@pytest.mark.parametrize("name,B,H,nb,csr,pad", CASES, ids=[c[0] for c in CASES])
def test_parity_user_csr(name, B, H, nb, csr, pad):
    L = 64 * nb
    rp, ci = csr
    w = workloads.custom(B, H, L, 0, 0, 0, seed=0, key_pad_tail=pad)
    q, k, v = workloads.make_qkv(w, data_seed=21)
    km = workloads.make_key_mask(w)
    lay = bsa.bsa_layout_from_csr(H, L, rp, ci)
    bsa.bsa_layout_upload(lay)
    dev = torch.device("cuda")
    out, lse = bsa.bsa_forward(q.to(dev), k.to(dev), v.to(dev), lay,
                               key_mask=None if km is None else km.to(dev))
    assert bsa.bsa_sync_status() == 0
    o_ref, lse_ref = OA.attention(q, k, v, _oracle_layout(H, L, rp, ci), key_mask=km)
    o, lg = out.float().cpu().numpy(), lse.cpu().numpy()
    assert np.all(np.isfinite(o))
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isneginf(lg), ~fin)
    assert np.all(o[~fin] == 0.0)
    assert np.abs(o - o_ref).max() <= O_TOL
    if fin.any():
        assert np.abs(lg[fin] - lse_ref[fin]).max() <= LSE_TOL
