"""The C++ layout builder (Philox4x64-10 written from its definition) against
the oracle's (numpy's Philox): bit-exact CSR on every benchmark shape and on a
grid of tiny shapes, plus invariants of the 128-row tile decomposition."""

import itertools

import numpy as np
import pytest

import workloads
from block_sparse_attention_bigbird_b200 import bsa
from oracle import layout as OL


def _compare(H, L, window, n_global, n_random, seed, explicit=None):
    lay = bsa.bsa_layout_build(H, L, 64, window, n_global, n_random, seed, globals=explicit)
    rp, ci = bsa.bsa_layout_csr(lay)
    ref = OL.build_layout(H, L, 64, window, n_global, n_random, seed, explicit_globals=explicit)
    assert np.array_equal(rp, ref["row_ptr"].astype(np.int32))
    assert np.array_equal(ci, ref["col_idx"])
    assert list(bsa.bsa_layout_globals(lay)) == ref["globals"]
    return lay, ref


@pytest.mark.parametrize("name", list(workloads.WORKLOADS))
def test_bit_exact_benchmark_shapes(name):
    w = workloads.get(name)
    H = 2 if w.nb > 1000 else w.H   # rows depend on (h, i) only; 2 heads suffice at L=131072
    _compare(H, w.L, w.window, w.n_global, w.n_random, w.seed)


def test_bit_exact_tiny_grid():
    for nb, win, ng, nr, seed in itertools.product(
            [1, 2, 3, 5, 17], [0, 1, 3], [0, 1, 2, 5], [0, 1, 4, 20], [0, 12345, 2**64 - 1]):
        _compare(3, 64 * nb, win, ng, nr, seed)


def test_bit_exact_explicit_globals():
    _compare(2, 64 * 40, 2, 0, 3, 7, explicit=[39, 3, 3, 17])
    _compare(2, 64 * 9, 1, 0, 2, 1, explicit=[])


def test_tile_decomposition():
    for name in ["c1", "c2", "c4"]:
        w = workloads.get(name)
        lay, ref = _compare(w.H, w.L, w.window, w.n_global, w.n_random, w.seed)
        pair_q, pair_ptr, pair_ent = bsa.bsa_layout_tiles(lay)
        g = set(ref["globals"])
        seen = []
        for a, b in pair_q:
            seen += [a] + ([b] if b >= 0 else [])
            if b >= 0:
                assert (a in g) == (b in g)
        assert sorted(seen) == list(range(w.nb))
        P = len(pair_q)
        for h in range(w.H):
            for p, (a, b) in enumerate(pair_q):
                ent = pair_ent[pair_ptr[h * P + p]:pair_ptr[h * P + p + 1]]
                cols = ent & 0xFFFFFF
                bits = ent >> 24
                ra = set(OL.row(ref, h, a).tolist())
                rb = set(OL.row(ref, h, b).tolist()) if b >= 0 else set()
                assert sorted(cols) == sorted(ra | rb) and len(set(cols)) == len(cols)
                for c, bt in zip(cols, bits):
                    assert bool(bt & 1) == (c in ra) and bool(bt & 2) == (c in rb)
                # order: blocks of both rows, then one-row blocks alternating a/b
                both = sorted(ra & rb)
                oa, ob = sorted(ra - rb), sorted(rb - ra)
                alt = [x for i in range(max(len(oa), len(ob)))
                       for x in (oa[i:i + 1] + ob[i:i + 1])]
                assert list(cols) == both + alt
