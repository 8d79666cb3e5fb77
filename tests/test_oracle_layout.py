"""Pins for the oracle layout builder (CPU only).

Each check ties the oracle to something other than itself: a published
known-answer vector, the page's own linspace expression evaluated by torch,
arithmetic counts that never build a row, and distribution properties of the
sampler.
"""

import collections
import json
import os

import numpy as np
import pytest
import torch

import workloads
from oracle import layout as OL


def _kat_rows(golden_dir):
    rows = []
    with open(os.path.join(golden_dir, "philox4x64_10_kat.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append([int(x, 16) for x in line.split()])
    return rows


def test_philox_known_answer(golden_dir):
    # numpy increments the 256-bit counter before producing a block, so start one
    # below the vector's counter (mod 2^256).
    for row in _kat_rows(golden_dir):
        ctr, key, expect = row[0:4], row[4:6], row[6:10]
        c = int(sum(x << (64 * i) for i, x in enumerate(ctr))) - 1
        c %= 1 << 256
        words = [(c >> (64 * i)) & (2**64 - 1) for i in range(4)]
        bg = np.random.Philox(counter=words, key=key)
        assert [int(x) for x in bg.random_raw(4)] == expect


def test_philox_stream_counter_convention():
    # The stream of (i, h) starts from counter [0, i, h, 0]; numpy bumps the
    # counter before each 4-word block, so the first block is Philox([1,i,h,0]).
    s = OL.philox_stream(7, 5, 3, 8)
    bg = np.random.Philox(key=[7, 0], counter=[0, 5, 3, 0])
    assert [int(x) for x in bg.random_raw(1)] == s[:1]
    assert [int(x) for x in bg.state["state"]["counter"]] == [1, 5, 3, 0]


@pytest.mark.parametrize("name", list(workloads.WORKLOADS))
def test_globals_match_page_linspace(name):
    w = workloads.get(name)
    g = OL.global_blocks(w.nb, w.n_global)
    page = sorted(set(torch.linspace(0, w.nb - 1, w.n_global).long().tolist()))
    assert g == page


def test_globals_literal_13_of_128():
    assert OL.global_blocks(128, 13) == [0, 10, 21, 31, 42, 52, 63, 74, 84, 95, 105, 116, 127]
    assert OL.global_blocks(256, 2) == [0, 255]
    assert OL.global_blocks(8, 1) == [0]
    assert OL.global_blocks(8, 0) == []
    assert OL.global_blocks(4, 9) == [0, 1, 2, 3]   # more globals than blocks


def test_window_clipping():
    assert OL.window_blocks(0, 8, 1) == [0, 1]
    assert OL.window_blocks(7, 8, 1) == [6, 7]
    assert OL.window_blocks(3, 8, 2) == [1, 2, 3, 4, 5]
    assert OL.window_blocks(0, 3, 5) == [0, 1, 2]


def _count_nnz_per_head(nb, w, g, r):
    """Row sizes from interval arithmetic only (no sets, no random draws)."""
    total = 0
    gs = sorted(g)
    for i in range(nb):
        if i in gs:
            total += nb
            continue
        lo, hi = max(0, i - w), min(nb - 1, i + w)
        n_wg = (hi - lo + 1) + sum(1 for x in gs if x < lo or x > hi)
        total += n_wg + min(r, nb - n_wg)
    return total


@pytest.mark.parametrize("name", list(workloads.WORKLOADS))
def test_layout_invariants_and_counts(name):
    w = workloads.get(name)
    H = min(w.H, 2) if w.nb > 1000 else w.H
    lay = OL.build_layout(H, w.L, w.block, w.window, w.n_global, w.n_random, w.seed)
    g = set(lay["globals"])
    nnz_head = _count_nnz_per_head(w.nb, w.window, g, w.n_random)
    assert lay["row_ptr"][-1] == H * nnz_head
    for h in range(H):
        for i in range(w.nb):
            r = [int(x) for x in OL.row(lay, h, i)]
            assert r == sorted(set(r))
            if i in g:
                assert r == list(range(w.nb))
                continue
            win = set(OL.window_blocks(i, w.nb, w.window))
            assert win | g <= set(r)
            rnd = set(r) - win - g
            m = w.nb - len(win | g)
            assert len(rnd) == min(w.n_random, m)


def test_nnz_literal_counts():
    # nnz per head of the five shapes, by interval arithmetic.
    expect = {"c1": 41, "c2": 622, "c3": 3046, "c4": 4604, "c5": 32720}
    for alias, n in expect.items():
        w = workloads.get(alias)
        g = set(OL.global_blocks(w.nb, w.n_global))
        assert _count_nnz_per_head(w.nb, w.window, g, w.n_random) == n


def test_layout_depends_on_head_and_seed():
    a = OL.build_layout(2, 64 * 64, 64, 1, 2, 3, 0)
    b = OL.build_layout(2, 64 * 64, 64, 1, 2, 3, 1)
    ra = [tuple(OL.row(a, 0, i)) for i in range(64)]
    rb = [tuple(OL.row(b, 0, i)) for i in range(64)]
    rh = [tuple(OL.row(a, 1, i)) for i in range(64)]
    assert ra != rb and ra != rh


def test_fisher_yates_marginals_uniform():
    # Each of m candidates must be drawn with probability r/m.
    m, r, n = 7, 3, 20000
    cand = list(range(100, 100 + m))
    counts = collections.Counter()
    for s in range(n):
        bg = np.random.Philox(key=[s, 0], counter=[0, 1, 2, 0])
        pick = OL.random_blocks(cand, r, [int(x) for x in bg.random_raw(r)])
        assert len(set(pick)) == r and set(pick) <= set(cand)
        counts.update(pick)
    for c in cand:
        assert abs(counts[c] / n - r / m) < 0.02


def test_fisher_yates_full_shuffle_uniform():
    # With r = m = 3 every one of the 6 orders must be equally likely.
    n = 12000
    counts = collections.Counter()
    for s in range(n):
        bg = np.random.Philox(key=[s, 0], counter=[0, 0, 0, 0])
        counts[tuple(OL.random_blocks([0, 1, 2], 3, [int(x) for x in bg.random_raw(3)]))] += 1
    assert len(counts) == 6
    for v in counts.values():
        assert abs(v / n - 1 / 6) < 0.02


def test_fewer_candidates_than_r_takes_all():
    lay = OL.build_layout(1, 6 * 64, 64, 1, 1, 10, 0)
    for i in range(1, 6):
        assert list(OL.row(lay, 0, i)) == list(range(6))


def test_density_matches_page_figures(golden_dir):
    with open(os.path.join(golden_dir, "page_figures.json")) as f:
        fig = json.load(f)
    # all-ones layout at L=512: block nnz x 64^2 equals the page's 262,144 weights
    lay = OL.build_layout(1, 512, 64, 8, 0, 0, 0)
    assert int(lay["row_ptr"][-1]) * 64 * 64 == fig["dense_weights_512"]["value"]
    lay = OL.build_layout(1, 2048, 64, 0, 32, 0, 0)   # every block global
    n = int(lay["row_ptr"][-1]) * 64 * 64
    ref = fig["dense_weights_2048_approx"]
    assert abs(n - ref["value"]) / ref["value"] < ref["rel_tol"]
