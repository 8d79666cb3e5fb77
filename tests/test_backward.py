"""The backward (bsa_backward): key-major tiles and argument checks on the CPU,
gradients against the fp64 oracle on the GPU.

GPU tolerance, per element, derived from the arithmetic: with w the oracle's sum
of absolute terms (P (|dP| + rowsum |dO||O|) times |K| or |Q| for dQ and dK,
P^T |dO| for dV), the kernel's roundings move a result by at most
  2^-9 w  (P and dS rounded to bf16 for the tensor cores)
+ 2^-8 w  (D taken from the bf16 O of the forward, itself within 2^-9)
+ ~1e-5 w (ex2.approx and the forward's fp32 lse)
before its own rounding to bf16 (2^-9 |ref|).  The test allows
|gpu - ref| <= 2^-6 w + 2^-8 |ref| + 1e-6, about twice that sum.
"""

import ctypes

import numpy as np
import pytest
import torch

import workloads
from block_sparse_attention_bigbird_b200 import bsa
from oracle import backward as OB
from oracle import layout as OL

W_TOL = 2.0 ** -6
R_TOL = 2.0 ** -8
A_TOL = 1e-6


def _transposed_rows(ref):
    """Row (h, j) of the transposed block mask: the query blocks attending key block j."""
    m = OL.block_mask(ref)  # [H, nb(query), nb(key)]
    return [[np.nonzero(m[h, :, j])[0].tolist() for j in range(ref["nb"])] for h in range(ref["H"])]


def _check_key_tiles(lay, ref):
    H, nb = ref["H"], ref["nb"]
    rows = _transposed_rows(ref)
    pair_k, pair_ptr, pair_ent = bsa.bsa_layout_key_tiles(lay)
    assert sorted(int(x) for x in pair_k.ravel() if x >= 0) == list(range(nb))
    P = len(pair_k)
    for h in range(H):
        for p, (a, b) in enumerate(pair_k):
            ent = pair_ent[pair_ptr[h * P + p]:pair_ptr[h * P + p + 1]]
            ra = set(rows[h][a])
            rb = set(rows[h][b]) if b >= 0 else set()
            if not ra and not rb:
                assert list(ent) == [0]
                continue
            cols, bits = ent & 0xFFFFFF, ent >> 24
            assert sorted(cols.tolist()) == sorted(ra | rb)
            for c, m in zip(cols.tolist(), bits.tolist()):
                assert m == (1 if c in ra else 0) | (2 if c in rb else 0)


@pytest.mark.parametrize("name", ["c1", "c2", "c4"])
def test_key_tiles_are_the_transposed_layout(name):
    w = workloads.get(name)
    lay = bsa.bsa_layout_build(w.H, w.L, 64, w.window, w.n_global, w.n_random, w.seed)
    ref = OL.build_layout(w.H, w.L, 64, w.window, w.n_global, w.n_random, w.seed)
    _check_key_tiles(lay, ref)
    # BigBird's global key blocks are attended by every query block: they pair together
    g = set(ref["globals"])
    pair_k, _, _ = bsa.bsa_layout_key_tiles(lay)
    for a, b in pair_k:
        if b >= 0:
            assert (a in g) == (b in g)


def test_key_tiles_of_a_caller_csr():
    H, nb = 2, 29
    rp, ci = workloads.make_block_csr(H, nb, seed=31, p_empty=0.2, p_full=0.1)
    lay = bsa.bsa_layout_from_csr(H, 64 * nb, rp, ci)
    r2, c2 = bsa.bsa_layout_csr(lay)
    ref = {"H": H, "L": 64 * nb, "block": 64, "nb": nb, "row_ptr": r2.astype(np.int64), "col_idx": c2}
    _check_key_tiles(lay, ref)


def _bwd(lay, **kw):
    a = dict(q=1 << 12, k=1 << 12, v=1 << 12, out=1 << 12, dout=1 << 12, lse=1 << 12, B=1, H=2, L=512, d=64,
             key_mask=None, scale=0.0, dq=1 << 12, dk=1 << 12, dv=1 << 12, ws=1 << 12, ws_bytes=1 << 30)
    a.update(kw)
    return bsa.lib.bsa_backward(a["q"], a["k"], a["v"], a["out"], a["dout"], a["lse"], a["B"], a["H"], a["L"],
                                a["d"], lay.handle if a.get("use_layout", True) else None, a["key_mask"],
                                ctypes.c_float(a["scale"]), a["dq"], a["dk"], a["dv"], a["ws"], a["ws_bytes"], None)


def test_backward_argument_errors_before_any_launch():
    lay = bsa.bsa_layout_build(2, 512, 64, 1, 1, 1, 0)
    for name in ("q", "k", "v", "out", "dout", "lse", "dq", "dk", "dv"):
        assert _bwd(lay, **{name: None}) == bsa.BSA_ERR_INVALID_ARG, name
    assert _bwd(lay, use_layout=False) == bsa.BSA_ERR_INVALID_ARG
    assert _bwd(lay, B=0) == bsa.BSA_ERR_INVALID_ARG
    assert _bwd(lay, d=128) == bsa.BSA_ERR_UNSUPPORTED
    assert _bwd(lay, H=3) == bsa.BSA_ERR_LAYOUT_MISMATCH
    assert _bwd(lay, dq=(1 << 12) + 8) == bsa.BSA_ERR_INVALID_ARG  # misaligned
    assert _bwd(lay, scale=float("inf")) == bsa.BSA_ERR_INVALID_ARG
    assert _bwd(lay, ws=None) == bsa.BSA_ERR_WORKSPACE
    assert _bwd(lay, ws_bytes=16) == bsa.BSA_ERR_WORKSPACE
    assert _bwd(lay) == bsa.BSA_ERR_LAYOUT_MISMATCH  # never uploaded


def test_backward_workspace_grows_with_batch():
    lay = bsa.bsa_layout_build(12, 4096, 64, 1, 2, 3, 0)
    w1, w2 = bsa.bsa_backward_workspace_bytes(lay, 1), bsa.bsa_backward_workspace_bytes(lay, 2)
    assert w1 % 256 == 0 and w2 > w1
    # at least D and lse2 for every row
    assert w1 >= 2 * 4 * 12 * 4096


# ------------------------------------------------------------------ GPU parity

def _gpu_grads(w, lay, key_mask, scale, data_seed=0, to_numpy=True):
    """Forward then backward on the GPU with the inputs bench.py's rank 0 uses
    (data seed 0, gradient seed 100)."""
    q, k, v = workloads.make_qkv(w, data_seed)
    do = workloads.make_grad(w, seed=data_seed + 100)
    dev = torch.device("cuda")
    qd, kd, vd, dod = q.to(dev), k.to(dev), v.to(dev), do.to(dev)
    kmd = key_mask.to(dev) if key_mask is not None else None
    out, lse = bsa.bsa_forward(qd, kd, vd, lay, key_mask=kmd, scale=scale)
    dq, dk, dv = bsa.bsa_backward(qd, kd, vd, out, dod, lse, lay, key_mask=kmd, scale=scale)
    assert bsa.bsa_sync_status() == 0
    grads = (dq, dk, dv)
    return (q, k, v, do), ([t.float().cpu().numpy() for t in grads] if to_numpy else grads)


def _check_grads(gpu, ref, mags):
    for name, g, r, m in zip(("dq", "dk", "dv"), gpu, ref, mags):
        assert np.all(np.isfinite(g)), name
        bound = W_TOL * m + R_TOL * np.abs(r) + A_TOL
        err = np.abs(g - r)
        worst = np.unravel_index(np.argmax(err - bound), err.shape)
        assert np.all(err <= bound), f"{name}: err {err[worst]} > bound {bound[worst]} at {worst}"
        # where the oracle is exactly zero (no attended key, or a key no query attends) so is the GPU
        assert np.all(g[(r == 0) & (m == 0)] == 0), name


GPU = [pytest.mark.gpu, pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

CASES = [
    # name, workload, scale
    ("tiny_b1h2l512", workloads.get("c1"), None),
    ("odd_blocks_ragged_tail", workloads.custom(2, 3, 64 * 13, 1, 1, 2, seed=5), None),
    ("two_globals_split", workloads.custom(1, 2, 64 * 64, 1, 2, 3, seed=1), None),
    ("key_padding_partial", workloads.custom(2, 2, 64 * 20, 1, 2, 2, seed=3, key_pad_tail=100), None),
    ("many_globals_split", workloads.custom(1, 2, 64 * 100, 2, 7, 4, seed=2), None),
    ("explicit_scale_sharp", workloads.custom(1, 2, 64 * 16, 1, 1, 2, k_mul=2.0), 0.3),
    ("single_block", workloads.custom(1, 1, 64, 0, 1, 0), None),
]


@pytest.mark.gpu
@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
@pytest.mark.parametrize("name,w,scale", CASES, ids=[c[0] for c in CASES])
def test_backward_parity(name, w, scale):
    lay = bsa.bsa_layout_build(w.H, w.L, 64, w.window, w.n_global, w.n_random, w.seed)
    bsa.bsa_layout_upload(lay)
    km = workloads.make_key_mask(w)
    (q, k, v, do), gpu = _gpu_grads(w, lay, km, scale)
    ref_lay = OL.build_layout(w.H, w.L, 64, w.window, w.n_global, w.n_random, w.seed)
    dq, dk, dv, mags = OB.attention_backward(q, k, v, do, ref_lay, key_mask=km, scale=scale, with_magnitude=True)
    _check_grads(gpu, (dq, dk, dv), mags)


@pytest.mark.gpu
@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
def test_backward_parity_caller_csr_with_empty_rows():
    H, nb = 2, 24
    rp, ci = workloads.make_block_csr(H, nb, seed=41, p_empty=0.2, p_full=0.1)
    w = workloads.custom(2, H, 64 * nb, 0, 0, 0, key_pad_tail=70)
    lay = bsa.bsa_layout_from_csr(H, w.L, rp, ci)
    bsa.bsa_layout_upload(lay)
    r2, c2 = bsa.bsa_layout_csr(lay)
    ref_lay = {"H": H, "L": w.L, "block": 64, "nb": nb, "row_ptr": r2.astype(np.int64), "col_idx": c2}
    km = workloads.make_key_mask(w)
    (q, k, v, do), gpu = _gpu_grads(w, lay, km, None)
    dq, dk, dv, mags = OB.attention_backward(q, k, v, do, ref_lay, key_mask=km, with_magnitude=True)
    _check_grads(gpu, (dq, dk, dv), mags)


@pytest.mark.gpu
@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
def test_backward_repeatable_and_workspace_reusable():
    w = workloads.custom(1, 2, 64 * 64, 1, 2, 3, seed=1)
    lay = bsa.bsa_layout_build(w.H, w.L, 64, w.window, w.n_global, w.n_random, w.seed)
    bsa.bsa_layout_upload(lay)
    _, g1 = _gpu_grads(w, lay, None, None)
    _, g2 = _gpu_grads(w, lay, None, None)
    for a, b in zip(g1, g2):
        assert np.array_equal(a, b)


@pytest.mark.gpu
@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
@pytest.mark.parametrize("name", ["c3", "c5"])
def test_backward_full_size_sampled(name):
    """Full benchmark shapes in the launch configuration ``bench.py --pass backward``
    times, checked on sampled rows: query rows (first, last, global, random) and key
    rows (random non-global ones; for long_b4h12l16384 also the global key blocks'
    first and last keys, which every query block attends; for genomic_b1h8l131072
    padded keys, whose gradients are zero)."""
    w = workloads.get(name)
    lay = bsa.bsa_layout_build(w.H, w.L, 64, w.window, w.n_global, w.n_random, w.seed)
    bsa.bsa_layout_upload(lay)
    km = workloads.make_key_mask(w)
    (q, k, v, do), (dq, dk, dv) = _gpu_grads(w, lay, km, None, to_numpy=False)
    ref_lay = OL.build_layout(w.H, w.L, 64, w.window, w.n_global, w.n_random, w.seed)
    g = ref_lay["globals"]
    rng = np.random.default_rng(7)
    non_global = np.setdiff1d(np.arange(w.nb), g)
    if w.key_pad_tail:
        non_global = non_global[non_global * 64 + 63 < w.L - w.key_pad_tail]
    # the genomic shape's oracle rows span 131072 keys each: one (b, h) keeps it to seconds
    pairs = [(0, 0), (w.B - 1, w.H - 1)] if w.L <= 16384 else [(w.B - 1, w.H - 1)]
    for n, (b, h) in enumerate(pairs):
        qt = {0, 63, 64, w.L - 1, g[0] * 64 + 5, g[-1] * 64 + 60}
        qt.update(int(x) * 64 + int(rng.integers(0, 64)) for x in rng.choice(non_global, 4, replace=False))
        kt = {int(x) * 64 + int(rng.integers(0, 64)) for x in rng.choice(non_global, 4, replace=False)}
        if name == "c3" and n == 0:
            kt.update({g[0] * 64, g[-1] * 64 + 63})
        if w.key_pad_tail:
            # padded keys of non-global blocks (a global key needs every query row of the oracle)
            pad_blocks = [x for x in range((w.L - w.key_pad_tail) // 64, w.nb) if x not in g]
            kt.update({w.L - w.key_pad_tail, pad_blocks[-1] * 64 + 63})
        qt, kt = sorted(qt), sorted(kt)
        rq, rk, rv, (mq, mk, mv) = OB.attention_backward_rows(q, k, v, do, ref_lay, b, h, qt, kt, key_mask=km)
        got = [t[b, h, idx].float().cpu().numpy() for t, idx in ((dq, qt), (dk, kt), (dv, kt))]
        _check_grads(got, (rq, rk, rv), (mq, mk, mv))
        if w.key_pad_tail:
            padded = [x for x, p in enumerate(kt) if p >= w.L - w.key_pad_tail]
            assert np.all(got[1][padded] == 0) and np.all(got[2][padded] == 0)
