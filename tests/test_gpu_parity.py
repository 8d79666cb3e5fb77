"""GPU parity: the CUDA path (through the C-ABI binding) against the fp64 oracle.

Tolerances: O max-abs <= 2e-2 and lse max-abs <= 1e-3 against the unrounded
fp64 oracle on the same bf16 inputs (O is bf16 on the GPU, so its own rounding
alone costs up to 2^-9 relative); layouts are compared bit-exactly in the
CPU tests.
"""

import math

import numpy as np
import pytest
import torch

import workloads
from oracle import attention as OA
from oracle import layout as OL

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

O_TOL = 2e-2
LSE_TOL = 1e-3


@pytest.fixture(scope="module")
def bsa():
    from block_sparse_attention_bigbird_b200 import bsa as _bsa
    return _bsa


def _run(bsa, w, key_mask=None, scale=None, data_seed=0, explicit_globals=None):
    q, k, v = workloads.make_qkv(w, data_seed)
    lay = bsa.bsa_layout_build(w.H, w.L, 64, w.window, w.n_global, w.n_random, w.seed,
                               globals=explicit_globals)
    bsa.bsa_layout_upload(lay)
    dev = torch.device("cuda")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    kmd = key_mask.to(dev) if key_mask is not None else None
    out, lse = bsa.bsa_forward(qd, kd, vd, lay, key_mask=kmd, scale=scale)
    assert bsa.bsa_sync_status() == 0
    ref_layout = OL.build_layout(w.H, w.L, 64, w.window, w.n_global, w.n_random, w.seed,
                                 explicit_globals=explicit_globals)
    return (q, k, v), lay, ref_layout, out.float().cpu().numpy(), lse.cpu().numpy()


def _check(o_gpu, lse_gpu, o_ref, lse_ref):
    assert np.all(np.isfinite(o_gpu))
    err_o = np.abs(o_gpu - o_ref).max()
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isneginf(lse_gpu), ~fin)
    err_l = np.abs(lse_gpu[fin] - lse_ref[fin]).max() if fin.any() else 0.0
    assert err_o <= O_TOL, f"O max-abs {err_o}"
    assert err_l <= LSE_TOL, f"lse max-abs {err_l}"
    return err_o, err_l


SMALL = [
    # name, workload, key padding tail, scale
    ("tiny_b1h2l512", workloads.get("c1"), 0, None),
    ("odd_blocks_ragged_tail", workloads.custom(2, 3, 64 * 13, 1, 1, 2, seed=5), 0, None),
    ("two_globals_split", workloads.custom(1, 2, 64 * 64, 1, 2, 3, seed=1), 0, None),
    ("many_globals_split_single", workloads.custom(1, 2, 64 * 100, 2, 7, 4, seed=2), 0, None),
    ("key_padding_partial", workloads.custom(2, 2, 64 * 20, 1, 2, 2, seed=3, key_pad_tail=100), 100, None),
    ("dense_window", workloads.custom(1, 2, 64 * 6, 8, 0, 0), 0, None),
    ("all_global", workloads.custom(1, 1, 64 * 70, 0, 70, 0), 0, None),
    ("explicit_scale_sharp", workloads.custom(1, 2, 64 * 16, 1, 1, 2, k_mul=2.0), 0, 0.3),
    ("no_random_no_global", workloads.custom(2, 2, 64 * 9, 0, 0, 0), 0, None),
    ("single_block", workloads.custom(1, 1, 64, 0, 1, 0), 0, None),
    # logits with std ~16 (scale 1): later chunks often exceed the running max by far
    ("huge_logits", workloads.custom(2, 2, 64 * 24, 2, 2, 3, seed=6, k_mul=2.0), 0, 1.0),
]


@pytest.mark.parametrize("name,w,pad,scale", SMALL, ids=[s[0] for s in SMALL])
def test_parity_small_full(bsa, name, w, pad, scale):
    km = workloads.make_key_mask(w) if pad else None
    (q, k, v), _, ref_lay, o, lse = _run(bsa, w, key_mask=km, scale=scale)
    o_ref, lse_ref = OA.attention(q, k, v, ref_lay, key_mask=km, scale=scale)
    _check(o, lse, o_ref, lse_ref)


def test_rising_scores_raise_the_running_max(bsa):
    # Key norms grow by 2^4 along the sequence, so later chunks of a row keep
    # exceeding the running max: the path that redoes a chunk with the larger max
    # and rescales l and O runs many times per row.
    w = workloads.custom(2, 2, 64 * 40, 2, 1, 3, seed=7)
    q, k, v = workloads.make_qkv(w)
    ramp = torch.exp2(4.0 * torch.arange(w.L, dtype=torch.float32) / w.L).view(1, 1, w.L, 1)
    k = (k.float() * ramp).to(torch.bfloat16)
    lay = bsa.bsa_layout_build(w.H, w.L, 64, w.window, w.n_global, w.n_random, w.seed)
    bsa.bsa_layout_upload(lay)
    out, lse = bsa.bsa_forward(q.cuda(), k.cuda(), v.cuda(), lay, scale=0.5)
    assert bsa.bsa_sync_status() == 0
    ref = OL.build_layout(w.H, w.L, 64, w.window, w.n_global, w.n_random, w.seed)
    o_ref, lse_ref = OA.attention(q, k, v, ref, scale=0.5)
    _check(out.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref)


def test_fully_masked_rows_give_zero_and_neg_inf(bsa):
    # window 0, no globals/random: block i attends block i only; mask block 2's keys.
    w = workloads.custom(1, 1, 64 * 5, 0, 0, 0)
    km = torch.ones((1, w.L), dtype=torch.uint8)
    km[0, 128:192] = 0
    (q, k, v), _, ref_lay, o, lse = _run(bsa, w, key_mask=km)
    assert np.all(o[0, 0, 128:192] == 0) and np.all(np.isneginf(lse[0, 0, 128:192]))
    o_ref, lse_ref = OA.attention(q, k, v, ref_lay, key_mask=km)
    _check(o, lse, o_ref, lse_ref)


def test_explicit_globals(bsa):
    w = workloads.custom(1, 2, 64 * 30, 1, 3, 2, seed=4)
    (q, k, v), _, ref_lay, o, lse = _run(bsa, w, explicit_globals=[29, 5, 11])
    o_ref, lse_ref = OA.attention(q, k, v, ref_lay)
    _check(o, lse, o_ref, lse_ref)


def _sample_tokens(w, globals_, rng, n_random_rows=48):
    toks = set()
    for g in globals_[:4]:
        toks.update([64 * g, 64 * g + 17, 64 * g + 63])
    toks.update([0, 63, 64, w.L - 64, w.L - 1])
    toks.update(rng.integers(0, w.L, n_random_rows).tolist())
    return sorted(toks)


@pytest.mark.parametrize("name", ["c2", "c3", "c4", "c5"])
def test_parity_full_size_sampled(bsa, name):
    """Full benchmark shapes in the launch configuration the benchmark times,
    checked on sampled rows (all head/batch pairs' first and last rows, rows of
    global blocks, and seeded random rows)."""
    w = workloads.get(name)
    km = workloads.make_key_mask(w)
    (q, k, v), _, ref_lay, o, lse = _run(bsa, w, key_mask=km)
    rng = np.random.default_rng(0)
    pairs = [(b, h) for b in range(w.B) for h in range(w.H)]
    pick = [pairs[i] for i in sorted(set([0, len(pairs) - 1] + rng.integers(0, len(pairs), 3).tolist()))]
    worst_o = worst_l = 0.0
    for b, h in pick:
        toks = _sample_tokens(w, ref_lay["globals"], rng)
        o_ref, lse_ref = OA.attention_rows(q, k, v, ref_lay, b, h, toks, key_mask=km)
        eo, el = _check(o[b, h, toks], lse[b, h, toks], o_ref, lse_ref)
        worst_o, worst_l = max(worst_o, eo), max(worst_l, el)
    # every row attends unpadded global block 0, so every lse is finite
    assert np.isfinite(lse).all()


FULL_HEADS = [
    # name, (b, h) pairs checked on every row, which query blocks ("all" or the
    # global blocks plus the blocks of the padded key tail and the 4 blocks before it)
    ("c3", [(0, 0), (3, 11)], "all"),
    ("c4", [(0, 9)], "all"),
    ("c5", [(0, 7)], "globals_and_tail"),
]


@pytest.mark.parametrize("name,pairs,which", FULL_HEADS, ids=[f[0] for f in FULL_HEADS])
def test_parity_full_heads(bsa, name, pairs, which):
    """Every row of whole heads at the benchmark shapes, as launched by the
    benchmark: all 256 query blocks of the first and last (b, h) of the L=16384
    shape; all 128 blocks of one head of the 13-global shape (13 global query
    blocks split across chunks and merged); and in the L=131072 shape with the
    padded key tail, the global query blocks plus every query block of the
    padded tail and the 4 before it (whose windows reach the padding)."""
    w = workloads.get(name)
    km = workloads.make_key_mask(w)
    (q, k, v), _, ref_lay, o, lse = _run(bsa, w, key_mask=km)
    if which == "all":
        blocks = list(range(w.nb))
    else:
        tail0 = (w.L - w.key_pad_tail) // w.block - 4
        blocks = sorted(set(int(g) for g in ref_lay["globals"]) | set(range(tail0, w.nb)))
    if name == "c4":
        assert len(ref_lay["globals"]) == 13
    o_ref, lse_ref = OA.attention(q, k, v, ref_lay, key_mask=km, query_blocks=blocks, pairs=pairs)
    rows = np.concatenate([np.arange(i * w.block, (i + 1) * w.block) for i in blocks])
    for b, h in pairs:
        _check(o[b, h, rows], lse[b, h, rows], o_ref[b, h, rows], lse_ref[b, h, rows])


def test_constant_v_gives_constant_output_everywhere(bsa):
    # A property that holds at any size: softmax rows sum to 1, so v == c gives
    # O == c up to the bf16 rounding of P (l is summed from the unrounded fp32 p).
    w = workloads.get("c3")
    q, k, _ = workloads.make_qkv(w)
    v = torch.full_like(q, 0.5)
    lay = bsa.bsa_layout_build(w.H, w.L, 64, w.window, w.n_global, w.n_random, w.seed)
    bsa.bsa_layout_upload(lay)
    out, lse = bsa.bsa_forward(q.cuda(), k.cuda(), v.cuda(), lay)
    assert bsa.bsa_sync_status() == 0
    dev = (out.float() - 0.5).abs().max().item()
    assert dev <= 4e-3, dev
    assert torch.isfinite(lse).all().item()


def test_deterministic_and_any_workspace_contents(bsa):
    """Two calls give bit-identical results, and a workspace full of garbage (as a
    call that ended in a device error could leave it) gives the same result as a
    zeroed one: each call clears the schedule counters it uses."""
    w = workloads.custom(2, 2, 64 * 64, 1, 2, 3, seed=1)
    q, k, v = [t.cuda() for t in workloads.make_qkv(w)]
    lay = bsa.bsa_layout_build(w.H, w.L, 64, w.window, w.n_global, w.n_random, w.seed)
    bsa.bsa_layout_upload(lay)
    n = bsa.bsa_workspace_bytes(lay, w.B)
    ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
    o1, l1 = bsa.bsa_forward(q, k, v, lay, workspace=ws)
    o2, l2 = bsa.bsa_forward(q, k, v, lay, workspace=ws)
    dirty = torch.full((n,), 0x5A, dtype=torch.uint8, device="cuda")
    o3, l3 = bsa.bsa_forward(q, k, v, lay, workspace=dirty)
    assert bsa.bsa_sync_status() == 0
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert torch.equal(o1, o3) and torch.equal(l1, l3)


def test_bounded_wait_reports_timeout_and_context_survives(bsa):
    bsa.bsa_debug_wait_timeout(2_000_000)   # 2 ms on a barrier nothing completes
    assert bsa.bsa_sync_status() == bsa.BSA_ERR_DEVICE_TIMEOUT
    assert bsa.bsa_sync_status() == 0        # status word was cleared
    x = torch.arange(10, device="cuda").sum().item()
    assert x == 45
