"""The forward at head dim 128 against the fp64 oracle (GPU), and the calls that
do not take it.

The pages' BigBird module splits its hidden size into heads of dim // heads
("BigBird 稀疏注意力机制解析", 代码实现); d = 128 is the other head size the
kernel supports.  The d = 128 kernel runs one pipeline per SM with the head dim
in two 64-column halves (Q, K and V loaded as two boxes per block, eight 16-deep
S MMA steps, two PV issuers, O in 128 TMEM columns).  The cases mirror the d = 64
parity set: ragged tiles, global rows long enough to be split and merged, a
partially padded key tail, an explicit scale with sharp scores, a rising key norm,
a caller CSR with empty and full rows, sampled rows at L = 16384, bit-identical
repeats and the allocation-free entry.  Tolerances are the d = 64 ones (O max-abs
2e-2, lse max-abs 1e-3).
"""

import numpy as np
import pytest
import torch

import workloads
from oracle import attention as OA
from oracle import layout as OL

O_TOL = 2e-2
LSE_TOL = 1e-3

gpu = [pytest.mark.gpu, pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def _check(o_gpu, lse_gpu, o_ref, lse_ref):
    assert np.all(np.isfinite(o_gpu))
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isneginf(lse_gpu), ~fin)
    assert np.all(o_gpu[~fin] == 0)
    assert np.abs(o_gpu - o_ref).max() <= O_TOL
    if fin.any():
        assert np.abs(lse_gpu[fin] - lse_ref[fin]).max() <= LSE_TOL


def test_backward_rejects_head_dim_128_before_device_work():
    from block_sparse_attention_bigbird_b200 import bsa
    lay = bsa.bsa_layout_build(1, 64 * 4, 64, 1, 1, 1, 0)
    fake = 1 << 20
    code = bsa.lib.bsa_backward(fake, fake, fake, fake, fake, fake, 1, 1, 64 * 4, 128, lay.handle, None, 0.0,
                                fake, fake, fake, fake, 1 << 20, None)
    assert code == bsa.BSA_ERR_UNSUPPORTED
    assert bsa.bsa_forward_workspace_bytes(lay, 2, 128) > bsa.bsa_forward_workspace_bytes(lay, 2, 64) or \
        bsa.bsa_forward_workspace_bytes(lay, 2, 128) == bsa.bsa_workspace_bytes(lay, 2)
    with pytest.raises(bsa.BsaError):
        bsa.bsa_forward_workspace_bytes(lay, 2, 96)


CASES = [
    ("odd_blocks_ragged_tail", workloads.custom(2, 3, 64 * 13, 1, 1, 2, seed=5, d=128), None, None),
    ("two_globals_split", workloads.custom(1, 2, 64 * 64, 1, 2, 3, seed=1, d=128), None, None),
    ("many_globals_split", workloads.custom(1, 2, 64 * 100, 2, 7, 4, seed=2, d=128), None, None),
    ("key_padding_partial", workloads.custom(2, 2, 64 * 20, 1, 2, 2, seed=3, key_pad_tail=100, d=128), None, None),
    ("explicit_scale_sharp", workloads.custom(1, 2, 64 * 16, 1, 1, 2, k_mul=2.0, d=128), 0.3, None),
    ("rising_key_norms", workloads.custom(2, 2, 64 * 40, 2, 1, 3, seed=7, d=128), 0.5, "ramp"),
    ("all_global", workloads.custom(1, 1, 64 * 70, 0, 70, 0, d=128), None, None),
]


@pytest.mark.parametrize("name,w,scale,mod", CASES, ids=[c[0] for c in CASES])
@pytest.mark.gpu
@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
def test_head_dim_128_matches_oracle(name, w, scale, mod):
    from block_sparse_attention_bigbird_b200 import bsa
    q, k, v = workloads.make_qkv(w)
    assert q.shape[-1] == 128
    if mod == "ramp":
        ramp = torch.exp2(4.0 * torch.arange(w.L, dtype=torch.float32) / w.L).view(1, 1, w.L, 1)
        k = (k.float() * ramp).to(torch.bfloat16)
    km = workloads.make_key_mask(w)
    lay = bsa.bsa_layout_build(w.H, w.L, 64, w.window, w.n_global, w.n_random, w.seed)
    bsa.bsa_layout_upload(lay)
    dev = torch.device("cuda")
    out, lse = bsa.bsa_forward(q.to(dev), k.to(dev), v.to(dev), lay,
                               key_mask=km.to(dev) if km is not None else None, scale=scale)
    assert bsa.bsa_sync_status() == 0
    ref = OL.build_layout(w.H, w.L, 64, w.window, w.n_global, w.n_random, w.seed)
    o_ref, l_ref = OA.attention(q, k, v, ref, key_mask=km, scale=scale)
    _check(out.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref)


@pytest.mark.gpu
@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
def test_head_dim_128_caller_csr_with_empty_and_full_rows():
    from block_sparse_attention_bigbird_b200 import bsa
    w = workloads.custom(2, 3, 64 * 24, 1, 1, 1, seed=4, d=128)
    q, k, v = workloads.make_qkv(w)
    rp, ci = workloads.make_block_csr(w.H, w.nb, seed=11, p_empty=0.2, p_full=0.15)
    lay = bsa.bsa_layout_from_csr(w.H, w.L, rp, ci)
    bsa.bsa_layout_upload(lay)
    r2, c2 = bsa.bsa_layout_csr(lay)
    dev = torch.device("cuda")
    out, lse = bsa.bsa_forward(q.to(dev), k.to(dev), v.to(dev), lay)
    assert bsa.bsa_sync_status() == 0
    ref = {"H": w.H, "L": w.L, "block": 64, "nb": w.nb, "row_ptr": np.asarray(r2, dtype=np.int64),
           "col_idx": np.asarray(c2, dtype=np.int32)}
    o_ref, l_ref = OA.attention(q, k, v, ref)
    _check(out.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref)


@pytest.mark.gpu
@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
def test_head_dim_128_long_sequence_sampled_repeatable_and_static():
    """L = 16384 with split global rows: every row of the global query blocks and of
    sampled other blocks of one head against the oracle; a second call equal bit for
    bit; the allocation-free entry equal to the workspace entry."""
    from block_sparse_attention_bigbird_b200 import bsa
    w = workloads.custom(2, 4, 16384, 2, 2, 3, seed=9, d=128)
    q, k, v = workloads.make_qkv(w)
    lay = bsa.bsa_layout_build(w.H, w.L, 64, w.window, w.n_global, w.n_random, w.seed)
    bsa.bsa_layout_upload(lay)
    dev = torch.device("cuda")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    out, lse = bsa.bsa_forward(qd, kd, vd, lay)
    out2, lse2 = bsa.bsa_forward(qd, kd, vd, lay)
    out3, lse3 = bsa.bsa_forward_static_ws(qd, kd, vd, lay)
    assert bsa.bsa_sync_status() == 0
    assert torch.equal(out, out2) and torch.equal(lse, lse2)
    assert torch.equal(out, out3) and torch.equal(lse, lse3)
    ref = OL.build_layout(w.H, w.L, 64, w.window, w.n_global, w.n_random, w.seed)
    rng = np.random.default_rng(3)
    blocks = sorted(set([0, w.nb - 1, 1, w.nb - 2] + list(rng.integers(2, w.nb - 2, 6))))
    for b, h in ((0, 0), (1, 3)):
        view = {"H": 1, "L": w.L, "block": 64, "nb": w.nb, "globals": ref["globals"],
                "row_ptr": ref["row_ptr"][h * w.nb:(h + 1) * w.nb + 1] - ref["row_ptr"][h * w.nb],
                "col_idx": ref["col_idx"][ref["row_ptr"][h * w.nb]:ref["row_ptr"][(h + 1) * w.nb]]}
        o_ref, l_ref = OA.attention(q[b:b + 1, h:h + 1], k[b:b + 1, h:h + 1], v[b:b + 1, h:h + 1], view,
                                    query_blocks=blocks)
        rows = np.concatenate([np.arange(64 * i, 64 * i + 64) for i in blocks])
        _check(out[b, h].float().cpu().numpy()[rows], lse[b, h].cpu().numpy()[rows],
               o_ref[0, 0][rows], l_ref[0, 0][rows])
