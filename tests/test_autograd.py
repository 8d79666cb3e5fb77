"""torch.autograd binding (block_sparse_attention).

CPU: the binding's plumbing with the library calls replaced by fakes built on
the fp64 oracle -- which arguments reach bsa_forward and bsa_backward, that the
incoming gradient reaches the backward, and that its results land in q.grad,
k.grad, v.grad.
GPU: the binding against direct C-ABI calls on the same inputs (bit-identical).
"""

import numpy as np
import pytest
import torch

import workloads
from block_sparse_attention_bigbird_b200 import autograd as AG
from block_sparse_attention_bigbird_b200 import bsa
from oracle import attention as OA
from oracle import backward as OB
from oracle import layout as OL


def test_plumbing_with_fake_library(monkeypatch):
    w = workloads.custom(2, 2, 64 * 4, 1, 1, 1, seed=2, key_pad_tail=10)
    q, k, v = (t.double().requires_grad_(True) for t in workloads.make_qkv(w))
    km = workloads.make_key_mask(w)
    ref = OL.build_layout(w.H, w.L, 64, w.window, w.n_global, w.n_random, w.seed)
    seen = {}

    def fake_forward(q_, k_, v_, layout, key_mask=None, scale=None):
        seen["fwd"] = (layout, key_mask, scale)
        o, lse = OA.attention(q_, k_, v_, ref, key_mask=key_mask, scale=scale)
        return torch.from_numpy(o), torch.from_numpy(lse)

    def fake_backward(q_, k_, v_, out, dout, lse, layout, key_mask=None, scale=None):
        seen["bwd"] = (layout, key_mask, scale, dout.clone())
        g = OB.attention_backward(q_, k_, v_, dout, ref, key_mask=key_mask, scale=scale)
        return tuple(torch.from_numpy(x) for x in g)

    monkeypatch.setattr(bsa, "bsa_forward", fake_forward)
    monkeypatch.setattr(bsa, "bsa_backward", fake_backward)
    layout = object()
    out, lse = AG.block_sparse_attention(q, k, v, layout, key_mask=km, scale=0.2, return_lse=True)
    assert not lse.requires_grad
    wgt = torch.from_numpy(np.random.default_rng(0).standard_normal(out.shape))
    (out * wgt).sum().backward()
    assert seen["fwd"][0] is layout and seen["fwd"][1] is km and seen["fwd"][2] == 0.2
    assert seen["bwd"][0] is layout and seen["bwd"][1] is km and seen["bwd"][2] == 0.2
    assert torch.equal(seen["bwd"][3], wgt)
    g = OB.attention_backward(q.detach(), k.detach(), v.detach(), wgt, ref, key_mask=km, scale=0.2)
    for t, r in zip((q, k, v), g):
        assert np.array_equal(t.grad.numpy(), r)


@pytest.mark.gpu
@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
def test_autograd_equals_direct_calls():
    w = workloads.custom(2, 2, 64 * 20, 1, 2, 2, seed=3, key_pad_tail=100)
    dev = torch.device("cuda")
    q, k, v = (t.to(dev) for t in workloads.make_qkv(w))
    do = workloads.make_grad(w, seed=5).to(dev)
    km = workloads.make_key_mask(w).to(dev)
    lay = bsa.bsa_layout_build(w.H, w.L, 64, w.window, w.n_global, w.n_random, w.seed)
    bsa.bsa_layout_upload(lay)
    out_d, lse_d = bsa.bsa_forward(q, k, v, lay, key_mask=km)
    dq_d, dk_d, dv_d = bsa.bsa_backward(q, k, v, out_d, do, lse_d, lay, key_mask=km)
    qa, ka, va = (t.clone().requires_grad_(True) for t in (q, k, v))
    out = AG.block_sparse_attention(qa, ka, va, lay, key_mask=km)
    out.backward(do)
    assert bsa.bsa_sync_status() == 0
    assert torch.equal(out, out_d)
    for got, ref in ((qa.grad, dq_d), (ka.grad, dk_d), (va.grad, dv_d)):
        assert torch.equal(got, ref)
