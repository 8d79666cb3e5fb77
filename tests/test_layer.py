"""BigBirdSelfAttention: QKV projection, block-sparse attention, output projection.

CPU: the layer with the library's kernels replaced by fakes built on the fp64
oracle, against a dense fp64 torch implementation of the same layer (masked
softmax attention over the expanded block mask) -- outputs and the gradients of
the input and of both projections.  This pins the head split, the q/k/v order of
the projection and the merge of heads.
GPU: the layer against the same steps spelled out with the binding (the same
arithmetic: equal up to the GEMM library's choice of algorithm, checked at 1 %
of the output's scale -- a wrong head split or q/k/v order is off by O(1)), and
a backward that reaches every weight.
"""

import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import workloads
from block_sparse_attention_bigbird_b200 import bsa
from block_sparse_attention_bigbird_b200.layer import BigBirdSelfAttention
from oracle import attention as OA
from oracle import backward as OB
from oracle import layout as OL


def _dense_reference(mod, x, lay, km):
    B, L, C = x.shape
    H = mod.num_heads
    q, k, v = mod.qkv(x).view(B, L, 3, H, 64).permute(2, 0, 3, 1, 4).unbind(0)
    s = (q @ k.transpose(-1, -2)) / math.sqrt(64)
    allowed = torch.from_numpy(np.repeat(np.repeat(OL.block_mask(lay), 64, axis=1), 64, axis=2))  # [H, L, L]
    allowed = allowed[None].expand(B, H, L, L)
    if km is not None:
        allowed = allowed & (torch.as_tensor(km) != 0)[:, None, None, :]
    p = torch.softmax(s.masked_fill(~allowed, -math.inf), dim=-1)
    o = (p @ v).transpose(1, 2).reshape(B, L, C)
    return mod.proj(o)


def test_layer_plumbing_with_fake_library(monkeypatch):
    B, H, L = 2, 2, 64 * 5
    w = workloads.custom(B, H, L, 1, 1, 1, seed=4, key_pad_tail=30)
    lay = OL.build_layout(H, L, 64, w.window, w.n_global, w.n_random, w.seed)

    class FakeLayout:
        def __init__(self):
            self.H, self.L = H, L

    def fake_build(H_, L_, block, window, n_global, n_random, seed, globals=None):
        assert (H_, L_, block, window, n_global, n_random, seed) == (H, L, 64, 1, 1, 1, 4)
        return FakeLayout()

    def fake_forward(q, k, v, layout, key_mask=None, scale=None):
        o, lse = OA.attention(q, k, v, lay, key_mask=key_mask, scale=scale)
        return torch.from_numpy(o), torch.from_numpy(lse)

    def fake_backward(q, k, v, out, dout, lse, layout, key_mask=None, scale=None):
        return tuple(torch.from_numpy(t) for t in OB.attention_backward(q, k, v, dout, lay, key_mask=key_mask,
                                                                          scale=scale))

    monkeypatch.setattr(bsa, "bsa_layout_build", fake_build)
    monkeypatch.setattr(bsa, "bsa_layout_upload", lambda layout, stream=None: None)
    monkeypatch.setattr(bsa, "bsa_forward", fake_forward)
    monkeypatch.setattr(bsa, "bsa_backward", fake_backward)
    torch.manual_seed(0)
    mod = BigBirdSelfAttention(H * 64, H, window=1, num_global=1, num_random=1, seed=4).double()
    ref = BigBirdSelfAttention(H * 64, H).double()
    ref.load_state_dict(mod.state_dict())
    km = workloads.make_key_mask(w).numpy()
    x = torch.randn(B, L, H * 64, dtype=torch.float64, requires_grad=True)
    x_ref = x.detach().clone().requires_grad_(True)
    y = mod(x, key_mask=torch.from_numpy(km))
    y_ref = _dense_reference(ref, x_ref, lay, km)
    assert torch.allclose(y, y_ref, rtol=0, atol=1e-10)
    g = torch.randn_like(y)
    y.backward(g)
    y_ref.backward(g)
    assert torch.allclose(x.grad, x_ref.grad, rtol=0, atol=1e-9)
    for (n, a), (_, b) in zip(mod.named_parameters(), ref.named_parameters()):
        assert torch.allclose(a.grad, b.grad, rtol=0, atol=1e-8), n


def test_layer_rejects_non_64_heads_and_blocks():
    with pytest.raises(ValueError):
        BigBirdSelfAttention(100, 2)
    with pytest.raises(ValueError):
        BigBirdSelfAttention(128, 2, block=96)


@pytest.mark.gpu
@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
def test_layer_equals_its_steps_spelled_out():
    B, H, L = 2, 4, 64 * 24
    dev = torch.device("cuda")
    torch.manual_seed(1)
    mod = BigBirdSelfAttention(H * 64, H, window=1, num_global=2, num_random=2, seed=3).to(dev, torch.bfloat16)
    x = torch.randn(B, L, H * 64, device=dev).to(torch.bfloat16).requires_grad_(True)
    km = torch.ones(B, L, dtype=torch.uint8, device=dev)
    km[1, -40:] = 0
    y = mod(x, key_mask=km)
    # the same steps with the binding
    lay = bsa.bsa_layout_build(H, L, 64, 1, 2, 2, 3)
    bsa.bsa_layout_upload(lay)
    q, k, v = F.linear(x.detach(), mod.qkv.weight, mod.qkv.bias).view(B, L, 3, H, 64).permute(2, 0, 3, 1, 4).unbind(0)
    o, _ = bsa.bsa_forward(q.contiguous(), k.contiguous(), v.contiguous(), lay, key_mask=km)
    y2 = F.linear(o.transpose(1, 2).reshape(B, L, H * 64), mod.proj.weight, mod.proj.bias)
    err = (y.detach().float() - y2.float()).abs().max().item()
    assert err <= 1e-2 * y2.float().abs().max().item(), err
    y.float().square().sum().backward()
    assert bsa.bsa_sync_status() == 0
    for t in (x.grad, mod.qkv.weight.grad, mod.qkv.bias.grad, mod.proj.weight.grad):
        assert torch.isfinite(t.float()).all() and t.float().abs().sum() > 0


@pytest.mark.gpu
@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
def test_layer_on_gpu_matches_fp64_dense_layer():
    """The bf16 layer on the GPU (cuBLAS projections, the library's attention and
    gradients) against the same layer evaluated in fp64 on the CPU from the same
    bf16 weights and inputs: dense masked softmax over the oracle's layout, with
    torch autograd for the gradients.  The bf16 rounding of q, k, v, O and y costs
    about 0.4 % of the output's scale here; the bounds leave a 5x margin, while a
    wrong head split, q/k/v order or gradient routing is off by O(1)."""
    B, H, L = 2, 4, 64 * 24
    dev = torch.device("cuda")
    torch.manual_seed(1)
    mod = BigBirdSelfAttention(H * 64, H, window=1, num_global=2, num_random=2, seed=3).to(dev, torch.bfloat16)
    ref = BigBirdSelfAttention(H * 64, H).double()
    ref.load_state_dict({n: t.detach().cpu().double() for n, t in mod.state_dict().items()})
    x = torch.randn(B, L, H * 64).to(torch.bfloat16)
    km = torch.ones(B, L, dtype=torch.uint8)
    km[1, -40:] = 0
    xg = x.to(dev).requires_grad_(True)
    y = mod(xg, key_mask=km.to(dev))
    (y.float().square().sum() * 0.5).backward()
    assert bsa.bsa_sync_status() == 0
    lay = OL.build_layout(H, L, 64, 1, 2, 2, 3)
    xr = x.double().requires_grad_(True)
    y_ref = _dense_reference(ref, xr, lay, km.numpy())
    scale = y_ref.abs().max().item()
    err = (y.detach().cpu().double() - y_ref).abs().max().item()
    assert err <= 2e-2 * scale, (err, scale)
    # the loss gradient dy = y of each side's own output, so the checks below
    # also carry the forward's rounding
    y_ref.backward(y_ref.detach())
    for got, want, name in ((xg.grad, xr.grad, "x"),
                            (mod.qkv.weight.grad, ref.qkv.weight.grad, "qkv.weight"),
                            (mod.qkv.bias.grad, ref.qkv.bias.grad, "qkv.bias"),
                            (mod.proj.weight.grad, ref.proj.weight.grad, "proj.weight"),
                            (mod.proj.bias.grad, ref.proj.bias.grad, "proj.bias")):
        g = got.detach().cpu().double()
        assert torch.isfinite(g).all(), name
        m = want.abs().max().item()
        e = (g - want).abs().max().item()
        assert e <= 5e-2 * m, (name, e, m)
