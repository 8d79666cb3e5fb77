"""The layer's projection kernels (bsa_qkv_projection, bsa_out_projection).

CPU:
  - argument checks of the C ABI that return before any device work;
  - the fused layer's two autograd functions with the library calls replaced by
    fakes on the fp64 oracle: outputs and every gradient against torch autograd
    of the same layer spelled out (this pins the q/k/v order and the head
    merge of the hand-written backward formulas).
GPU: each kernel against the fp64 oracle on shapes with ragged row tiles
(L not a multiple of 128), partial column tiles (N not a multiple of 256,
N < 256), with and without bias; sampled rows at the long shape
(B=4, L=16384, 12 heads); bit-identical repeats; and the fused layer against the
fp64 dense layer.

Tolerance (from the arithmetic): the products of bf16 inputs are exact in fp32,
the K-term fp32 sum errs by at most K 2^-24 sum|terms| (the oracle's magnitude),
and the final rounding to bf16 by 2^-9 |result|; the bound used is
2^-8 |ref| + K 2^-23 magnitude.
"""

import ctypes

import numpy as np
import pytest
import torch

from block_sparse_attention_bigbird_b200 import bsa
from block_sparse_attention_bigbird_b200 import layer as LY
from oracle import projection as OP

gpu = [pytest.mark.gpu, pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


# ---------------------------------------------------------------- CPU
def test_abi_rejects_bad_arguments_before_device_work():
    fake = 1 << 20  # an aligned non-null pointer value that is never dereferenced
    out = bsa.lib.bsa_out_projection
    assert out(None, fake, None, 1, 1, 64, 64, fake, None) == bsa.BSA_ERR_INVALID_ARG
    assert out(fake, fake, None, 1, 1, 64, 100, fake, None) == bsa.BSA_ERR_INVALID_ARG  # N % 64
    assert out(fake, fake, None, 0, 1, 64, 64, fake, None) == bsa.BSA_ERR_INVALID_ARG
    assert out(fake + 8, fake, None, 1, 1, 64, 64, fake, None) == bsa.BSA_ERR_INVALID_ARG  # alignment
    qkv = bsa.lib.bsa_qkv_projection
    assert qkv(fake, fake, None, 1, 64, 0, fake, fake, fake, None) == bsa.BSA_ERR_INVALID_ARG
    assert qkv(fake, fake, None, 1, 0, 1, fake, fake, fake, None) == bsa.BSA_ERR_INVALID_ARG
    assert qkv(fake, fake, None, 1, 64, 1, fake, None, fake, None) == bsa.BSA_ERR_INVALID_ARG
    assert qkv(fake, fake, fake + 4, 1, 64, 1, fake, fake, fake, None) == bsa.BSA_ERR_INVALID_ARG


def test_fused_autograd_functions_with_fake_library(monkeypatch):
    def fake_qkv(x, w, b, H, q=None, k=None, v=None, stream=None):
        return tuple(torch.from_numpy(t.copy()) for t in OP.qkv_projection(x, w, b, H))

    def fake_out(o, w, b=None, y=None, stream=None):
        return torch.from_numpy(OP.out_projection(o, w, b))

    monkeypatch.setattr(bsa, "bsa_qkv_projection", fake_qkv)
    monkeypatch.setattr(bsa, "bsa_out_projection", fake_out)
    torch.manual_seed(3)
    B, L, H = 2, 5, 3
    C = 64 * H
    x = torch.randn(B, L, C, dtype=torch.float64, requires_grad=True)
    w = torch.randn(3 * C, C, dtype=torch.float64, requires_grad=True)
    b = torch.randn(3 * C, dtype=torch.float64, requires_grad=True)
    wo = torch.randn(C, C, dtype=torch.float64, requires_grad=True)
    bo = torch.randn(C, dtype=torch.float64, requires_grad=True)
    mix = torch.randn(3, dtype=torch.float64)

    def run(qkv_fn, out_fn):
        q, k, v = qkv_fn(x, w, b)
        o = (mix[0] * q + mix[1] * k * k + mix[2] * v.sin())  # touches q, k and v differently
        return out_fn(o, wo, bo)

    def ref_qkv(x_, w_, b_):
        y = torch.nn.functional.linear(x_, w_, b_).view(B, L, 3, H, 64).permute(2, 0, 3, 1, 4)
        return y[0], y[1], y[2]

    def ref_out(o, w_, b_):
        return torch.nn.functional.linear(o.transpose(1, 2).reshape(B, L, C), w_, b_)

    y = run(lambda *a: LY._QKVProjection.apply(*a, H), LY._OutProjection.apply)
    g = torch.randn_like(y)
    grads = torch.autograd.grad(y, (x, w, b, wo, bo), g)
    y_ref = run(ref_qkv, ref_out)
    grads_ref = torch.autograd.grad(y_ref, (x, w, b, wo, bo), g)
    assert torch.allclose(y, y_ref, rtol=0, atol=1e-10)
    for a, r in zip(grads, grads_ref):
        assert torch.allclose(a, r, rtol=1e-12, atol=1e-9)


# ---------------------------------------------------------------- GPU
def _bf16(rng, *shape, scale=1.0):
    return torch.from_numpy(rng.standard_normal(shape) * scale).to(torch.bfloat16)


def _assert_close(got, ref, mag, K):
    got = got.detach().float().cpu().double().numpy()
    tol = 2.0 ** -8 * np.abs(ref) + K * 2.0 ** -23 * mag
    bad = np.abs(got - ref) > tol
    assert not bad.any(), (np.abs(got - ref).max(), int(bad.sum()))


QKV_CASES = [(1, 64, 1, True), (2, 320, 3, True), (2, 256, 12, False), (3, 192, 2, True), (1, 1000, 5, False)]


@pytest.mark.parametrize("B,L,H,with_bias", QKV_CASES)
@pytest.mark.gpu
@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
def test_qkv_projection_matches_oracle(B, L, H, with_bias):
    rng = np.random.default_rng(100 + B * 7 + L + H)
    C = 64 * H
    x, w = _bf16(rng, B, L, C), _bf16(rng, 3 * C, C, scale=C ** -0.5)
    b = _bf16(rng, 3 * C) if with_bias else None
    dev = torch.device("cuda")
    q, k, v = bsa.bsa_qkv_projection(x.to(dev), w.to(dev), b.to(dev) if b is not None else None)
    assert bsa.bsa_sync_status() == 0
    refs = OP.qkv_projection(x, w, b, H)
    mags = OP.magnitude_qkv(x, w, b, H)
    for got, ref, mag in zip((q, k, v), refs, mags):
        assert tuple(got.shape) == (B, H, L, 64)
        _assert_close(got, ref, mag, C)


OUT_CASES = [(1, 1, 64, 64, True), (2, 3, 320, 192, True), (2, 12, 256, 768, False), (1, 2, 200, 576, True),
             (2, 4, 128, 1024, False)]


@pytest.mark.parametrize("B,H,L,N,with_bias", OUT_CASES)
@pytest.mark.gpu
@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
def test_out_projection_matches_oracle(B, H, L, N, with_bias):
    rng = np.random.default_rng(200 + B * 5 + H + L + N)
    o, w = _bf16(rng, B, H, L, 64), _bf16(rng, N, 64 * H, scale=(64 * H) ** -0.5)
    b = _bf16(rng, N) if with_bias else None
    dev = torch.device("cuda")
    y = bsa.bsa_out_projection(o.to(dev), w.to(dev), b.to(dev) if b is not None else None)
    assert bsa.bsa_sync_status() == 0
    assert tuple(y.shape) == (B, L, N)
    _assert_close(y, OP.out_projection(o, w, b), OP.magnitude_out(o, w, b), 64 * H)


@pytest.mark.gpu
@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
def test_projections_at_the_long_shape_on_sampled_rows_and_repeatable():
    B, L, H = 4, 16384, 12
    C = 64 * H
    rng = np.random.default_rng(7)
    dev = torch.device("cuda")
    x, w, b = _bf16(rng, B, L, C), _bf16(rng, 3 * C, C, scale=C ** -0.5), _bf16(rng, 3 * C)
    wo, bo = _bf16(rng, C, C, scale=C ** -0.5), _bf16(rng, C)
    xd, wd, bd, wod, bod = (t.to(dev) for t in (x, w, b, wo, bo))
    q, k, v = bsa.bsa_qkv_projection(xd, wd, bd)
    y = bsa.bsa_out_projection(v, wod, bod)
    q2, k2, v2 = bsa.bsa_qkv_projection(xd, wd, bd)
    y2 = bsa.bsa_out_projection(v2, wod, bod)
    assert bsa.bsa_sync_status() == 0
    for a, a2 in ((q, q2), (k, k2), (v, v2), (y, y2)):
        assert torch.equal(a, a2)
    # rows at both ends of every batch element, at tile edges and at random
    rows = sorted(set([0, 1, 127, 128, 255, L - 129, L - 128, L - 1] + list(rng.integers(0, L, 40))))
    xs = x[:, rows]  # [B, R, C]
    ref = OP.qkv_projection(xs, w, b, H)
    mag = OP.magnitude_qkv(xs, w, b, H)
    for got, r, m in zip((q, k, v), ref, mag):
        _assert_close(got[:, :, rows], r, m, C)
    vs = v[:, :, rows].cpu()  # the kernel's own v rows are the output projection's input
    _assert_close(y[:, rows], OP.out_projection(vs, wo, bo), OP.magnitude_out(vs, wo, bo), C)


@pytest.mark.gpu
@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
def test_fused_layer_matches_fp64_dense_layer():
    """The fused bf16 layer (library projections and attention) against the layer
    in fp64 from the same bf16 weights and inputs, outputs and gradients, at the
    bounds of the unfused layer's test (bf16 rounding of q, k, v, O and y costs
    about 0.4 % of the output's scale)."""
    import test_layer as TL
    from oracle import layout as OL
    B, H, L = 2, 4, 64 * 24
    dev = torch.device("cuda")
    torch.manual_seed(1)
    mod = LY.BigBirdSelfAttention(H * 64, H, window=1, num_global=2, num_random=2, seed=3,
                                  fused=True).to(dev, torch.bfloat16)
    ref = LY.BigBirdSelfAttention(H * 64, H).double()
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
    y_ref = TL._dense_reference(ref, xr, lay, km.numpy())
    scale = y_ref.abs().max().item()
    err = (y.detach().cpu().double() - y_ref).abs().max().item()
    assert err <= 2e-2 * scale, (err, scale)
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
