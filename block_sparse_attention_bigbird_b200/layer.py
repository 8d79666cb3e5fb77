"""BigBird self-attention layer: QKV projection, block-sparse attention, output
projection.

The layer the pages build around the attention: one linear map of the hidden
states to q, k, v ("BigBird 稀疏注意力机制解析", 代码实现: ``self.qkv =
nn.Linear(dim, dim * 3)``, split into heads), the attention over the BigBird
layout, and an output projection ("BERT 稀疏注意力机制入门指南", PyTorch 实现:
``self.proj = nn.Linear(dim, dim)``).  The two projections are plain dense GEMMs
(torch, i.e. cuBLAS) by default; the attention and its gradients are the
library's kernels through ``block_sparse_attention``.

With ``fused=True`` (bf16 on an sm_100 device) the forward runs the library's
own projection kernels instead, with the head split and merge inside them:
``bsa_qkv_projection`` writes q, k and v straight into the attention's
[B, H, L, 64] layout, and ``bsa_out_projection`` reads the attention output in
that layout through its tile loads.  So the layer's forward is three library
kernels (four with the split-row merge) and no transposes.  The projections'
gradients are plain GEMMs in torch.
"""

from __future__ import annotations

from typing import Optional

import torch

from . import bsa
from .autograd import block_sparse_attention


class _QKVProjection(torch.autograd.Function):
    """q, k, v = heads of x W^T + b by the library kernel; gradients by torch GEMMs."""

    @staticmethod
    def forward(ctx, x, weight, bias, num_heads):
        x, weight = x.contiguous(), weight.contiguous()
        q, k, v = bsa.bsa_qkv_projection(x, weight, bias.contiguous() if bias is not None else None, num_heads)
        ctx.save_for_backward(x, weight)
        ctx.has_bias = bias is not None
        return q, k, v

    @staticmethod
    def backward(ctx, dq, dk, dv):
        x, weight = ctx.saved_tensors
        B, L, C = x.shape
        H = C // 64
        grads = [torch.zeros((B, H, L, 64), dtype=x.dtype, device=x.device) if g is None else g
                 for g in (dq, dk, dv)]
        # the projection's output gradient [B, L, 3C]: the heads merged back in q, k, v order
        dy = torch.stack(grads, 0).permute(1, 3, 0, 2, 4).reshape(B, L, 3 * C)
        dx = dy @ weight
        dw = dy.reshape(-1, 3 * C).t() @ x.reshape(-1, C)
        db = dy.sum((0, 1)) if ctx.has_bias else None
        return dx, dw, db, None


class _OutProjection(torch.autograd.Function):
    """y = merge_heads(o) W^T + b by the library kernel; gradients by torch GEMMs."""

    @staticmethod
    def forward(ctx, o, weight, bias):
        o, weight = o.contiguous(), weight.contiguous()
        y = bsa.bsa_out_projection(o, weight, bias.contiguous() if bias is not None else None)
        ctx.save_for_backward(o, weight)
        ctx.has_bias = bias is not None
        return y

    @staticmethod
    def backward(ctx, dy):
        o, weight = ctx.saved_tensors
        B, H, L, d = o.shape
        N = weight.shape[0]
        dy = dy.contiguous()
        do = (dy @ weight).view(B, L, H, d).permute(0, 2, 1, 3).contiguous()
        dw = dy.reshape(-1, N).t() @ o.permute(0, 2, 1, 3).reshape(-1, H * d)
        db = dy.sum((0, 1)) if ctx.has_bias else None
        return do, dw, db


class BigBirdSelfAttention(torch.nn.Module):
    """x [B, L, dim] -> [B, L, dim] with ``num_heads`` heads of 64.

    block (a multiple of 64), window, num_global, num_random and seed define the
    BigBird layout of each sequence length (see bsa_layout_build); it is built
    and uploaded on first use per (length, device).  ``key_mask`` in forward is
    uint8 [B, L], 1 = keep.  ``fused``: run the projections with the library's
    kernels (bf16 CUDA inputs and parameters only).
    """

    HEAD_DIM = 64

    def __init__(self, dim: int, num_heads: int, window: int = 1, num_global: int = 2, num_random: int = 3,
                 seed: int = 0, bias: bool = True, out_proj: bool = True, block: int = 64, fused: bool = False):
        super().__init__()
        if dim != num_heads * self.HEAD_DIM:
            raise ValueError(f"dim must be num_heads * {self.HEAD_DIM}")
        if block < 64 or block % 64:
            raise ValueError("block must be a multiple of 64")
        self.num_heads, self.block, self.fused = num_heads, block, fused
        self.window, self.num_global, self.num_random, self.seed = window, num_global, num_random, seed
        self.qkv = torch.nn.Linear(dim, 3 * dim, bias=bias)
        self.proj = torch.nn.Linear(dim, dim, bias=bias) if out_proj else None
        self._layouts = {}

    def layout(self, L: int, device: torch.device) -> "bsa.Layout":
        key = (L, str(device))
        lay = self._layouts.get(key)
        if lay is None:
            lay = bsa.bsa_layout_build(self.num_heads, L, self.block, self.window, self.num_global,
                                       self.num_random, self.seed)
            bsa.bsa_layout_upload(lay)
            self._layouts[key] = lay
        return lay

    def forward(self, x: torch.Tensor, key_mask: Optional[torch.Tensor] = None) -> torch.Tensor:
        B, L, C = x.shape
        H, d = self.num_heads, self.HEAD_DIM
        if self.fused:
            if x.dtype != torch.bfloat16 or not x.is_cuda or self.qkv.weight.dtype != torch.bfloat16:
                raise ValueError("the fused layer takes bf16 CUDA inputs and parameters")
            q, k, v = _QKVProjection.apply(x, self.qkv.weight, self.qkv.bias, H)
            o = block_sparse_attention(q, k, v, self.layout(L, x.device), key_mask=key_mask)
            if self.proj is None:
                return o.transpose(1, 2).reshape(B, L, C)
            return _OutProjection.apply(o, self.proj.weight, self.proj.bias)
        # [B, L, 3C] -> three [B, H, L, d] contiguous tensors
        q, k, v = self.qkv(x).view(B, L, 3, H, d).permute(2, 0, 3, 1, 4).unbind(0)
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        o = block_sparse_attention(q, k, v, self.layout(L, x.device), key_mask=key_mask)
        o = o.transpose(1, 2).reshape(B, L, C)
        return self.proj(o) if self.proj is not None else o
