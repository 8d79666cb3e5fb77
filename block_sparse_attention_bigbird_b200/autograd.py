"""torch.autograd binding of the block-sparse attention.

``block_sparse_attention(q, k, v, layout)`` runs bsa_forward and records a node
whose backward runs bsa_backward, so the kernels take part in an ordinary
training step (the pages train BigBird-style models: "BERT 稀疏注意力机制入门指南",
生产环境部署建议; "BigBird 稀疏注意力机制解析", 避坑指南).  It is argument
marshalling only: both directions are the library's kernels.
"""

from __future__ import annotations

from typing import Optional

import torch

from . import bsa


class _BlockSparseAttention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, layout, key_mask, scale):
        out, lse = bsa.bsa_forward(q, k, v, layout, key_mask=key_mask, scale=scale)
        ctx.save_for_backward(q, k, v, out, lse, key_mask)
        ctx.layout = layout
        ctx.scale = scale
        ctx.mark_non_differentiable(lse)
        return out, lse

    @staticmethod
    def backward(ctx, dout, _dlse):
        q, k, v, out, lse, key_mask = ctx.saved_tensors
        dq, dk, dv = bsa.bsa_backward(q, k, v, out, dout.contiguous(), lse, ctx.layout, key_mask=key_mask,
                                      scale=ctx.scale)
        return dq, dk, dv, None, None, None


def block_sparse_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, layout: "bsa.Layout",
                           key_mask: Optional[torch.Tensor] = None, scale: Optional[float] = None,
                           return_lse: bool = False):
    """O = softmax(q k^T * scale restricted to the layout) v, differentiable in q, k, v.

    q, k, v: contiguous bf16 CUDA tensors [B, H, L, 64]; layout: an uploaded
    bsa.Layout for this H and L; key_mask: optional uint8 [B, L] (1 = keep);
    scale: None for 1/sqrt(64).  Returns O (bf16), and lse (fp32 [B, H, L], not
    differentiable) when ``return_lse``.
    """
    out, lse = _BlockSparseAttention.apply(q, k, v, layout, key_mask, scale)
    return (out, lse) if return_lse else out
