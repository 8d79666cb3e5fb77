"""BigBird self-attention layer: QKV projection, block-sparse attention, output
projection.

The layer the pages build around the attention: one linear map of the hidden
states to q, k, v ("BigBird 稀疏注意力机制解析", 代码实现: ``self.qkv =
nn.Linear(dim, dim * 3)``, split into heads), the attention over the BigBird
layout, and an output projection ("BERT 稀疏注意力机制入门指南", PyTorch 实现:
``self.proj = nn.Linear(dim, dim)``).  The two projections are plain dense GEMMs
(torch, i.e. cuBLAS); the attention and its gradients are the library's kernels
through ``block_sparse_attention``.  The projections are not fused into the
attention kernels.
"""

from __future__ import annotations

from typing import Optional

import torch

from . import bsa
from .autograd import block_sparse_attention


class BigBirdSelfAttention(torch.nn.Module):
    """x [B, L, dim] -> [B, L, dim] with ``num_heads`` heads of 64.

    block (a multiple of 64), window, num_global, num_random and seed define the
    BigBird layout of each sequence length (see bsa_layout_build); it is built
    and uploaded on first use per (length, device).  ``key_mask`` in forward is
    uint8 [B, L], 1 = keep.
    """

    HEAD_DIM = 64

    def __init__(self, dim: int, num_heads: int, window: int = 1, num_global: int = 2, num_random: int = 3,
                 seed: int = 0, bias: bool = True, out_proj: bool = True, block: int = 64):
        super().__init__()
        if dim != num_heads * self.HEAD_DIM:
            raise ValueError(f"dim must be num_heads * {self.HEAD_DIM}")
        if block < 64 or block % 64:
            raise ValueError("block must be a multiple of 64")
        self.num_heads, self.block = num_heads, block
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
        # [B, L, 3C] -> three [B, H, L, d] contiguous tensors
        q, k, v = self.qkv(x).view(B, L, 3, H, d).permute(2, 0, 3, 1, 4).unbind(0)
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        o = block_sparse_attention(q, k, v, self.layout(L, x.device), key_mask=key_mask)
        o = o.transpose(1, 2).reshape(B, L, C)
        return self.proj(o) if self.proj is not None else o
