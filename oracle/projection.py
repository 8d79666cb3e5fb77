"""Oracle of the layer's two projections in fp64 (numpy).  TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import this module.  It shares no code with the CUDA library.

Definitions followed:
  [BigBird] "BigBird 稀疏注意力机制解析", 代码实现 -- the module maps the hidden
      states with one linear layer ``self.qkv = nn.Linear(dim, dim * 3)`` and
      splits the result into q, k and v and then into heads.
  [Primer] "BERT 稀疏注意力机制入门指南", PyTorch 实现 -- after the attention the
      heads are concatenated and mapped by ``self.proj = nn.Linear(dim, dim)``.

Reading: a linear layer computes y = x W^T + b with W stored [out, in].  The
3·dim outputs of the QKV layer are read as three consecutive groups of dim
(q, then k, then v), each of H consecutive heads of 64 features, which is the
split the BigBird module's reshape to (3, heads, head_dim) makes.  Merging the
heads is its inverse: feature 64 h + j of a token is O[b, h, l, j].
"""

from __future__ import annotations

import numpy as np

HEAD_DIM = 64


def _as_f64(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def linear(x, w, b=None) -> np.ndarray:
    """y = x W^T + b over the last axis of x ([BigBird] / [Primer]: nn.Linear)."""
    y = _as_f64(x) @ _as_f64(w).T
    if b is not None:
        y = y + _as_f64(b)
    return y


def split_heads(y: np.ndarray, H: int):
    """[B, L, 3·64H] -> q, k, v each [B, H, L, 64] ([BigBird]: reshape to (3, heads, 64))."""
    B, L, F = y.shape
    assert F == 3 * H * HEAD_DIM
    t = y.reshape(B, L, 3, H, HEAD_DIM).transpose(2, 0, 3, 1, 4)
    return t[0], t[1], t[2]


def merge_heads(o) -> np.ndarray:
    """[B, H, L, 64] -> [B, L, 64H]: feature 64 h + j is head h's j ([Primer]: concatenation)."""
    o = _as_f64(o)
    B, H, L, d = o.shape
    return o.transpose(0, 2, 1, 3).reshape(B, L, H * d)


def qkv_projection(x, w, b, H: int):
    """q, k, v [B, H, L, 64] of the QKV layer applied to x [B, L, 64H]."""
    return split_heads(linear(x, w, b), H)


def out_projection(o, w, b=None) -> np.ndarray:
    """y [B, L, N] = merge_heads(o) W^T + b."""
    return linear(merge_heads(o), w, b)


def magnitude_qkv(x, w, b, H: int):
    """Per output element, sum of |x_c w_c| + |b|: the scale of its rounding error."""
    return split_heads(linear(np.abs(_as_f64(x)), np.abs(_as_f64(w)), None if b is None else np.abs(_as_f64(b))), H)


def magnitude_out(o, w, b=None) -> np.ndarray:
    """The same for the output projection."""
    return linear(np.abs(merge_heads(o)), np.abs(_as_f64(w)), None if b is None else np.abs(_as_f64(b)))
