"""Thin ctypes binding of libbsa.so (the C ABI in include/bsa.h).

Argument marshalling only: every step of the forward runs in the library's
CUDA kernels.  PyTorch supplies device memory and the current stream.  If the
shared library is missing this module raises at import; there is no fallback.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libbsa.so")

BSA_OK = 0
BSA_ERR_INVALID_ARG = -1
BSA_ERR_UNSUPPORTED = -2
BSA_ERR_CUDA = -3
BSA_ERR_LAYOUT_MISMATCH = -4
BSA_ERR_DEVICE_TIMEOUT = -5
BSA_ERR_OOM = -6
BSA_ERR_WORKSPACE = -7
BSA_ERR_STATIC_WORKSPACE = -8
STATIC_WORKSPACE_BYTES = 32 * 1024 * 1024  # BSA_STATIC_WORKSPACE_BYTES in include/bsa.h
SPLIT_THRESHOLD = 48  # BSA_SPLIT_THRESHOLD in include/bsa.h: longer tile unions are split

# name -> (restype, argtypes); mirrors include/bsa.h
_SIGNATURES = {
    "bsa_layout_build": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                        ctypes.c_int, ctypes.c_int, ctypes.c_uint64,
                                        ctypes.POINTER(ctypes.c_int32),
                                        ctypes.POINTER(ctypes.c_void_p)]),
    "bsa_layout_build_tokens": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                               ctypes.c_int, ctypes.c_uint64, ctypes.POINTER(ctypes.c_int32),
                                               ctypes.POINTER(ctypes.c_void_p)]),
    "bsa_layout_token_masks": (ctypes.c_int, [ctypes.c_void_p, ctypes.POINTER(ctypes.c_int),
                                              ctypes.POINTER(ctypes.c_void_p)]),
    "bsa_layout_from_csr": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                           ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int32),
                                           ctypes.POINTER(ctypes.c_void_p)]),
    "bsa_layout_csr": (ctypes.c_int, [ctypes.c_void_p, ctypes.POINTER(ctypes.c_void_p),
                                      ctypes.POINTER(ctypes.c_void_p), ctypes.POINTER(ctypes.c_int64),
                                      ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)]),
    "bsa_layout_globals": (ctypes.c_int, [ctypes.c_void_p, ctypes.POINTER(ctypes.c_void_p),
                                          ctypes.POINTER(ctypes.c_int)]),
    "bsa_layout_tiles": (ctypes.c_int, [ctypes.c_void_p, ctypes.POINTER(ctypes.c_void_p),
                                        ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_void_p),
                                        ctypes.POINTER(ctypes.c_void_p), ctypes.POINTER(ctypes.c_int64)]),
    "bsa_layout_upload": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p]),
    "bsa_layout_free": (None, [ctypes.c_void_p]),
    "bsa_workspace_bytes": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int,
                                           ctypes.POINTER(ctypes.c_size_t)]),
    "bsa_forward_workspace_bytes": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                                                   ctypes.POINTER(ctypes.c_size_t)]),
    "bsa_forward": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                                   ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                                   ctypes.c_void_p, ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p,
                                   ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "bsa_forward_static_ws": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                                             ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                                             ctypes.c_void_p, ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p,
                                             ctypes.c_void_p]),
    "bsa_layout_key_tiles": (ctypes.c_int, [ctypes.c_void_p, ctypes.POINTER(ctypes.c_void_p),
                                            ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_void_p),
                                            ctypes.POINTER(ctypes.c_void_p), ctypes.POINTER(ctypes.c_int64)]),
    "bsa_backward_workspace_bytes": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int,
                                                    ctypes.POINTER(ctypes.c_size_t)]),
    "bsa_backward": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                    ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                    ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_float,
                                    ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                    ctypes.c_size_t, ctypes.c_void_p]),
    "bsa_qkv_projection": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                                          ctypes.c_void_p, ctypes.c_void_p]),
    "bsa_out_projection": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                                          ctypes.c_void_p]),
    "bsa_sync_status": (ctypes.c_int, [ctypes.c_void_p]),
    "bsa_strerror": (ctypes.c_char_p, [ctypes.c_int]),
    "bsa_debug_wait_timeout": (ctypes.c_int, [ctypes.c_uint64, ctypes.c_void_p]),
}


def _load() -> ctypes.CDLL:
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"{_LIB_PATH} is missing; build it with "
                          "`python -m block_sparse_attention_bigbird_b200.build`")
    lib = ctypes.CDLL(_LIB_PATH)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()
LIB_PATH = _LIB_PATH


class BsaError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {bsa_strerror(code)} ({code})")
        self.code = code


def bsa_strerror(code: int) -> str:
    return lib.bsa_strerror(int(code)).decode()


def _check(code: int, what: str) -> None:
    if code != BSA_OK:
        raise BsaError(code, what)


def _stream_ptr(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


class Layout:
    """Owner of a bsa_layout*; freed with the object."""

    def __init__(self, handle: int, H: int, L: int):
        self._h = ctypes.c_void_p(handle)
        self.H = H
        self.L = L
        self._workspaces = {}

    @property
    def handle(self) -> ctypes.c_void_p:
        return self._h

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value and lib is not None:   # lib is None at interpreter exit
            lib.bsa_layout_free(h)
            self._h = ctypes.c_void_p(0)


def bsa_layout_build(H: int, L: int, block: int = 64, window: int = 1, n_global: int = 2,
                     n_random: int = 3, seed: int = 0, globals=None) -> Layout:
    out = ctypes.c_void_p()
    gptr = None
    if globals is not None:
        g = np.ascontiguousarray(np.asarray(globals, dtype=np.int32))
        n_global = int(g.size)
        gptr = g.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    _check(lib.bsa_layout_build(H, L, block, window, n_global, n_random,
                                ctypes.c_uint64(seed & 0xFFFFFFFFFFFFFFFF), gptr, ctypes.byref(out)),
           "bsa_layout_build")
    return Layout(out.value, H, L)


def bsa_layout_build_tokens(H: int, L: int, window: int, n_global: int = 0, n_random: int = 0, seed: int = 0,
                            global_tokens=None) -> Layout:
    """A BigBird layout with its window and global set in tokens (see bsa.h)."""
    out = ctypes.c_void_p()
    gptr = None
    if global_tokens is not None:
        g = np.ascontiguousarray(np.asarray(global_tokens, dtype=np.int32))
        n_global = int(g.size)
        gptr = g.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    _check(lib.bsa_layout_build_tokens(H, L, window, n_global, n_random,
                                       ctypes.c_uint64(seed & 0xFFFFFFFFFFFFFFFF), gptr, ctypes.byref(out)),
           "bsa_layout_build_tokens")
    return Layout(out.value, H, L)


def bsa_layout_token_masks(layout: Layout):
    """(window in tokens, uint64 [L / 64] global-token bits) of a token-level layout."""
    w, gb = ctypes.c_int(), ctypes.c_void_p()
    _check(lib.bsa_layout_token_masks(layout.handle, ctypes.byref(w), ctypes.byref(gb)), "bsa_layout_token_masks")
    bits = np.ctypeslib.as_array(ctypes.cast(gb, ctypes.POINTER(ctypes.c_uint64)), (layout.L // 64,)).copy()
    return w.value, bits


def bsa_layout_from_csr(H: int, L: int, row_ptr, col_idx, block: int = 64) -> Layout:
    """Layout from a caller's block CSR (rows head-major; see bsa_layout_from_csr in bsa.h)."""
    rp = np.ascontiguousarray(np.asarray(row_ptr, dtype=np.int32))
    ci = np.ascontiguousarray(np.asarray(col_idx, dtype=np.int32))
    if rp.ndim != 1 or rp.size != H * (L // block if block > 0 else 0) + 1:
        raise BsaError(BSA_ERR_INVALID_ARG, "bsa_layout_from_csr: row_ptr must hold H * L / block + 1 entries")
    if int(rp[-1]) > ci.size:
        raise BsaError(BSA_ERR_INVALID_ARG, "bsa_layout_from_csr: col_idx is shorter than row_ptr[-1]")
    out = ctypes.c_void_p()
    cptr = ci.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)) if ci.size else None
    _check(lib.bsa_layout_from_csr(H, L, block, rp.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), cptr,
                                   ctypes.byref(out)), "bsa_layout_from_csr")
    return Layout(out.value, H, L)


def bsa_layout_csr(layout: Layout):
    """(row_ptr int32 [H*nb+1], col_idx int32 [nnz]) as numpy copies."""
    rp, ci = ctypes.c_void_p(), ctypes.c_void_p()
    nnz, nb, H = ctypes.c_int64(), ctypes.c_int(), ctypes.c_int()
    _check(lib.bsa_layout_csr(layout.handle, ctypes.byref(rp), ctypes.byref(ci), ctypes.byref(nnz),
                              ctypes.byref(nb), ctypes.byref(H)), "bsa_layout_csr")
    n_rows = H.value * nb.value + 1
    row_ptr = np.ctypeslib.as_array(ctypes.cast(rp, ctypes.POINTER(ctypes.c_int32)), (n_rows,)).copy()
    col_idx = (np.ctypeslib.as_array(ctypes.cast(ci, ctypes.POINTER(ctypes.c_int32)), (nnz.value,)).copy()
               if nnz.value else np.zeros(0, np.int32))
    return row_ptr, col_idx


def bsa_layout_globals(layout: Layout) -> np.ndarray:
    gp, n = ctypes.c_void_p(), ctypes.c_int()
    _check(lib.bsa_layout_globals(layout.handle, ctypes.byref(gp), ctypes.byref(n)), "bsa_layout_globals")
    if n.value == 0:
        return np.zeros(0, np.int32)
    return np.ctypeslib.as_array(ctypes.cast(gp, ctypes.POINTER(ctypes.c_int32)), (n.value,)).copy()


def bsa_layout_tiles(layout: Layout):
    """(pair_q [n_pairs, 2], pair_ptr [H*n_pairs+1], pair_ent [n_ent] uint32) as numpy copies."""
    pq, pp, pe = ctypes.c_void_p(), ctypes.c_void_p(), ctypes.c_void_p()
    n_pairs, n_ent = ctypes.c_int(), ctypes.c_int64()
    _check(lib.bsa_layout_tiles(layout.handle, ctypes.byref(pq), ctypes.byref(n_pairs), ctypes.byref(pp),
                                ctypes.byref(pe), ctypes.byref(n_ent)), "bsa_layout_tiles")
    P = n_pairs.value
    pair_q = np.ctypeslib.as_array(ctypes.cast(pq, ctypes.POINTER(ctypes.c_int32)), (2 * P,)).copy()
    pair_ptr = np.ctypeslib.as_array(ctypes.cast(pp, ctypes.POINTER(ctypes.c_int32)),
                                     (layout.H * P + 1,)).copy()
    pair_ent = np.ctypeslib.as_array(ctypes.cast(pe, ctypes.POINTER(ctypes.c_uint32)), (n_ent.value,)).copy()
    return pair_q.reshape(P, 2), pair_ptr, pair_ent


def bsa_layout_key_tiles(layout: Layout):
    """(pair_k [n_pairs, 2], pair_ptr [H*n_pairs+1], pair_ent [n_ent] uint32) of the key-major tiles."""
    pq, pp, pe = ctypes.c_void_p(), ctypes.c_void_p(), ctypes.c_void_p()
    n_pairs, n_ent = ctypes.c_int(), ctypes.c_int64()
    _check(lib.bsa_layout_key_tiles(layout.handle, ctypes.byref(pq), ctypes.byref(n_pairs), ctypes.byref(pp),
                                    ctypes.byref(pe), ctypes.byref(n_ent)), "bsa_layout_key_tiles")
    P = n_pairs.value
    pair_k = np.ctypeslib.as_array(ctypes.cast(pq, ctypes.POINTER(ctypes.c_int32)), (2 * P,)).copy()
    pair_ptr = np.ctypeslib.as_array(ctypes.cast(pp, ctypes.POINTER(ctypes.c_int32)),
                                     (layout.H * P + 1,)).copy()
    pair_ent = np.ctypeslib.as_array(ctypes.cast(pe, ctypes.POINTER(ctypes.c_uint32)), (n_ent.value,)).copy()
    return pair_k.reshape(P, 2), pair_ptr, pair_ent


def bsa_layout_upload(layout: Layout, stream=None) -> None:
    _check(lib.bsa_layout_upload(layout.handle, ctypes.c_void_p(_stream_ptr(stream))), "bsa_layout_upload")
    layout._workspaces.clear()


def bsa_workspace_bytes(layout: Layout, B: int) -> int:
    n = ctypes.c_size_t()
    _check(lib.bsa_workspace_bytes(layout.handle, B, ctypes.byref(n)), "bsa_workspace_bytes")
    return n.value


def bsa_forward_workspace_bytes(layout: Layout, B: int, d: int) -> int:
    n = ctypes.c_size_t()
    _check(lib.bsa_forward_workspace_bytes(layout.handle, B, d, ctypes.byref(n)), "bsa_forward_workspace_bytes")
    return n.value


def _workspace(layout: Layout, B: int, device, d: int = 64):
    import torch
    key = (str(device), B, d)
    ws = layout._workspaces.get(key)
    if ws is None:
        ws = torch.empty(bsa_forward_workspace_bytes(layout, B, d), dtype=torch.uint8, device=device)
        layout._workspaces[key] = ws
    return ws


def bsa_forward(q, k, v, layout: Layout, key_mask=None, scale: Optional[float] = None, out=None,
                lse=None, workspace=None, stream=None):
    """O (bf16 [B,H,L,d]) and lse (fp32 [B,H,L]) of the block-sparse attention.

    q, k, v: contiguous bf16 CUDA tensors [B, H, L, d], d = 64 or 128.  key_mask: optional
    uint8 CUDA tensor [B, L] (1 = keep).  workspace: optional uint8 CUDA tensor
    of at least bsa_workspace_bytes(layout, B) bytes, any contents; when
    omitted a cached one of the layout is used (not safe for concurrent calls
    on different streams with the same layout).
    """
    import torch
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous() or t.dim() != 4:
            raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor [B, H, L, d]")
    if q.shape != k.shape or q.shape != v.shape:
        raise ValueError("q, k, v shapes differ")
    B, H, L, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, L), dtype=torch.float32, device=q.device)
    if key_mask is not None:
        if key_mask.dtype != torch.uint8 or tuple(key_mask.shape) != (B, L) or not key_mask.is_contiguous():
            raise ValueError("key_mask must be a contiguous uint8 tensor [B, L]")
    if workspace is None:
        workspace = _workspace(layout, B, q.device, d)
    code = lib.bsa_forward(q.data_ptr(), k.data_ptr(), v.data_ptr(), B, H, L, d, layout.handle,
                           key_mask.data_ptr() if key_mask is not None else None,
                           ctypes.c_float(scale if scale is not None else 0.0), out.data_ptr(),
                           lse.data_ptr(), workspace.data_ptr(), workspace.numel(),
                           ctypes.c_void_p(_stream_ptr(stream)))
    _check(code, "bsa_forward")
    return out, lse


def bsa_forward_static_ws(q, k, v, layout: Layout, key_mask=None, scale: Optional[float] = None,
                          out=None, lse=None, stream=None):
    """bsa_forward for callers that cannot allocate device memory.

    The library's built-in scratch buffer (STATIC_WORKSPACE_BYTES per device)
    replaces the workspace; nothing is allocated by the call itself (``out`` and
    ``lse`` must then be given by such a caller).  Calls on one device share that
    buffer: serialise them.  Raises BsaError(BSA_ERR_STATIC_WORKSPACE) when the
    problem needs more scratch than the buffer holds.
    """
    import torch
    B, H, L, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, L), dtype=torch.float32, device=q.device)
    code = lib.bsa_forward_static_ws(q.data_ptr(), k.data_ptr(), v.data_ptr(), B, H, L, d, layout.handle,
                                     key_mask.data_ptr() if key_mask is not None else None,
                                     ctypes.c_float(scale if scale is not None else 0.0), out.data_ptr(),
                                     lse.data_ptr(), ctypes.c_void_p(_stream_ptr(stream)))
    _check(code, "bsa_forward_static_ws")
    return out, lse


def bsa_backward_workspace_bytes(layout: Layout, B: int) -> int:
    n = ctypes.c_size_t()
    _check(lib.bsa_backward_workspace_bytes(layout.handle, B, ctypes.byref(n)), "bsa_backward_workspace_bytes")
    return n.value


def bsa_backward(q, k, v, out, dout, lse, layout: Layout, key_mask=None, scale: Optional[float] = None,
                 dq=None, dk=None, dv=None, workspace=None, stream=None):
    """dq, dk, dv (bf16 [B,H,L,64]) of the block-sparse attention for dL/dO = ``dout``.

    q, k, v, out, dout: contiguous bf16 CUDA tensors [B, H, L, 64]; out and lse
    (fp32 [B, H, L]) are the forward's results for the same inputs, layout,
    key_mask and scale.  workspace: optional uint8 CUDA tensor of at least
    bsa_backward_workspace_bytes(layout, B) bytes (no clearing needed); when
    omitted a cached one of the layout is used.
    """
    import torch
    for name, t in (("q", q), ("k", k), ("v", v), ("out", out), ("dout", dout)):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous() or t.dim() != 4:
            raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor [B, H, L, d]")
        if t.shape != q.shape:
            raise ValueError(f"{name} shape differs from q")
    B, H, L, d = q.shape
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, L) or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous fp32 tensor [B, H, L]")
    if key_mask is not None:
        if key_mask.dtype != torch.uint8 or tuple(key_mask.shape) != (B, L) or not key_mask.is_contiguous():
            raise ValueError("key_mask must be a contiguous uint8 tensor [B, L]")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if workspace is None:
        key = ("bwd", str(q.device), B)
        workspace = layout._workspaces.get(key)
        if workspace is None:
            workspace = torch.empty(bsa_backward_workspace_bytes(layout, B), dtype=torch.uint8, device=q.device)
            layout._workspaces[key] = workspace
    code = lib.bsa_backward(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), dout.data_ptr(),
                            lse.data_ptr(), B, H, L, d, layout.handle,
                            key_mask.data_ptr() if key_mask is not None else None,
                            ctypes.c_float(scale if scale is not None else 0.0), dq.data_ptr(), dk.data_ptr(),
                            dv.data_ptr(), workspace.data_ptr(), workspace.numel(),
                            ctypes.c_void_p(_stream_ptr(stream)))
    _check(code, "bsa_backward")
    return dq, dk, dv


def _check_bf16(name, t, dim):
    import torch
    if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous() or t.dim() != dim:
        raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor of {dim} dimensions")


def bsa_qkv_projection(x, weight, bias=None, num_heads: Optional[int] = None, q=None, k=None, v=None,
                       stream=None):
    """q, k, v = the heads of x W^T + bias, each bf16 [B, H, L, 64].

    x: bf16 [B, L, C] with C = 64 H; weight: bf16 [3C, C] (rows: the q features,
    then k, then v; within each, head h's 64 features at 64 h); bias: bf16 [3C]
    or None.  The library's tcgen05 GEMM writes the three outputs in the head
    layout directly.
    """
    import torch
    _check_bf16("x", x, 3)
    _check_bf16("weight", weight, 2)
    B, L, C = x.shape
    H = num_heads if num_heads is not None else C // 64
    if C != 64 * H or tuple(weight.shape) != (3 * C, C):
        raise ValueError("x must be [B, L, 64 H] and weight [3 C, C]")
    if bias is not None:
        _check_bf16("bias", bias, 1)
        if bias.numel() != 3 * C:
            raise ValueError("bias must have 3 C elements")
    outs = []
    for t in (q, k, v):
        outs.append(torch.empty((B, H, L, 64), dtype=torch.bfloat16, device=x.device) if t is None else t)
    code = lib.bsa_qkv_projection(x.data_ptr(), weight.data_ptr(), bias.data_ptr() if bias is not None else None,
                                  B, L, H, outs[0].data_ptr(), outs[1].data_ptr(), outs[2].data_ptr(),
                                  ctypes.c_void_p(_stream_ptr(stream)))
    _check(code, "bsa_qkv_projection")
    return tuple(outs)


def bsa_out_projection(o, weight, bias=None, y=None, stream=None):
    """y = merge_heads(o) W^T + bias, bf16 [B, L, N].

    o: bf16 [B, H, L, 64] (the attention output); weight: bf16 [N, 64 H] with N
    a multiple of 64; bias: bf16 [N] or None.  The heads are merged by the
    GEMM's own tile loads.
    """
    import torch
    _check_bf16("o", o, 4)
    _check_bf16("weight", weight, 2)
    B, H, L, d = o.shape
    N = weight.shape[0]
    if d != 64 or weight.shape[1] != 64 * H:
        raise ValueError("o must be [B, H, L, 64] and weight [N, 64 H]")
    if bias is not None:
        _check_bf16("bias", bias, 1)
        if bias.numel() != N:
            raise ValueError("bias must have N elements")
    if y is None:
        y = torch.empty((B, L, N), dtype=torch.bfloat16, device=o.device)
    code = lib.bsa_out_projection(o.data_ptr(), weight.data_ptr(), bias.data_ptr() if bias is not None else None,
                                  B, H, L, N, y.data_ptr(), ctypes.c_void_p(_stream_ptr(stream)))
    _check(code, "bsa_out_projection")
    return y


def bsa_sync_status(stream=None) -> int:
    """Synchronises the stream; returns (and clears) the device status word."""
    return lib.bsa_sync_status(ctypes.c_void_p(_stream_ptr(stream)))


def bsa_debug_wait_timeout(timeout_ns: int, stream=None) -> None:
    _check(lib.bsa_debug_wait_timeout(ctypes.c_uint64(timeout_ns), ctypes.c_void_p(_stream_ptr(stream))),
           "bsa_debug_wait_timeout")


def header_symbols() -> list[str]:
    """Function names declared in include/bsa.h (parsed from the header text)."""
    import re
    hdr = os.path.join(os.path.dirname(os.path.dirname(_LIB_PATH)), "include", "bsa.h")
    with open(hdr) as f:
        text = f.read()
    return sorted(set(re.findall(r"^\s*(?:int|void|const char\*)\s+(bsa_\w+)\s*\(", text, re.M)))
