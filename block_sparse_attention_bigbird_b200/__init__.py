"""BigBird block-sparse attention for B200 (sm_100a): forward and gradients.

The compute lives in libbsa.so (C ABI, include/bsa.h); ``bsa`` is its thin
ctypes binding and ``autograd.block_sparse_attention`` its torch.autograd form.
Attributes are resolved lazily so that the build module can be imported before
the library exists; any other attribute access loads the library and fails
loudly if it is missing.
"""

from __future__ import annotations

import importlib

__all__ = ["bsa_layout_build", "bsa_layout_from_csr", "bsa_layout_csr", "bsa_layout_globals",
           "bsa_layout_tiles", "bsa_layout_key_tiles", "bsa_layout_upload", "bsa_workspace_bytes",
           "bsa_forward", "bsa_backward", "bsa_backward_workspace_bytes", "bsa_sync_status",
           "bsa_strerror", "bsa_debug_wait_timeout", "bsa_forward_static_ws", "Layout", "BsaError",
           "block_sparse_attention", "BigBirdSelfAttention"]


def __getattr__(name):
    if name == "block_sparse_attention":
        return getattr(importlib.import_module(".autograd", __name__), name)
    if name == "BigBirdSelfAttention":
        return getattr(importlib.import_module(".layer", __name__), name)
    if name in __all__:
        return getattr(importlib.import_module(".bsa", __name__), name)
    raise AttributeError(name)
