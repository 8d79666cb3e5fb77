"""BigBird block-sparse attention forward for B200 (sm_100a).

The compute lives in libbsa.so (C ABI, include/bsa.h); ``bsa`` is its thin
ctypes binding.  Attributes are resolved lazily so that the build module can be
imported before the library exists; any other attribute access loads the
library and fails loudly if it is missing.
"""

from __future__ import annotations

import importlib

__all__ = ["bsa_layout_build", "bsa_layout_csr", "bsa_layout_globals", "bsa_layout_tiles",
           "bsa_layout_upload", "bsa_workspace_bytes", "bsa_forward", "bsa_sync_status",
           "bsa_strerror", "bsa_debug_wait_timeout", "bsa_forward_static_ws", "Layout", "BsaError"]


def __getattr__(name):
    if name in __all__:
        return getattr(importlib.import_module(".bsa", __name__), name)
    raise AttributeError(name)
