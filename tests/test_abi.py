"""The C-ABI library loads, exports every declared symbol, and rejects bad
arguments with status codes before touching a GPU (runs without one)."""

import ctypes
import subprocess

import pytest

from block_sparse_attention_bigbird_b200 import bsa


def test_exports_every_header_symbol():
    names = bsa.header_symbols()
    assert "bsa_forward" in names and "bsa_layout_build" in names and len(names) >= 10
    for n in names:
        assert hasattr(bsa.lib, n), n
    dyn = subprocess.run(["nm", "-D", "--defined-only", bsa.LIB_PATH], capture_output=True,
                         text=True).stdout
    for n in names:
        assert f" T {n}\n" in dyn, n


def test_binding_constants_match_header():
    import os
    import re
    hdr = open(os.path.join(os.path.dirname(bsa.LIB_PATH), "..", "include", "bsa.h")).read()
    defs = dict(re.findall(r"#define (BSA_\w+) \(?(\d+)u?", hdr))
    assert int(defs["BSA_SPLIT_THRESHOLD"]) == bsa.SPLIT_THRESHOLD
    m = re.search(r"#define BSA_STATIC_WORKSPACE_BYTES \((\d+)u \* (\d+)u \* (\d+)u\)", hdr)
    assert int(m.group(1)) * int(m.group(2)) * int(m.group(3)) == bsa.STATIC_WORKSPACE_BYTES


def test_strerror_covers_codes():
    for code in range(0, -8, -1):
        assert bsa.bsa_strerror(code) != "unknown status"
    assert bsa.bsa_strerror(-99) == "unknown status"


@pytest.mark.parametrize("args,code", [
    (dict(H=0, L=512), bsa.BSA_ERR_INVALID_ARG),
    (dict(H=1, L=500), bsa.BSA_ERR_INVALID_ARG),
    (dict(H=1, L=512, block=32), bsa.BSA_ERR_UNSUPPORTED),
    (dict(H=1, L=512, window=-1), bsa.BSA_ERR_INVALID_ARG),
    (dict(H=1, L=512, n_random=-2), bsa.BSA_ERR_INVALID_ARG),
    (dict(H=1, L=512, globals=[0, 8]), bsa.BSA_ERR_INVALID_ARG),
])
def test_layout_build_rejects(args, code):
    with pytest.raises(bsa.BsaError) as e:
        bsa.bsa_layout_build(**args)
    assert e.value.code == code


def test_layout_build_null_out():
    assert bsa.lib.bsa_layout_build(1, 512, 64, 1, 1, 1, 0, None, None) == bsa.BSA_ERR_INVALID_ARG


def _fwd(layout, **kw):
    lay = layout
    a = dict(q=1 << 12, k=1 << 12, v=1 << 12, B=1, H=lay.H, L=lay.L, d=64, key_mask=None, scale=0.0,
             out=1 << 12, lse=1 << 12, ws=1 << 12, ws_bytes=1 << 30)
    a.update(kw)
    return bsa.lib.bsa_forward(a["q"], a["k"], a["v"], a["B"], a["H"], a["L"], a["d"],
                               lay.handle if a.get("use_layout", True) else None, a["key_mask"],
                               ctypes.c_float(a["scale"]), a["out"], a["lse"], a["ws"], a["ws_bytes"],
                               None)


def test_forward_argument_errors_before_any_launch():
    lay = bsa.bsa_layout_build(2, 512, 64, 1, 1, 1, 0)
    assert _fwd(lay, q=None) == bsa.BSA_ERR_INVALID_ARG
    assert _fwd(lay, out=None) == bsa.BSA_ERR_INVALID_ARG
    assert _fwd(lay, lse=None) == bsa.BSA_ERR_INVALID_ARG
    assert _fwd(lay, use_layout=False) == bsa.BSA_ERR_INVALID_ARG
    assert _fwd(lay, B=0) == bsa.BSA_ERR_INVALID_ARG
    assert _fwd(lay, d=96) == bsa.BSA_ERR_UNSUPPORTED  # the forward takes d = 64 or 128
    assert _fwd(lay, d=32) == bsa.BSA_ERR_UNSUPPORTED
    assert _fwd(lay, H=3) == bsa.BSA_ERR_LAYOUT_MISMATCH
    assert _fwd(lay, L=1024) == bsa.BSA_ERR_LAYOUT_MISMATCH
    assert _fwd(lay, q=(1 << 12) + 2) == bsa.BSA_ERR_INVALID_ARG          # misaligned
    assert _fwd(lay, scale=float("nan")) == bsa.BSA_ERR_INVALID_ARG
    assert _fwd(lay, ws=None) == bsa.BSA_ERR_WORKSPACE
    assert _fwd(lay, ws=(1 << 12) + 64) == bsa.BSA_ERR_WORKSPACE          # not 256-aligned
    assert _fwd(lay, ws_bytes=16) == bsa.BSA_ERR_WORKSPACE
    assert _fwd(lay) == bsa.BSA_ERR_LAYOUT_MISMATCH                       # never uploaded


def test_workspace_bytes_grows_with_batch():
    lay = bsa.bsa_layout_build(12, 16384, 64, 2, 2, 3, 0)
    w1, w4 = bsa.bsa_workspace_bytes(lay, 1), bsa.bsa_workspace_bytes(lay, 4)
    assert w1 % 256 == 0 and w4 > w1
    with pytest.raises(bsa.BsaError):
        bsa.bsa_workspace_bytes(lay, 0)
