"""bsa_forward_static_ws: the forward for callers that cannot allocate device
memory (a host runtime that owns every allocation, a plugin without an
allocator hook, a path where cudaMalloc would synchronise the device).  It runs
the same kernel with the library's built-in scratch buffer instead of a
caller-provided workspace.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test.
"""

import ctypes

import numpy as np
import pytest
import torch

import workloads
from block_sparse_attention_bigbird_b200 import bsa

O_TOL = 2e-2
LSE_TOL = 1e-3


def test_static_entry_rejects_bad_arguments_without_a_gpu():
    lay = bsa.bsa_layout_build(2, 512, 64, 1, 1, 1, 0)
    fwd = bsa.lib.bsa_forward_static_ws
    a = 1 << 12
    assert fwd(None, a, a, 1, 2, 512, 64, lay.handle, None, ctypes.c_float(0), a, a, None) == bsa.BSA_ERR_INVALID_ARG
    assert fwd(a, a, a, 1, 2, 512, 96, lay.handle, None, ctypes.c_float(0), a, a, None) == bsa.BSA_ERR_UNSUPPORTED
    assert fwd(a, a, a, 1, 3, 512, 64, lay.handle, None, ctypes.c_float(0), a, a, None) == bsa.BSA_ERR_LAYOUT_MISMATCH


@pytest.mark.gpu
@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
def test_static_workspace_matches_workspace_forward_on_two_calls():
    # global rows split across chunks (partial records + merge) and partial key
    # padding (key bits): every region of the scratch buffer is exercised.  Both
    # entry points run the same kernels on the same schedule, and each output is
    # written by one fixed sequence of operations whatever CTA takes it, so the
    # results must be bit-identical; the first result is also checked against the
    # fp64 oracle.
    from oracle import attention as OA
    from oracle import layout as OL
    w = workloads.custom(2, 3, 64 * 64, 1, 2, 3, seed=1, key_pad_tail=100)
    qc, kc, vc = workloads.make_qkv(w)
    q, k, v = qc.cuda(), kc.cuda(), vc.cuda()
    kmc = workloads.make_key_mask(w)
    km = kmc.cuda()
    lay = bsa.bsa_layout_build(w.H, w.L, 64, w.window, w.n_global, w.n_random, w.seed)
    bsa.bsa_layout_upload(lay)
    assert 0 < bsa.bsa_workspace_bytes(lay, w.B) <= bsa.STATIC_WORKSPACE_BYTES
    o_ws, lse_ws = bsa.bsa_forward(q, k, v, lay, key_mask=km)
    assert bsa.bsa_sync_status() == 0
    for call in range(2):
        out = torch.empty_like(q)
        lse = torch.empty((w.B, w.H, w.L), dtype=torch.float32, device="cuda")
        bsa.bsa_forward_static_ws(q, k, v, lay, key_mask=km, out=out, lse=lse)
        assert bsa.bsa_sync_status() == 0
        assert torch.equal(out, o_ws), f"call {call}: O differs from the workspace entry point"
        assert torch.equal(lse, lse_ws), f"call {call}: lse differs from the workspace entry point"
    ref = OL.build_layout(w.H, w.L, 64, w.window, w.n_global, w.n_random, w.seed)
    o_ref, lse_ref = OA.attention(qc, kc, vc, ref, key_mask=kmc)
    o, l = out.float().cpu().numpy(), lse.cpu().numpy()
    assert np.abs(o - o_ref).max() <= O_TOL
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(l), fin)
    assert np.abs(l[fin] - lse_ref[fin]).max() <= LSE_TOL


@pytest.mark.gpu
@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
def test_static_workspace_rejects_problems_beyond_its_size():
    # every block global: 2048 split tiles of 8 chunks, far beyond the buffer
    H, L = 16, 16384
    lay = bsa.bsa_layout_build(H, L, 64, 0, L // 64, 0, 0)
    bsa.bsa_layout_upload(lay)
    assert bsa.bsa_workspace_bytes(lay, 1) > bsa.STATIC_WORKSPACE_BYTES
    q = torch.zeros((1, H, L, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(bsa.BsaError) as e:
        bsa.bsa_forward_static_ws(q, q, q, lay)
    assert e.value.code == bsa.BSA_ERR_STATIC_WORKSPACE
    assert bsa.bsa_sync_status() == 0
