"""Multi-rank host logic on CPU with two gloo ranks (no GPU).

A forward, and a backward, split by batch element across ranks, each rank
computing its shard (here with the fp64 oracle, since no GPU is present), must
reproduce the single-process result once gathered -- the gradients of one batch
element, dK and dV included, depend on that element alone; the timing reduction
must return the maximum over ranks.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import workloads
from block_sparse_attention_bigbird_b200 import sharding
from oracle import attention as OA
from oracle import backward as OB
from oracle import layout as OL


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, queue):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = workloads.custom(3, 2, 64 * 6, 1, 1, 2, seed=3)
        q, k, v = workloads.make_qkv(w)
        lay = OL.build_layout(w.H, w.L, 64, w.window, w.n_global, w.n_random, w.seed)
        b0, b1 = sharding.batch_shard(w.B, rank, world)
        o, lse = OA.attention(q[b0:b1], k[b0:b1], v[b0:b1], lay)
        shards = [None] * world
        dist.all_gather_object(shards, (b0, b1, o, lse))
        slowest = sharding.max_over_ranks(0.5 + rank, world)
        if rank == 0:
            queue.put((shards, slowest))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_batch_shard_covers_exactly():
    for B in range(0, 9):
        for world in range(1, 5):
            spans = [sharding.batch_shard(B, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == B
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1


def test_two_gloo_ranks_reproduce_single_process():
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, queue)) for r in range(2)]
    for pr in procs:
        pr.start()
    shards, slowest = queue.get(timeout=120)
    for pr in procs:
        pr.join(timeout=120)
        assert pr.exitcode == 0
    assert slowest == 1.5
    w = workloads.custom(3, 2, 64 * 6, 1, 1, 2, seed=3)
    q, k, v = workloads.make_qkv(w)
    lay = OL.build_layout(w.H, w.L, 64, w.window, w.n_global, w.n_random, w.seed)
    o_ref, lse_ref = OA.attention(q, k, v, lay)
    o = np.concatenate([s[2] for s in sorted(shards, key=lambda x: x[0])])
    lse = np.concatenate([s[3] for s in sorted(shards, key=lambda x: x[0])])
    assert np.array_equal(o, o_ref) and np.array_equal(lse, lse_ref)


def _worker_bwd(rank, world, port, queue):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = workloads.custom(3, 2, 64 * 5, 1, 1, 1, seed=4, key_pad_tail=20)
        q, k, v = workloads.make_qkv(w)
        do = workloads.make_grad(w, seed=7)
        km = workloads.make_key_mask(w)
        lay = OL.build_layout(w.H, w.L, 64, w.window, w.n_global, w.n_random, w.seed)
        b0, b1 = sharding.batch_shard(w.B, rank, world)
        grads = OB.attention_backward(q[b0:b1], k[b0:b1], v[b0:b1], do[b0:b1], lay, key_mask=km[b0:b1])
        shards = [None] * world
        dist.all_gather_object(shards, (b0, b1, grads))
        if rank == 0:
            queue.put(shards)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_backward_reproduce_single_process():
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker_bwd, args=(r, 2, port, queue)) for r in range(2)]
    for pr in procs:
        pr.start()
    shards = queue.get(timeout=120)
    for pr in procs:
        pr.join(timeout=120)
        assert pr.exitcode == 0
    w = workloads.custom(3, 2, 64 * 5, 1, 1, 1, seed=4, key_pad_tail=20)
    q, k, v = workloads.make_qkv(w)
    do = workloads.make_grad(w, seed=7)
    km = workloads.make_key_mask(w)
    lay = OL.build_layout(w.H, w.L, 64, w.window, w.n_global, w.n_random, w.seed)
    ref = OB.attention_backward(q, k, v, do, lay, key_mask=km)
    shards = sorted(shards, key=lambda x: x[0])
    for i in range(3):
        got = np.concatenate([s[2][i] for s in shards])
        assert np.array_equal(got, ref[i])


def _worker_heads(rank, world, port, queue):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # one long-ish sequence (B = 1), its heads split across the ranks; each rank
        # builds its own layout from its heads' rows with the library's CSR builder
        from block_sparse_attention_bigbird_b200 import bsa
        w = workloads.custom(1, 5, 64 * 12, 1, 2, 2, seed=9, key_pad_tail=30)
        q, k, v = workloads.make_qkv(w)
        km = workloads.make_key_mask(w)
        full = bsa.bsa_layout_build(w.H, w.L, 64, w.window, w.n_global, w.n_random, w.seed)
        rp, ci = bsa.bsa_layout_csr(full)
        h0, h1 = sharding.head_shard(w.H, rank, world)
        srp, sci = sharding.head_rows(rp, ci, w.nb, h0, h1)
        mine = bsa.bsa_layout_from_csr(h1 - h0, w.L, srp, sci)
        r2, c2 = bsa.bsa_layout_csr(mine)
        lay = {"H": h1 - h0, "L": w.L, "block": 64, "nb": w.nb, "row_ptr": r2.astype(np.int64), "col_idx": c2}
        o, lse = OA.attention(q[:, h0:h1], k[:, h0:h1], v[:, h0:h1], lay, key_mask=km)
        shards = [None] * world
        dist.all_gather_object(shards, (h0, h1, o, lse))
        if rank == 0:
            queue.put(shards)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_head_shard_rows_and_two_gloo_ranks_reproduce_single_process():
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker_heads, args=(r, 2, port, queue)) for r in range(2)]
    for pr in procs:
        pr.start()
    shards = queue.get(timeout=120)
    for pr in procs:
        pr.join(timeout=120)
        assert pr.exitcode == 0
    w = workloads.custom(1, 5, 64 * 12, 1, 2, 2, seed=9, key_pad_tail=30)
    q, k, v = workloads.make_qkv(w)
    km = workloads.make_key_mask(w)
    lay = OL.build_layout(w.H, w.L, 64, w.window, w.n_global, w.n_random, w.seed)
    o_ref, lse_ref = OA.attention(q, k, v, lay, key_mask=km)
    shards = sorted(shards, key=lambda x: x[0])
    assert [s[:2] for s in shards] == [(0, 3), (3, 5)]
    assert np.array_equal(np.concatenate([s[2] for s in shards], axis=1), o_ref)
    assert np.array_equal(np.concatenate([s[3] for s in shards], axis=1), lse_ref)


@pytest.mark.gpu
@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
@pytest.mark.parametrize("world", [2, 3])
def test_head_sharded_layouts_on_the_gpu_reproduce_the_full_run(world):
    """The work each rank of a head-sharded job does, run shard after shard on one
    GPU: every rank builds its layout from its heads' CSR rows
    (sharding.head_rows -> bsa_layout_from_csr) and runs the forward and the
    backward on its heads' slices.  Put back together, the shards equal the
    single-layout run bit for bit (a head's tiles, entries and schedule do not
    depend on the other heads) and the fp64 oracle within the parity tolerances."""
    from block_sparse_attention_bigbird_b200 import bsa
    from test_backward import _check_grads
    from test_gpu_parity import _check
    # global query rows long enough to be split into chunks, and a padded key tail
    w = workloads.custom(2, 5, 64 * 64, 1, 2, 3, seed=9, key_pad_tail=30)
    qc, kc, vc = workloads.make_qkv(w)
    doc = workloads.make_grad(w, seed=100)
    kmc = workloads.make_key_mask(w)
    dev = torch.device("cuda")
    q, k, v, do, km = (t.to(dev) for t in (qc, kc, vc, doc, kmc))
    full = bsa.bsa_layout_build(w.H, w.L, 64, w.window, w.n_global, w.n_random, w.seed)
    bsa.bsa_layout_upload(full)
    o_full, lse_full = bsa.bsa_forward(q, k, v, full, key_mask=km)
    g_full = bsa.bsa_backward(q, k, v, o_full, do, lse_full, full, key_mask=km)
    rp, ci = bsa.bsa_layout_csr(full)
    outs = []
    for rank in range(world):
        h0, h1 = sharding.head_shard(w.H, rank, world)
        srp, sci = sharding.head_rows(rp, ci, w.nb, h0, h1)
        mine = bsa.bsa_layout_from_csr(h1 - h0, w.L, srp, sci)
        bsa.bsa_layout_upload(mine)
        qs, ks, vs, dos = (t[:, h0:h1].contiguous() for t in (q, k, v, do))
        o, lse = bsa.bsa_forward(qs, ks, vs, mine, key_mask=km)
        outs.append((o, lse) + tuple(bsa.bsa_backward(qs, ks, vs, o, dos, lse, mine, key_mask=km)))
    assert bsa.bsa_sync_status() == 0
    got = [torch.cat([s[i] for s in outs], dim=1) for i in range(5)]
    for a, b in zip(got, (o_full, lse_full) + tuple(g_full)):
        assert torch.equal(a, b)
    ref = OL.build_layout(w.H, w.L, 64, w.window, w.n_global, w.n_random, w.seed)
    o_ref, lse_ref = OA.attention(qc, kc, vc, ref, key_mask=kmc)
    _check(got[0].float().cpu().numpy(), got[1].cpu().numpy(), o_ref, lse_ref)
    dq, dk, dv, mags = OB.attention_backward(qc, kc, vc, doc, ref, key_mask=kmc, with_magnitude=True)
    _check_grads([t.float().cpu().numpy() for t in got[2:]], (dq, dk, dv), mags)
