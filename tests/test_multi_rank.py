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


# ---------------------------------------------------------------- query-block sharding
def test_query_block_shard_covers_and_balances():
    for (H, nb, window, n_global, n_random, seed) in ((3, 40, 1, 2, 3, 5), (2, 64, 2, 4, 2, 1), (1, 9, 0, 1, 0, 2)):
        lay = OL.build_layout(H, nb * 64, 64, window, n_global, n_random, seed)
        rp = lay["row_ptr"]
        per_block = (rp[1:] - rp[:-1]).reshape(H, nb).sum(axis=0)
        total = int(per_block.sum())
        for world in range(1, 7):
            spans = [sharding.query_block_shard(rp, nb, H, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == nb
            assert all(a[1] == b[0] and a[0] <= a[1] for a, b in zip(spans, spans[1:]))
            for a, b in spans:  # no rank exceeds an even share by more than one query block's work
                assert int(per_block[a:b].sum()) <= -(-total // world) + int(per_block.max())


def test_query_rows_keep_exactly_the_range():
    H, nb = 3, 20
    lay = OL.build_layout(H, nb * 64, 64, 1, 2, 3, 4)
    rp, ci = lay["row_ptr"], lay["col_idx"]
    r2, c2 = sharding.query_rows(rp, ci, nb, H, 4, 11)
    assert r2.shape == rp.shape and r2[0] == 0
    for h in range(H):
        for i in range(nb):
            x = h * nb + i
            got = list(c2[r2[x]:r2[x + 1]])
            assert got == (list(ci[rp[x]:rp[x + 1]]) if 4 <= i < 11 else [])


def _worker_queries(rank, world, port, queue):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # one sequence, its query blocks split across the ranks; K and V whole on every rank
        w = workloads.custom(1, 3, 64 * 12, 1, 2, 2, seed=11, key_pad_tail=30)
        q, k, v = workloads.make_qkv(w)
        do = workloads.make_grad(w, seed=5)
        km = workloads.make_key_mask(w)
        full = OL.build_layout(w.H, w.L, 64, w.window, w.n_global, w.n_random, w.seed)
        q0, q1 = sharding.query_block_shard(full["row_ptr"], w.nb, w.H, rank, world)
        rp, ci = sharding.query_rows(full["row_ptr"], full["col_idx"], w.nb, w.H, q0, q1)
        mine = {"H": w.H, "L": w.L, "block": 64, "nb": w.nb, "row_ptr": rp.astype(np.int64), "col_idx": ci}
        o, lse = OA.attention(q, k, v, mine, key_mask=km)
        dq, dk, dv = OB.attention_backward(q, k, v, do, mine, key_mask=km)
        dkv = torch.from_numpy(np.stack([dk, dv]))
        sharding.sum_over_ranks(dkv, world)  # the backward's one exchange
        rows = slice(64 * q0, 64 * q1)
        shards = [None] * world
        dist.all_gather_object(shards, (q0, q1, o[:, :, rows], lse[:, :, rows], dq[:, :, rows],
                                        bool(np.all(o[:, :, :64 * q0] == 0) and np.all(o[:, :, 64 * q1:] == 0))))
        if rank == 0:
            queue.put((shards, dkv.numpy()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_query_block_shards_on_two_gloo_ranks_reproduce_single_process():
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker_queries, args=(r, 2, port, queue)) for r in range(2)]
    for pr in procs:
        pr.start()
    shards, dkv = queue.get(timeout=120)
    for pr in procs:
        pr.join(timeout=120)
        assert pr.exitcode == 0
    w = workloads.custom(1, 3, 64 * 12, 1, 2, 2, seed=11, key_pad_tail=30)
    q, k, v = workloads.make_qkv(w)
    do = workloads.make_grad(w, seed=5)
    km = workloads.make_key_mask(w)
    lay = OL.build_layout(w.H, w.L, 64, w.window, w.n_global, w.n_random, w.seed)
    o_ref, lse_ref = OA.attention(q, k, v, lay, key_mask=km)
    dq_ref, dk_ref, dv_ref = OB.attention_backward(q, k, v, do, lay, key_mask=km)
    shards = sorted(shards, key=lambda s: s[0])
    assert shards[0][0] == 0 and shards[-1][1] == w.nb and shards[0][1] == shards[1][0]
    assert all(s[5] for s in shards)  # rows a rank does not own come out zero there
    # a row's output and dQ depend on its own layout row alone: bit for bit
    assert np.array_equal(np.concatenate([s[2] for s in shards], axis=2), o_ref)
    assert np.array_equal(np.concatenate([s[3] for s in shards], axis=2), lse_ref)
    assert np.array_equal(np.concatenate([s[4] for s in shards], axis=2), dq_ref)
    # dK and dV are sums over query rows, added across ranks in another order
    for got, ref in ((dkv[0], dk_ref), (dkv[1], dv_ref)):
        assert np.abs(got - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max())


@pytest.mark.gpu
@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
@pytest.mark.parametrize("world", [2, 3])
def test_query_sharded_layouts_on_the_gpu_match_the_oracle(world):
    """The work each rank of a query-block-sharded job does, run shard after shard
    on one GPU: every rank's layout keeps its query blocks' rows
    (sharding.query_rows -> bsa_layout_from_csr over the full length), the forward
    and backward read the whole q, k, v.  Each rank's own rows of O, lse and dQ,
    and dK, dV summed over the ranks in fp32, match the fp64 oracle within the
    parity tolerances; rows a rank does not own come out as empty rows (O = 0,
    lse = -inf)."""
    from block_sparse_attention_bigbird_b200 import bsa
    from test_backward import _check_grads
    from test_gpu_parity import _check
    w = workloads.custom(2, 3, 64 * 64, 1, 2, 3, seed=9, key_pad_tail=30)
    qc, kc, vc = workloads.make_qkv(w)
    doc = workloads.make_grad(w, seed=100)
    kmc = workloads.make_key_mask(w)
    dev = torch.device("cuda")
    q, k, v, do, km = (t.to(dev) for t in (qc, kc, vc, doc, kmc))
    full = bsa.bsa_layout_build(w.H, w.L, 64, w.window, w.n_global, w.n_random, w.seed)
    rp, ci = bsa.bsa_layout_csr(full)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.L), dtype=torch.float32, device=dev)
    dq = torch.empty_like(q)
    dk = torch.zeros(q.shape, dtype=torch.float32, device=dev)
    dv = torch.zeros_like(dk)
    for rank in range(world):
        q0, q1 = sharding.query_block_shard(rp, w.nb, w.H, rank, world)
        srp, sci = sharding.query_rows(rp, ci, w.nb, w.H, q0, q1)
        mine = bsa.bsa_layout_from_csr(w.H, w.L, srp, sci)
        bsa.bsa_layout_upload(mine)
        o_r, lse_r = bsa.bsa_forward(q, k, v, mine, key_mask=km)
        dq_r, dk_r, dv_r = bsa.bsa_backward(q, k, v, o_r, do, lse_r, mine, key_mask=km)
        rows = slice(64 * q0, 64 * q1)
        o[:, :, rows], lse[:, :, rows], dq[:, :, rows] = o_r[:, :, rows], lse_r[:, :, rows], dq_r[:, :, rows]
        dk += dk_r.float()
        dv += dv_r.float()
        other = torch.ones(w.L, dtype=torch.bool, device=dev)
        other[rows] = False
        assert torch.all(o_r[:, :, other] == 0) and torch.all(torch.isneginf(lse_r[:, :, other]))
    assert bsa.bsa_sync_status() == 0
    ref = OL.build_layout(w.H, w.L, 64, w.window, w.n_global, w.n_random, w.seed)
    o_ref, lse_ref = OA.attention(qc, kc, vc, ref, key_mask=kmc)
    _check(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref)
    dq_o, dk_o, dv_o, mags = OB.attention_backward(qc, kc, vc, doc, ref, key_mask=kmc, with_magnitude=True)
    _check_grads([dq.float().cpu().numpy(), dk.cpu().numpy(), dv.cpu().numpy()], (dq_o, dk_o, dv_o), mags)
