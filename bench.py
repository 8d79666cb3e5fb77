"""Benchmark: BigBird block-sparse attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {ours,reference}]
                    [--workload NAME]

Metric: effective TFLOP/s counted over the layout's non-zero 64x64 blocks
(4 * 64 * 64 * d flop per (b, h, query block, key block); fully key-padded
blocks excluded), and its fraction of the measured B200 dense bf16 peak.

One step = one bsa_forward over one batch of the workload (inputs resident in
HBM).  Weak scaling: under torchrun every rank runs its own batch of the same
shape (its own data seed); there is no data-path collective, only a barrier and
a max-over-ranks reduction of the timings.  Rank 0 prints one JSON line.

``--impl reference`` times the CPU oracle (fp64 masked-dense, as it stands) on
the host cores, each step a bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads  # noqa: E402
from block_sparse_attention_bigbird_b200 import sharding  # noqa: E402

METRIC = "block-sparse attn fwd TFLOP/s (non-zero blocks) and % of B200 bf16 peak"
UNIT = "TFLOP/s"
FLOP_PER_BLOCK = 4 * 64 * 64 * 64
DEFAULT_WORKLOAD = "long_b4h12l16384"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "hbm_gbs": 6650.0, "bf16_tflops_sustained": 1400.0}


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p, "measured"
    except OSError:
        return FALLBACK_PEAKS, "fallback"


# The sources the forward kernel is compiled from (its own file and what it includes).
FWD_SOURCES = ("bsa_fwd_sm100.cu", "bsa_internal.h", "bsa_wait.cuh", "bsa_host_cuda.h", "sm100_ptx.cuh")


def _source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "block_sparse_attention_bigbird_b200", "csrc")
    for name in FWD_SOURCES:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    with open(os.path.join(ROOT, "include", "bsa.h"), "rb") as f:
        h.update(b"bsa.h" + f.read())
    return h.hexdigest()[:16]


def _traffic_for(workload: str):
    """DRAM bytes per launch from a committed ncu summary of the CURRENT kernel source."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except OSError:
        return None
    e = d.get(workload)
    if not e or e.get("source_hash") != _source_hash():
        return None
    return e.get("dram_bytes_per_launch")


def _dead_from(w):
    """First key block whose 64 keys are all padded (None when nothing is padded)."""
    if not w.key_pad_tail:
        return None
    return (w.L - w.key_pad_tail + 63) // 64


METRIC_BWD = ("block-sparse attn bwd TFLOP/s (non-zero blocks, five 64x64x64 products each) "
              "and % of B200 bf16 peak")
FLOP_PER_BLOCK_BWD = 5 * 2 * 64 * 64 * 64  # S, dP, dV, dK, dQ: 2.5x the forward's


def _has_split_rows(lay) -> bool:
    """Whether bsa_forward launches its split-row merge for this layout."""
    from block_sparse_attention_bigbird_b200 import bsa
    _, pair_ptr, _ = bsa.bsa_layout_tiles(lay)
    return bool(np.any(np.diff(pair_ptr) > bsa.SPLIT_THRESHOLD))


def _ex2_ceiling(nnz_eff, kernel_ms, dev, peaks) -> dict:
    """The second ceiling of this d = 64 forward: one ex2 per attended score (64 x 64
    per non-zero block) on an ex2 unit that retires 16 results per clock per SM,
    taken at the GPU's maximum SM clock."""
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    mhz = float(peaks.get("sm_max_mhz", 1965.0))
    peak = 16.0 * sms * mhz * 1e6 / 1e9          # G ex2 / s
    achieved = nnz_eff * 64 * 64 / (kernel_ms * 1e-3) / 1e9
    return {"bound": "alu (ex2 unit)", "achieved": achieved, "peak": peak, "unit": "Gex2/s",
            "frac": achieved / peak, "peak_source": f"16 per clock per SM x {sms} SMs x {mhz:.0f} MHz"}


def _nnz_eff(w, row_ptr, col_idx) -> int:
    """Blocks over all (b, h, i, j), minus those whose 64 keys are all padded."""
    per_batch = int(len(col_idx))
    dead = _dead_from(w)
    if dead is not None:
        per_batch -= int(np.count_nonzero(col_idx >= dead))
    return w.B * per_batch


def _mma_useful_frac(w, lay, nnz_eff) -> float:
    """Useful non-zero blocks / 64x64 block-equivalents the forward's MMAs compute.

    Each union entry of a 128-row tile costs an M=128 S MMA and PV MMA over one 64-key
    block: two 64x64 block-equivalents, of which a one-half entry (attended by one of
    the tile's two query blocks) uses one.  Entries of fully padded key blocks are
    dropped by the kernel and not counted."""
    from block_sparse_attention_bigbird_b200 import bsa
    _, pair_ptr, pair_ent = bsa.bsa_layout_tiles(lay)
    cols = pair_ent & 0xFFFFFF
    dead = _dead_from(w)
    issued_per_batch = int(len(cols) if dead is None else np.count_nonzero(cols < dead))
    return nnz_eff / (2.0 * w.B * issued_per_batch)


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons in a background thread."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.samples = []
        self._stop = threading.Event()
        self._proc = None
        sel = str(device_index)
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            sel = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            pass
        self._cmd = ["nvidia-smi", "-i", sel, f"--query-gpu={self.FIELDS}",
                     "--format=csv,noheader,nounits", "-lms", "100"]
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        try:
            self._proc = subprocess.Popen(self._cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                          text=True)
        except OSError:
            return
        for line in self._proc.stdout:
            if self._stop.is_set():
                break
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                self.samples.append((time.time(), float(parts[0]), float(parts[1]), parts[3:8]))
            except ValueError:
                continue

    def start(self):
        self._t.start()
        return self

    def stop(self):
        self._stop.set()
        if self._proc is not None:
            self._proc.terminate()
            try:
                self._proc.wait(timeout=5)
            except Exception:
                self._proc.kill()
        self._t.join(timeout=5)

    def summary(self, t0: float, t1: float, t_timed0: float):
        win = [s for s in self.samples if t0 <= s[0] <= t1]
        if not win:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "note": "no nvidia-smi samples"}
        names = ["active_mask", "hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        reasons = set()
        for s in win:
            for n, v in zip(names[1:], s[3][1:]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(s[1] for s in win),
                "sm_max_mhz": max(s[2] for s in win), "reasons": sorted(reasons),
                "samples": len(win), "samples_in_timed_region": sum(1 for s in win if s[0] >= t_timed0),
                "window": "settle run + timed region"}


def _dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if args.gpus > 1 and world == 1:
        raise SystemExit("--gpus N > 1 needs torchrun (one process per GPU)")
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def _barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()


def _config(w, nnz_eff, world):
    return {"workload": w.name, "B": w.B, "H": w.H, "L": w.L, "d": w.d, "block": w.block,
            "window": w.window, "n_global": w.n_global, "n_random": w.n_random,
            "key_pad_tail": w.key_pad_tail, "nnz_blocks_per_rank": nnz_eff,
            "global_batch": w.B * world, "seq_len": w.L, "parallelism": f"dp{world}",
            "l2": "inputs larger than L2 (q,k,v %d MB + out %d MB per step vs 126 MB L2)"
                  % (3 * w.B * w.H * w.L * w.d * 2 >> 20, w.B * w.H * w.L * w.d * 2 >> 20)}


# ----------------------------------------------------------------------------- CPU oracle
def _oracle_heads(w):
    from oracle import layout as OL
    return OL.build_layout(w.H, w.L, w.block, w.window, w.n_global, w.n_random, w.seed)


def _head_view(lay, h):
    nb = lay["nb"]
    rp = lay["row_ptr"][h * nb:(h + 1) * nb + 1]
    return {"H": 1, "L": lay["L"], "block": lay["block"], "nb": nb, "globals": lay["globals"],
            "row_ptr": rp - rp[0], "col_idx": lay["col_idx"][rp[0]:rp[-1]]}


def _oracle_cores():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        n = max((i.get("num_threads", 0) for i in info if i.get("user_api") == "blas"), default=0)
        if n:
            return n
    except Exception:
        pass
    return os.cpu_count()


def _oracle_sample(w, lay, q, k, v, km, h, n_blocks):
    """Oracle on query blocks [0, n_blocks) of (b=0, head h); returns (seconds, flop counted)."""
    from oracle import attention as OA
    view = _head_view(lay, h)
    rp, ci = view["row_ptr"], view["col_idx"]
    nnz = int(rp[n_blocks])
    dead = _dead_from(w)
    if dead is not None:
        nnz -= int(np.count_nonzero(ci[:rp[n_blocks]] >= dead))
    sl = slice(h, h + 1)
    kmask = None if km is None else km[0:1]
    t0 = time.perf_counter()
    OA.attention(q[0:1, sl], k[0:1, sl], v[0:1, sl], view, key_mask=kmask,
                 query_blocks=range(n_blocks))
    return time.perf_counter() - t0, nnz * FLOP_PER_BLOCK


def run_reference(args, w, world, rank):
    if rank != 0:
        return
    lay = _oracle_heads(w)
    q, k, v = workloads.make_qkv(w, 0)
    km = workloads.make_key_mask(w)
    nb = w.nb
    n_blocks = max(1, min(nb, int(os.environ.get("BSA_REF_BLOCKS", "8"))))
    backward = args.pass_ == "backward"
    layer = args.pass_ == "layer"
    if backward:
        do = workloads.make_grad(w, seed=100)
        sample_fn = lambda h: _oracle_bwd_sample(w, lay, q, k, v, do, km, h, n_blocks)  # noqa: E731
    elif layer:
        lp = _layer_params(w, seed=0)
        sample_fn = lambda h: _oracle_layer_sample(w, lay, *lp, km, h, n_blocks)  # noqa: E731
    else:
        sample_fn = lambda h: _oracle_sample(w, lay, q, k, v, km, h, n_blocks)  # noqa: E731
    for s in range(args.warmup):
        sample_fn(s % w.H)
    tot_t = tot_f = 0.0
    for s in range(args.steps):
        dt, fl = sample_fn(s % w.H)
        tot_t += dt
        tot_f += fl
    val = tot_f / tot_t / 1e12
    cores = _oracle_cores()
    if layer:
        sample = (f"per step: head step%H of batch 0: q for query blocks 0..{n_blocks - 1}, k and v for every "
                  f"row, attention on those blocks, the head's share of the output projection (fp64)")
    else:
        sample = (f"per step: {'gradients from ' if backward else ''}query blocks 0..{n_blocks - 1} of batch 0, "
                  f"head step%H ({n_blocks * 64} of {w.L} query rows), fp64 masked-dense")
    metric = METRIC_BWD if backward else (METRIC_LAYER if layer else METRIC)
    line = {"impl": "reference", "metric": metric, "value": val, "unit": UNIT,
            "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": _config(w, None, world),
            "cpu_baseline": {"value": val, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- GPU arm
def run_ours(args, w, world, rank, local):
    from block_sparse_attention_bigbird_b200 import bsa
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    km = workloads.make_key_mask(w)
    t_lay = time.perf_counter()
    lay = bsa.bsa_layout_build(w.H, w.L, w.block, w.window, w.n_global, w.n_random, w.seed)
    layout_build_ms = (time.perf_counter() - t_lay) * 1e3
    row_ptr, col_idx = bsa.bsa_layout_csr(lay)
    heads = args.shard == "heads"
    queries = args.shard == "queries"
    if queries:
        # strong scaling over query-block ranges: every rank reads the whole q, k, v
        # of the sequence and computes its own range of query blocks (all heads)
        q0, q1 = sharding.query_block_shard(row_ptr, w.nb, w.H, rank, world)
        total_flop = _nnz_eff(w, row_ptr, col_idx) * FLOP_PER_BLOCK
        row_ptr, col_idx = sharding.query_rows(row_ptr, col_idx, w.nb, w.H, q0, q1)
        lay = bsa.bsa_layout_from_csr(w.H, w.L, row_ptr, col_idx)
        q, k, v = workloads.make_qkv(w, data_seed=0)
    elif heads:
        # strong scaling over heads: every rank takes its heads of the same sequence
        # (the genomic shape has one batch element) and a layout of those heads' rows
        if world > w.H:
            raise SystemExit(f"--shard heads needs at most {w.H} ranks")
        h0, h1 = sharding.head_shard(w.H, rank, world)
        total_flop = _nnz_eff(w, row_ptr, col_idx) * FLOP_PER_BLOCK
        row_ptr, col_idx = sharding.head_rows(row_ptr, col_idx, w.nb, h0, h1)
        lay = bsa.bsa_layout_from_csr(h1 - h0, w.L, row_ptr, col_idx)
        q, k, v = (t[:, h0:h1].contiguous() for t in workloads.make_qkv(w, data_seed=0))
    else:
        q, k, v = workloads.make_qkv(w, data_seed=rank)
    torch.zeros(1, device=dev)  # the context exists before the upload is timed
    torch.cuda.synchronize(dev)
    t_up = time.perf_counter()
    bsa.bsa_layout_upload(lay)
    torch.cuda.synchronize(dev)
    layout_upload_ms = (time.perf_counter() - t_up) * 1e3
    H_r = q.shape[1]
    nnz_eff = _nnz_eff(w, row_ptr, col_idx)
    flop_step = nnz_eff * FLOP_PER_BLOCK
    # work of the whole job per step: every rank's own batch (weak), or one sequence's heads (strong)
    strong = heads or queries
    job_flop = total_flop if strong else world * flop_step
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    kmd = km.to(dev) if km is not None else None
    out = torch.empty_like(qd)
    lse = torch.empty((w.B, H_r, w.L), dtype=torch.float32, device=dev)
    ws = torch.zeros(bsa.bsa_workspace_bytes(lay, w.B), dtype=torch.uint8, device=dev)
    # forward, plus the key-bit kernel with a key mask and the merge with split rows
    launches_per_step = 1 + (1 if km is not None else 0) + (1 if _has_split_rows(lay) else 0)

    def step():
        bsa.bsa_forward(qd, kd, vd, lay, key_mask=kmd, out=out, lse=lse, workspace=ws, stream=stream)

    sampler = ClockSampler(local).start() if rank == 0 else None
    for _ in range(max(3, args.warmup)):
        step()
    _barrier(world)
    if bsa.bsa_sync_status(stream) != 0:
        raise RuntimeError("device status error during warm-up")
    # settle run so clock samples reflect the loaded GPU (untimed)
    t_settle = time.time()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    step()
    e1.record(stream)
    torch.cuda.synchronize()
    per = max(e0.elapsed_time(e1), 1e-3)
    for _ in range(int(min(4000, 1500.0 / per))):
        step()
    # ---- timed region: exactly K steps
    _barrier(world)
    t_timed0 = time.time()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for i in range(args.steps):
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    end.record(stream)
    _barrier(world)
    t_timed1 = time.time()
    status = bsa.bsa_sync_status(stream)
    if status != 0:
        raise RuntimeError(f"device status {status} in the timed region")
    total_ms = sharding.max_over_ranks(start.elapsed_time(end), world)
    kernel_ms = sharding.max_over_ranks(sum(a.elapsed_time(b) for a, b in ev) / args.steps, world)
    clocks = sampler.summary(t_settle, t_timed1, t_timed0) if sampler else None
    if sampler:
        sampler.stop()

    # ---- the same step with L2 flushed before each one (a 256 MB write, outside the
    # events): every K/V block comes from HBM the first time a step reads it
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    cold = []
    for _ in range(10):
        flush.fill_(1)
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        c0.record(stream)
        step()
        c1.record(stream)
        cold.append((c0, c1))
    torch.cuda.synchronize(dev)
    cold_ms = sharding.max_over_ranks(sorted(a.elapsed_time(b) for a, b in cold)[len(cold) // 2], world)
    del flush

    # ---- end to end through the public API.  Every step copies its inputs from
    # pinned host memory and reads its result back.  Device tensors are double-
    # buffered and three streams (host->device, forward, device->host) overlap step
    # i's input copy with step i-1's forward and step i-2's read-back.
    e2e_steps = max(4, min(args.steps, 20))
    qh, kh, vh = q.pin_memory(), k.pin_memory(), v.pin_memory()
    kmh = km.pin_memory() if km is not None else None
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    lse_h = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    h2d = 3 * qh.numel() * qh.element_size() + (kmh.numel() if kmh is not None else 0)
    d2h = out_h.numel() * out_h.element_size() + lse_h.numel() * 4
    bufs = [(qd, kd, vd, kmd, out, lse),
            (torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd),
             torch.empty_like(kmd) if kmd is not None else None, torch.empty_like(out), torch.empty_like(lse))]
    h2d_s, d2h_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event(), torch.cuda.Event()]    # slot's inputs landed
    ev_fwd = [torch.cuda.Event(), torch.cuda.Event()]   # slot's forward finished
    ev_out = [torch.cuda.Event(), torch.cuda.Event()]   # slot's result read back

    def e2e_step(i):
        sl = i % 2
        qs, ks, vs, kms, outs, lses = bufs[sl]
        if i >= 2:
            h2d_s.wait_event(ev_fwd[sl])                 # the forward that read these inputs
        with torch.cuda.stream(h2d_s):
            qs.copy_(qh, non_blocking=True)
            ks.copy_(kh, non_blocking=True)
            vs.copy_(vh, non_blocking=True)
            if kmh is not None:
                kms.copy_(kmh, non_blocking=True)
        ev_in[sl].record(h2d_s)
        stream.wait_event(ev_in[sl])
        if i >= 2:
            stream.wait_event(ev_out[sl])                # this slot's previous result is read back
        bsa.bsa_forward(qs, ks, vs, lay, key_mask=kms, out=outs, lse=lses, workspace=ws, stream=stream)
        ev_fwd[sl].record(stream)
        d2h_s.wait_event(ev_fwd[sl])
        with torch.cuda.stream(d2h_s):
            out_h.copy_(outs, non_blocking=True)
            lse_h.copy_(lses, non_blocking=True)
        ev_out[sl].record(d2h_s)

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    _barrier(world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    h2d_s.wait_event(a)
    d2h_s.wait_event(a)
    for i in range(e2e_steps):
        e2e_step(i)
    stream.wait_event(ev_out[(e2e_steps - 1) % 2])
    stream.wait_event(ev_out[(e2e_steps - 2) % 2])
    b.record(stream)
    _barrier(world)
    e2e_ms = sharding.max_over_ranks(a.elapsed_time(b) / e2e_steps, world)
    if bsa.bsa_sync_status(stream) != 0:
        raise RuntimeError("device status error in the end-to-end run")

    ms_per_step = total_ms / args.steps
    value = job_flop / (ms_per_step * 1e-3) / 1e12
    peaks, peak_src = _peaks()
    achieved = flop_step / (kernel_ms * 1e-3) / 1e12
    peak = float(peaks["bf16_tflops"])
    traffic = _traffic_for(w.name) if not strong or world == 1 else None
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = _cpu_baseline(w)
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "strong" if strong else "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded randn, see workloads.py)",
        "config": dict(_config(w, nnz_eff, world),
                       **({"parallelism": f"{args.shard}{world}", "global_batch": w.B} if strong else {})),
        "pct_of_peak": 100.0 * value / world / peak,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": UNIT,
                     "frac": achieved / peak, "traffic": traffic,
                     "kernel": "bsa_fwd_kernel (+ bsa_merge_kernel when the layout has split rows)",
                     "peak_source": f"{peak_src} bf16 burst",
                     "frac_of_sustained": achieved / float(peaks.get("bf16_tflops_sustained", peak)),
                     "mma_useful_frac": _mma_useful_frac(w, lay, nnz_eff),
                     "ex2": _ex2_ceiling(nnz_eff, kernel_ms, dev, peaks)},
        "e2e": {"value": job_flop / (e2e_ms * 1e-3) / 1e12, "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "pipelining": "double-buffered device tensors; host->device copy, forward and "
                              "device->host read on three streams, overlapped across steps"},
        "gpu_launches": launches_per_step * args.steps,
        "cold_l2": {"ms_per_step": cold_ms, "value": job_flop / (cold_ms * 1e-3) / 1e12, "unit": UNIT,
                    "how": "median of 10 steps, each after a 256 MB write that evicts L2"},
        "host_layout": {"build_ms": layout_build_ms, "upload_ms": layout_upload_ms,
                        "note": "once per (H, L, layout parameters); not part of a step"},
        "clocks": clocks,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)


def _bwd_launches(lay, masked: bool) -> int:
    """Kernels one bsa_backward call enqueues: key bits (with a mask), D and lse,
    dQ, dK/dV, and the split-tile sums of dQ and of dK and dV when there are any."""
    from block_sparse_attention_bigbird_b200 import bsa
    _, qp, _ = bsa.bsa_layout_tiles(lay)
    _, kp, _ = bsa.bsa_layout_key_tiles(lay)
    n = 3 + (1 if masked else 0)
    n += 1 if np.any(np.diff(qp) > bsa.SPLIT_THRESHOLD) else 0
    n += 2 if np.any(np.diff(kp) > bsa.SPLIT_THRESHOLD) else 0
    return n


def _oracle_bwd_sample(w, lay, q, k, v, do, km, h, n_blocks):
    """Oracle gradients from query blocks [0, n_blocks) of (b=0, head h); (seconds, flop)."""
    from oracle import backward as OB
    view = _head_view(lay, h)
    rp, ci = view["row_ptr"], view["col_idx"]
    nnz = int(rp[n_blocks])
    dead = _dead_from(w)
    if dead is not None:
        nnz -= int(np.count_nonzero(ci[:rp[n_blocks]] >= dead))
    sl = slice(h, h + 1)
    kmask = None if km is None else km[0:1]
    t0 = time.perf_counter()
    OB.attention_backward(q[0:1, sl], k[0:1, sl], v[0:1, sl], do[0:1, sl], view, key_mask=kmask,
                          query_blocks=range(n_blocks))
    return time.perf_counter() - t0, nnz * FLOP_PER_BLOCK_BWD


def run_backward(args, w, world, rank, local):
    """Backward pass: one bsa_backward call per step on inputs resident in HBM."""
    from block_sparse_attention_bigbird_b200 import bsa
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    q, k, v = workloads.make_qkv(w, data_seed=rank)
    do = workloads.make_grad(w, seed=100 + rank)
    km = workloads.make_key_mask(w)
    lay = bsa.bsa_layout_build(w.H, w.L, w.block, w.window, w.n_global, w.n_random, w.seed)
    bsa.bsa_layout_upload(lay)
    row_ptr, col_idx = bsa.bsa_layout_csr(lay)
    nnz_eff = _nnz_eff(w, row_ptr, col_idx)
    flop_step = nnz_eff * FLOP_PER_BLOCK_BWD
    qd, kd, vd, dod = q.to(dev), k.to(dev), v.to(dev), do.to(dev)
    kmd = km.to(dev) if km is not None else None
    out, lse = bsa.bsa_forward(qd, kd, vd, lay, key_mask=kmd, stream=stream)
    dq, dk, dv = torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd)
    ws = torch.empty(bsa.bsa_backward_workspace_bytes(lay, w.B), dtype=torch.uint8, device=dev)
    launches_per_step = _bwd_launches(lay, km is not None)

    def step(qs=qd, ks=kd, vs=vd, outs=out, dos=dod, lses=lse, gq=dq, gk=dk, gv=dv):
        bsa.bsa_backward(qs, ks, vs, outs, dos, lses, lay, key_mask=kmd, dq=gq, dk=gk, dv=gv, workspace=ws,
                         stream=stream)

    sampler = ClockSampler(local).start() if rank == 0 else None
    for _ in range(max(3, args.warmup)):
        step()
    _barrier(world)
    if bsa.bsa_sync_status(stream) != 0:
        raise RuntimeError("device status error during warm-up")
    t_settle = time.time()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    step()
    e1.record(stream)
    torch.cuda.synchronize()
    per = max(e0.elapsed_time(e1), 1e-3)
    for _ in range(int(min(2000, 1500.0 / per))):
        step()
    _barrier(world)
    t_timed0 = time.time()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(args.steps):
        step()
    end.record(stream)
    _barrier(world)
    t_timed1 = time.time()
    if bsa.bsa_sync_status(stream) != 0:
        raise RuntimeError("device status error in the timed region")
    total_ms = sharding.max_over_ranks(start.elapsed_time(end), world)
    clocks = sampler.summary(t_settle, t_timed1, t_timed0) if sampler else None
    if sampler:
        sampler.stop()

    # end to end through the public API, one step after another on one stream:
    # the step's six inputs from pinned host memory, the backward, the three
    # gradients back to pinned host memory
    e2e_steps = max(3, min(args.steps, 10))
    hosts = [t.detach().to("cpu").pin_memory() for t in (qd, kd, vd, out, dod, lse)]
    outs_h = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (dq, dk, dv)]
    h2d = sum(t.numel() * t.element_size() for t in hosts) + (km.numel() if km is not None else 0)
    d2h = sum(t.numel() * t.element_size() for t in outs_h)
    devs = [torch.empty_like(t) for t in (qd, kd, vd, out, dod, lse)]
    _barrier(world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(e2e_steps):
        for dst, src in zip(devs, hosts):
            dst.copy_(src, non_blocking=True)
        step(*devs)
        for dst, src in zip(outs_h, (dq, dk, dv)):
            dst.copy_(src, non_blocking=True)
    b.record(stream)
    _barrier(world)
    e2e_ms = sharding.max_over_ranks(a.elapsed_time(b) / e2e_steps, world)
    if bsa.bsa_sync_status(stream) != 0:
        raise RuntimeError("device status error in the end-to-end run")

    ms_per_step = total_ms / args.steps
    value = world * flop_step / (ms_per_step * 1e-3) / 1e12
    peaks, peak_src = _peaks()
    achieved = flop_step / (ms_per_step * 1e-3) / 1e12
    peak = float(peaks["bf16_tflops"])
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        lay_o = _oracle_heads(w)
        budget = float(os.environ.get("BSA_CPU_BUDGET_S", "12"))
        tot_t = tot_f = 0.0
        n_blocks, h = min(w.nb, 8), 0
        while tot_t < budget and h < w.H:
            dt, fl = _oracle_bwd_sample(w, lay_o, q, k, v, do, km, h, n_blocks)
            tot_t, tot_f, h = tot_t + dt, tot_f + fl, h + 1
        cpu = {"value": tot_f / tot_t / 1e12, "unit": UNIT, "cores": _oracle_cores(), "kind": "oracle",
               "sample": f"gradients from query blocks 0..{n_blocks - 1} of batch 0, heads 0..{h - 1} "
                         f"({tot_t:.1f} s of fp64 masked-dense)"}
    if rank != 0:
        return
    line = {
        "metric": METRIC_BWD, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded randn, see workloads.py)",
        "config": dict(_config(w, nnz_eff, world), **{"pass": "backward"}),
        "pct_of_peak": 100.0 * value / world / peak,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": UNIT,
                     "frac": achieved / peak, "traffic": None,
                     "kernel": "the whole bsa_backward step (prep, dQ, dK/dV and split-tile sums)",
                     "peak_source": f"{peak_src} bf16 burst"},
        "e2e": {"value": world * flop_step / (e2e_ms * 1e-3) / 1e12, "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "pipelining": "none: copies in, backward, copies out on one stream"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)


METRIC_LAYER = "BigBird layer forward TFLOP/s (dense projections + attention on non-zero blocks)"


def _layer_params(w, seed):
    """x [B, L, C] and the two projections' bf16 weights and biases (C = 64 H), seeded."""
    g = torch.Generator().manual_seed(seed)
    C = w.H * w.d
    x = torch.randn(w.B, w.L, C, generator=g).to(torch.bfloat16)
    wq = (torch.randn(3 * C, C, generator=g) * C ** -0.5).to(torch.bfloat16)
    bq = (torch.randn(3 * C, generator=g) * 0.1).to(torch.bfloat16)
    wo = (torch.randn(C, C, generator=g) * C ** -0.5).to(torch.bfloat16)
    bo = (torch.randn(C, generator=g) * 0.1).to(torch.bfloat16)
    return x, wq, bq, wo, bo


def _oracle_layer_sample(w, lay, x, wq, bq, wo, bo, km, h, n_blocks):
    """The layer's work for head h of batch 0 on query blocks [0, n_blocks): the oracle's
    q, k, v of that head (k, v for every key row), its attention on those query blocks
    and the head's share of the output projection; returns (seconds, flop)."""
    from oracle import attention as OA
    from oracle import projection as OP
    C = w.H * w.d
    rows = n_blocks * 64
    view = _head_view(lay, h)
    rp, ci = view["row_ptr"], view["col_idx"]
    nnz = int(rp[n_blocks])
    dead = _dead_from(w)
    if dead is not None:
        nnz -= int(np.count_nonzero(ci[:rp[n_blocks]] >= dead))
    kmask = None if km is None else km[0:1]
    t0 = time.perf_counter()
    sl = [slice(i * C + h * 64, i * C + h * 64 + 64) for i in range(3)]
    xq = x[0].double().numpy()
    qh = np.zeros((w.L, 64))
    qh[:rows] = OP.linear(xq[:rows], wq[sl[0]], bq[sl[0]])
    kh = OP.linear(xq, wq[sl[1]], bq[sl[1]])
    vh = OP.linear(xq, wq[sl[2]], bq[sl[2]])
    o, _ = OA.attention(qh[None, None], kh[None, None], vh[None, None], view, key_mask=kmask,
                        query_blocks=range(n_blocks))
    OP.linear(o[0, 0, :rows], wo[:, h * 64:(h + 1) * 64])
    dt = time.perf_counter() - t0
    flop = 2 * 64 * C * (rows + 2 * w.L) + nnz * FLOP_PER_BLOCK + 2 * rows * 64 * C
    return dt, flop


def run_layer(args, w, world, rank, local):
    """The fused BigBird layer forward: bsa_qkv_projection, bsa_forward, bsa_out_projection."""
    from block_sparse_attention_bigbird_b200 import bsa
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    if w.d != 64:
        raise SystemExit("the layer pass needs d = 64")
    C = w.H * w.d
    x, wq, bq, wo, bo = _layer_params(w, seed=rank)
    km = workloads.make_key_mask(w)
    lay = bsa.bsa_layout_build(w.H, w.L, w.block, w.window, w.n_global, w.n_random, w.seed)
    bsa.bsa_layout_upload(lay)
    row_ptr, col_idx = bsa.bsa_layout_csr(lay)
    nnz_eff = _nnz_eff(w, row_ptr, col_idx)
    flop_qkv = 2 * w.B * w.L * C * 3 * C
    flop_att = nnz_eff * FLOP_PER_BLOCK
    flop_out = 2 * w.B * w.L * C * C
    flop_step = flop_qkv + flop_att + flop_out
    xd, wqd, bqd, wod, bod = (t.to(dev) for t in (x, wq, bq, wo, bo))
    kmd = km.to(dev) if km is not None else None
    q, k, v = (torch.empty((w.B, w.H, w.L, 64), dtype=torch.bfloat16, device=dev) for _ in range(3))
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.L), dtype=torch.float32, device=dev)
    y = torch.empty((w.B, w.L, C), dtype=torch.bfloat16, device=dev)
    ws = torch.zeros(bsa.bsa_workspace_bytes(lay, w.B), dtype=torch.uint8, device=dev)
    launches_per_step = 2 + 1 + (1 if km is not None else 0) + (1 if _has_split_rows(lay) else 0)

    def part_qkv(xs=xd):
        bsa.bsa_qkv_projection(xs, wqd, bqd, q=q, k=k, v=v, stream=stream)

    def part_att():
        bsa.bsa_forward(q, k, v, lay, key_mask=kmd, out=o, lse=lse, workspace=ws, stream=stream)

    def part_out():
        bsa.bsa_out_projection(o, wod, bod, y=y, stream=stream)

    def step(xs=xd):
        part_qkv(xs)
        part_att()
        part_out()

    def timed(fn, n):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / n

    sampler = ClockSampler(local).start() if rank == 0 else None
    for _ in range(max(3, args.warmup)):
        step()
    _barrier(world)
    if bsa.bsa_sync_status(stream) != 0:
        raise RuntimeError("device status error during warm-up")
    t_settle = time.time()
    per = max(timed(step, 1), 1e-3)
    for _ in range(int(min(2000, 1500.0 / per))):
        step()
    _barrier(world)
    t_timed0 = time.time()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(args.steps):
        step()
    end.record(stream)
    _barrier(world)
    t_timed1 = time.time()
    if bsa.bsa_sync_status(stream) != 0:
        raise RuntimeError("device status error in the timed region")
    total_ms = sharding.max_over_ranks(start.elapsed_time(end), world)
    # each part alone, the same number of launches, right after the timed region
    n_part = max(3, args.steps)
    ms_parts = {"qkv_projection": timed(part_qkv, n_part), "attention": timed(part_att, n_part),
                "out_projection": timed(part_out, n_part)}
    clocks = sampler.summary(t_settle, t_timed1, t_timed0) if sampler else None
    if sampler:
        sampler.stop()
    if bsa.bsa_sync_status(stream) != 0:
        raise RuntimeError("device status error in the per-part timing")

    # end to end through the public API: x from pinned host memory, the layer, y back
    e2e_steps = max(3, min(args.steps, 10))
    xh = x.pin_memory()
    yh = torch.empty(y.shape, dtype=y.dtype).pin_memory()
    xbuf = torch.empty_like(xd)
    _barrier(world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(e2e_steps):
        xbuf.copy_(xh, non_blocking=True)
        step(xbuf)
        yh.copy_(y, non_blocking=True)
    b.record(stream)
    _barrier(world)
    e2e_ms = sharding.max_over_ranks(a.elapsed_time(b) / e2e_steps, world)
    if bsa.bsa_sync_status(stream) != 0:
        raise RuntimeError("device status error in the end-to-end run")

    ms_per_step = total_ms / args.steps
    value = world * flop_step / (ms_per_step * 1e-3) / 1e12
    peaks, peak_src = _peaks()
    peak = float(peaks["bf16_tflops"])
    kern = {}
    for name, fl in (("qkv_projection", flop_qkv), ("attention", flop_att), ("out_projection", flop_out)):
        t = ms_parts[name]
        kern[name] = {"ms": t, "tflops": fl / (t * 1e-3) / 1e12, "frac": fl / (t * 1e-3) / 1e12 / peak,
                      "share": t / sum(ms_parts.values())}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        lay_o = _oracle_heads(w)
        budget = float(os.environ.get("BSA_CPU_BUDGET_S", "12"))
        tot_t = tot_f = 0.0
        n_blocks, h = min(w.nb, 8), 0
        while tot_t < budget and h < w.H:
            dt, fl = _oracle_layer_sample(w, lay_o, x, wq, bq, wo, bo, km, h, n_blocks)
            tot_t, tot_f, h = tot_t + dt, tot_f + fl, h + 1
        cpu = {"value": tot_f / tot_t / 1e12, "unit": UNIT, "cores": _oracle_cores(), "kind": "oracle",
               "sample": f"heads 0..{h - 1} of batch 0: q for query blocks 0..{n_blocks - 1}, k and v for "
                         f"every row, attention on those blocks, the head's share of the output projection "
                         f"({tot_t:.1f} s of fp64)"}
    if rank != 0:
        return
    att = kern["attention"]
    line = {
        "metric": METRIC_LAYER, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded randn hidden states and weights, see bench._layer_params)",
        "config": dict(_config(w, nnz_eff, world), **{"pass": "layer", "dim": C}),
        "pct_of_peak": 100.0 * value / world / peak,
        "kernels": kern,
        "roofline": {"bound": "tensor", "achieved": att["tflops"], "peak": peak, "unit": UNIT,
                     "frac": att["frac"], "traffic": None,
                     "kernel": "bsa_fwd_kernel (the layer's largest share; the projections are in 'kernels')",
                     "peak_source": f"{peak_src} bf16 burst"},
        "e2e": {"value": world * flop_step / (e2e_ms * 1e-3) / 1e12, "unit": UNIT,
                "h2d_bytes_per_step": x.numel() * 2, "d2h_bytes_per_step": y.numel() * 2, "ms_per_step": e2e_ms,
                "pipelining": "none: x in, the layer, y out on one stream"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)


def _cpu_baseline(w):
    lay = _oracle_heads(w)
    q, k, v = workloads.make_qkv(w, 0)
    km = workloads.make_key_mask(w)
    budget = float(os.environ.get("BSA_CPU_BUDGET_S", "12"))
    tot_t = tot_f = 0.0
    n_blocks = min(w.nb, 16)
    h = 0
    while tot_t < budget and h < w.H:
        dt, fl = _oracle_sample(w, lay, q, k, v, km, h, n_blocks)
        tot_t += dt
        tot_f += fl
        h += 1
    return {"value": tot_f / tot_t / 1e12, "unit": UNIT, "cores": _oracle_cores(), "kind": "oracle",
            "sample": f"query blocks 0..{n_blocks - 1} of batch 0 for heads 0..{h - 1} "
                      f"({h * n_blocks * 64} query rows, {tot_t:.1f} s of fp64 masked-dense)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--pass", dest="pass_", choices=["forward", "backward", "layer"], default="forward",
                    help="forward (the default benchmark), the backward pass, or the fused layer forward "
                         "(QKV projection, attention, output projection)")
    ap.add_argument("--shard", choices=["batch", "heads", "queries"], default="batch",
                    help="forward over N ranks: each rank its own batch (weak scaling, the default) "
                         "or the heads, or the query-block ranges, of one batch split across ranks "
                         "(strong scaling)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    w = workloads.get(args.workload)
    if args.impl == "reference":
        # rank 0 alone times the CPU oracle; the other ranks exit without work
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, w, world, rank)
        return
    world, rank, local = _dist_setup(args)
    try:
        runner = {"backward": run_backward, "layer": run_layer}.get(args.pass_, run_ours)
        runner(args, w, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            if dist.is_initialized():
                dist.destroy_process_group()


if __name__ == "__main__":
    main()
