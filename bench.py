"""Benchmark of the S2O prefill hot path on B200 (one JSON line on rank 0).

A step is one pass of the whole hot path — index build (stripe pooling, both orderings, block
scores, early-stop lists) then the fused gather-attention — over one synthetic Llama-3.1-8B-shaped
128K layer (32 query / 8 KV heads, d = 128, S = 2048, B = 128, τ = 0.01), inputs resident in HBM.
Q alone is 1.07 GB, larger than the 126 MB L2, so no flush is needed between steps.

Metric (the pages' headline): sparse prefill attention time and effective TFLOP/s at 128K, with
sparsity and MSE, against the bf16 peak. ``value`` is the effective (dense-causal-equivalent)
TFLOP/s of the whole job: N GPUs × 4·d·N(N+1)/2·Hq FLOPs ÷ the slowest rank's step time.

Multi-GPU (``torchrun``): by default every rank runs its own independent layer (weak scaling);
with ``--parallel heads`` one layer is split by KV head (rank r takes the KV heads g with
g mod N = r and their query heads; strong scaling). Heads shard with no exchange, so no data-path
collective is used; NCCL carries the barrier, the max-over-ranks timing and, in the head split,
one optional all-gather of O reported beside the step.

``--impl reference`` times the CPU oracle (the only reference arm this project has) on rank 0
only: each step is one bounded sample of the same workload (one KV group's index build and the
attention of 2048 random rows per head by default); ``ms_per_step`` is the sample's wall time and
``value`` the layer's work over the sample's time scaled to the whole layer.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import gen  # noqa: E402

METRIC = "sparse prefill attention ms & effective TFLOPS @128K (sparsity, MSE) vs bf16 peak"
UNIT = "TFLOP/s (dense-causal-equivalent)"
WORKLOAD = "llama-128k"


# DRAM bytes per launch of the dominant kernel (the attention local pass), from an ncu capture of
# that kernel (dram__bytes_read.sum + dram__bytes_write.sum on llama-32k, scaled by the tile count
# to llama-128k). Valid only for the kernel source it was taken on: reported as null once
# s2o_attn.cu changes.
ATTN_TRAFFIC = {"src_sha256_16": "0eeeddd21e4b9762", "workload": "llama-128k",
                "bytes_per_launch": (403.441408e6 + 232.880128e6) * 4}


def attention_traffic(workload):
    import hashlib
    path = os.path.join(ROOT, "long_context_sparse_stripe_b200", "csrc", "s2o_attn.cu")
    with open(path, "rb") as f:
        sha = hashlib.sha256(f.read()).hexdigest()[:16]
    if sha != ATTN_TRAFFIC["src_sha256_16"] or workload != ATTN_TRAFFIC["workload"]:
        return None
    return ATTN_TRAFFIC["bytes_per_launch"]


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p.get("bf16_tflops", 1590.0), p.get("hbm_gbs", 6650.0), "measured"
    return 1590.0, 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples taken while the timed region runs.

    The sampler is started and confirmed running before the region opens; only samples whose
    arrival time falls inside [mark_start, mark_end] are kept."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, period_ms: int = 20):
        self.gpu, self.period = gpu_index, period_ms
        self.proc, self.samples, self.t0, self.t1 = None, [], None, None

    def _reader(self):
        for ln in self.proc.stdout:
            if ln.strip():
                self.samples.append((time.perf_counter(), ln))

    def __enter__(self):
        import threading
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", str(self.period)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return self
        threading.Thread(target=self._reader, daemon=True).start()
        deadline = time.perf_counter() + 5.0
        while not self.samples and time.perf_counter() < deadline:
            time.sleep(0.01)
        return self

    def mark_start(self):
        self.t0 = time.perf_counter()

    def mark_end(self):
        self.t1 = time.perf_counter()

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sms, maxes, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for t, ln in list(self.samples):
            if self.t0 is None or self.t1 is None or not (self.t0 <= t <= self.t1):
                continue
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sms.append(float(f[1]))
                maxes.append(float(f[2]))
            except ValueError:
                continue
            for name, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sms:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": float(np.median(sms)), "sm_max_mhz": max(maxes),
                "reasons": sorted(reasons), "samples": len(sms)}


def dist_setup(n_gpus: int, backend: str = "nccl"):
    """One process per GPU (torchrun's RANK / LOCAL_RANK / WORLD_SIZE / MASTER_*): the process
    group for the barriers and the max-over-ranks times; None when the job has one rank. The
    tests drive the same code with the gloo backend on the host."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=timedelta(seconds=600),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=timedelta(seconds=60))
        return dist, rank, world, local
    return None, 0, 1, 0


def layer_seed(w, rank: int) -> int:
    """Seed of the independent layer rank `rank` runs (weak scaling: one layer per GPU)."""
    return w.seed + 100 * rank


def whole_job_value(flops_per_layer: float, world: int, ms_step: float) -> float:
    """Whole-job TFLOP/s: every rank's layer over the slowest rank's step time."""
    return flops_per_layer * world / (ms_step * 1e-3) / 1e12


def max_over_ranks(dist, x: float, device) -> float:
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def cpu_oracle_sample(w, q, k, v, max_rows=2048, seed=0):
    """The oracle as it stands on a bounded sample: one KV group (G query heads) — its index build
    in full and the attention of `max_rows` random query rows per head — extrapolated to the whole
    layer. Returns (seconds for the full layer, description, threads)."""
    import oracle
    G = w.n_q_heads // w.n_kv_heads
    sub = w.replace(n_q_heads=G, n_kv_heads=1)
    qs, ks, vs = q[:, :G].contiguous(), k[:, :1].contiguous(), v[:, :1].contiguous()
    cfg = oracle.config(sub)
    threads = oracle.threads()
    t0 = time.perf_counter()
    idx = oracle.build_indices(cfg, qs, ks, n_threads=threads)
    t_idx = time.perf_counter() - t0
    rng = np.random.default_rng(seed)
    rows = np.sort(np.concatenate([h * w.seq_len + rng.choice(w.seq_len, max_rows, replace=False)
                                   for h in range(G)]))
    t0 = time.perf_counter()
    oracle.attention(cfg, qs, ks, vs, idx, rows=rows, n_threads=threads)
    t_attn = time.perf_counter() - t0
    groups = w.n_kv_heads * w.batch
    full = groups * (t_idx + t_attn * (w.seq_len / max_rows))
    desc = (f"index build of 1 KV group ({G} query heads) in full ({t_idx:.2f} s) + attention of "
            f"{max_rows} random rows per head ({t_attn:.2f} s), extrapolated x{groups} groups and "
            f"x{w.seq_len / max_rows:.0f} rows")
    return full, desc, threads


def workload_config(name, w, world, parallel="replica"):
    """The bench line's ``config`` (the same keys on both arms)."""
    par = (f"one layer split by KV head over {world} GPUs" if parallel == "heads"
           else f"independent layer per GPU x{world}")
    return {"workload": name, "batch": w.batch, "n_q_heads": w.n_q_heads,
            "n_kv_heads": w.n_kv_heads, "seq_len": w.seq_len, "head_dim": w.head_dim,
            "segment_len": w.segment_len, "block_size": w.block_size, "tau": w.tau,
            "query_perm": w.query_perm, "parallelism": par,
            "l2": "inputs larger than L2 (Q is 1.07 GB); no flush"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = gen.workload(args.workload, tau=args.tau)
    q, k, v = gen.make_inputs(w)
    times, walls, desc, threads = [], [], "", 0
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        full, desc, threads = cpu_oracle_sample(w, q, k, v, max_rows=args.ref_rows, seed=i)
        if i >= args.warmup:
            times.append(full)
            walls.append(time.perf_counter() - t0)
    sec = float(np.median(times))
    value = w.dense_causal_flops / sec / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        # Each step runs one bounded sample of the layer: ms_per_step is the time a step really
        # took; `value` is the layer's work over the sample's time scaled to the whole layer
        # (layer_ms_extrapolated), since the sample stands for that share of the layer.
        "ms_per_step": float(np.median(walls)) * 1e3,
        "ms_per_step_kind": "one bounded sample of the layer per step (wall time of the sample)",
        "layer_ms_extrapolated": sec * 1e3,
        "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(args.workload, w, args.gpus, args.parallel),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_s2o(args):
    import long_context_sparse_stripe_b200 as s2o

    dist, rank, world, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = gen.workload(args.workload, tau=args.tau)
    if args.parallel == "heads":
        # One layer split by KV head: this rank's KV heads g (g mod world = rank) with their
        # query heads; no data-path collective (strong scaling).
        from long_context_sparse_stripe_b200 import shard
        q, k, v = shard.shard_inputs(*gen.make_inputs(w), rank, world)
        wr = shard.shard_config(w, rank, world)
        job_flops = w.dense_causal_flops
    else:
        # Each rank runs its own independent layer (weak scaling).
        q, k, v = gen.make_inputs(w.replace(seed=layer_seed(w, rank)))
        wr = w
        job_flops = w.dense_causal_flops * world
    cfg = s2o.Config.of(wr)
    qd, kd, vd = (t.to(dev) for t in (q, k, v))
    o = torch.empty_like(qd)
    idx = s2o.alloc_indices(cfg, dev)
    # With room for the permuted copy of K and V, which the library makes when it pays.
    ws = s2o.alloc_prefill_workspace(cfg, dev)
    stream = torch.cuda.current_stream(dev)

    nvtx = torch.cuda.nvtx  # named ranges for a timeline profiler; no-ops without one

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        with nvtx.range("s2o index build"):
            s2o.build_indices(cfg, qd, kd, out=idx, ws=ws)
        if ev is not None:
            ev[1].record(stream)
        with nvtx.range("s2o attention"):
            s2o.attention_prefill_with_indices_ws(cfg, qd, kd, vd, idx, ws, out=o)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if s2o.check_device_status(dev) != 0:
        raise RuntimeError("device timeout during warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(dev)
    launches0 = s2o.kernel_launch_count()
    with ClockSampler(local) as clocks:
        clocks.mark_start()
        start.record(stream)
        for i in range(args.steps):
            step(evs[i])
        end.record(stream)
        torch.cuda.synchronize(dev)
        clocks.mark_end()
    launches = s2o.kernel_launch_count() - launches0
    if dist is not None:
        dist.barrier()
    status = s2o.check_device_status(dev)
    total_ms = start.elapsed_time(end)
    index_ms = float(np.mean([e[0].elapsed_time(e[1]) for e in evs]))
    attn_ms = float(np.mean([e[1].elapsed_time(e[2]) for e in evs]))
    ms_step = max_over_ranks(dist, total_ms / args.steps, dev)
    attn_ms_max = max_over_ranks(dist, attn_ms, dev)

    stats = s2o.index_stats(cfg, idx, ws)
    tile_flops = 4.0 * w.block_size * w.block_size * w.head_dim
    # Tile products the attention kernel executes (local pass: every segment's causal triangle in
    # original order; permuted pass: the selected blocks, packed when most are selected), and the
    # tiles of (query, key) pairs the method attends (pairs / B²).
    work = s2o.attention_work(cfg, idx, ws)
    local_pass, permuted_pass = work.local_pass_tiles, work.permuted_unit_tiles
    kernel_tiles = work.unit_tiles
    useful_tiles = stats.pairs / float(w.block_size ** 2)
    exec_flops = kernel_tiles * tile_flops
    peak, hbm_peak, peak_kind = measured_peaks()

    # Dense causal baseline on the same inputs, and the MSE of the S2O output against it.
    od = torch.empty_like(qd)
    s2o.dense_causal_prefill(cfg, qd, kd, vd, out=od)
    torch.cuda.synchronize(dev)
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    d0.record(stream)
    for _ in range(args.dense_steps):
        s2o.dense_causal_prefill(cfg, qd, kd, vd, out=od)
    d1.record(stream)
    torch.cuda.synchronize(dev)
    dense_ms = d0.elapsed_time(d1) / args.dense_steps
    mse = float(((o.float() - od.float()) ** 2).mean().item())
    del od

    # End to end through the public call with host buffers: every step copies its Q/K/V from
    # pinned host memory to the device, runs the prefill and reads O back, pipelined as a serving
    # loop runs it: step k's inputs go up on one copy stream while step k-1 computes, and step k's
    # output comes down on another while step k+1 computes (the two PCIe directions are
    # independent); device inputs and outputs are double-buffered. The timed region holds every
    # step's copies, the pipeline's fill and its drain.
    qh, kh, vh = (t.pin_memory() for t in (q, k, v))
    oh = torch.empty(q.shape, dtype=torch.bfloat16).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in (qh, kh, vh))
    d2h = oh.numel() * oh.element_size()
    ins = [(qd, kd, vd), tuple(torch.empty_like(t) for t in (qd, kd, vd))]
    outs = [o, torch.empty_like(o)]
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    loaded, computed, read = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    n_e2e = args.e2e_steps
    torch.cuda.synchronize(dev)
    if dist is not None:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    up.wait_stream(stream)
    down.wait_stream(stream)
    for step in range(n_e2e):
        b = step % 2
        with torch.cuda.stream(up):
            if step >= 2:
                up.wait_event(computed[b])  # step - 2 has finished reading these inputs
            for dst, src in zip(ins[b], (qh, kh, vh)):
                dst.copy_(src, non_blocking=True)
            loaded[b].record(up)
        stream.wait_event(loaded[b])
        if step >= 2:
            stream.wait_event(read[b])  # step - 2's output has been read back
        qb, kb, vb = ins[b]
        s2o.attention_prefill(cfg, qb, kb, vb, out=outs[b], idx=idx, ws=ws)
        computed[b].record(stream)
        with torch.cuda.stream(down):
            down.wait_event(computed[b])
            oh.copy_(outs[b], non_blocking=True)
            read[b].record(down)
    stream.wait_stream(up)
    stream.wait_stream(down)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(dist, e0.elapsed_time(e1) / n_e2e, dev)
    del ins, outs
    gather_ms = None
    if args.parallel == "heads" and dist is not None:
        # Assembling the whole O on every GPU, if a caller wants it: one NCCL all-gather of the
        # shards (not part of the step; the step's output stays sharded).
        from long_context_sparse_stripe_b200 import shard
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        full_o = shard.gather_output(o, w.n_q_heads, w.n_kv_heads, rank, world, dist)
        g1.record(stream)
        torch.cuda.synchronize(dev)
        gather_ms = max_over_ranks(dist, g0.elapsed_time(g1), dev)
        del full_o

    line = None
    if rank == 0:
        achieved = exec_flops / (attn_ms_max * 1e-3) / 1e12
        line = {
            "metric": METRIC,
            "value": whole_job_value(job_flops, 1, ms_step),
            "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_step,
            "higher_is_better": True,
            "scaling": "strong" if args.parallel == "heads" else "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": workload_config(args.workload, w, world, args.parallel),
            "s2o_ms": ms_step, "index_ms": index_ms, "attention_ms": attn_ms,
            "index_fraction_of_attention": index_ms / attn_ms,
            "dense_ms": dense_ms, "speedup_vs_dense": dense_ms / ms_step,
            "pair_sparsity": stats.pair_sparsity,
            "tile_density": stats.executed_tiles * w.block_size ** 2 * 1.0 / stats.causal_pairs,
            "executed_tiles": stats.executed_tiles, "local_tiles": stats.local_tiles,
            "selected_tiles": stats.selected_tiles,
            "kernel_tiles": {"local_pass": local_pass, "permuted_pass": permuted_pass,
                             "permuted_loaded": work.permuted_loaded_tiles,
                             "packed_streams": work.packed,
                             "executed_over_attended": kernel_tiles / useful_tiles},
            "mse_vs_dense": mse,
            "exec_tflops": achieved,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak,
                         "unit": "TFLOP/s", "frac": achieved / peak,
                         "traffic": attention_traffic(args.workload),
                         "kernel": "s2o_attention_kernel<128,128> (" + (
                             ("packed permuted pass + merging local pass" if work.packed else
                              "gathered permuted pass + merging local pass") if work.merged else
                             "local pass + permuted pass, the path without the merge") + ")",
                         "peak_source": f"{peak_kind} bf16 (burst)"},
            "e2e": {"value": whole_job_value(job_flops, 1, e2e_ms), "unit": UNIT,
                    "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "steps": n_e2e,
                    "schedule": "pipelined: H2D of step k+1 and D2H of step k-1 overlap step k's "
                                "prefill (double-buffered device inputs and outputs)"},
            "gpu_launches": launches,
            "o_all_gather_ms": gather_ms,
            "clocks": clocks.summary(),
            "device_status": s2o.STATUS.get(status, status),
        }
    if dist is not None:
        dist.barrier()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        full, desc, threads = cpu_oracle_sample(w, q, k, v, max_rows=args.ref_rows)
        line["cpu_baseline"] = {"value": w.dense_causal_flops / full / 1e12, "unit": UNIT,
                                "cores": threads, "kind": "oracle", "sample": desc}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


def run_sweep(args):
    """Per-configuration report (not the headline line): the llama-32k layer, the llama-128k layer
    at three thresholds, the qwen-128k ablations (threshold, segment length, query permutation off)
    and the 32-layer stack. One JSON line per configuration on stdout."""
    import long_context_sparse_stripe_b200 as s2o

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peak = measured_peaks()[0]
    cache = {}

    def events():
        return torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def measure(w, reps=5, dense=True):
        key = (w.name, w.seed, w.seq_len, w.stripe_frac)
        if key not in cache:
            cache.clear()
            cache[key] = tuple(t.to(dev) for t in gen.make_inputs(w))
        qd, kd, vd = cache[key]
        cfg = s2o.Config.of(w)
        idx, o = s2o.alloc_indices(cfg, dev), torch.empty_like(qd)
        ws = s2o.alloc_prefill_workspace(cfg, dev)
        for _ in range(2):
            s2o.build_indices(cfg, qd, kd, out=idx, ws=ws)
            s2o.attention_prefill_with_indices_ws(cfg, qd, kd, vd, idx, ws, out=o)
        a0, a1 = events()
        b0, b1 = events()
        a0.record()
        for _ in range(reps):
            s2o.build_indices(cfg, qd, kd, out=idx, ws=ws)
        a1.record()
        b0.record()
        for _ in range(reps):
            s2o.attention_prefill_with_indices_ws(cfg, qd, kd, vd, idx, ws, out=o)
        b1.record()
        torch.cuda.synchronize()
        index_ms, attn_ms = a0.elapsed_time(a1) / reps, b0.elapsed_time(b1) / reps
        stats = s2o.index_stats(cfg, idx, ws)
        work = s2o.attention_work(cfg, idx, ws)
        local_pass, permuted_pass = work.local_pass_tiles, work.permuted_unit_tiles
        tile_flops = 4.0 * w.block_size ** 2 * w.head_dim
        useful = stats.pairs / float(w.block_size ** 2)
        row = {"workload": w.name, "tau": w.tau, "segment_len": w.segment_len,
               "query_perm": w.query_perm, "shared_key_order": w.shared_key_order,
               "int4_centroids": w.int4_centroids,
               "stripe_frac": w.stripe_frac,
               "pair_sparsity": stats.pair_sparsity,
               "tile_density": stats.executed_tiles * w.block_size ** 2 / stats.causal_pairs,
               "selected_tiles": stats.selected_tiles,
               "kernel_tiles": {"local_pass": local_pass, "permuted_pass": permuted_pass,
                                "permuted_loaded": work.permuted_loaded_tiles,
                                "packed_streams": work.packed,
                                "executed_over_attended": (local_pass + permuted_pass) / useful},
               "index_ms": index_ms, "attention_ms": attn_ms,
               "index_fraction_of_attention": index_ms / attn_ms,
               "exec_tflops": (local_pass + permuted_pass) * tile_flops / (attn_ms * 1e-3) / 1e12,
               "effective_tflops": w.dense_causal_flops / ((index_ms + attn_ms) * 1e-3) / 1e12}
        row["exec_frac_of_peak"] = row["exec_tflops"] / peak
        if dense:
            od = torch.empty_like(qd)
            s2o.dense_causal_prefill(cfg, qd, kd, vd, out=od)
            d0, d1 = events()
            d0.record()
            s2o.dense_causal_prefill(cfg, qd, kd, vd, out=od)
            d1.record()
            torch.cuda.synchronize()
            row["dense_ms"] = d0.elapsed_time(d1)
            row["mse_vs_dense"] = float(((o.float() - od.float()) ** 2).mean().item())
            del od
        if s2o.check_device_status(dev) != 0:
            raise RuntimeError("device timeout")
        return row

    def measure_online(w, reps=3):
        """The measured-share early stop (labelled variant) against the same lists run in full on
        the same path (local pass, then the permuted pass over gathered list streams), and the
        default path with a workspace."""
        key = (w.name, w.seed, w.seq_len, w.stripe_frac)
        if key not in cache:
            cache.clear()
            cache[key] = tuple(t.to(dev) for t in gen.make_inputs(w))
        qd, kd, vd = cache[key]
        cfg = s2o.Config.of(w)
        ws = s2o.alloc_prefill_workspace(cfg, dev)
        idx = s2o.build_indices(cfg, qd, kd, ws=ws)
        o_full, o_stop, o_ws = (torch.empty_like(qd) for _ in range(3))
        runs = {"full_lists": lambda: s2o.attention_prefill_with_indices(cfg, qd, kd, vd, idx,
                                                                         out=o_full),
                "online_stop": lambda: s2o.attention_prefill_online_stop(cfg, qd, kd, vd, idx,
                                                                         out=o_stop),
                "default_with_workspace": lambda: s2o.attention_prefill_with_indices_ws(
                    cfg, qd, kd, vd, idx, ws, out=o_ws)}
        row = {"workload": w.name, "tau": w.tau, "variant": "online stop (measured share)"}
        stop = None
        for name, fn in runs.items():
            r = fn()
            if name == "online_stop":
                stop = r[1]
            fn()
            e0, e1 = events()
            e0.record()
            for _ in range(reps):
                fn()
            e1.record()
            torch.cuda.synchronize()
            row[name + "_ms"] = e0.elapsed_time(e1) / reps
        row["listed_blocks"] = int(idx.sel_cnt.long().sum().item())
        row["kept_blocks"] = int(stop.long().sum().item())
        row["cut_lists"] = int((stop < idx.sel_cnt).sum().item())
        od = torch.empty_like(qd)
        s2o.dense_causal_prefill(cfg, qd, kd, vd, out=od)
        torch.cuda.synchronize()
        row["mse_vs_dense"] = {k: float(((o.float() - od.float()) ** 2).mean().item())
                               for k, o in (("full_lists", o_full), ("online_stop", o_stop))}
        if s2o.check_device_status(dev) != 0:
            raise RuntimeError("device timeout")
        return row

    configs = [gen.workload("llama-32k")]
    # Labelled strong-stripe workload (beside the specified ones): the permuted pass at the
    # selection density the pages report.
    configs += [gen.workload("llama-128k-strong", tau=t) for t in (0.005, 0.01, 0.02)]
    configs += [gen.workload("llama-128k", tau=t) for t in (0.005, 0.01, 0.02)]
    qwen = gen.workload("qwen-128k")
    configs += [qwen.replace(tau=t) for t in (0.001, 0.005, 0.01, 0.02)]
    configs += [qwen.replace(segment_len=s) for s in (1024, 4096)]
    configs += [qwen.replace(query_perm=0)]
    # Labelled variant beside the specified configurations: one key ordering per KV head.
    configs += [gen.workload("llama-128k").replace(shared_key_order=1),
                qwen.replace(tau=0.001, shared_key_order=1)]
    # Labelled variant: 4-bit key centroids for the block scores (alone and with the above).
    configs += [gen.workload("llama-128k").replace(int4_centroids=1),
                gen.workload("llama-128k").replace(shared_key_order=1, int4_centroids=1)]
    if args.sweep_filter:
        keep = args.sweep_filter.split(",")
        configs = [w for w in configs if any(f"{w.name}@{w.tau}".startswith(k) for k in keep)]
    for w in configs:
        print(json.dumps({"config": measure(w)}), flush=True)
    online = [gen.workload("llama-128k-strong", tau=t) for t in (0.005, 0.01, 0.02)]
    online += [gen.workload("qwen-128k", tau=0.001)]
    if args.sweep_filter:
        online = [w for w in online if any(f"online:{w.name}@{w.tau}".startswith(k) for k in keep)]
    for w in online:
        print(json.dumps({"online_stop": measure_online(w)}), flush=True)
    if args.sweep_filter and "stack" not in args.sweep_filter.split(","):
        return 0
    stack = [measure(gen.layer_workload(l), reps=2, dense=(l % 8 == 7)) for l in range(32)]
    tot_i = sum(r["index_ms"] for r in stack)
    tot_a = sum(r["attention_ms"] for r in stack)
    print(json.dumps({"stack32": {
        "layers": 32, "index_ms_total": tot_i, "attention_ms_total": tot_a,
        "index_fraction_of_attention": tot_i / tot_a,
        "pair_sparsity_mean": float(np.mean([r["pair_sparsity"] for r in stack])),
        "mse_vs_dense_layers_7_15_23_31": [r["mse_vs_dense"] for r in stack if "mse_vs_dense" in r],
        "effective_tflops": sum(gen.layer_workload(l).dense_causal_flops for l in range(32))
        / ((tot_i + tot_a) * 1e-3) / 1e12}}), flush=True)
    return 0


def run_layer(args):
    """End-to-end-shaped prefill (not the headline line): one Llama-3.1-8B-shaped decoder layer
    with random weights at the bench workload's attention shape, S2O attention against the dense
    causal baseline, CUDA events. A 32-layer prefill is 32 such layers (embedding and output head
    left out). One JSON line on stdout."""
    import long_context_sparse_stripe_b200 as s2o

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = gen.workload(args.workload, tau=args.tau)
    shape = gen.LAYER_8B
    host = gen.make_layer(w, shape)
    wts = {k: v.to(dev) for k, v in host.items()}
    x0 = wts.pop("x")
    cfg = s2o.Config.of(w)
    H, I, rows = w.n_q_heads * w.head_dim, shape.intermediate, w.batch * w.seq_len
    qkvw = (w.n_q_heads + 2 * w.n_kv_heads) * w.head_dim
    gemm_flops = 2.0 * rows * (H * qkvw + H * H + H * 2 * I + I * H)
    peak = measured_peaks()[0]
    out = {}
    for dense in (False, True):
        ws = torch.empty(s2o.layer_workspace_size(cfg, shape, dense), dtype=torch.uint8,
                         device=dev)
        x = torch.empty_like(x0)
        reps = 3
        for _ in range(1):
            x.copy_(x0)
            s2o.layer_prefill(cfg, shape, wts, x, ws=ws, dense=dense)
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        # the copy that restores x each repetition is timed on its own and subtracted
        c0.record()
        for _ in range(reps):
            x.copy_(x0)
        c1.record()
        e0.record()
        for _ in range(reps):
            x.copy_(x0)
            s2o.layer_prefill(cfg, shape, wts, x, ws=ws, dense=dense)
        e1.record()
        torch.cuda.synchronize(dev)
        ms = (e0.elapsed_time(e1) - c0.elapsed_time(c1)) / reps
        out["dense" if dense else "s2o"] = ms
        del ws
        torch.cuda.empty_cache()
    attn_dense = w.dense_causal_flops
    line = {"layer": {
        "workload": w.name, "tau": w.tau, "hidden": H, "intermediate": I,
        "weights": "random N(0, 1/fan_in), seeded", "status": s2o.check_device_status(dev),
        "s2o_layer_ms": out["s2o"], "dense_layer_ms": out["dense"],
        "e2e_speedup_vs_dense_attention": out["dense"] / out["s2o"],
        "projection_tflop_per_layer": gemm_flops / 1e12,
        "dense_attention_tflop_per_layer": attn_dense / 1e12,
        "dense_layer_tflops": (gemm_flops + attn_dense) / (out["dense"] * 1e-3) / 1e12,
        "prefill_32_layers_ms": {"s2o": 32 * out["s2o"], "dense": 32 * out["dense"]},
        "peak_bf16_tflops": peak,
    }}
    print(json.dumps(line), flush=True)
    return 0


def run_gemm(args):
    """The decoder layer's projection GEMM alone (not the headline line): C = A·B (+ C) for one
    shape, bf16 with fp32 accumulation, CUDA events; one JSON line."""
    import long_context_sparse_stripe_b200 as s2o

    torch.cuda.set_device(0)
    m, n, k = (int(x) for x in args.gemm.split(","))
    g = torch.Generator(device="cuda").manual_seed(0)
    a = torch.randn(m, k, device="cuda", generator=g).to(torch.bfloat16)
    b = (torch.randn(k, n, device="cuda", generator=g) / k ** 0.5).to(torch.bfloat16)
    c = torch.empty(m, n, device="cuda", dtype=torch.bfloat16)
    for _ in range(args.warmup):
        s2o.gemm_bf16(a, b, c, accumulate=args.accumulate)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        s2o.gemm_bf16(a, b, c, accumulate=args.accumulate)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    tflops = 2.0 * m * n * k / (ms * 1e-3) / 1e12
    peak = measured_peaks()[0]
    print(json.dumps({"gemm": {"m": m, "n": n, "k": k, "accumulate": args.accumulate, "ms": ms,
                               "tflops": tflops, "frac_of_measured_peak": tflops / peak,
                               "status": s2o.check_device_status()}}), flush=True)
    return 0


def run_profile_target(args):
    """A short fixed sequence for profiler captures (not a bench line): one index build, then
    `--steps` attention calls and one dense-baseline call. Without `--ws-mode` each call is the
    path without a workspace (the local pass, then the permuted pass); with it, a call with a
    prefill workspace in that permuted-copy mode launches, in order, the merge path's permuted
    pass (gathered), its packed form, the merging local pass, the plain local pass and the plain
    permuted pass, of which the device-side decision lets one path run."""
    import long_context_sparse_stripe_b200 as s2o

    torch.cuda.set_device(0)
    # A profiler replays each captured launch dozens of times with instrumented counter passes;
    # an instrumented pass can stretch the attention kernel's in-kernel waits far beyond their
    # normal microseconds, so the bound on each wait is raised for captures.
    s2o.set_wait_limit_ns(60_000_000_000)
    w = gen.workload(args.workload, tau=args.tau)
    if args.heads:
        hq, hkv = (int(x) for x in args.heads.split(","))
        w = w.replace(n_q_heads=hq, n_kv_heads=hkv)
    q, k, v = (t.cuda() for t in gen.make_inputs(w))
    cfg = s2o.Config.of(w)
    idx = s2o.build_indices(cfg, q, k)
    o = torch.empty_like(q)
    ws = None
    if args.ws_mode >= 0:
        s2o.set_permuted_copy(args.ws_mode)
        ws = s2o.alloc_prefill_workspace(cfg)
    for _ in range(args.steps):
        if ws is None:
            s2o.attention_prefill_with_indices(cfg, q, k, v, idx, out=o)
        else:
            s2o.attention_prefill_with_indices_ws(cfg, q, k, v, idx, ws, out=o)
    s2o.dense_causal_prefill(cfg, q, k, v, out=o)
    torch.cuda.synchronize()
    if s2o.check_device_status() != 0:
        raise RuntimeError("device timeout")
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="s2o", choices=["s2o", "reference"])
    ap.add_argument("--parallel", default="replica", choices=["replica", "heads"],
                    help="N > 1: an independent layer per GPU (replica, weak scaling) or one "
                         "layer split by KV head (heads, strong scaling)")
    ap.add_argument("--tau", type=float, default=0.01)
    ap.add_argument("--workload", default=WORKLOAD, choices=sorted(gen.WORKLOADS),
                    help="bench lines use the default; smaller workloads serve profiling")
    ap.add_argument("--dense-steps", type=int, default=2)
    ap.add_argument("--e2e-steps", type=int, default=12)
    ap.add_argument("--ref-rows", type=int, default=2048)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ws-mode", type=int, default=-1,
                    help="profile target only: call with a prefill workspace in this mode")
    ap.add_argument("--heads", default="",
                    help="profile target only: 'Hq,Hkv' (the first KV groups of the workload)")
    ap.add_argument("--sweep", action="store_true",
                    help="per-configuration report (one JSON line per configuration)")
    ap.add_argument("--sweep-filter", default="",
                    help="sweep only: comma-separated 'workload@tau' prefixes (and 'stack')")
    ap.add_argument("--layer", action="store_true",
                    help="end-to-end-shaped decoder layer, S2O vs dense attention (one JSON line)")
    ap.add_argument("--gemm", default="",
                    help="'M,N,K': time the decoder layer's projection GEMM alone (one JSON line)")
    ap.add_argument("--accumulate", action="store_true", help="--gemm: C += A·B")
    ap.add_argument("--profile-target", action="store_true",
                    help="run a short fixed call sequence for profiler captures; print nothing")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "s2o":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.gemm:
        return run_gemm(args)
    if args.profile_target:
        return run_profile_target(args)
    if args.sweep:
        return run_sweep(args)
    if args.layer:
        return run_layer(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_s2o(args)


if __name__ == "__main__":
    sys.exit(main())
