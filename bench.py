#!/usr/bin/env python
"""Decode-step throughput of the Self-Indexing KVCache hot path on B200.

One step = one sikv_decode (compressed-domain LUT-GEMV scoring, exact top-k,
fused dequant + sparse attention over 64 sinks + k selected tokens) of a
whole batch, with the query redrawn every step.  Default workload: batch 4,
32 query / 8 KV heads, head_dim 128, 131072 cached tokens per sequence,
k = 2048 (bf16 K/V, fp32 arithmetic).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl sikv|reference]

Prints one JSON line (rank 0).  Timing: K steps captured in one CUDA graph and
timed with CUDA events on the launching stream, barrier + synchronize on both
sides, max over ranks.  No step finds its inputs in L2: the encoded cache is
replicated R times (R * bytes-per-step > 2 * L2) and step i reads replica
i mod R.  Multi-GPU runs shard the sequences (weak scaling, no collective on
the data path): every rank decodes its own batch.
"""

from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import sikv_inputs as gen  # noqa: E402

METRIC = "decode steps/s at 128K ctx (sparse attn+scoring); achieved HBM GB/s vs peak"
UNIT = "decode steps/s"
PROFILED = {
    "score": ("score_kernel_long_context_b4_n131072.md", ("score_device.cuh", "score.cu", "sikv_common.cuh")),
    "decode_fused": ("decode_fused_kernel_long_context_b4_n131072.md",
                     ("score_device.cuh", "decode_common.cuh", "decode_fused.cu", "sikv_common.cuh")),
    "decode_cluster": ("decode_cluster_kernel_long_context_b4_n131072.md",
                       ("score_device.cuh", "decode_common.cuh", "decode_cluster.cu", "sikv_common.cuh")),
}
KERNEL_OF_PATH = {1: ("decode_cluster", "decode_cluster_kernel (score + top-k + sparse attention, one cluster "
                                        "per segment)"),
                  2: ("decode_fused", "decode_fused_kernel (score + top-k + sparse attention, cooperative)")}


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2560)
    ap.add_argument("--warmup", type=int, default=16)
    ap.add_argument("--impl", choices=("sikv", "reference"), default="sikv")
    ap.add_argument("--config", type=int, default=2, help="workload index (2: B=4, N=131072)")
    ap.add_argument("--replicas", type=int, default=0, help="cache replicas (0: enough to defeat L2)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="oracle CPU-baseline budget")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extreme-encode", action="store_true", help="skip the 512K-key encoder leg")
    ap.add_argument("--no-all-core-oracle", action="store_true", help="skip the all-core oracle figure")
    return ap.parse_args(argv)


# ----------------------------------------------------------------------------
# workload arithmetic (bytes per step, the roofline numerator)
# ----------------------------------------------------------------------------

def step_bytes(w: gen.Workload, value_row_bytes: int | None = None) -> int:
    """Algorithmic HBM bytes of one decode step.

    Per (sequence, KV head): the n = N - S code rows (16 B each), the k
    selected value rows (D x 2 B, or ``value_row_bytes`` each when they are
    read as 2-bit rows), the S sink key and value rows, and the 8 KB codebook.
    """
    eb = 4 if w.dtype == "f32" else 2
    vrow = w.head_dim * eb if value_row_bytes is None else value_row_bytes
    tot = 0
    for b in range(w.batch):
        n = max(w.seq_lens[b] - w.num_sinks, 0)
        s = min(w.num_sinks, w.seq_lens[b])
        per_head = 16 * n + w.topk[b] * vrow + s * 2 * w.head_dim * eb + 32 * 16 * 4 * 4
        tot += per_head * w.num_kv_heads
    return tot


def score_bytes(w: gen.Workload) -> int:
    """Algorithmic bytes of the scoring kernel: code rows read, codebook read, fp32 scores written."""
    tot = 0
    for b in range(w.batch):
        n = max(w.seq_lens[b] - w.num_sinks, 0)
        tot += (16 * n + 4 * w.seq_lens[b] + 8192) * w.num_kv_heads
    return tot


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "MEASURED_PEAKS.json"
    except (OSError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}, "fallback"


def kernel_source_hash(kernel: str) -> str:
    h = hashlib.sha256()
    for name in PROFILED[kernel][1]:
        with open(os.path.join(ROOT, "long_context_decode_sikv_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str):
    """DRAM bytes per launch of a kernel from its committed ncu summary.

    Returns None when the summary is missing or was taken on different kernel
    sources than the ones being timed.
    """
    path = os.path.join(ROOT, "profiles", PROFILED[kernel][0])
    try:
        txt = open(path).read()
    except OSError:
        return None
    vals = {}
    for line in txt.splitlines():
        if line.startswith("- bench_traffic_"):
            k, _, v = line[2:].partition(":")
            vals[k.strip()] = v.strip()
    if vals.get("bench_traffic_source_hash") != kernel_source_hash(kernel):
        return None
    try:
        return float(vals["bench_traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


# ----------------------------------------------------------------------------
# clocks during the timed region (NVML reads only)
# ----------------------------------------------------------------------------

class ClockSampler:
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting"}

    def __init__(self, torch_device):
        self.samples, self.reasons, self.ok = [], set(), False
        self.max_mhz = None
        self._stop = threading.Event()
        try:
            import pynvml
            import torch

            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(torch_device)
            handle = None
            uuid = getattr(props, "uuid", None)
            if uuid is not None:
                try:
                    handle = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + str(uuid)).encode())
                except Exception:
                    handle = None
            if handle is None:
                vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
                ids = [x for x in vis.split(",") if x.strip()]
                idx = int(ids[torch_device.index]) if ids and ids[torch_device.index].strip().isdigit() \
                    else torch_device.index
                handle = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.nv, self.h = pynvml, handle
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report it instead of clocks
            self.err = repr(e)

    def _run(self):
        nv = self.nv
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = get_reasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "NVML unavailable"}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ----------------------------------------------------------------------------
# distributed plumbing
# ----------------------------------------------------------------------------

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def shard_workload(w: gen.Workload, rank: int) -> gen.Workload:
    """Rank r decodes its own batch of sequences (independent seeds)."""
    from dataclasses import replace

    return w if rank == 0 else replace(w, seed=w.seed + 1000 * rank, name=w.name)


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device="cuda" if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


# ----------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline leg and the reference arm)
# ----------------------------------------------------------------------------

def oracle_decode_seconds(w: gen.Workload, budget_s: float, max_iters: int, token_frac: float = 1.0):
    """Time the oracle's decode step on one (sequence 0, KV head 0) segment.

    Returns (seconds per whole-batch step, description of the sample, threads).
    The oracle is O(n) in the scored tokens, so a prefix sample of
    ``token_frac`` of the segment is scaled back by 1 / token_frac, and one
    segment is scaled to all B * Hkv segments of the step.
    """
    import oracle
    from threadpoolctl import threadpool_limits

    hi = gen.head_inputs(w, 0, 0)
    n_full = w.seq_lens[0]
    n_tok = max(w.num_sinks + 1, int(round(w.num_sinks + token_frac * (n_full - w.num_sinks))))
    frac = (n_tok - w.num_sinks) / max(n_full - w.num_sinks, 1)
    K = gen.storage_to_f64(hi.keys[:n_tok], w.dtype)
    V = gen.storage_to_f64(hi.values[:n_tok], w.dtype)
    mu, code, cent, _ = oracle.encode_keys(K, w.num_sinks)
    k = max(1, int(round(w.topk[0] * frac)))
    k = min(k, n_tok - w.num_sinks)
    times = []
    with threadpool_limits(limits=1):
        t_end = time.perf_counter() + budget_s
        for it in range(max_iters):
            q = gen.storage_to_f64(gen.head_queries(w, 0, 0, it, hi.mean_dir), w.dtype)
            t0 = time.perf_counter()
            oracle.decode_step(q, K, V, mu, cent, code, k, w.num_sinks)
            times.append(time.perf_counter() - t0)
            if time.perf_counter() > t_end and len(times) >= 2:
                break
    per_seg = statistics.mean(times) / frac
    desc = (f"oracle decode_step (fp64 numpy, 1 thread) on sequence 0 / KV head 0 of the workload, "
            f"{len(times)} query draws over {n_tok - w.num_sinks} of {n_full - w.num_sinks} scored tokens "
            f"(k={k}), scaled by tokens and by the {w.segments} segments of a step")
    return per_seg * w.segments, desc, 1, times


def _oracle_steps_worker(cfg, segs, warmup, steps, start, results):
    """One worker process of the whole-step oracle run: regenerates and
    encodes its segments (not timed), then decodes them for every step with
    that step's query, single-threaded, timing the ``steps`` steps after the
    common start barrier."""
    import oracle
    from threadpoolctl import threadpool_limits

    w = gen.config(cfg)
    data = []
    for (b, h) in segs:
        hi = gen.head_inputs(w, b, h, steps=tuple(range(warmup + steps)))
        K = gen.storage_to_f64(hi.keys, w.dtype)
        V = gen.storage_to_f64(hi.values, w.dtype)
        mu, code, cent, _ = oracle.encode_keys(K, w.num_sinks)
        qs = [gen.storage_to_f64(hi.queries[i], w.dtype) for i in range(warmup + steps)]
        data.append((K, V, mu, code, cent, qs, w.topk[b]))
    with threadpool_limits(limits=1):
        for i in range(warmup):
            for (K, V, mu, code, cent, qs, k) in data:
                oracle.decode_step(qs[i], K, V, mu, cent, code, k, w.num_sinks)
        start.wait()
        t0 = time.perf_counter()
        for i in range(warmup, warmup + steps):
            for (K, V, mu, code, cent, qs, k) in data:
                oracle.decode_step(qs[i], K, V, mu, cent, code, k, w.num_sinks)
        results.put(time.perf_counter() - t0)


def oracle_whole_steps(cfg: int, steps: int, warmup: int, max_workers: int | None = None):
    """The oracle on whole decode steps (every segment of the batch, the query
    redrawn every step), its segments spread over spawned worker processes,
    one single-threaded worker per available core (at most one per segment).

    Returns (seconds per step, workers, description).  The step time is the
    slowest worker's time over the timed steps divided by their number: a
    step is done when its last segment is."""
    import multiprocessing as mp

    w = gen.config(cfg)
    cores = len(os.sched_getaffinity(0))
    segs = [(b, h) for b in range(w.batch) for h in range(w.num_kv_heads)]
    workers = max(1, min(cores, len(segs), max_workers or len(segs)))
    parts = [segs[i::workers] for i in range(workers)]
    ctx = mp.get_context("spawn")
    start = ctx.Barrier(workers)
    results = ctx.Queue()
    procs = [ctx.Process(target=_oracle_steps_worker, args=(cfg, part, warmup, steps, start, results))
             for part in parts]
    for pr in procs:
        pr.start()
    elapsed = [results.get() for _ in procs]
    for pr in procs:
        pr.join()
    per_step = max(elapsed) / steps
    desc = (f"oracle decode_step (fp64 numpy, single-threaded per process) on whole steps: all "
            f"{len(segs)} (sequence, KV head) segments of the workload, {steps} timed steps after {warmup} "
            f"warm-up, queries redrawn every step; segments spread over {workers} worker processes "
            f"({cores} cores available)")
    return per_step, workers, desc


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    w = gen.config(args.config)
    steps, warmup = max(1, args.steps), max(0, min(args.warmup, 2))
    per_step, workers, desc = oracle_whole_steps(args.config, steps, warmup)
    value = 1.0 / per_step
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1, "steps": steps,
        "warmup": warmup, "ms_per_step": per_step * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, replicas=0),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": workers, "kind": "oracle", "sample": desc,
                         "cores_available": len(os.sched_getaffinity(0))},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w: gen.Workload, replicas: int) -> dict:
    return {"workload": w.name, "batch": w.batch, "q_heads": w.num_q_heads, "kv_heads": w.num_kv_heads,
            "head_dim": w.head_dim, "seq_len": w.max_seq_len, "topk": w.max_topk, "sinks": w.num_sinks,
            "io_dtype": w.dtype, "queries": "redrawn every step",
            "l2": (f"{replicas} rotating replicas of the encoded cache; step i reads replica i mod {replicas}, "
                   f"so each step's inputs were last touched >2x L2 bytes earlier") if replicas else None}


# ----------------------------------------------------------------------------
# the CUDA arm
# ----------------------------------------------------------------------------

def run_sikv(args):
    import torch

    import long_context_decode_sikv_b200 as sk

    rank, world, local = dist_env()
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)

    w = shard_workload(gen.config(args.config), rank)
    bt = gen.make_batch(w, steps=(0,))
    p = sk.make_params(w.dtype, w.batch, w.num_q_heads, w.num_kv_heads, w.max_seq_len, w.num_sinks, w.max_topk)
    K = sk.to_device(bt.K, w.dtype, dev)
    V = sk.to_device(bt.V, w.dtype, dev)
    seq = torch.from_numpy(bt.seq_lens).to(dev)
    kk = torch.from_numpy(bt.topk).to(dev)
    dirs = bt.mean_dirs
    del bt

    # prefill encoder (timed on its own, reported as an extra)
    base = sk.SikvCache(p, K, V, seq)
    base.encode()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(3):
        base.encode()
    e1.record()
    torch.cuda.synchronize()
    enc_ms = e0.elapsed_time(e1) / 3
    base.check()
    k_bytes = K.numel() * K.element_size()

    # replicas of the encoded cache so that no step's inputs sit in L2
    sb = step_bytes(w)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    R = args.replicas or max(2, math.ceil(2 * l2 / sb) + 1)
    reps = [base]
    for _ in range(R - 1):
        c = sk.SikvCache(p, K.clone(), V.clone(), seq)
        c.mu.copy_(base.mu)
        c.codes.copy_(base.codes)
        c.codebook.copy_(base.codebook)
        reps.append(c)
    ws = base.ws_decode

    # queries redrawn every step
    total = args.warmup + args.steps
    qs_host = np.stack([gen.step_queries(w, s, dirs) for s in range(total)])
    qs = sk.to_device(qs_host, w.dtype, dev)
    out = torch.empty((w.batch, w.num_q_heads, w.head_dim), dtype=p.torch_dtype, device=dev)
    scores = torch.empty((w.batch, w.num_kv_heads, w.max_seq_len), dtype=torch.float32, device=dev)
    idx = torch.empty((w.batch, w.num_kv_heads, w.max_topk), dtype=torch.int32, device=dev)

    def decode_step(i):
        c = reps[i % R]
        sk.sikv_decode(p, qs[i], c.K, c.V, c.codes, c.codebook, c.mu, seq, kk, out, workspace=ws)

    def score_only(i):
        c = reps[i % R]
        sk.sikv_score(p, qs[i], c.codes, c.codebook, c.mu, seq, scores, workspace=ws)

    def topk_only(i):
        sk.sikv_topk(p, scores, seq, kk, idx, workspace=ws)

    def attn_only(i):
        c = reps[i % R]
        sk.sikv_sparse_attn(p, qs[i], c.K, c.V, c.codes, c.codebook, c.mu, idx, kk, seq, out, workspace=ws)

    stream = torch.cuda.Stream(device=dev)

    def graph_of(fn, lo, hi):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(lo, hi):
                fn(i)
        return g

    def timed(g):
        barrier(world)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            a.record(stream)
            g.replay()
            b.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        return a.elapsed_time(b)

    # warm-up (eager, also sets kernel attributes before capture)
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            decode_step(i)
    torch.cuda.synchronize()
    ws.check()

    g_dec = graph_of(decode_step, args.warmup, total)
    sampler = ClockSampler(dev)
    with sampler:
        reps_ms = [max_over_ranks(timed(g_dec), world) for _ in range(5)]
    ws.check()
    ms = statistics.median(reps_ms)
    del g_dec
    # the graph's last step left its output in `out`: an eager call on the
    # same query and replica must give the same bytes
    graph_out = out.clone()
    with torch.cuda.stream(stream):
        decode_step(total - 1)
    torch.cuda.synchronize()
    last_step_identical = bool(torch.equal(graph_out, out))

    # the other single-launch kernel on the same steps, for comparison
    resolved = int(sk.lib().sikv_decode_resolved_path(ctypes.byref(p)))
    alt_ms, alt_name = None, None
    alt_path = 2 if resolved == 1 else (1 if resolved == 2 else 0)
    if alt_path:
        p_alt = sk.make_params(w.dtype, w.batch, w.num_q_heads, w.num_kv_heads, w.max_seq_len, w.num_sinks,
                               w.max_topk, decode_path=alt_path)
        if int(sk.lib().sikv_decode_resolved_path(ctypes.byref(p_alt))) == alt_path:
            def alt_step(i):
                c = reps[i % R]
                sk.sikv_decode(p_alt, qs[i], c.K, c.V, c.codes, c.codebook, c.mu, seq, kk, out, workspace=ws)

            with torch.cuda.stream(stream):
                for i in range(args.warmup):
                    alt_step(i)
            g = graph_of(alt_step, args.warmup, total)
            alt_ms = max_over_ranks(timed(g), world)
            alt_name = KERNEL_OF_PATH[alt_path][0]
            del g
            ws.check()

    # per-kernel breakdown over the same steps (dominant kernel timed live)
    torch.cuda.synchronize()
    g = graph_of(score_only, args.warmup, total)
    ms_score = max_over_ranks(timed(g), world)
    del g
    g = graph_of(topk_only, args.warmup, total)
    ms_topk = max_over_ranks(timed(g), world)
    del g
    g = graph_of(attn_only, args.warmup, total)
    ms_attn = max_over_ranks(timed(g), world)
    del g
    ws.check()

    # comparison baselines on the same workload and replicas (not the method):
    # full-precision scoring of every token and dense attention over every token
    n_cmp = min(args.steps, 32)
    dout = torch.empty_like(out)
    ws_dscore = sk.Workspace(256, dev, stream)
    ws_dattn = sk.Workspace(sk.workspace_size("dense_attn", p), dev, stream)

    def dense_score_only(i):
        c = reps[i % R]
        sk.sikv_dense_score(p, qs[i], c.K, seq, scores, workspace=ws_dscore, stream=stream)

    def dense_attn_only(i):
        c = reps[i % R]
        sk.sikv_dense_attn(p, qs[i], c.K, c.V, seq, dout, workspace=ws_dattn, stream=stream)

    with torch.cuda.stream(stream):
        for i in range(2):
            dense_score_only(i)
            dense_attn_only(i)
    g = graph_of(dense_score_only, args.warmup, args.warmup + n_cmp)
    us_dscore = 1e3 * max_over_ranks(timed(g), world) / n_cmp
    del g
    g = graph_of(dense_attn_only, args.warmup, args.warmup + n_cmp)
    us_dattn = 1e3 * max_over_ranks(timed(g), world) / n_cmp
    del g
    ws_dscore.check()
    ws_dattn.check()
    kv_bytes = K.numel() * K.element_size()
    comparison = {
        "note": "own dense kernels on the same GPU and replicas; not the method",
        "dense_score_us": us_dscore, "lut_score_us": 1e3 * ms_score / args.steps,
        "retrieval_speedup_lut_vs_dense": us_dscore / (1e3 * ms_score / args.steps),
        "dense_attention_us": us_dattn, "sikv_decode_us": 1e3 * ms / args.steps,
        "decode_speedup_sikv_vs_dense_attention": us_dattn / (1e3 * ms / args.steps),
        "dense_attention_GB_per_s": 2 * kv_bytes / (us_dattn / 1e6) / 1e9,
        "dense_score_GB_per_s": kv_bytes / (us_dscore / 1e6) / 1e9,
        # the same ratios against the dense kernels' HBM bound (all of K, or of
        # K and V, read once at the measured copy peak): independent of how
        # good the dense kernels are
        "dense_attention_roofline_us": 2 * kv_bytes / (float(measured_peaks()[0]["hbm_gbs"]) * 1e3),
        "decode_speedup_sikv_vs_dense_attention_roofline":
            2 * kv_bytes / (float(measured_peaks()[0]["hbm_gbs"]) * 1e3) / (1e3 * ms / args.steps),
        "dense_score_roofline_us": kv_bytes / (float(measured_peaks()[0]["hbm_gbs"]) * 1e3),
        "retrieval_speedup_lut_vs_dense_score_roofline":
            kv_bytes / (float(measured_peaks()[0]["hbm_gbs"]) * 1e3) / (1e3 * ms_score / args.steps),
    }

    # 2-bit values: the same steps with the selected tokens' values read from
    # 48-byte 2-bit rows (sinks keep full precision); not the headline, whose
    # values stay in the storage dtype
    for c in reps:
        c.quantize_values(stream=stream)
    torch.cuda.synchronize()

    def decode_qv_step(i):
        c = reps[i % R]
        sk.sikv_decode_qv(p, qs[i], c.K, c.V, c.vq, c.codes, c.codebook, c.mu, seq, kk, out, workspace=ws,
                          stream=stream)

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            decode_qv_step(i)
    torch.cuda.synchronize()
    g = graph_of(decode_qv_step, args.warmup, total)
    ms_qv = max_over_ranks(timed(g), world)
    del g
    ws.check()
    sb_qv = step_bytes(w, value_row_bytes=48)
    values_2bit = {
        "decode_us": 1e3 * ms_qv / args.steps, "steps_per_s": world * args.steps / (ms_qv / 1e3),
        "algorithmic_bytes_per_step": sb_qv, "GB_per_s": sb_qv / (ms_qv / 1e3 / args.steps) / 1e9,
        "frac_of_hbm": sb_qv / (ms_qv / 1e3 / args.steps) / 1e9 / float(measured_peaks()[0]["hbm_gbs"]),
        "value_bytes_per_selected_token": 48,
        "note": "selected tokens' V as 2-bit rows (groups of 32 channels, fp16 min and step); sinks in bf16",
    }
    for c in reps:
        c.vq = None

    # clustering: the one-pass sign-pattern codebook (the whole prefill
    # encoder, mean pass included) against 20 Lloyd's k-means iterations on the
    # same points (mean given), both on this GPU with this library's kernels
    init = torch.from_numpy(gen.kmeans_init(w, w.seq_lens)).to(dev)
    km_codes, km_cb, km_cnt = torch.empty_like(base.codes), torch.empty_like(base.codebook), torch.empty_like(base.counts)
    ws_km = sk.Workspace(sk.workspace_size("kmeans", p), dev, stream)

    def kmeans20():
        sk.sikv_kmeans_codebook(p, K, seq, base.mu, init, km_codes, km_cb, km_cnt, iters=20, workspace=ws_km,
                                stream=stream)

    with torch.cuda.stream(stream):
        kmeans20()
    torch.cuda.synchronize()
    barrier(world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        a.record(stream)
        for _ in range(2):
            kmeans20()
        b.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    km_ms = max_over_ranks(a.elapsed_time(b), world) / 2
    ws_km.check()
    # bound-based: per k-means iteration the assignment reads K and writes the
    # codes, the accumulation reads K and the codes; the one-pass encoder
    # reads K twice (mean, then codes and cluster sums) and writes the codes
    kb, cb_ = K.numel() * K.element_size(), base.codes.numel()
    hbm = float(measured_peaks()[0]["hbm_gbs"]) * 1e9
    km_bound_ms = 20 * (2 * kb + 2 * cb_) / hbm * 1e3
    enc_bound_ms = (2 * kb + cb_) / hbm * 1e3
    comparison.update({
        "kmeans20_roofline_ms": km_bound_ms, "one_pass_encode_roofline_ms": enc_bound_ms,
        "clustering_speedup_roofline": km_bound_ms / enc_bound_ms,
        "one_pass_encode_ms": enc_ms, "kmeans20_ms": km_ms,
        "clustering_speedup_one_pass_vs_kmeans20": km_ms / enc_ms,
        "kmeans_iteration_us": 1e3 * km_ms / 20,
        "kmeans_iteration_key_GB_per_s": K.numel() * K.element_size() / (km_ms / 20 / 1e3) / 1e9,
    })
    del km_codes, km_cb, km_cnt, ws_km

    # end to end through the public API: every step is one
    # sikv_decode_host_plan_run call (a DecodeHostPlan per cache replica,
    # created before the timed region) on that step's query and output in
    # page-locked host memory; each call copies the query in over the host
    # link, decodes, and copies the output back
    e2e = None
    if not args.no_e2e:
        qh = torch.from_numpy(qs_host.view(np.int16) if w.dtype == "bf16" else qs_host)
        qh = (qh.view(torch.bfloat16) if w.dtype == "bf16" else qh).pin_memory()
        oh = torch.empty((total,) + tuple(out.shape), dtype=out.dtype).pin_memory()
        ws_host = sk.Workspace(sk.workspace_size("decode_host", p), dev, stream)
        plans = [sk.DecodeHostPlan(p, c.K, c.V, c.codes, c.codebook, c.mu, seq, kk, workspace=ws_host, stream=stream)
                 for c in reps]
        for i in range(args.warmup):
            plans[i % R](qh[i], oh[i])
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            a.record(stream)
            for i in range(args.warmup, total):
                plans[i % R](qh[i], oh[i])
            b.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        ms_e2e = max_over_ranks(a.elapsed_time(b), world)
        ws_host.check()
        e2e = {"value": world * args.steps / (ms_e2e / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": int(qh[0].numel() * qh.element_size()),
               "d2h_bytes_per_step": int(oh[0].numel() * oh.element_size()),
               "api": "sikv_decode_host_plan_run (C ABI) on page-locked host buffers, one call per step: "
                      "a graph captured at plan creation (query copy kernel, decode, output copy kernel) "
                      "re-pointed at the step's buffers and launched"}

    # prefill encoder at the extreme-context shape (B=1, 32/8 heads, 512K keys
    # per head, the same generator with drift): keys encoded per second over
    # all 512K x 8 keys, and GB/s over its algorithmic bytes (two reads of K
    # plus the code rows written)
    encode_extreme = None
    if args.config == 2 and world == 1 and not args.no_extreme_encode:
        from concurrent.futures import ThreadPoolExecutor

        del reps, base, K, V
        torch.cuda.empty_cache()
        w4 = gen.config(4)
        n4 = w4.max_seq_len
        with ThreadPoolExecutor(min(8, os.cpu_count() or 1)) as ex:
            keys = list(ex.map(lambda h: gen.head_inputs(w4, 0, h).keys, range(w4.num_kv_heads)))
        K4 = sk.to_device(np.stack(keys)[None], w4.dtype, dev)
        del keys
        p4 = sk.make_params(w4.dtype, 1, w4.num_q_heads, w4.num_kv_heads, n4, w4.num_sinks, w4.max_topk)
        c4 = sk.SikvCache(p4, K4, K4, torch.full((1,), n4, dtype=torch.int32, device=dev))
        c4.encode()
        torch.cuda.synchronize()
        a4, b4 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a4.record()
        for _ in range(3):
            c4.encode()
        b4.record()
        torch.cuda.synchronize()
        c4.check()
        ms4 = a4.elapsed_time(b4) / 3
        keys4 = w4.num_kv_heads * n4
        bytes4 = 2 * K4.numel() * K4.element_size() + c4.codes.numel()
        encode_extreme = {"workload": w4.name, "keys": keys4, "ms": ms4, "keys_per_s": keys4 / (ms4 / 1e3),
                          "GB_per_s": bytes4 / (ms4 / 1e3) / 1e9,
                          "frac_of_hbm": bytes4 / (ms4 / 1e3) / 1e9 / float(measured_peaks()[0]["hbm_gbs"]),
                          "algorithmic_bytes": bytes4,
                          "note": "mean, sign codes and one-pass codebook of every key (sikv_encode_keys)"}
        del c4, K4
        torch.cuda.empty_cache()

    peaks, peak_src = measured_peaks()
    peak = float(peaks["hbm_gbs"])
    score_launch_s = ms_score / 1e3 / args.steps
    score_gbs = score_bytes(w) / score_launch_s / 1e9
    step_s = ms / 1e3 / args.steps
    step_gbs = sb / step_s / 1e9
    launches = int(sk.lib().sikv_decode_launches(ctypes.byref(p)))
    if launches == 1 and resolved in KERNEL_OF_PATH:
        # one single-launch kernel per step: the timed graph holds exactly one
        # launch per step, so its average duration is the step time
        kname, kdesc = KERNEL_OF_PATH[resolved]
        roofline = {"bound": "hbm", "kernel": kdesc,
                    "achieved": step_gbs, "peak": peak, "unit": "GB/s", "frac": step_gbs / peak,
                    "traffic": profiled_traffic(kname), "algorithmic_bytes_per_launch": sb,
                    "peak_source": f"{peak_src} hbm_gbs (copy, of measured)"}
    else:
        roofline = {"bound": "hbm", "kernel": "score_kernel (LUT-GEMV scoring)", "achieved": score_gbs,
                    "peak": peak, "unit": "GB/s", "frac": score_gbs / peak, "traffic": profiled_traffic("score"),
                    "algorithmic_bytes_per_launch": score_bytes(w),
                    "peak_source": f"{peak_src} hbm_gbs (copy, of measured)"}

    line = {
        "metric": METRIC, "value": world * args.steps / (ms / 1e3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": workload_config(w, R),
        "roofline": roofline,
        "score_kernel_roofline": {"achieved": score_gbs, "peak": peak, "unit": "GB/s", "frac": score_gbs / peak,
                                  "algorithmic_bytes_per_launch": score_bytes(w)},
        "step_roofline": {"achieved": step_gbs, "peak": peak, "unit": "GB/s", "frac": step_gbs / peak,
                          "frac_of_8000_nominal": step_gbs / 8000.0,
                          "algorithmic_bytes_per_step": sb,
                          "formula": "per (seq, kv head): 16*(N-S) code bytes + k*D*2 V bytes + S*2*D*2 sink "
                                     "K/V bytes + 8 KB codebook"},
        "timed_replays": {"runs": len(reps_ms), "ms_per_step_median": ms / args.steps,
                          "ms_per_step_min": min(reps_ms) / args.steps, "ms_per_step_max": max(reps_ms) / args.steps,
                          "last_step_output_identical_to_eager_call": last_step_identical},
        "breakdown_us_per_step": {"decode": 1e3 * ms / args.steps, "score": 1e3 * ms_score / args.steps,
                                  "topk": 1e3 * ms_topk / args.steps, "sparse_attn": 1e3 * ms_attn / args.steps,
                                  **({f"decode_{alt_name}": 1e3 * alt_ms / args.steps} if alt_ms else {})},
        "encode": {"ms": enc_ms, "keys_per_s": w.batch * w.num_kv_heads * w.max_seq_len / (enc_ms / 1e3),
                   "GB_per_s_2reads": 2 * k_bytes / (enc_ms / 1e3) / 1e9},
        "comparison": comparison,
        "values_2bit": values_2bit,
        "clocks": sampler.summary(),
        "gpu_launches": launches * args.steps,
        "e2e": e2e,
        "encode_extreme_context": encode_extreme,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        per_step, desc, cores, times = oracle_decode_seconds(w, args.cpu_seconds, 10_000)
        line["cpu_baseline"] = {"value": 1.0 / per_step, "unit": UNIT, "cores": cores, "kind": "oracle",
                                "sample": desc, "cores_available": len(os.sched_getaffinity(0))}
        if not args.no_all_core_oracle:
            per_all, workers, desc_all = oracle_whole_steps(args.config, steps=2, warmup=1)
            line["cpu_baseline"]["all_cores"] = {"value": 1.0 / per_all, "unit": UNIT, "cores": workers,
                                                 "sample": desc_all}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_sikv(args)


if __name__ == "__main__":
    sys.exit(main())
