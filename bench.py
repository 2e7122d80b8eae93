#!/usr/bin/env python3
"""Benchmark of one CSA2 decode layer-group step (Hierarchical Sparse Indexer
over an FP4 main-KV cache) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl b200|reference]

A step is one pass of the whole decode path over one batch: Full indexer scan,
pool selection, the Full layer's Top-512, the two Reindex layers' Top-512 and
six sparse-attention layers (1 Full + 2 Reindex + 3 Reuse), replayed as one
CUDA graph.  Default workload: 4 decode queries, each over its own
1,048,576-position cache (64 needles per request).  Multi-GPU (torchrun): every
rank owns its own batch of requests (weak scaling, no data-path collective);
timings are the max over ranks.

Rank 0 prints one JSON line.  `value` is queries/s of the whole job with the
cache resident in HBM; `e2e` is the same metric with the step's inputs copied
from pinned host memory and the outputs read back every step; `roofline`
rates the dominant kernel (the Full scan) against the measured copy bandwidth;
`cpu_baseline` times the float64 oracle on a bounded sample.
`--impl reference` times that oracle as the reference arm.

`--workload prefill_256k_q8192` measures the encoder-style causal prefill
chunk instead (8,192 queries over 262,144 m=2 entries: the causal prefill
indexer, then six attention layers over its Top-512); its line rates the
indexer against the FP8 tensor-core peak.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from kv_cache_decode_index_b200 import workloads as W  # noqa: E402

METRIC = "CSA2 decode queries/s per layer group at 1M ctx; achieved HBM GB/s vs 8 TB/s"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
IK_ROW_BYTES = 129     # 128 FP8 codes + 1 exponent byte
IK4_ROW_BYTES = 72     # FP4 indexer: 64 E2M1 code bytes + 8 E4M3 scales
KV_ROW_BYTES = 288     # 256 E2M1 bytes + 32 E4M3 scales
POOL_ENTRY_BYTES = 4


# --------------------------------------------------------------- host logic --

def env_rank():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def rank_workload(wl, rank: int):
    """Each rank serves its own requests: same shapes, its own seeded data."""
    return wl if rank == 0 else W.scaled(wl, seed=wl.seed + 1000 * rank)


def alg_bytes(wl, lengths=None, ik_row_bytes=IK_ROW_BYTES):
    """Algorithmic HBM bytes of one step and of one Full-scan launch.

    Per request: the Full scan reads every visible indexer-K row (129 B); each
    Reindex layer reads the pool's rows (<= 16,384 x 129 B); every layer
    gathers its Top-k main-KV rows (<= 512 x 288 B); the pool is read once per
    selecting layer (2048 x 4 B).  Score / block-max round trips and the
    queries and outputs are implementation traffic and are not counted."""
    n = W.ctx_lengths(wl) if lengths is None else np.asarray(lengths)
    n_ri = sum(1 for m in wl.modes if m == "Ri")
    P = wl.pool_blocks or 0
    cand = np.minimum(n, P * 8) if P else n
    scan = int((ik_row_bytes * n).sum())
    step = scan + int((n_ri * ik_row_bytes * cand).sum()) + \
        int((len(wl.modes) * KV_ROW_BYTES * np.minimum(n, wl.topk)).sum()) + \
        (POOL_ENTRY_BYTES * P * (1 + n_ri) * len(n) if P else 0)
    return step, scan


def append_rows(wl, dev):
    """(kv_new [B,512], ik_new [B,128], pos [B]) of each request's newest row:
    its last visible position, regenerated from the workload's seeds."""
    import torch
    last = W.ctx_lengths(wl) - 1
    kv = np.stack([W.rows_at(wl, b, [last[b]], "kv")[0] for b in range(wl.batch)]).astype(np.float32)
    ik = np.stack([W.rows_at(wl, b, [last[b]], "ik")[0] for b in range(wl.batch)]).astype(np.float32)
    return (torch.from_numpy(kv).to(dev), torch.from_numpy(ik).to(dev),
            torch.from_numpy(last.astype(np.int32)).to(dev))


def io_bytes(wl):
    """Host<->device bytes of one end-to-end step: indexer queries and head
    weights of every non-Reuse layer, main queries (and the appended rows with
    their positions, for workloads with an append) in; attention outputs out."""
    B, H = wl.batch, wl.heads
    n_idx = len(wl.index_layers)
    h2d = n_idx * B * (32 * 128 * 4 + 32 * 4) + len(wl.modes) * B * H * 512 * 2
    if wl.append:
        h2d += B * (512 + 128 + 1) * 4
    d2h = len(wl.modes) * B * H * 512 * 2
    return h2d, d2h


def measured_peak_hbm():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def scan_kernel_hash(fp4=False):
    h = hashlib.sha256()
    names = ("k_index_fp4.cu", "fp4.cuh") if fp4 else ("k_index.cu", "index_common.cuh")
    for name in names + ("scan_units.cuh", "common.cuh"):
        with open(os.path.join(ROOT, "kv_cache_decode_index_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def scan_traffic_per_launch(workload_name, fp4=False):
    """DRAM bytes per Full-scan launch from the committed ncu summary, or None
    when the summary is missing or was taken on a different kernel source."""
    path = os.path.join(ROOT, "profiles", "index_full_fp4_traffic.txt" if fp4 else "index_full_traffic.txt")
    try:
        fields = dict(line.split(":", 1) for line in open(path).read().splitlines() if ":" in line)
    except OSError:
        return None
    if fields.get("kernel_source_hash", "").strip() != scan_kernel_hash(fp4):
        return None
    if fields.get("workload", "").strip() != workload_name:
        return None
    try:
        return float(fields["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clock / throttle sampling (every 200 ms) while the GPU works."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", self.gpu_id], stdout=open(self.path, "w"),
                                         stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        return parse_clock_samples(open(self.path).read())


def parse_clock_samples(text):
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    sm, mx, reasons, n = [], [], set(), 0
    for line in text.splitlines():
        parts = [p.strip() for p in line.split(",")]
        if len(parts) < 9:
            continue
        try:
            sm.append(float(parts[1]))
            mx.append(float(parts[2]))
        except ValueError:
            continue
        n += 1
        for name, flag in zip(names, parts[5:9]):
            if flag.lower() == "active":
                reasons.add(name)
    return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
            "reasons": sorted(reasons), "samples": n}


def describe(wl):
    n = W.ctx_lengths(wl)
    ctx = f"{int(n[0]):,}-position" if len(set(n.tolist())) == 1 else "ragged"
    modes = {"F": 0, "Ri": 0, "Ru": 0}
    for m in wl.modes:
        modes[m] += 1
    pool = f"pool {wl.pool_blocks}x8, " if wl.pool_blocks else "no pool, "
    return (f"{wl.name}: {wl.batch} decode queries x {ctx} contexts, {modes['F']} Full + {modes['Ri']} Reindex + "
            f"{modes['Ru']} Reuse, {pool}Top-{wl.topk}, {wl.heads} heads d512"
            + (f", {wl.needles} needles/request" if wl.needles else ""))


def base_line(args, wl, world, value, ms):
    return {"metric": METRIC, "value": value, "unit": "queries/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "fp8", "data": "synthetic",
            "config": {"workload": describe(wl), "batch_per_gpu": wl.batch, "global_batch": wl.batch * world,
                       "ctx": int(W.ctx_lengths(wl).max()), "page_size": wl.page_size,
                       "parallelism": f"replicas{world}" if world > 1 else "single",
                       "l2": "inputs larger than L2 (the Full scan streams 135 MB of indexer K per query)",
                       "graph": "one CUDA graph per step"}}


# ------------------------------------------------------------ oracle sample --

def oracle_sample(wl, b: int = 0, prepared=None):
    """Time the float64 oracle on one query of the workload: its whole decode
    step (Full scan, pool, Full/Reindex/Reuse Top-512, six attention layers).
    The cache rows are the oracle's own quantisation of the generated rows;
    main-KV rows are prepared for the positions the step gathers."""
    from oracle import csa2 as C
    from oracle import formats as F
    n = int(W.ctx_lengths(wl)[b])
    if prepared is None:
        codes, exp = F.quantize_indexer(W.request_rows(wl, b, n, "ik"))
        q_idx = [None if m == "Ru" else W.index_query(wl, l)[0][b] for l, m in enumerate(wl.modes)]
        w_idx = [None if m == "Ru" else W.index_query(wl, l)[1][b] for l, m in enumerate(wl.modes)]
        q_main = [W.main_query(wl, l)[b].float().numpy() for l in range(len(wl.modes))]
        sel = np.unique(np.concatenate([t[t >= 0] for t in
                                        C.decode_group(wl.modes, q_idx, w_idx, codes, exp, n, wl.pool_blocks,
                                                       wl.topk)["topk"]]))
        kvc = np.zeros((n, 256), np.uint8)
        kvs = np.zeros((n, 32), np.uint8)
        kvc[sel], kvs[sel] = F.quantize_main_kv(W.rows_at(wl, b, sel, "kv"))
        prepared = (codes, exp, q_idx, w_idx, q_main, kvc, kvs, n)
    codes, exp, q_idx, w_idx, q_main, kvc, kvs, n = prepared
    t0 = time.perf_counter()
    out = C.decode_group(wl.modes, q_idx, w_idx, codes, exp, n, wl.pool_blocks, wl.topk)
    for layer in range(len(wl.modes)):
        C.sparse_attention(q_main[layer], kvc, kvs, out["topk"][layer], wl.scale)
    return time.perf_counter() - t0, prepared


def cpu_cores():
    """Threads the oracle's numpy BLAS calls use (the rest of the oracle is
    single-threaded numpy)."""
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        blas = [i["num_threads"] for i in info if i.get("user_api") == "blas"]
        if blas:
            return max(blas)
    except Exception:
        pass
    return 1


def cpu_host():
    """The host the CPU baseline ran on: logical CPUs and the CPU model."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"nproc": os.cpu_count(), "cpu_model": model}


# --------------------------------------------------------------- b200 arm ----

def run_b200(args):
    import torch
    import torch.distributed as dist
    from datetime import timedelta

    rank, world, local = env_rank()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)
    if local == 0:
        from kv_cache_decode_index_b200 import build as _build
        _build.build()
    if world > 1:
        dist.barrier()
    from kv_cache_decode_index_b200 import csa2
    from kv_cache_decode_index_b200.fill import build_cache

    wl = rank_workload(selected_workload(args), rank)
    t0 = time.time()
    fp4 = args.indexer == "fp4"
    cache = build_cache(wl, csa2, fp4_indexer=fp4, append_last=wl.append)
    log(rank, f"cache filled in {time.time() - t0:.1f}s ({cache.kv_codes.numel() * 417 / 256 / 1e9:.2f} GB)")

    q_idx, w_idx, q_main = [], [], []
    for layer, m in enumerate(wl.modes):
        if m == "Ru":
            q_idx.append(None)
            w_idx.append(None)
        else:
            q, w = W.index_query(wl, layer)
            q_idx.append(torch.from_numpy(q).to(dev))
            w_idx.append(torch.from_numpy(w).to(dev))
        q_main.append(W.main_query(wl, layer).to(dev))
    out = [torch.empty_like(m) for m in q_main]
    group = csa2.DecodeGroup(cache, wl.modes, wl.heads, wl.topk, wl.pool_blocks, wl.scale,
                             ik4=cache.ik4 if fp4 else None)
    # workloads with an append: every step first appends each request's newest
    # row (its last position, left out of the filled cache) through the
    # quantise-on-append kernel
    append = append_rows(wl, dev) if wl.append else None

    # ---- warm-up (eager), then capture one step as a graph ----
    for _ in range(args.warmup):
        group.step(q_idx, w_idx, q_main, out, append=append)
    torch.cuda.synchronize()
    # The timed graph has no events between launches (an event between two
    # kernels would cut their programmatic-dependent-launch link); a second
    # graph with events around every launch gives the per-launch durations.
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        group.step(q_idx, w_idx, q_main, out, append=append)
    timing = {name: (torch.cuda.Event(enable_timing=True, external=True),
                     torch.cuda.Event(enable_timing=True, external=True))
              for name in group.launch_names(append is not None)}
    tgraph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(tgraph):
        group.step(q_idx, w_idx, q_main, out, timing=timing, append=append)
    graph.replay()
    tgraph.replay()
    torch.cuda.synchronize()
    st, word = csa2.get_error(cache)
    if st != csa2.OK:
        raise RuntimeError(f"device error during warm-up: {word}")

    gpu_id = torch.cuda.get_device_properties(dev).uuid
    sampler = ClockSampler(f"GPU-{gpu_id}" if not str(gpu_id).startswith("GPU-") else str(gpu_id))
    sampler.start()
    # keep the GPU busy ~0.5 s so the clock sampler sees it under load, then time K steps
    t_busy = time.time()
    while time.time() - t_busy < 0.5:
        for _ in range(50):
            graph.replay()
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        graph.replay()
    e1.record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = e0.elapsed_time(e1) / args.steps
    ms = max_over_ranks(ms, dev, world)

    # ---- launch durations, from events recorded inside the graph on each
    # launch's own stream (one synchronised replay per sample) ----
    per_launch = {name: [] for name in timing}
    for _ in range(args.steps):
        tgraph.replay()
        torch.cuda.synchronize()
        for name, (a, b) in timing.items():
            per_launch[name].append(a.elapsed_time(b))
    scan_ms = per_launch["scan"]
    clocks = sampler.stop()

    # ---- end to end: pinned host inputs -> device, step, outputs -> host ----
    h2d, d2h = io_bytes(wl)
    e2e_value = e2e_serial = None
    if not args.no_e2e:
        piped_ms, serial_ms = e2e_step_ms(args, group, q_idx, w_idx, q_main, out, dev, world, append)
        e2e_value = world * wl.batch / (max_over_ranks(piped_ms, dev, world) / 1e3)
        e2e_serial = world * wl.batch / (max_over_ranks(serial_ms, dev, world) / 1e3)

    st, word = csa2.get_error(cache)
    if st != csa2.OK:
        raise RuntimeError(f"device error during the timed run: {word}")

    step_bytes, scan_bytes = alg_bytes(wl, ik_row_bytes=IK4_ROW_BYTES if fp4 else IK_ROW_BYTES)
    scan_avg_ms = statistics.mean(scan_ms)
    peak, peak_src = measured_peak_hbm()
    achieved = scan_bytes / (scan_avg_ms / 1e3) / 1e9
    traffic = scan_traffic_per_launch(wl.name, fp4)
    if rank == 0:
        value = world * wl.batch / (ms / 1e3)
        line = base_line(args, wl, world, value, ms)
        if fp4:
            line["dtype"] = "fp4"
            line["config"]["indexer"] = "FP4 (E2M1 + E4M3 per 16) indexer K and Q, 72 B/position"
        step_gbs = step_bytes / (ms / 1e3) / 1e9
        line.update({
            "alg_bytes_per_step": step_bytes,
            "step_hbm_gbs": step_gbs,
            "step_frac_of_8tbs": step_gbs / NOMINAL_HBM_GBS,
            "step_frac_of_measured": step_gbs / peak,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                         "traffic": traffic,
                         "kernel": "csa2 index_full_fp4 (Full indexer scan, FP4 indexer K, 72 B/position)" if fp4
                         else "csa2 index_full (Full indexer scan)",
                         "kernel_ms": scan_avg_ms, "alg_bytes_per_launch": scan_bytes,
                         "peak_source": f"{peak_src} copy bandwidth (MEASURED_PEAKS.json hbm_gbs, burst)"},
            "e2e": {"value": e2e_value, "unit": "queries/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "how": "DecodeGroup.step per step; one packed pinned host-to-device copy of all the step's inputs "
                           "and one device-to-host copy of all its outputs every step, inside the timed region; two "
                           "buffer slots and one copy stream per direction overlap step i+1's upload and step i-1's "
                           "download with step i",
                    "serial_value": e2e_serial},
            "gpu_launches": (group.launches_per_step + (0 if append is None else (2 if fp4 else 1))) * args.steps,
            "launch_ms": {name: statistics.mean(v) for name, v in per_launch.items()},
            "clocks": clocks,
        })
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline_entry(wl, fp4)
        print(json.dumps(line), flush=True)
    del graph, tgraph
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


PREFILL_METRIC = "CSA2 causal prefill chunk queries/s (indexer + 6 attention layers); indexer FP8 TFLOP/s"


def prefill_flops(wl):
    """Algorithmic FP8 MMA FLOPs of the prefill indexer: 2 * 32 heads * 128 per
    visible (query, entry) pair."""
    vis = np.minimum((W.prefill_positions(wl).astype(np.int64) + 1) // W.prefill_ratio(wl), wl.ctx)
    return 2.0 * 32 * 128 * float(vis.sum())


def measured_peak_fp8():
    """Dense FP8 tensor peak: the measured cuBLAS bf16 burst x 2 (the nominal
    FP8 : BF16 ratio), else the fallback bf16 figure x 2."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return 2.0 * float(json.load(f)["bf16_tflops"]), "measured bf16 burst x 2 (nominal FP8/BF16 ratio)"
    except (OSError, KeyError, ValueError):
        return 2.0 * 1590.0, "fallback bf16 x 2 (nominal FP8/BF16 ratio)"


def prefill_oracle_sample(wl, n_q: int = 2):
    """Float64 oracle of n_q prefill queries (Top-512 over all visible entries
    plus six attention layers each); returns seconds per query."""
    from oracle import csa2 as C
    from oracle import formats as F
    codes, exp = F.quantize_indexer(W.request_rows(wl, 0, wl.ctx, "ik"))
    q, w = W.index_query(wl, 0, rows=n_q)
    pos = W.prefill_positions(wl)[:n_q]
    qm = [W.main_query(wl, l, rows=n_q).float().numpy() for l in range(len(wl.modes))]
    t0 = time.perf_counter()
    for j in range(n_q):
        t = C.prefill_topk(q[j], w[j], codes, exp, int(pos[j]), wl.topk, W.prefill_ratio(wl))
        kvc, kvs = F.quantize_main_kv(W.rows_at(wl, 0, t, "kv"))
        for layer in range(len(wl.modes)):
            C.sparse_attention(qm[layer][j], kvc, kvs, np.arange(len(t)), wl.scale)
    return (time.perf_counter() - t0) / n_q


def run_prefill(args):
    """The causal prefill chunk: per step, the prefill indexer (FP8 GEMM with
    streaming Top-512) and six attention layers over its Top-512."""
    import torch
    rank, world, local = env_rank()
    if world > 1:
        raise SystemExit("the prefill measurement runs on one GPU")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    from kv_cache_decode_index_b200 import build as _build
    _build.build()
    from kv_cache_decode_index_b200 import csa2
    from kv_cache_decode_index_b200.fill import build_cache

    wl = selected_workload(args)
    cache = build_cache(wl, csa2)
    n = wl.prefill_queries
    pos = torch.from_numpy(W.prefill_positions(wl)).to(dev)
    q, w = W.index_query(wl, 0)
    tq = [torch.from_numpy(q).to(dev)] + [None] * (len(wl.modes) - 1)
    tw = [torch.from_numpy(w).to(dev)] + [None] * (len(wl.modes) - 1)
    qm = [W.main_query(wl, l).to(dev) for l in range(len(wl.modes))]
    out = [torch.empty_like(m) for m in qm]
    group = csa2.PrefillGroup(cache, 0, wl.modes, wl.heads, n, wl.topk, W.prefill_ratio(wl), wl.scale)
    for _ in range(args.warmup):
        group.step(pos, tq, tw, qm, out)
    torch.cuda.synchronize()
    st, word = csa2.get_error(cache)
    if st != csa2.OK:
        raise RuntimeError(f"device error during warm-up: {word}")
    gpu_id = str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(gpu_id if gpu_id.startswith("GPU-") else f"GPU-{gpu_id}")
    sampler.start()
    names = group.launch_names()
    timing = {k: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for k in names}
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    per_launch = {k: [] for k in names}
    step_ms = []
    for _ in range(args.steps):
        torch.cuda.synchronize()
        e0.record()
        group.step(pos, tq, tw, qm, out, timing=timing)
        e1.record()
        torch.cuda.synchronize()
        step_ms.append(e0.elapsed_time(e1))
        for k, (a, b) in timing.items():
            per_launch[k].append(a.elapsed_time(b))
    clocks = sampler.stop()
    st, word = csa2.get_error(cache)
    if st != csa2.OK:
        raise RuntimeError(f"device error during the timed run: {word}")
    ms = statistics.mean(step_ms)
    idx_ms = statistics.mean(per_launch["topk0"])
    flops = prefill_flops(wl)
    peak, peak_src = measured_peak_fp8()
    achieved = flops / (idx_ms / 1e3) / 1e12
    e2e_value = None
    h2d = pos.numel() * 4 + q.nbytes + w.nbytes + sum(t.numel() * 2 for t in qm)
    d2h = n * wl.topk * 4 + sum(t.numel() * 2 for t in out)
    if not args.no_e2e:
        hp, hq, hw = pos.cpu().pin_memory(), tq[0].cpu().pin_memory(), tw[0].cpu().pin_memory()
        hm = [t.cpu().pin_memory() for t in qm]
        ho = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in out]
        hk = torch.empty(n, wl.topk, dtype=torch.int32, pin_memory=True)
        torch.cuda.synchronize()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record()
        for _ in range(args.steps):
            pos.copy_(hp, non_blocking=True)
            tq[0].copy_(hq, non_blocking=True)
            tw[0].copy_(hw, non_blocking=True)
            for dst, src in zip(qm, hm):
                dst.copy_(src, non_blocking=True)
            group.step(pos, tq, tw, qm, out)
            hk.copy_(group.topk[0], non_blocking=True)
            for dst, src in zip(ho, out):
                dst.copy_(src, non_blocking=True)
        a1.record()
        torch.cuda.synchronize()
        e2e_value = n / (a0.elapsed_time(a1) / args.steps / 1e3)
    line = {"metric": PREFILL_METRIC, "value": n / (ms / 1e3), "unit": "queries/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "fp8", "data": "synthetic",
            "config": {"workload": f"{wl.name}: {n} causal prefill queries over {wl.ctx:,} m={W.prefill_ratio(wl)} "
                                   f"entries, 1 Full + {len(wl.modes) - 1} Reuse, Top-{wl.topk}, {wl.heads} heads d512",
                       "parallelism": "single", "l2": "indexer K (34 MB) is L2-resident by design; main KV rows "
                                                     "gathered per query"},
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "traffic": None, "kernel": "csa2 prefill_index (FP8 GEMM + "
                         "streaming Top-512)", "kernel_ms": idx_ms, "flops_per_launch": flops,
                         "peak_source": peak_src},
            "e2e": {"value": e2e_value, "unit": "queries/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "how": "PrefillGroup.step per step; every step copies its inputs (positions, the Full layer's "
                           "indexer query and weights, every layer's main query) from pinned host memory and its "
                           "outputs (the Top-k and every layer's attention output) back, inside the timed region, "
                           "in order on the calling stream"},
            "gpu_launches": group.launches_per_step * args.steps,
            "launch_ms": {k: statistics.mean(v) for k, v in per_launch.items()},
            "clocks": clocks}
    if not args.no_cpu_baseline:
        spq = prefill_oracle_sample(wl)
        line["cpu_baseline"] = {"value": 1.0 / spq, "unit": "queries/s", "cores": cpu_cores(), **cpu_host(), "kind": "oracle",
                                "sample": f"2 of the {n} queries: float64 oracle Top-512 over all visible entries "
                                          f"and six attention layers, {spq:.1f} s per query"}
    print(json.dumps(line), flush=True)


def e2e_step_ms(args, group, q_idx, w_idx, q_main, out, dev, world, append=None):
    """Milliseconds per step end to end through DecodeGroup.step with host
    buffers.  Every step copies all of its inputs from pinned host memory
    (packed: one host-to-device copy) and all of its outputs back (one
    device-to-host copy), inside the timed region.  Two slots of device
    buffers, each with its own captured step, and one copy stream per
    direction let step i+1's upload and step i-1's download overlap step i."""
    import torch
    import torch.distributed as dist
    app = list(append) if append is not None else []
    ins = [t for t in q_idx + w_idx + q_main if t is not None] + app
    nbytes = lambda t: t.numel() * t.element_size()
    in_bytes, out_bytes = sum(nbytes(t) for t in ins), sum(nbytes(t) for t in out)
    h_in = torch.empty(in_bytes, dtype=torch.uint8, pin_memory=True)
    off = 0
    for t in ins:
        h_in[off:off + nbytes(t)].copy_(t.reshape(-1).view(torch.uint8).cpu())
        off += nbytes(t)
    h_out = [torch.empty(out_bytes, dtype=torch.uint8, pin_memory=True) for _ in range(2)]

    def carve(buf, like):
        views, off = [], 0
        for t in like:
            views.append(buf[off:off + nbytes(t)].view(t.dtype).view(t.shape))
            off += nbytes(t)
        return views

    slots = []
    for _ in range(2):
        d_in = torch.empty(in_bytes, dtype=torch.uint8, device=dev)
        d_out = torch.empty(out_bytes, dtype=torch.uint8, device=dev)
        it_in = iter(carve(d_in, ins))
        sq = [None if t is None else next(it_in) for t in q_idx]
        sw = [None if t is None else next(it_in) for t in w_idx]
        sm = [next(it_in) for _ in q_main]
        sa = tuple(next(it_in) for _ in app) if app else None
        so = carve(d_out, out)
        d_in.copy_(h_in)
        group.step(sq, sw, sm, so, append=sa)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            group.step(sq, sw, sm, so, append=sa)
        slots.append((d_in, d_out, g))
    comp = torch.cuda.current_stream(dev)
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    in_ready = [torch.cuda.Event() for _ in range(2)]
    done = [torch.cuda.Event() for _ in range(2)]
    out_read = [torch.cuda.Event() for _ in range(2)]
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for it in range(args.warmup + args.steps):
        sl = it % 2
        if it == args.warmup:
            torch.cuda.synchronize()
            if world > 1:
                dist.barrier()
            a0.record(comp)
            up.wait_event(a0)
        d_in, d_out, g = slots[sl]
        with torch.cuda.stream(up):
            if it >= 2:
                up.wait_event(done[sl])          # step it-2 is done with this slot's inputs
            d_in.copy_(h_in, non_blocking=True)
            in_ready[sl].record(up)
        comp.wait_event(in_ready[sl])
        if it >= 2:
            comp.wait_event(out_read[sl])        # step it-2's outputs have been read back
        g.replay()
        done[sl].record(comp)
        with torch.cuda.stream(down):
            down.wait_event(done[sl])
            h_out[sl].copy_(d_out, non_blocking=True)
            out_read[sl].record(down)
    comp.wait_stream(down)
    a1.record(comp)
    torch.cuda.synchronize()
    pipelined = a0.elapsed_time(a1) / args.steps
    # the same copies and step back to back, with a host synchronisation per
    # step (no overlap): reported beside the pipelined figure
    d_in, d_out, g = slots[0]
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    a0.record(comp)
    for _ in range(args.steps):
        d_in.copy_(h_in, non_blocking=True)
        g.replay()
        h_out[0].copy_(d_out, non_blocking=True)
        comp.synchronize()
    a1.record(comp)
    torch.cuda.synchronize()
    del slots
    return pipelined, a0.elapsed_time(a1) / args.steps


def max_over_ranks(x: float, dev, world: int) -> float:
    """Max of a per-rank timing over all ranks (NCCL on GPUs, gloo on CPU)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def oracle_sample_fp4(wl, b: int = 0):
    """Time the float64 oracle of the FP4 indexer variant on one query: FP4
    scores of every position, pool, Full/Reindex/Reuse Top-k, six attention
    layers (main-KV rows prepared for the gathered positions only)."""
    from oracle import csa2 as C
    from oracle import formats as F
    n = int(W.ctx_lengths(wl)[b])
    codes, scales = F.quantize_indexer_fp4(W.request_rows(wl, b, n, "ik"))
    qw = [None if m == "Ru" else (W.index_query(wl, l)[0][b], W.index_query(wl, l)[1][b])
          for l, m in enumerate(wl.modes)]
    q_main = [W.main_query(wl, l)[b].float().numpy() for l in range(len(wl.modes))]
    t0 = time.perf_counter()
    s = C.indexer_scores_fp4(qw[0][0], qw[0][1], codes, scales)
    pool = C.pool_select(C.block_max(s, n), wl.pool_blocks)
    cand = C.pool_positions(pool, n)
    topk, cur = [], None
    for l, m in enumerate(wl.modes):
        if m == "F":
            cur = C.top_k_ascending(cand, s[cand], wl.topk)
        elif m == "Ri":
            cur = C.top_k_ascending(cand, C.indexer_scores_fp4(qw[l][0], qw[l][1], codes[cand], scales[cand]),
                                    wl.topk)
        topk.append(cur)
    t_sel = time.perf_counter() - t0
    sel = np.unique(np.concatenate([t[t >= 0] for t in topk]))
    kvc = np.zeros((n, 256), np.uint8)
    kvs = np.zeros((n, 32), np.uint8)
    kvc[sel], kvs[sel] = F.quantize_main_kv(W.rows_at(wl, b, sel, "kv"))
    t1 = time.perf_counter()
    for layer in range(len(wl.modes)):
        C.sparse_attention(q_main[layer], kvc, kvs, topk[layer], wl.scale)
    return t_sel + time.perf_counter() - t1


CPU_SAMPLE_S = 10.0   # oracle work the default run's CPU baseline times (seconds)


def cpu_baseline_entry(wl, fp4=False):
    if fp4:
        secs = oracle_sample_fp4(wl, 0)
        return {"value": 1.0 / secs, "unit": "queries/s", "cores": cpu_cores(), **cpu_host(), "kind": "oracle",
                "sample": f"1 of the {wl.batch} queries of one step (request 0, full "
                          f"{int(W.ctx_lengths(wl)[0]):,}-position context): float64 numpy oracle of the FP4 "
                          f"indexer variant, whole layer-group step, {secs:.1f} s"}
    # request 0's query, timed repeatedly until about 10 s of oracle work (at most 8 runs)
    secs, prepared = oracle_sample(wl, 0)
    runs = [secs]
    while sum(runs) < CPU_SAMPLE_S and len(runs) < 8:
        runs.append(oracle_sample(wl, 0, prepared)[0])
    total = sum(runs)
    return {"value": len(runs) / total, "unit": "queries/s", "cores": cpu_cores(), **cpu_host(), "kind": "oracle",
            "sample": f"1 of the {wl.batch} queries of one step (request 0, full {int(W.ctx_lengths(wl)[0]):,}-position "
                      f"context), timed {len(runs)} times: float64 numpy oracle, whole layer-group step, "
                      f"{total:.1f} s in all"}


# ---------------------------------------------------------- reference arm ----

REFERENCE_TIME_BOX_S = 120   # wall-clock bound of the reference arm's timed queries


def run_reference(args):
    """The float64 oracle as the reference arm: each step is one query of the
    workload (cycling over the batch's requests), timed on the host cores."""
    rank, world, _ = env_rank()
    if rank != 0:
        return
    wl = selected_workload(args)
    t_box = time.perf_counter()
    if wl.prefill_queries:
        times = []
        for _ in range(args.steps):   # one prefill query per step, inside the time box
            times.append(prefill_oracle_sample(wl, 1))
            if time.perf_counter() - t_box > REFERENCE_TIME_BOX_S:
                break
        ms = 1e3 * sum(times) / len(times)
        line = {"metric": PREFILL_METRIC, "value": 1e3 / ms, "unit": "queries/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
                "config": {"workload": wl.name},
                "cpu_baseline": {"value": 1e3 / ms, "unit": "queries/s", "cores": cpu_cores(), **cpu_host(), "kind": "oracle",
                                 "sample": f"one prefill query per step, float64 oracle; {len(times)} of the "
                                           f"{args.steps} steps timed inside a {REFERENCE_TIME_BOX_S} s box"},
                "timed_steps": len(times),
                "e2e": {"value": 1e3 / ms, "unit": "queries/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return
    # The oracle has nothing to warm up beyond building a request's inputs:
    # one warm-up query, then timed queries (requests cycled) until K are done
    # or the time box is spent.
    prepared = {}
    times = []
    warm = min(args.warmup, 1)
    for it in range(warm + args.steps):
        b = it % wl.batch
        secs, prepared[b] = oracle_sample(wl, b, prepared.get(b))
        if it >= warm:
            times.append(secs)
            if time.perf_counter() - t_box > REFERENCE_TIME_BOX_S:
                break
    ms = 1e3 * sum(times) / len(times)
    value = 1e3 / ms
    line = base_line(args, wl, world, value, ms)
    line.update({"impl": "reference", "dtype": "f64",
                 "cpu_baseline": {"value": value, "unit": "queries/s", "cores": cpu_cores(), **cpu_host(), "kind": "oracle",
                                  "sample": f"one query per step (requests cycled), full context, float64 numpy "
                                            f"oracle of the whole layer-group step; {len(times)} of the {args.steps} "
                                            f"steps timed inside a {REFERENCE_TIME_BOX_S} s box after {warm} "
                                            f"warm-up query"},
                 "timed_steps": len(times),
                 "e2e": {"value": value, "unit": "queries/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}})
    print(json.dumps(line), flush=True)


def selected_workload(args):
    wl = W.WORKLOADS[args.workload]
    changes = {}
    if args.batch:
        changes["batch"] = args.batch
    if args.ctx:
        changes["ctx"] = args.ctx
    if args.prefill_queries:
        changes["prefill_queries"] = args.prefill_queries
    return W.scaled(wl, **changes) if changes else wl


def log(rank, msg):
    if rank == 0:
        print(f"[bench] {msg}", file=sys.stderr, flush=True)


def main(argv=None):
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=["b200", "reference"], default="b200")
    p.add_argument("--workload", default="group_1m_b4", choices=sorted(W.WORKLOADS))
    p.add_argument("--batch", type=int, default=0, help="override the workload's batch (profiling cases)")
    p.add_argument("--ctx", type=int, default=0, help="override the workload's context length (profiling cases)")
    p.add_argument("--prefill-queries", type=int, default=0,
                   help="override the number of prefill queries (profiling cases)")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--indexer", choices=["fp8", "fp4"], default="fp8",
                   help="indexer K format of the decode workloads (fp4: the FP4 indexer variant)")
    args = p.parse_args(argv)
    if args.warmup < 3:
        p.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    elif W.WORKLOADS[args.workload].prefill_queries:
        run_prefill(args)
    else:
        run_b200(args)


if __name__ == "__main__":
    main()
