"""Benchmark: compressed decode attention on the 7B-shaped GQA workload at 3.5% KV.

Workload (one step = one decode-attention call for the whole batch):
  B = 32 sequences, 28 query / 4 KV heads (GQA 7), d = 128, T = 32,768 tokens per sequence,
  coarsened by this library's own kernels to 8 sink + N = 1,091 equal-variation nodes + 48
  recent entries per KV head (regime-walk keys with 200 regimes, N(0,1) values, bf16). One
  query row per query head: 896 query rows per step.
  The caches of L layers (distinct seeds, 76 MB each) are built once; step i decodes layer
  i % L, so consecutive steps never find their cache in the 126 MB L2.

Output: one JSON line (rank 0) with the decode throughput (`value`, query rows/s), the decode
op's achieved HBM bandwidth against the measured copy peak (`roofline`), an end-to-end figure
with pinned host queries / outputs copied every step (`e2e`), the SM clocks sampled during the
timed region, the CPU oracle timed on the host (`cpu_baseline`), the coarsener's own
throughput on the 8 x 4 x 131,072-token workload (`coarsen`), decode with the diagonal closure
(`diagonal_closure`), streaming appends (`streaming_append`), and decode on the 1.5B-shaped
10.5K-token and the ragged paged 2% workloads (`other_decode`).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Multi-GPU (torchrun, one rank per GPU): every rank decodes its own batch (weak scaling, no
collective on the data path); the timed duration is the max over ranks.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import tempfile
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode-attn query-rows/s & HBM GB/s (% of peak), 7B GQA shape, 3.5% KV"
UNIT = "query-rows/s"
WORKLOAD = "gqa7_32k_decode_3p5pct"
COARSEN_WORKLOAD = "coarsen_131k"
FALLBACK_HBM_GBS = 6650.0


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            p = json.load(fh)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def _source_sha(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


DECODE_SOURCES = ["compressed_decode_attention_equal_b200/csrc/decode.cu",
                  "compressed_decode_attention_equal_b200/csrc/skv_common.cuh",
                  "compressed_decode_attention_equal_b200/csrc/skv_internal.h"]
COARSEN_SOURCES = ["compressed_decode_attention_equal_b200/csrc/coarsen.cu",
                   "compressed_decode_attention_equal_b200/csrc/skv_common.cuh",
                   "compressed_decode_attention_equal_b200/csrc/skv_internal.h"]


def _profile_traffic(summary: str, sources):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on the current source."""
    path = os.path.join(ROOT, "profiles", summary)
    try:
        text = open(path).read()
    except OSError:
        return None
    m_sha = re.search(r"source_sha256_16:\s*([0-9a-f]+)", text)
    m_b = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
    if not m_sha or not m_b or m_sha.group(1) != _source_sha(sources):
        return None
    return float(m_b.group(1))


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples taken while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, flags in rows for i, f in enumerate(flags) if f.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------
# workload set-up (untimed)
# ---------------------------------------------------------------------------
def build_layer_caches(w, layers: int, device, closure: str = "scalar"):
    import torch
    import compressed_decode_attention_equal_b200 as skv
    import workloads
    T_list = workloads.seq_lengths(w)
    N_list = workloads.segment_counts(w, T_list)
    pages = [skv.pages_for(T, N, workloads.N_SINK, workloads.N_RECENT) for T, N in zip(T_list, N_list)]
    table, num_pages = workloads.page_assignment(w.B, w.Hkv, pages, w.shuffle_pages, w.seed)
    table = table.to(device)
    ws = torch.zeros(skv.coarsen_workspace_bytes(w.Hkv, w.d, T_list, N_list, workloads.N_SINK, workloads.N_RECENT),
                     dtype=torch.uint8, device=device)
    caches, coarsen_ms = [], []
    for layer in range(layers):
        wl = dataclasses.replace(w, seed=w.seed + 1000 * layer)
        k, v, _ = workloads.make_kv(wl, device, T_list=T_list)
        pool = skv.NodePool(num_pages, w.d, w.torch_dtype, device=device, closure=closure)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        lens = skv.coarsen(k, v, w.Hkv, T_list, N_list, workloads.N_SINK, workloads.N_RECENT, wl.seed, pool, table,
                           workspace=ws)
        e1.record()
        torch.cuda.synchronize()
        coarsen_ms.append(e0.elapsed_time(e1))
        st, flags = skv.workspace_error(ws)
        if st != 0:
            raise RuntimeError(f"coarsening raised device flags {flags}")
        q = workloads.make_queries(wl, device)
        caches.append(dict(pool=pool, lens=lens, q=q, seed=wl.seed))
        del k, v
    torch.cuda.empty_cache()
    return caches, table, T_list, N_list, coarsen_ms


def algorithmic_decode_bytes(w, lens_list, closure: str = "scalar"):
    """HBM bytes one decode call must move: every entry's key, value and (alpha, beta) once (and its
    per-dimension variances with the diagonal closure), the queries once, the outputs and lse once."""
    ent = sum(int(x) for x in lens_list)
    node = (3 if closure == "diagonal" else 2) * w.d * 2 + 8
    rows = w.B * w.R * w.Hq
    return ent * node + rows * w.d * 2 * 2 + rows * 4, ent


def _graph_steps(fn, steps: int, start: int = 0):
    """Capture `fn(start + i)` for i in [0, steps) into one CUDA graph."""
    import torch
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            for i in range(steps):
                fn(start + i)
    torch.cuda.current_stream().wait_stream(s)
    return g


# ---------------------------------------------------------------------------
# ranks (one process per GPU under torchrun; every rank takes the same collective steps)
# ---------------------------------------------------------------------------
def rank_workload(w, rank: int, world: int):
    """The batch a rank decodes: the same shapes, an independent seed per rank (weak scaling;
    no data-path collective)."""
    if world <= 1:
        return w
    return dataclasses.replace(w, seed=w.seed + 100000 * rank)


def max_over_ranks(x: float, device, world: int) -> float:
    """The largest x over all ranks (the job's duration is set by its slowest rank)."""
    if world <= 1:
        return x
    import torch
    t = torch.tensor([x], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_step: int, world: int, steps: int, ms: float) -> float:
    """Whole-job units per second: every rank's units over the max-over-ranks time."""
    return units_per_step * world * steps / (ms / 1e3)


def init_ranks(backend: str, device, world: int, timeout_s: int = 120):
    """One process group per job (short timeout: ranks that wait on a dead peer end with an
    error); NCCL binds the rank's device."""
    if world <= 1:
        return
    import datetime
    import torch
    kw = {"device_id": device} if backend == "nccl" else {}
    torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)


def finish_ranks(world: int):
    if world <= 1:
        return
    import torch
    torch.distributed.barrier()
    torch.distributed.destroy_process_group()


GRAPH_MAX_STEPS = 20000   # calls per captured graph; longer regions replay several graphs back to back


def region_graphs(fn, steps: int):
    """Graphs that together run exactly `steps` calls fn(0) .. fn(steps - 1), in order."""
    graphs, done = [], 0
    while done < steps:
        n = min(GRAPH_MAX_STEPS, steps - done)
        graphs.append(_graph_steps(fn, n, done))
        done += n
    return graphs


def summarise_regions(times_ms, steps: int):
    """Per-call statistics (us) over the timed regions of `steps` calls each."""
    per = sorted(t / steps * 1e3 for t in times_ms)
    n = len(per)
    return {"regions": n, "steps_per_region": steps, "median_us": statistics.median(per), "min_us": per[0],
            "max_us": per[-1], "p10_us": per[int(0.1 * (n - 1))], "p90_us": per[int(0.9 * (n - 1))]}


def time_regions(fn, steps: int, dist_on: bool, regions: int, flush=None):
    """Device time (ms) of `regions` timed regions, each EXACTLY `steps` calls fn(0..steps-1)
    replayed from CUDA graphs and bracketed by a barrier (multi-rank) and a synchronize on both
    sides. Between regions (outside the timed interval) `flush`, a buffer larger than L2, is read
    (a sum) so that no region starts with the previous region's data in L2; reading leaves clean
    lines behind, so the timed calls pay no write-back of the flush."""
    import torch
    graphs = region_graphs(fn, steps)
    for g in graphs:
        g.replay()   # the first replay uploads the graph
    torch.cuda.synchronize()
    times = []
    for _ in range(regions):
        if flush is not None:
            flush.sum()
        torch.cuda.synchronize()
        if dist_on:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for g in graphs:
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        if dist_on:
            torch.distributed.barrier()
        times.append(e0.elapsed_time(e1))
    del graphs
    return times


def l2_flush_buffer(device):
    import torch
    return torch.zeros(64 << 20, dtype=torch.float32, device=device)   # 256 MB, twice the 126 MB L2 (read)


def coarsen_stage(device, reps: int = 5, batch: int | None = None):
    """Coarsener throughput on the 8 x 4 x 131,072-token workload (tokens/s, GB/s of raw KV);
    `batch` < 8 takes the first sequences only (a profiling case)."""
    import torch
    import compressed_decode_attention_equal_b200 as skv
    import workloads
    w = workloads.WORKLOADS[COARSEN_WORKLOAD]
    if batch is not None:
        w = dataclasses.replace(w, B=batch)
    T_list = workloads.seq_lengths(w)
    N_list = workloads.segment_counts(w, T_list)
    k, v, _ = workloads.make_kv(w, device, T_list=T_list)
    pages = [skv.pages_for(T, N, workloads.N_SINK, workloads.N_RECENT) for T, N in zip(T_list, N_list)]
    table, num_pages = workloads.page_assignment(w.B, w.Hkv, pages, False, w.seed)
    table = table.to(device)
    pool = skv.NodePool(num_pages, w.d, w.torch_dtype, device=device)
    lens = torch.empty(w.B, w.Hkv, dtype=torch.int32, device=device)
    ws = torch.zeros(skv.coarsen_workspace_bytes(w.Hkv, w.d, T_list, N_list, workloads.N_SINK, workloads.N_RECENT),
                     dtype=torch.uint8, device=device)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)

    def call(**opts):
        skv.coarsen(k, v, w.Hkv, T_list, N_list, workloads.N_SINK, workloads.N_RECENT, w.seed, pool, table,
                    lens=lens, workspace=ws, **opts)

    def timed(**opts):
        for _ in range(2):
            call(**opts)
        torch.cuda.synchronize()
        times = []
        for _ in range(reps):
            flush.zero_()                      # evict the raw KV from L2 between calls
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            call(**opts)
            e1.record()
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1))
        st, flags = skv.workspace_error(ws)
        if st != 0:
            raise RuntimeError(f"coarsening raised device flags {flags}")
        return statistics.median(times)

    ms_weighted = timed(representative="variation")
    ms_centred = timed(center_keys=True)
    ms_tensor = timed(projection="tensor")
    ms = timed()
    tokens = sum(T_list) * w.Hkv
    raw_bytes = 2 * tokens * w.d * 2
    ent = int(lens.sum())
    node_bytes = ent * (2 * w.d * 2 + 8)
    alg = raw_bytes + node_bytes
    peak, src = _peaks()
    middle = sum(max(0, T - workloads.N_SINK - workloads.N_RECENT) for T in T_list) * w.Hkv
    fma = middle * 16 * 2 * w.d
    sm_clock_ghz = 1.965
    alu_peak_tfma = 148 * 128 * sm_clock_ghz / 1000.0
    del k, v, flush
    torch.cuda.empty_cache()
    return {
        "workload": COARSEN_WORKLOAD, "ms": ms, "tokens_per_s": tokens / (ms / 1e3),
        "raw_kv_gbs": raw_bytes / (ms / 1e3) / 1e9,
        "roofline": {"bound": "hbm", "achieved": alg / (ms / 1e3) / 1e9, "peak": peak, "unit": "GB/s",
                     "frac": alg / (ms / 1e3) / 1e9 / peak, "peak_source": src, "traffic": _profile_traffic(
                         "coarsen_131k_summary.md", COARSEN_SOURCES), "algorithmic_bytes": alg},
        "projection_alu": {"fma_per_call": fma, "achieved_tfma_s": fma / (ms / 1e3) / 1e12,
                           "peak_tfma_s_at_max_clock": alu_peak_tfma},
        "frac_of_8tbs": alg / (ms / 1e3) / 8e12,
        "variation_weighted": {"ms": ms_weighted, "tokens_per_s": tokens / (ms_weighted / 1e3),
                               "frac": alg / (ms_weighted / 1e3) / 1e9 / peak,
                               "note": "same call with the variation-weighted segment representative"},
        "centred_keys": {"ms": ms_centred, "tokens_per_s": tokens / (ms_centred / 1e3),
                         "frac": alg / (ms_centred / 1e3) / 1e9 / peak,
                         "note": "same call with common-mode mean removal (one more read of the keys)"},
        "tensor_projection": {
            "ms": ms_tensor, "tokens_per_s": tokens / (ms_tensor / 1e3),
            "roofline": {"bound": "hbm", "achieved": alg / (ms_tensor / 1e3) / 1e9, "peak": peak, "unit": "GB/s",
                         "frac": alg / (ms_tensor / 1e3) / 1e9 / peak, "peak_source": src,
                         "algorithmic_bytes": alg},
            "note": "same call with the tensor-core bf16 projection option (steps checked stage by stage, not "
                    "bit-exact with the fixed fp32 recipe)"},
    }


def cpu_baseline(w, caches, table, budget_s: float = 12.0):
    """The fp64 CPU oracle decoding the same cache (nodes read back from the GPU) on the host
    cores: whole batches of one layer, repeated until `budget_s` of work."""
    import numpy as np
    import torch
    import compressed_decode_attention_equal_b200 as skv
    import oracle

    class U:
        def __init__(self, kt, vt, al, be):
            self.kt, self.vt, self.alpha, self.beta = kt, vt, al, be

    c = caches[0]
    units = []
    for b in range(w.B):
        row = []
        for h in range(w.Hkv):
            kt, vt, al, be = skv.read_entries(c["pool"], table, c["lens"], b, h)
            row.append(U(kt.double().cpu().numpy(), vt.double().cpu().numpy(), al.double().cpu().numpy(),
                         be.double().cpu().numpy()))
        units.append(row)
    q = c["q"].double().cpu().numpy()
    threads = os.cpu_count() or 1
    rows = 0
    t0 = time.perf_counter()
    reps = 0
    while True:
        oracle.decode(q, units, threads=threads)
        rows += w.B * w.R * w.Hq
        reps += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": rows / dt, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{reps} full decode batches of one layer ({w.B} x {w.Hq} query rows over "
                      f"{int(c['lens'].sum())} entries), fp64, nodes read back from the GPU"}


def diagonal_closure_stage(w, device, layers: int, steps: int = 1000, regions: int = 3):
    """Decode with the diagonal closure (per-dimension variances in every node) on the same workload:
    layer caches coarsened into diagonal pools, graph replays, CUDA events (rank 0 only)."""
    import torch
    import compressed_decode_attention_equal_b200 as skv
    caches, table, _, _, _ = build_layer_caches(w, layers, device, closure="diagonal")
    L = len(caches)
    alg, _ = algorithmic_decode_bytes(w, [int(caches[0]["lens"].sum())], closure="diagonal")
    outs = [torch.empty_like(c["q"]) for c in caches]
    lses = [torch.empty(w.B, w.R, w.Hq, dtype=torch.float32, device=device) for _ in caches]
    ws = torch.zeros(skv.decode_workspace_bytes(w.B, w.R, w.Hq, w.Hkv, w.d, table.shape[2]), dtype=torch.uint8,
                     device=device)

    def step(i):
        c = caches[i % L]
        skv.decode_attn(c["q"], w.Hkv, c["pool"], table, c["lens"], out=outs[i % L], lse=lses[i % L], workspace=ws)

    for i in range(3 * L):
        step(i)
    torch.cuda.synchronize()
    st, flags = skv.workspace_error(ws)
    if st != 0:
        raise RuntimeError(f"diagonal-closure decode raised device flags {flags}")
    stats = summarise_regions(time_regions(step, steps, False, regions, flush=l2_flush_buffer(device)), steps)
    us = stats["median_us"]
    peak, src = _peaks()
    del caches
    torch.cuda.empty_cache()
    return {"us_per_call": us, "query_rows_per_s": w.B * w.R * w.Hq / (us * 1e-6),
            "achieved_gbs": alg / (us * 1e-6) / 1e9, "frac": alg / (us * 1e-6) / 1e9 / peak,
            "algorithmic_bytes_per_launch": alg, "timing": stats,
            "note": "same workload and call with diagonal-closure pools (per-dimension key variances)"}


def other_decode_stage(device, steps: int = 1000, regions: int = 3):
    """Decode on the two other decode workloads, each cache built by the coarsener and replayed from
    CUDA graphs (rank 0 only):
    - gqa6_10k5_prefill_decode: 1 sequence, 2 KV heads, 421 entries each, a 0.45 MB cache, so the
      call is latency-bound (reported in us); the cache is copied into enough pools to exceed L2
      and the copies rotate.
    - gqa7_ragged_paged_2pct: 128 sequences of log-uniform lengths, 4 query rows per sequence,
      shuffled page tables; HBM-bound. Two independently seeded caches (each larger than L2) rotate."""
    import torch
    import compressed_decode_attention_equal_b200 as skv
    import workloads
    peak, _ = _peaks()
    res = {}
    for name, layers in (("gqa6_10k5_prefill_decode", 1), ("gqa7_ragged_paged_2pct", 2)):
        w = workloads.WORKLOADS[name]
        caches, table, _, _, _ = build_layer_caches(w, layers, device)
        base = caches[0]
        copies = -(-(256 << 20) // base["pool"].nbytes()) if layers == 1 else 1
        if copies > 1:
            pools = []
            for _ in range(copies):
                p = skv.NodePool(base["pool"].num_pages, w.d, w.torch_dtype, device=device)
                p.pages.copy_(base["pool"].pages)
                pools.append(p)
            caches = [dict(base, pool=p) for p in pools]
        L = len(caches)
        alg, ent = algorithmic_decode_bytes(w, [int(caches[0]["lens"].sum())])
        outs = [torch.empty_like(c["q"]) for c in caches]
        lses = [torch.empty(w.B, w.R, w.Hq, dtype=torch.float32, device=device) for _ in caches]
        ws = torch.zeros(skv.decode_workspace_bytes(w.B, w.R, w.Hq, w.Hkv, w.d, table.shape[2]), dtype=torch.uint8,
                         device=device)

        def step(i):
            c = caches[i % L]
            skv.decode_attn(c["q"], w.Hkv, c["pool"], table, c["lens"], out=outs[i % L], lse=lses[i % L],
                            workspace=ws)

        for i in range(L + 3):
            step(i)
        torch.cuda.synchronize()
        st, flags = skv.workspace_error(ws)
        if st != 0:
            raise RuntimeError(f"{name}: decode raised device flags {flags}")
        stats = summarise_regions(time_regions(step, steps, False, regions, flush=l2_flush_buffer(device)), steps)
        us = stats["median_us"]
        rows = w.B * w.R * w.Hq
        res[name] = {"us_per_call": us, "query_rows_per_call": rows, "query_rows_per_s": rows / (us * 1e-6),
                     "entries_per_call": ent, "algorithmic_bytes_per_launch": alg,
                     "achieved_gbs": alg / (us * 1e-6) / 1e9, "frac": alg / (us * 1e-6) / 1e9 / peak,
                     "timing": stats, "l2": f"{L} caches of {base['pool'].nbytes() / 1e6:.2f} MB pool each, rotated"}
        del caches, outs, lses, base
        torch.cuda.empty_cache()
    return res


def stream_stage(w, device, steps: int = 1000, distinct: int = 60, regions: int = 3):
    """Streaming coarsening on the decode workload: skv_stream_init on the prompts, then appends of
    one token per unit replayed from CUDA graphs (rank 0 only). The append is latency-bound (one CTA
    per unit, a 4,096-FMA projection chain and O(N) merge search per call)."""
    import torch
    import compressed_decode_attention_equal_b200 as skv
    import workloads
    T_list = workloads.seq_lengths(w)
    N_list = workloads.segment_counts(w, T_list)
    cap = skv.stream_capacity(N_list, workloads.N_SINK, workloads.N_RECENT)
    table, num_pages = workloads.page_assignment(w.B, w.Hkv, [-(-cap // 16)] * w.B, w.shuffle_pages, w.seed)
    table = table.to(device)
    k, v, _ = workloads.make_kv(w, device, T_list=T_list)
    pool = skv.NodePool(num_pages, w.d, w.torch_dtype, device=device)
    t0 = time.perf_counter()
    lens, state, ws = skv.stream_init(k, v, w.Hkv, T_list, N_list, workloads.N_SINK, workloads.N_RECENT, w.seed,
                                      pool, table)
    torch.cuda.synchronize()
    init_s = time.perf_counter() - t0
    del k, v
    g = torch.Generator(device=device).manual_seed(w.seed + 5)
    new_k = (torch.randn(distinct, w.B, w.Hkv, w.d, generator=g, device=device)).to(w.torch_dtype)
    new_v = (torch.randn(distinct, w.B, w.Hkv, w.d, generator=g, device=device)).to(w.torch_dtype)

    def step(i):
        skv.stream_append(new_k[i % distinct], new_v[i % distinct], N_list, workloads.N_SINK, workloads.N_RECENT,
                          pool, table, lens, state, ws)

    for i in range(distinct):
        step(i)
    torch.cuda.synchronize()
    stats = summarise_regions(time_regions(step, steps, False, regions), steps)
    st, flags = skv.workspace_error(ws)
    if st != 0:
        raise RuntimeError(f"streaming append raised device flags {flags}")
    us = stats["median_us"]
    units = w.B * w.Hkv
    del pool, state
    torch.cuda.empty_cache()
    return {"us_per_append": us, "tokens_per_s": units / (us * 1e-6), "units": units, "timing": stats,
            "init_s_host_clock": init_s,
            "note": "one token appended to every (sequence, KV head) unit per call, N = "
                    f"{N_list[0]} nodes per unit, graphs of {distinct} calls"}


# ---------------------------------------------------------------------------
# arms
# ---------------------------------------------------------------------------
def bench_config(w, world: int):
    """The `config` object of the JSON line: the workload, its sizes and how L2 is kept out of the
    timing. Both arms print this same object."""
    return {"workload": WORKLOAD, "batch": w.B, "q_heads": w.Hq, "kv_heads": w.Hkv, "d": w.d, "context": w.T,
            "middle_nodes": w.N, "entries_per_head": workloads_entries(w), "query_rows_per_step": w.B * w.R * w.Hq,
            "parallelism": f"dp{world}" if world > 1 else "single",
            "l2": "inputs larger than L2: 6 layer caches of 76.8 MB decoded in rotation (a call's pages were "
                  "last read 5 calls and 384 MB of pages earlier, and are read evict-first); timing_l2_flushed "
                  "repeats the regions with a 256 MB buffer read before each",
            "timing": "CUDA graphs of back-to-back decode calls; CUDA events around each region of exactly "
                      "`steps` calls; median over the regions, then max over ranks"}


def workloads_entries(w) -> int:
    import workloads
    return workloads.N_SINK + w.N + workloads.N_RECENT


def e2e_pipeline(w, caches, table, ws, outs, lses, device):
    """The end-to-end step through the public API with host buffers, pipelined the way a caller
    overlaps transfers with compute: step i's queries are copied from pinned host memory on an
    upload stream, the decode runs on the compute stream once they have landed, and out / lse are
    copied back to pinned host memory on a download stream. Buffers rotate over the L layer
    slots, so step i + 1's upload and step i - 1's download overlap step i's kernel; each reuse of
    a slot waits for the previous user of that slot. One cudaMemcpyAsync per buffer."""
    import torch
    import compressed_decode_attention_equal_b200 as skv
    L = len(caches)
    q_host = [c["q"].cpu().pin_memory() for c in caches]
    out_host = [torch.empty_like(q, device="cpu").pin_memory() for q in q_host]
    lse_host = [torch.empty(w.B, w.R, w.Hq, dtype=torch.float32).pin_memory() for _ in caches]
    q_dev = [torch.empty_like(c["q"]) for c in caches]
    up, down = torch.cuda.Stream(device), torch.cuda.Stream(device)
    h2d_done = [torch.cuda.Event() for _ in range(L)]
    k_done = [torch.cuda.Event() for _ in range(L)]
    d2h_done = [torch.cuda.Event() for _ in range(L)]

    def step(i, start):
        """Step i of a captured sequence that began at step `start` (slot waits reach back only to
        steps of the same capture; a graph completes before the next one starts)."""
        j = i % L
        main = torch.cuda.current_stream()
        if i - L >= start:
            up.wait_event(k_done[j])            # step i - L's kernel has read q_dev[j]
        with torch.cuda.stream(up):
            q_dev[j].copy_(q_host[j], non_blocking=True)
            h2d_done[j].record(up)
        main.wait_event(h2d_done[j])
        if i - L >= start:
            main.wait_event(d2h_done[j])        # step i - L's outputs have left outs[j]
        c = caches[j]
        skv.decode_attn(q_dev[j], w.Hkv, c["pool"], table, c["lens"], out=outs[j], lse=lses[j], workspace=ws)
        k_done[j].record(main)
        down.wait_event(k_done[j])
        with torch.cuda.stream(down):
            out_host[j].copy_(outs[j], non_blocking=True)
            lse_host[j].copy_(lses[j], non_blocking=True)
            d2h_done[j].record(down)

    def fork(main):
        up.wait_stream(main)
        down.wait_stream(main)

    def join(main):
        main.wait_stream(up)
        main.wait_stream(down)

    h2d = q_host[0].numel() * q_host[0].element_size()
    d2h = out_host[0].numel() * out_host[0].element_size() + lse_host[0].numel() * 4
    return step, fork, join, out_host, h2d, d2h


def time_e2e_regions(step, fork, join, steps: int, dist_on: bool, regions: int, flush=None):
    """time_regions for the pipelined end-to-end step: each captured graph forks the side streams
    at its start and joins them at its end, so a region ends only when its last download has
    landed."""
    import torch

    def graph(n, start):
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                fork(s)
                for i in range(n):
                    step(start + i, start)
                join(s)
        torch.cuda.current_stream().wait_stream(s)
        return g

    graphs, done = [], 0
    while done < steps:
        n = min(GRAPH_MAX_STEPS, steps - done)
        graphs.append(graph(n, done))
        done += n
    for g in graphs:
        g.replay()
    torch.cuda.synchronize()
    times = []
    for _ in range(regions):
        if flush is not None:
            flush.sum()
        torch.cuda.synchronize()
        if dist_on:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for g in graphs:
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        if dist_on:
            torch.distributed.barrier()
        times.append(e0.elapsed_time(e1))
    del graphs
    return times


def run_ours(args, rank: int, world: int, device):
    import torch
    import compressed_decode_attention_equal_b200 as skv
    import workloads

    dist_on = world > 1
    w = workloads.WORKLOADS[WORKLOAD]
    w = rank_workload(w, rank, world)   # each rank decodes its own, independently seeded batch
    caches, table, T_list, N_list, coarsen_ms = build_layer_caches(w, args.layers, device)
    L = len(caches)
    rows_per_step = w.B * w.R * w.Hq
    alg_bytes, ent = algorithmic_decode_bytes(w, [int(c["lens"].sum()) for c in caches][:1])
    outs = [torch.empty_like(c["q"]) for c in caches]
    lses = [torch.empty(w.B, w.R, w.Hq, dtype=torch.float32, device=device) for _ in caches]
    ws = torch.zeros(skv.decode_workspace_bytes(w.B, w.R, w.Hq, w.Hkv, w.d, table.shape[2]), dtype=torch.uint8,
                     device=device)
    flush = l2_flush_buffer(device)

    def step(i):
        c = caches[i % L]
        skv.decode_attn(c["q"], w.Hkv, c["pool"], table, c["lens"], out=outs[i % L], lse=lses[i % L], workspace=ws)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    st, flags = skv.workspace_error(ws)
    if st != 0:
        raise RuntimeError(f"decode raised device flags {flags}")

    sampler = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    if sampler:
        sampler.start()
    times = time_regions(step, args.steps, dist_on, args.regions)
    # the same regions with L2 emptied before each (the first call of a region then also fetches the
    # kernel's code, the page table, lens and queries from DRAM): reported beside the value
    cold = summarise_regions(time_regions(step, args.steps, dist_on, args.regions, flush=flush), args.steps)
    clocks = sampler.stop() if sampler else None
    stats = summarise_regions(times, args.steps)
    ms = max_over_ranks(stats["median_us"] * args.steps / 1e3, device, world)   # median region, slowest rank
    ms_per_step = ms / args.steps
    value = job_throughput(rows_per_step, world, args.steps, ms)

    # end to end through the public API with host buffers, transfers pipelined with the kernels
    e2e_step, e2e_fork, e2e_join, out_host, h2d, d2h = e2e_pipeline(w, caches, table, ws, outs, lses, device)
    e2e_steps = max(L, args.steps)
    e2e_regions = max(3, min(args.regions, 10))
    e2e_stats = summarise_regions(time_e2e_regions(e2e_step, e2e_fork, e2e_join, e2e_steps, dist_on, e2e_regions),
                                  e2e_steps)
    e2e_ms = max_over_ranks(e2e_stats["median_us"] * e2e_steps / 1e3, device, world)
    # the timed copies are real: the last step's outputs landed in host memory
    torch.cuda.synchronize()
    last = (e2e_steps - 1) % L
    assert torch.equal(out_host[last], outs[last].cpu())

    result = None
    if rank == 0:
        peak, src = _peaks()
        achieved = alg_bytes / (ms_per_step / 1e3) / 1e9
        launches_per_step = 1   # one decode kernel per call
        sm_ghz = clocks["sm_mhz"] / 1e3 if clocks else None
        result = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic: regime-walk keys, N(0,1) values and queries, coarsened on the GPU by this library",
            "config": bench_config(w, world),
            "timing": dict(stats, note=f"{args.regions} timed regions of exactly {args.steps} calls; value uses "
                                       "the median region (max over ranks)",
                           us_x_sm_ghz=stats["median_us"] * sm_ghz if sm_ghz else None),
            "timing_l2_flushed": dict(cold, note="the same regions, each after a 256 MB buffer read (rank 0)"),
            "entries_per_step": ent,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                         "traffic": _profile_traffic("decode_gqa7_32k_summary.md", DECODE_SOURCES),
                         "peak_source": f"{src} HBM copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"
                         if src == "measured" else "fallback 6.65 TB/s",
                         "frac_of_8tbs": achieved / 8000.0, "algorithmic_bytes_per_launch": alg_bytes,
                         "kernel": "k_decode_split (one launch per call), time per call"},
            "e2e": {"value": job_throughput(rows_per_step, world, e2e_steps, e2e_ms), "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                    "timing": e2e_stats,
                    "note": "pinned host queries in and out / lse back every step through the public API; "
                            "uploads and downloads on their own streams overlap the neighbouring steps' kernels"},
            "gpu_launches": launches_per_step * args.steps,
            "gpu_launches_note": "decode kernels per timed region (one per step)",
            "clocks": clocks,
            "coarsen_build_ms_per_layer": coarsen_ms,
        }
    return result, caches, table, w


def run_reference(args, rank: int, world: int = 1):
    """The oracle on the host cores, on this arm's workload, metric and unit (rank 0 only; under
    torchrun the other ranks exit without work)."""
    if rank != 0:
        return None
    import concurrent.futures
    import numpy as np
    import oracle
    import workloads
    w = workloads.WORKLOADS[WORKLOAD]
    rng = np.random.default_rng(w.seed)
    # the oracle decodes units whose entries have the workload's shape: E = 8 + 1091 + 48 per head
    E = workloads.N_SINK + w.N + workloads.N_RECENT
    T, N = w.T, w.N
    sizes = np.full(N, (T - workloads.N_SINK - workloads.N_RECENT) // N)
    sizes[: (T - workloads.N_SINK - workloads.N_RECENT) % N] += 1
    mass = np.concatenate([np.ones(workloads.N_SINK), sizes, np.ones(workloads.N_RECENT)])

    class U:
        pass

    def unit():
        u = U()
        u.kt = rng.standard_normal((E, w.d)) * 3
        u.vt = rng.standard_normal((E, w.d))
        u.alpha = np.log(mass)
        u.beta = rng.random(E) * 1e-3
        return u

    units = [[unit() for _ in range(w.Hkv)] for _ in range(w.B)]
    q = rng.standard_normal((w.B, w.R, w.Hq, w.d))
    # The oracle's unit of work is one query row against its KV head's E entries. A step decodes
    # the next `n` rows of the batch in order (sequence, KV head, the head group's rows), cycling,
    # one oracle call per KV head touched, spread over the host cores.
    G = w.Hq // w.Hkv
    per_unit = w.R * G
    total = w.B * w.Hkv * per_unit

    def unit_rows(k):
        b, h = divmod(k, w.Hkv)
        return q[b, :, h * G:(h + 1) * G, :].reshape(per_unit, w.d)

    def step(start, n, ex):
        jobs, i = [], start
        while i < start + n:
            k, off = divmod(i % total, per_unit)
            take = min(start + n - i, per_unit - off)
            jobs.append((k, off, take))
            i += take
        def one(job):
            k, off, take = job
            u = units[k // w.Hkv][k % w.Hkv]
            oracle.decode_rows(unit_rows(k)[off:off + take], u.kt, u.vt, u.alpha, u.beta)
        list(ex.map(one, jobs))
        return len(jobs)

    threads = os.cpu_count() or 1
    with concurrent.futures.ThreadPoolExecutor(threads) as ex:
        # calibrate on one KV head's rows: warmup + steps are sized to end in about a minute
        t0 = time.perf_counter()
        step(0, per_unit, ex)
        per_row = max((time.perf_counter() - t0) / per_unit, 1e-6)
        budget = args.ref_seconds / max(1, args.steps + args.warmup)
        n = int(max(1, min(total, budget / per_row)))
        pos, used = 0, 1
        for _ in range(args.warmup):
            step(pos, n, ex)
            pos += n
        t0 = time.perf_counter()
        for _ in range(args.steps):
            used = max(used, step(pos, n, ex))
            pos += n
        dt = time.perf_counter() - t0
    rows = n * args.steps
    value = rows / dt
    cores = min(threads, used)
    return {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": dt * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic entries with the workload's shape", "impl": "reference",
        "config": bench_config(w, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{n} of the batch's {total} query rows per step, each against {E} entries"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def free_port() -> int:
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def relaunch_command(args_argv, gpus: int, port: int):
    """The torch.distributed.run command that runs this script as `gpus` ranks on this node."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={gpus}",
            "--master-addr=127.0.0.1", f"--master-port={port}", os.path.abspath(__file__), *args_argv]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000, help="calls per timed region")
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--regions", type=int, default=30, help="timed regions of --steps calls (median reported)")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--layers", type=int, default=6)
    ap.add_argument("--ref-seconds", type=float, default=60.0,
                    help="reference arm: host seconds that warm-up plus steps are sized to")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-coarsen", action="store_true")
    ap.add_argument("--no-diagonal", action="store_true", help="skip the diagonal-closure decode timing")
    ap.add_argument("--no-stream", action="store_true", help="skip the streaming-append timing")
    ap.add_argument("--no-other", action="store_true", help="skip the decode timing on the other two workloads")
    ap.add_argument("--only", choices=["coarsen", "diagonal", "stream", "other"],
                    help="run this single-GPU stage alone (no headline line; a profiling aid)")
    ap.add_argument("--coarsen-batch", type=int, default=None,
                    help="sequences of the coarsening workload (default all 8; fewer for a profiling case)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus < 1 or args.regions < 1 or args.steps < 1:
        ap.error("--gpus, --regions and --steps must be >= 1")

    if "WORLD_SIZE" not in os.environ:
        if args.gpus > 1:
            # one process per GPU: run this script as --gpus ranks under torch.distributed.run
            rc = subprocess.call(relaunch_command(sys.argv[1:], args.gpus, free_port()))
            raise SystemExit(rc)
        world = 1
    else:
        world = int(os.environ["WORLD_SIZE"])
        if world != args.gpus:
            raise SystemExit(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}; launch one rank per GPU")
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return

    import torch
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    init_ranks("nccl", device, world)
    from compressed_decode_attention_equal_b200 import build
    build.build()
    if args.only:
        import workloads
        w = workloads.WORKLOADS[WORKLOAD]
        stage = {"coarsen": lambda: coarsen_stage(device, batch=args.coarsen_batch),
                 "diagonal": lambda: diagonal_closure_stage(w, device, args.layers, steps=args.steps),
                 "stream": lambda: stream_stage(w, device, steps=args.steps),
                 "other": lambda: other_decode_stage(device, steps=args.steps)}[args.only]
        print(json.dumps({"stage": args.only, "result": stage()}), flush=True)
        return
    res, caches, table, w = run_ours(args, rank, world, device)
    # the single-GPU characterisations and the CPU baseline run at N = 1 only: under torchrun the
    # other ranks would hold their GPUs idle at the closing barrier meanwhile
    if rank == 0 and world == 1:
        if not args.no_coarsen:
            res["coarsen"] = coarsen_stage(device, batch=args.coarsen_batch)
        if not args.no_diagonal:
            res["diagonal_closure"] = diagonal_closure_stage(w, device, args.layers)
        if not args.no_stream:
            res["streaming_append"] = stream_stage(w, device)
        if not args.no_other:
            res["other_decode"] = other_decode_stage(device)
        if not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline(w, caches, table)
    if rank == 0:
        print(json.dumps(res), flush=True)
    finish_ranks(world)


if __name__ == "__main__":
    main()
