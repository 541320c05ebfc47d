"""Benchmark of the MLA latent-KV decode step on B200 (one JSON line on rank 0).

A step is one pass of the whole decode path over one batch: latent append,
absorbed queries, split-KV decode, split combine, output projection.  The
default workload is the DeepSeek-V3-shaped decode (batch 64, ragged cached
lengths U[1024, 8192] + 1 new token each, 64-token pages in shuffled order,
seed 0): the configuration on which the decode roofline target is stated.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   # the fp64 oracle on the host cores
  python bench.py --workload v3_b4_long --shards 2   # also the sequence split

Besides the eager step the line carries `e2e` (pinned host inputs and
outputs through `DecodeLayer.run_from_host`), `graph_replay` (the step
recorded once as a CUDA graph and replayed) and, with `--shards N`,
`sequence_split` (each shard's decode and the merge, timed on one GPU).

Timing: every step is bracketed by CUDA events on the stream the library
launches on; the L2 is flushed before every step, outside the events (a
256 MiB write, then a 256 MiB read so the written-back lines do not land in
the next step); K steps run between a barrier + synchronize on both sides; with
N > 1 processes (torchrun), each rank runs its own replica of the workload
(weak scaling, no collective on the data path) and the step time is the max
over ranks.
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
import threading
import time
from pathlib import Path

import torch

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

from mla_synth import WORKLOADS, device_inputs, generate  # noqa: E402

DEFAULT_WORKLOAD = "v3_b64_ragged1k_8k"
L2_FLUSH_BYTES = 256 << 20


# ----------------------------------------------------------------- helpers

def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), \
        int(os.environ.get("LOCAL_RANK", 0))


def rank_seed(base_seed: int, rank: int) -> int:
    """Each rank's replica draws its own inputs (weak scaling)."""
    return base_seed + rank


def max_over_ranks(value: float, device=None) -> float:
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, device=None) -> float:
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def measured_peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}


# The sources the decode kernel is built from: a recorded DRAM traffic figure
# is only reported while none of them has changed since it was measured.
DECODE_SOURCES = ("common.cuh", "sm100.cuh", "decode_plan.cuh", "decode_pair.cuh")


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for name in DECODE_SOURCES:
        h.update((ROOT / "mla_latent_kv_39_b200" / "csrc" / name).read_bytes())
    return h.hexdigest()[:16]


def decode_flops(wl, data) -> float:
    """Tensor work of one decode call: per query row and visible cached row,
    2 H (d_c + d_r) for the scores and 2 H d_c for P V."""
    sh = wl.shape
    per_row = 2 * sh.n_heads * (sh.d_c + sh.d_r) + 2 * sh.n_heads * sh.d_c
    seq = data.seq_lens.to(torch.int64)
    visible = int((seq * wl.n_q).sum()) - wl.batch * (wl.n_q * (wl.n_q - 1) // 2)   # sum over rows of L - n_q + j + 1
    return float(per_row) * visible


def decode_roofline(wl, data, cache_bytes: int, dec_s: float, peaks, traffic):
    """Roofline of the decode call.  Its floor is max(cache bytes / HBM peak,
    tensor work / bf16 peak): one query token per sequence (decode) sits at
    the HBM / tensor ridge and is quoted against HBM; several causal query
    tokens per sequence (multi-token decode, chunked prefill) multiply the
    tensor work per cached byte and are quoted against the tensor peak once
    that term is the larger."""
    flops = decode_flops(wl, data)
    hbm_s = cache_bytes / (peaks["hbm_gbs"] * 1e9)
    tensor_s = flops / (peaks["bf16_tflops"] * 1e12)
    kernel = "mla_decode_packed_planned call (the pair decode kernel; its split plan runs beside the query projections)"
    if wl.fp8_cache:
        kernel = ("mla_cache_dequant_fp8 + mla_decode_packed_planned calls (the step's E4M3 pages expanded "
                  "into a bf16 scratch cache, then the pair decode)")
    if wl.n_q > 1 and tensor_s > hbm_s:
        achieved = flops / dec_s / 1e12
        return {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / peaks["bf16_tflops"], "traffic": traffic, "kernel": kernel,
                "algorithmic_flops_per_launch": flops, "algorithmic_bytes_per_launch": cache_bytes,
                "hbm_floor_us": hbm_s * 1e6, "tensor_floor_us": tensor_s * 1e6, "peak_source": peaks["source"]}
    achieved = cache_bytes / dec_s / 1e9
    return {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"], "frac_of_nominal_8tbs": achieved / NOMINAL_HBM_GBS,
            "traffic": traffic, "kernel": kernel, "algorithmic_bytes_per_launch": cache_bytes,
            "algorithmic_flops_per_launch": flops, "hbm_floor_us": hbm_s * 1e6, "tensor_floor_us": tensor_s * 1e6,
            "peak_source": peaks["source"]}


def recorded_traffic(workload: str):
    """DRAM bytes per decode launch from the committed ncu summary, if the
    kernel sources are unchanged since it was taken (else None)."""
    p = ROOT / "profiles" / "decode_traffic.json"
    if not p.exists():
        return None
    d = json.loads(p.read_text())
    if d.get("source_hash") != kernel_source_hash() or d.get("workload") != workload:
        return None
    return d.get("dram_bytes_per_launch")


class ClockSampler:
    """SM clock and throttle reasons of this process's GPU, sampled through NVML
    (the library nvidia-smi reads) every 5 ms while the timed region runs."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, index: int, period_s: float = 0.005):
        self.index, self.period, self.rows, self.err = index, period_s, [], None
        self.max_mhz = None
        self._stop = threading.Event()
        try:  # NVML start-up takes longer than a short timed region: do it first
            self.nv, self.h = self._handle()
            self.max_mhz = self.nv.nvmlDeviceGetMaxClockInfo(self.h, self.nv.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: report unsampled
            self.nv, self.err = None, repr(e)

    def _handle(self):
        import pynvml
        pynvml.nvmlInit()
        u = bytes(torch.cuda.get_device_properties(self.index).uuid.bytes).hex()
        uuid = f"GPU-{u[0:8]}-{u[8:12]}-{u[12:16]}-{u[16:20]}-{u[20:32]}"
        return pynvml, pynvml.nvmlDeviceGetHandleByUUID(uuid)

    def _run(self):
        if self.nv is None:
            return
        nv, h = self.nv, self.h
        try:
            while True:  # at least one sample, even for a very short region
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.rows.append((sm, reasons))
                if self._stop.wait(self.period):
                    break
        except Exception as e:
            self.err = repr(e)

    def __enter__(self):
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        self.thread.join(timeout=5)

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "error": self.err}
        reasons = sorted({name for _, r in self.rows for bit, name in self.REASONS.items() if r & bit})
        return {"sm_mhz": statistics.median(sm for sm, _ in self.rows), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.rows)}


def percentiles(xs):
    """p50 / p95 / p99 of a list of per-step times (nearest rank)."""
    v = sorted(xs)
    if not v:
        return None
    pick = lambda q: v[min(len(v) - 1, max(0, math.ceil(q * len(v)) - 1))]
    return {"p50": pick(0.50), "p95": pick(0.95), "p99": pick(0.99)}


NOMINAL_HBM_GBS = 8000.0  # spec-sheet HBM3e bandwidth the target is also quoted against


# ----------------------------------------------------------------- CPU oracle

def oracle_sample(wl, budget_s: float = 15.0, max_seqs: int = 64, data=None, W=None, first: int = 0):
    """Time the fp64 oracle (decompressed order) on whole sequences of ``wl``
    until ``budget_s`` of CPU time is spent; returns (tokens/s, sample text, cores)."""
    import numpy as np
    import oracle
    data = data if data is not None else generate(wl)
    shape = wl.shape
    W = W if W is not None else {k: oracle.to64(v) for k, v in data.weights.items()}
    done_tok, t_spent, seqs = 0, 0.0, 0
    for i in range(min(wl.batch, max_seqs)):
        b = (first + i) % wl.batch
        s, e = int(data.row_offsets[b]), int(data.row_offsets[b + 1])
        rows = oracle.to64(data.cached_rows[s:e]) if data.cached_rows is not None else None
        toks = slice(b * wl.n_q, (b + 1) * wl.n_q)
        t0 = time.perf_counter()
        if wl.fp8_cache:      # the values the stored E4M3 codes and row scales stand for
            rows = oracle.e4m3_value(data.cached_codes[s:e].numpy()) * oracle.to64(data.cached_scale[s:e])[:, None]
        if rows is None:
            c, kr = oracle.latent_rows(data.x_cached[s:e], W["W_DKV"], W["W_KR"], np.arange(e - s),
                                       shape.rope_theta, shape.dtype)
        else:
            c, kr = rows[:, :shape.d_c], rows[:, shape.d_c:]
        pos = data.new_positions().numpy()[toks]
        oracle.decode_step(shape, W, oracle.to64(data.x_new[toks]), pos, [c], [kr], wl.n_q,
                           order="decompressed", cache_dtype="fp8" if wl.fp8_cache else None)
        t_spent += time.perf_counter() - t0
        done_tok += wl.n_q
        seqs += 1
        if t_spent >= budget_s:
            break
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    threads = torch.get_num_threads()
    sample = (f"{seqs} of {wl.batch} sequences ({done_tok} query tokens, full decode step: append, "
              f"queries, decompressed attention over all heads, output projection) in {t_spent:.1f} s")
    return done_tok / t_spent, sample, min(cores, max(threads, 1))


# ----------------------------------------------------------------- main arms

METRIC = "MLA decode tokens/s and latent-KV GB/s (% of HBM roofline), 1 B200"


def run_reference(args):
    """The fp64 oracle on the host cores, on the same workload.  Each step is a
    bounded sample of that workload: whole sequences (all their query
    tokens) until the step's CPU-time budget is spent; the line reports what
    was actually timed (tokens and seconds of the timed steps)."""
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import oracle
    wl = WORKLOADS[args.workload]
    data = generate(wl)
    W = {k: oracle.to64(v) for k, v in data.weights.items()}
    n = args.steps + args.warmup
    step_budget = max(30.0, min(180.0, 6.0 * n)) / n
    tokens, seconds, samples = 0, 0.0, []
    cores = 1
    for i in range(n):
        t0 = time.perf_counter()
        tps, sample, cores = oracle_sample(wl, budget_s=step_budget, max_seqs=wl.batch, data=data, W=W,
                                           first=i)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            tokens += int(round(tps * dt)) if tps else 0
            seconds += dt
            samples.append(sample)
    value = tokens / seconds if seconds > 0 else 0.0
    sample = (f"{args.steps} timed steps, each whole sequences of {wl.name} until {step_budget:.1f} s of CPU "
              f"work: {tokens} query tokens in {seconds:.1f} s (full decode step per token: append, queries, "
              f"decompressed attention over all heads, output projection)")
    line = {
        "impl": "reference",
        "metric": METRIC,
        "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1000.0 * seconds / max(args.steps, 1),
        "tokens_per_step": tokens / max(args.steps, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": wl.name, "batch": wl.batch, "n_q": wl.n_q},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def measure_sequence_split(layer, dev, wl, n_shards: int, steps: int, flush_l2):
    """The sequence split across GPUs, its device work emulated on this GPU:
    each shard's decode (its pages only, one query per row, then its
    (o_lat, lse)) timed on its own, and the merge of the shards' pairs.  On
    n_shards GPUs the shards run at once, so the split decode takes the
    slowest shard plus the exchange (not run here: one GPU) plus the merge."""
    import mla_latent_kv_39_b200 as mla
    cfg, rows = layer.dcfg, wl.n_tok
    if not layer.packed:
        return {"shards": n_shards, "unavailable": "the sequence split decodes the packed bf16 query"}
    plan = mla.shard_plan(dev["block_table"].cpu(), dev["seq_lens"].cpu(), wl.n_q, wl.shape.block_size, n_shards)
    caches = [mla.Cache(dev["pool"], t.to(dev["pool"].device)) for t in plan.block_tables]
    lens = [x.to(dev["pool"].device) for x in plan.seq_lens]
    ws = torch.empty(mla.mla_decode_workspace_size(cfg, rows, 1, 0), dtype=torch.uint8, device=dev["pool"].device)
    H, d_c = cfg.n_heads, cfg.d_c
    o_parts = torch.empty(n_shards, rows, H, d_c, dtype=torch.float32, device=ws.device)
    lse_parts = torch.empty(n_shards, rows, H, dtype=torch.float32, device=ws.device)
    o = torch.empty(rows, H, d_c, dtype=torch.float32, device=ws.device)
    shard_ms = [[] for _ in range(n_shards)]
    merge_ms = []
    for it in range(steps + 2):
        for r in range(n_shards):
            flush_l2()
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
            ev[0].record()
            mla.decode_shard(cfg, layer.q_packed, rows, caches[r], lens[r], ws, o_parts[r], lse_parts[r])
            ev[1].record()
            torch.cuda.synchronize()
            if it >= 2:
                shard_ms[r].append(ev[0].elapsed_time(ev[1]))
        flush_l2()   # also keeps the GPU busy while the host enqueues the timed launch
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        ev[0].record()
        mla.mla_merge_shards(cfg, o_parts, lse_parts, o)
        ev[1].record()
        torch.cuda.synchronize()
        if it >= 2:
            merge_ms.append(ev[0].elapsed_time(ev[1]))
    mla.check_device_error()
    per_shard = [statistics.median(m) for m in shard_ms]
    return {"shards": n_shards, "shard_decode_ms": per_shard, "slowest_shard_ms": max(per_shard),
            "merge_ms": statistics.median(merge_ms),
            "exchange_bytes_per_gpu": int(rows * H * (d_c + 1) * 4),
            "note": "each shard's decode timed alone on one GPU (L2 flushed before); on one GPU per shard they "
                    "run at once, plus an all-gather of the exchange bytes"}


def run_ours(args):
    rank, world, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)

    import mla_latent_kv_39_b200 as mla

    base = WORKLOADS[args.workload]
    import dataclasses
    wl = dataclasses.replace(base, seed=rank_seed(base.seed, rank))
    data = generate(wl)
    dev = device_inputs(data, device)
    cfg = mla.Config.from_shape(wl.shape, split_query=wl.split_query, fp8_cache=wl.fp8_cache)
    cache = mla.Cache(dev["pool"], dev["block_table"], dev["row_scale"])
    layer = mla.DecodeLayer(cfg, dev["weights"], cache, wl.batch, wl.n_q, args.max_workers)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    clean = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)

    def flush_l2():
        # Overwrite L2 with a buffer larger than it, then read another one so
        # the dirty lines are written back here rather than inside the step.
        flush.fill_(1)
        clean.sum()
    stream = torch.cuda.current_stream()
    x, seq_idx, pos, seq_lens = dev["x_new"], dev["seq_idx"], dev["pos"], dev["seq_lens"]
    # every step appends the same positions again (the appended rows are rewritten identically)

    def one_step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        layer.append_and_queries(x, seq_idx, pos, seq_lens=seq_lens)   # the split plan beside the projections
        if ev is not None:
            ev[1].record(stream)
        layer.decode(seq_lens, planned=layer.packed)
        if ev is not None:
            ev[2].record(stream)
        if not layer.fused_out:     # bf16: the split merge runs inside the W_UV projection
            layer.combine()
        layer.project()
        if ev is not None:
            ev[3].record(stream)

    for _ in range(args.warmup):
        flush_l2()
        one_step()
    torch.cuda.synchronize()
    mla.check_device_error()

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize()

    events = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    launches0 = mla.mla_kernel_launches()
    barrier()
    wall0 = time.perf_counter()
    with ClockSampler(local) as clocks:
        for k in range(args.steps):
            flush_l2()
            one_step(events[k])
        barrier()
    wall = time.perf_counter() - wall0
    launches = mla.mla_kernel_launches() - launches0
    mla.check_device_error()
    step_ms = [e[0].elapsed_time(e[3]) for e in events]
    dec_ms = [e[1].elapsed_time(e[2]) for e in events]
    total_ms = max_over_ranks(sum(step_ms), device)
    tokens = sum_over_ranks(float(wl.n_tok * args.steps), device)
    value = tokens / (total_ms / 1000.0)

    # end to end through the public API with host (pinned) buffers
    x_h = data.x_new.pin_memory()
    seq_idx_h = data.new_seq_idx().pin_memory()
    pos_h = data.new_positions().pin_memory()
    seq_lens_h = data.seq_lens.to(torch.int32).pin_memory()
    y_h = torch.empty(layer.y.shape, dtype=layer.y.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in (x_h, seq_idx_h, pos_h, seq_lens_h))
    d2h = y_h.numel() * y_h.element_size()
    # K steps back to back through the public API, pipelined the way a serving
    # loop runs them: step k + 1's inputs go up and step k's y comes down on a
    # copy stream while step k computes.  No L2 flush here: one step touches
    # the whole cache and all weights (hundreds of MB, far beyond the 126 MB L2).
    y_hs = [torch.empty(layer.y.shape, dtype=layer.y.dtype).pin_memory() for _ in range(args.steps)]
    host_in = [(x_h, seq_idx_h, pos_h, seq_lens_h)] * args.steps
    layer.run_from_host(host_in[:max(1, args.warmup)], y_hs[:max(1, args.warmup)], stream=stream)
    e2e_ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    barrier()
    e2e_ev[0].record(stream)
    layer.run_from_host(host_in, y_hs, stream=stream)
    e2e_ev[1].record(stream)
    barrier()
    e2e_ms = max_over_ranks(e2e_ev[0].elapsed_time(e2e_ev[1]), device)
    e2e_value = tokens / (e2e_ms / 1000.0)

    # the same step replayed from a CUDA graph (launches and the side-stream
    # fork / join recorded once, no host work per step), L2 flushed between
    graph = layer.capture_step(x, seq_idx, pos, seq_lens)
    for _ in range(args.warmup):
        flush_l2()
        graph.replay()
    g_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    barrier()
    for k in range(args.steps):
        flush_l2()
        g_ev[k][0].record(stream)
        graph.replay()
        g_ev[k][1].record(stream)
    barrier()
    graph_ms = [a.elapsed_time(b) for a, b in g_ev]
    graph_total = max_over_ranks(sum(graph_ms), device)
    del graph
    mla.check_device_error()

    split = None
    if args.shards > 1 and world == 1:
        split = measure_sequence_split(layer, dev, wl, args.shards, max(3, min(args.steps, 10)), flush_l2)

    peaks = measured_peaks()
    cache_bytes = int(data.seq_lens.sum()) * wl.cache_row_bytes
    dec_avg_s = statistics.mean(dec_ms) / 1000.0
    achieved = cache_bytes / dec_avg_s / 1e9
    traffic = recorded_traffic(wl.name)
    roof = decode_roofline(wl, data, cache_bytes, dec_avg_s, peaks, traffic)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return 0

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        tps, sample, cores = oracle_sample(wl, budget_s=args.cpu_budget, max_seqs=wl.batch)
        cpu = {"value": tps, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample}
    ms_per_step = total_ms / args.steps
    line = {
        "metric": METRIC,
        "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if wl.shape.dtype == "bf16" else "f32",
        "data": "synthetic (seeded; random-init weights of the V3 layer shape)",
        "config": {"workload": wl.name, "batch": wl.batch, "n_q": wl.n_q,
                   "cached_len": (f"{int(data.cached_len.min())}..{int(data.cached_len.max())}"),
                   "cache_rows": int(data.seq_lens.sum()), "block_size": wl.shape.block_size,
                   "page_order": "shuffled" if wl.shuffled_blocks else "in order",
                   "l2": "flushed before every step outside the timed events (256 MiB write, then a 256 MiB read)",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "cache_format": "e4m3 codes + fp32 row scale" if wl.fp8_cache else wl.shape.dtype},
        "latent_kv_gbs": achieved,
        "decode_ms": statistics.mean(dec_ms),
        "step_ms_percentiles": percentiles(step_ms),
        "decode_ms_percentiles": percentiles(dec_ms),
        "roofline": roof,
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / args.steps,
                "mode": "pinned host inputs and outputs, copies overlapped with the neighbouring steps; "
                        "no L2 flush (each step touches the whole cache and all weights)"},
        "graph_replay": {"value": tokens / (graph_total / 1000.0), "unit": "tokens/s",
                         "ms_per_step": graph_total / args.steps, "step_ms_percentiles": percentiles(graph_ms),
                         "mode": "the step captured once as a CUDA graph (capture_step) and replayed; "
                                 "L2 flushed outside the timed events"},
        "gpu_launches": launches,
        "clocks": clocks.summary(),
        "wall_s_timed_region": wall,
        "cpu_baseline": cpu,
        **({"sequence_split": split} if split is not None else {}),
    }
    print(json.dumps(line), flush=True)
    return 0


def parse(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--max-workers", type=int, default=0)
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--shards", type=int, default=0,
                    help="also time the sequence split across this many GPUs (emulated on one: each shard's "
                         "decode alone, and the merge)")
    return ap.parse_args(argv)


def main(argv=None):
    args = parse(argv)
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
