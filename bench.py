"""Benchmark of the paged KV-cache hot path on B200: one step = pa_reshape_and_cache
(the step's new K/V into the pool) + pa_decode (paged attention over the pool),
through the C ABI of libpa_b200.so, on seeded synthetic inputs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload llama8b]
    python bench.py --impl reference ...        # the fp64 CPU oracle, timed on host cores
    torchrun --nproc-per-node N bench.py --gpus N ...   (one independent replica per GPU)

Prints ONE JSON line (rank 0). value = algorithmic bytes of all ranks' steps /
max-over-ranks device time, in GB/s.
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
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

DEFAULT_WORKLOAD = "llama8b"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM traffic per pa_decode launch measured by ncu (dram__bytes_read.sum +
# dram__bytes_write.sum summed over the launch's kernels), keyed by workload, with
# the hash of the kernel sources it was measured on. A different hash -> null.
NCU_TRAFFIC = {
    # dram__bytes_read.sum + dram__bytes_write.sum over the kernels of one pa_decode call (mean
    # of three calls), from one ncu capture per workload (commands in profiles/); valid only for
    # the kernel sources they were taken on
    "llama8b": {"source_hash": "14d5107606101b9d", "bytes_per_launch": 654_760_000},
    "llama70b_long": {"source_hash": "14d5107606101b9d", "bytes_per_launch": 1_352_130_000},
    "spec_verify": {"source_hash": "14d5107606101b9d", "bytes_per_launch": 414_730_000},
    "prefix_sharing": {"source_hash": "14d5107606101b9d", "bytes_per_launch": 210_150_000},
    "sliding_window": {"source_hash": "14d5107606101b9d", "bytes_per_launch": 273_290_000},
    "llama8b_fp8": {"source_hash": "14d5107606101b9d", "bytes_per_launch": 280_710_000},
}

# the same for one pa_copy_blocks launch of a copy workload (keyed by COPY_SOURCES' hash;
# mean of three 2048-pair launches: the writes still in L2 when a launch ends are not
# counted, so the traffic sits below the algorithmic bytes)
NCU_COPY_TRAFFIC = {
    "cow_bulk": {"source_hash": "d46ea268e31f8d30", "bytes_per_launch": 211_644_000},
}


# ------------------------------------------------------------------ accounting

def kv_bytes_per_token(layers: int, kv_heads: int, head_dim: int, bytes_per_value: int = 2) -> int:
    """KV-cache bytes per token of a model: K and V, every layer and kv head."""
    return 2 * layers * kv_heads * head_dim * bytes_per_value


def decode_bytes(w, unique: bool = True) -> int:
    """Algorithmic bytes of one pa_decode call: the K/V of every visible token (shared
    physical slots counted once when `unique`), q, out, the used block-table
    entries and context_lens."""
    bs = w.block_size
    win = getattr(w, "window", 0)
    # the first position any query row of a sequence sees (its first row's window start)
    lo = [max(0, int(c) - w.q_per_seq - win + 1) if win > 0 else 0 for c in w.context_lens]
    if unique:
        ranges = {}   # physical block -> offset ranges [s, e) some sequence sees
        for b in range(w.num_seqs):
            ctx = int(w.context_lens[b])
            tbl = w.block_tables[b]
            for j in range(lo[b] // bs, -(-ctx // bs)):
                s, e = max(lo[b], j * bs) - j * bs, min(ctx, (j + 1) * bs) - j * bs
                ranges.setdefault(int(tbl[j]), []).append((s, e))
        tokens = 0
        for rs in ranges.values():   # a slot seen by several sequences counts once
            end = 0
            for s, e in sorted(rs):
                s = max(s, end)
                if e > s:
                    tokens += e - s
                    end = e
    else:
        tokens = int(sum(int(c) - l for c, l in zip(w.context_lens, lo)))
    kv = tokens * w.num_kv_heads * w.head_dim * kv_elem_bytes(w) * 2
    qo = 2 * w.num_seqs * w.q_per_seq * w.num_q_heads * w.head_dim * 2
    tables = int(sum(-(-int(c) // bs) - l // bs for c, l in zip(w.context_lens, lo))) * 4
    return kv + qo + tables + w.num_seqs * 4


def kv_elem_bytes(w) -> int:
    """Bytes of one cached K or V element: 2 (bf16) or 1 (an E4M3 code)."""
    return 1 if getattr(w, "kv_dtype", "bf16") == "fp8_e4m3" else 2


def cache_write_bytes(w) -> int:
    """K and V rows read (bf16) and written (bf16 or E4M3), plus the slot mapping."""
    elems = w.num_kv_heads * w.head_dim
    return w.num_tokens * (2 * elems * (2 + kv_elem_bytes(w)) + 8)


def prefill_flops(w) -> int:
    """QK^T and PV multiply-adds of a chunked-prefill step: chunk token i of sequence b sees
    ctx_b - qlen_b + i + 1 keys, for every query head."""
    vis = 0
    for c, q in zip(w.context_lens, w.query_lens):
        c, q = int(c), int(q)
        vis += q * (c - q) + q * (q + 1) // 2
    return 4 * w.head_dim * w.num_q_heads * vis


def prefill_bytes(w) -> int:
    """Bytes a chunked-prefill step must move at least once: the K/V of every sequence's
    context, q and out, the used table entries, context_lens and query_start."""
    kv = int(w.context_lens.astype(np.int64).sum()) * w.num_kv_heads * w.head_dim * 2 * 2
    qo = 2 * w.num_tokens * w.num_q_heads * w.head_dim * 2
    tables = int(sum(-(-int(c) // w.block_size) for c in w.context_lens)) * 4
    return kv + qo + tables + 4 * w.num_seqs + 4 * (w.num_seqs + 1)


def decode_flops(w) -> int:
    """QK^T and PV multiply-adds over the visible keys of every query row."""
    vis = 0
    for b in range(w.num_seqs):
        ctx = int(w.context_lens[b])
        vis += sum(ctx - w.q_per_seq + i + 1 for i in range(w.q_per_seq))
    return 4 * w.head_dim * (w.num_q_heads // w.num_kv_heads) * w.num_kv_heads * vis


# the sources each kernel family is compiled from (the decode kernels share nothing with
# the block copy, so a change to one leaves the other's measured traffic valid)
DECODE_SOURCES = ("pa_api.cpp", "pa_device.cuh", "pa_internal.h", "pa_kernels.cu", "pa_prefill.cuh",
                  "pa_static_scratch.cu", "pa_tcgen05.cuh")
COPY_SOURCES = ("pa_copy.cu",)
FP8_SOURCES = ("pa_fp8.cu",)   # the FP8 cache write (timed inside the llama8b_fp8 step)


def source_hash(names=DECODE_SOURCES) -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "paged_kv_cache_399_b200", "csrc")
    for name in sorted(names):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return dict(PEAKS_FALLBACK, source="fallback")


# ------------------------------------------------------------------ ranks

BASE_SEEDS = {"tiny": 1000, "llama8b": 1001, "llama70b_long": 1002, "prefix_sharing": 1003,
              "spec_verify": 1004, "cow_fork": 1005, "cow_bulk": 1006, "sliding_window": 1007,
              "llama8b_fp8": 1008, "chunked_prefill": 1009}


def rank_seed(workload: str, rank: int) -> int:
    """Weak scaling: every rank decodes its own replica of the workload, own seed."""
    return BASE_SEEDS[workload] + 100 * rank


def reduce_over_ranks(value: float, op: str, dist=None, device=None) -> float:
    """max / sum of a per-rank float over the default process group (no-op alone)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return float(t.item())


def aggregate_throughput(bytes_per_step_per_rank: float, steps: int, max_ms: float, world: int) -> float:
    """Whole-job GB/s: all ranks' bytes over the slowest rank's device time."""
    return world * bytes_per_step_per_rank * steps / (max_ms * 1e-3) / 1e9


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi samples of this GPU's clocks and throttle reasons while timing."""

    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, device_index: int):
        import torch
        self.uuid = None
        try:
            u = torch.cuda.get_device_properties(device_index).uuid
            self.uuid = "GPU-" + str(u)
        except Exception:
            pass
        self.proc = None
        self.lines = []

    def __enter__(self):
        cmd = ["nvidia-smi", f"--query-gpu={','.join(self.FIELDS)}", "--format=csv,noheader,nounits",
               "-lms", "100"]
        if self.uuid:
            cmd += ["-i", self.uuid]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)  # nvidia-smi's start-up and first sample, before the work it watches
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]
        return False

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ GPU arm

# The decode configurations every default run also times on the same box, beside the
# headline workload (µs/call per config is half of the metric).
PER_CONFIG = ("tiny", "llama8b", "llama70b_long", "prefix_sharing", "spec_verify", "sliding_window",
              "llama8b_fp8")
PREFILL_CONFIG = ("chunked_prefill",)
# the 75 % bar of the measured copy bandwidth holds on the three bandwidth-scale configs
BAR_CONFIGS = ("llama8b", "llama70b_long", "prefix_sharing")


def _device_inputs(w, dev):
    """The step's per-call inputs in one device buffer (and one pinned host buffer for the
    end-to-end leg, so a step's host->device traffic is a single copy), plus the pools."""
    import torch
    parts = [("query", w.query), ("key", w.key), ("value", w.value),
             ("slots", torch.from_numpy(w.slot_mapping)), ("tables", torch.from_numpy(w.block_tables)),
             ("ctx", torch.from_numpy(w.context_lens))]
    offsets, total = {}, 0
    for name, t in parts:
        offsets[name] = total
        total += (t.numel() * t.element_size() + 255) // 256 * 256
    h_in = torch.empty(total, dtype=torch.uint8, pin_memory=True)
    d_in = torch.empty(total, dtype=torch.uint8, device=dev)
    views = {}
    for name, t in parts:
        n = t.numel() * t.element_size()
        h_in[offsets[name]:offsets[name] + n].copy_(t.contiguous().view(-1).view(torch.uint8))
        views[name] = d_in[offsets[name]:offsets[name] + n].view(t.dtype).view(t.shape)
    d_in.copy_(h_in)
    views["h_in"], views["d_in"], views["in_bytes"] = h_in, d_in, total
    views["key_cache"] = w.key_cache.to(dev)
    views["value_cache"] = w.value_cache.to(dev)
    views["out"] = torch.empty_like(views["query"])
    return views


def _plan_for(pa, w, args):
    # a caller that batches parallel samples of one prompt knows it: ask for prefix sharing
    share = bool(w.shared_groups) and not args.no_share_prefix
    return pa.pa_decode_plan(w.num_seqs, w.q_per_seq, w.num_q_heads, w.num_kv_heads, w.head_dim,
                             w.max_blocks_per_seq, share_prefix=share, sliding_window=w.window,
                             path={"auto": 0, "single": 1, "tile": 2, "tcgen05": 3}[args.path],
                             split_blocks=args.split_blocks,
                             schedule={"auto": 0, "grid": 1, "persistent": 2}[args.schedule],
                             kv_cache_dtype=pa.PA_KV_FP8_E4M3 if w.kv_dtype == "fp8_e4m3" else pa.PA_KV_BF16)


def _hot_path(pa, w, v, plan, ws, stream):
    """The step's two calls for this workload's pools: (cache write, decode), each taking no
    arguments, prepared once on these buffers (pa.PreparedCacheWrite / pa.PreparedDecode, as a
    step loop that reuses its buffers calls them). FP8 pools take the FP8 cache write and
    pa_decode_fp8. decode(s) on another stream (a graph capture) takes the per-call pa_decode."""
    fp8 = w.kv_dtype == "fp8_e4m3"
    scales = {"k_scale": w.k_scale, "v_scale": w.v_scale} if fp8 else {}
    write = pa.PreparedCacheWrite(v["key"], v["value"], v["key_cache"], v["value_cache"], v["slots"],
                                  stream=stream, **scales)
    prepared = pa.PreparedDecode(v["out"], v["query"], v["key_cache"], v["value_cache"], v["tables"], v["ctx"],
                                 w.q_per_seq, w.scale, plan=plan, workspace=ws, stream=stream, **scales)

    def decode(s=stream):
        if s is stream:
            prepared()
        elif fp8:
            pa.pa_decode_fp8(v["out"], v["query"], v["key_cache"], v["value_cache"], v["tables"], v["ctx"],
                             w.q_per_seq, w.scale, w.k_scale, w.v_scale, plan=plan, workspace=ws, stream=s)
        else:
            pa.pa_decode(v["out"], v["query"], v["key_cache"], v["value_cache"], v["tables"], v["ctx"],
                         w.q_per_seq, w.scale, plan=plan, workspace=ws, stream=s)
    return write, decode


def _ncu_traffic(name):
    rec = NCU_TRAFFIC.get(name)
    if rec and rec.get("source_hash") == source_hash():
        return rec["bytes_per_launch"]
    return None


def _time_calls(pa, w, v, plan, ws, stream, calls, barrier, flush=None):
    """CUDA-event times of `calls` pa_decode calls (each after the step's cache write, events
    on the launching stream around the decode only), queued behind a sleep kernel so that the
    host's own time per call (the binding, the C entry point) never leaves the GPU idle inside
    an interval: their mean and median in ms, the device time of a call; the mean of the same
    calls made one after another with nothing queued (host-paced: an interval then also holds
    whatever the GPU waits for the host's next launch); the median
    of the same calls made cold, with `flush` (a buffer twice the L2 size) read before each
    step outside the events (None without `flush`): a read leaves L2 holding clean lines of
    the buffer, where a write would leave dirty lines whose write-back the decode would pay
    for; the calls without host overhead: one CUDA graph of 20
    back-to-back calls, replayed (µs per call, None when capture is unavailable); and the mean
    event time of the step's cache writes (ms), timed apart from the decode."""
    import torch
    write, decode = _hot_path(pa, w, v, plan, ws, stream)
    barrier()
    def per_call(queued):
        # one event between the write and the decode ends the one and starts the other
        triples = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(calls)]
        if queued:   # about 5 ms of GPU time: the host enqueues every call before the GPU reaches them
            torch.cuda._sleep(10_000_000)
        for c, a, b in triples:
            c.record(stream)
            write()
            a.record(stream)
            decode()
            b.record(stream)
        barrier()
        return [a.elapsed_time(b) for _, a, b in triples], [c.elapsed_time(a) for c, a, _ in triples]
    times, writes = per_call(True)
    decode_ms, median_ms = statistics.mean(times), statistics.median(times)
    write_ms = statistics.mean(writes)
    paced_ms = statistics.mean(per_call(False)[0])
    cold_ms = None
    if flush is not None:
        pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(calls)]
        sink = torch.empty((), dtype=flush.dtype, device=flush.device)
        for a, b in pairs:
            torch.amax(flush, dim=0, out=sink)
            write()
            a.record(stream)
            decode()
            b.record(stream)
        barrier()
        cold_ms = statistics.median(a.elapsed_time(b) for a, b in pairs)
    graph_us = None
    try:
        per_graph, reps = 20, max(1, calls // 20)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for _ in range(per_graph):
                decode(None)   # the capture stream
        graph.replay()
        barrier()
        g0 = torch.cuda.Event(enable_timing=True)
        g1 = torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for _ in range(reps):
            graph.replay()
        g1.record(stream)
        barrier()
        graph_us = g0.elapsed_time(g1) * 1e3 / (reps * per_graph)
        del graph
    except Exception as exc:  # capture is a measurement aid: report why it is missing
        print(f"graph timing unavailable: {exc}", file=sys.stderr)
    return decode_ms, median_ms, cold_ms, graph_us, write_ms, paced_ms


def measure_config(name, args, dev, stream, peaks):
    """One decode configuration on this GPU: µs per pa_decode call (CUDA events, and
    graph-replayed), GB/s of its algorithmic bytes, the fraction of the measured copy
    bandwidth, its plan, the ncu traffic (when taken on these sources) and the clocks."""
    import torch
    from paged_kv_cache_399_b200 import pa, workloads
    w = workloads.make(name, seed=rank_seed(name, 0))
    v = _device_inputs(w, dev)
    plan = _plan_for(pa, w, args)
    ws_bytes = pa.pa_decode_workspace_size(plan, w.num_seqs, w.q_per_seq, w.num_q_heads,
                                           w.num_kv_heads, w.head_dim, w.max_blocks_per_seq)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev) if ws_bytes else None

    def barrier():
        torch.cuda.synchronize(dev)

    write, decode = _hot_path(pa, w, v, plan, ws, stream)
    for _ in range(max(3, args.warmup)):
        write()
        decode()
    barrier()
    assert pa.pa_get_device_error(reset=True, stream=stream) == 0
    flush = torch.zeros(2 * L2_BYTES, dtype=torch.uint8, device=dev)
    sampler = ClockSampler(dev.index)
    with sampler:
        decode_ms, median_ms, cold_ms, graph_us, write_ms, paced_ms = _time_calls(
            pa, w, v, plan, ws, stream, args.config_calls, barrier, flush)
    assert pa.pa_get_device_error(reset=True, stream=stream) == 0
    del flush
    dec_bytes = decode_bytes(w)
    gbs = dec_bytes / (decode_ms * 1e-3) / 1e9
    rec = {
        "workload": w.describe(),
        "calls": args.config_calls,
        "decode_us_per_call": round(decode_ms * 1e3, 3),
        "decode_us_per_call_median": round(median_ms * 1e3, 3),
        # the same calls made one after another with nothing queued ahead of them
        "decode_us_per_call_host_paced": round(paced_ms * 1e3, 3),
        # L2 filled with another buffer (one twice its size read) before every step, outside the events
        "decode_us_per_call_cold": round(cold_ms * 1e3, 3),
        "frac_cold": round(dec_bytes / (cold_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
        "decode_us_per_call_graph": None if graph_us is None else round(graph_us, 3),
        "decode_alg_bytes": dec_bytes,
        "decode_logical_bytes": decode_bytes(w, unique=False),
        "decode_gbs": round(gbs, 2),
        "frac": round(gbs / peaks["hbm_gbs"], 4),
        "frac_graph": None if graph_us is None else round(dec_bytes / (graph_us * 1e-6) / 1e9 / peaks["hbm_gbs"], 4),
        "plan": plan.as_dict(),
        "ncu_traffic": _ncu_traffic(name),
        "cache_write_us_per_call": round(write_ms * 1e3, 3),
        "cache_write_bytes": cache_write_bytes(w),
        "clocks": sampler.summary(),
    }
    if name in BAR_CONFIGS:
        rec["bar_us_at_75pct"] = round(dec_bytes / (0.75 * peaks["hbm_gbs"] * 1e9) * 1e6, 2)
    del v, ws
    torch.cuda.empty_cache()
    return rec


NCU_PREFILL_TRAFFIC = {
    # dram__bytes_read.sum + dram__bytes_write.sum of one pa_prefill launch (mean of three),
    # valid only for the kernel sources it was taken on
    "chunked_prefill": {"source_hash": "14d5107606101b9d", "bytes_per_launch": 142_000_000},
}


def measure_prefill(name, args, dev, stream, peaks):
    """The chunked-prefill step (pa_reshape_and_cache of the chunks' K/V + pa_prefill): µs
    per pa_prefill call (CUDA events, and graph-replayed), its TFLOP/s against the measured
    sustained bf16 tensor peak, and its bytes over the copy bandwidth."""
    import torch
    from paged_kv_cache_399_b200 import pa, workloads
    w = workloads.PREFILL_WORKLOADS[name](seed=rank_seed(name, 0))
    parts = {"query": w.query, "key": w.key, "value": w.value}
    v = {k: t.to(dev) for k, t in parts.items()}
    v["slots"] = torch.from_numpy(w.slot_mapping).to(dev)
    v["tables"] = torch.from_numpy(w.block_tables).to(dev)
    v["ctx"] = torch.from_numpy(w.context_lens).to(dev)
    v["qstart"] = torch.from_numpy(w.query_start).to(dev)
    v["key_cache"] = w.key_cache.to(dev)
    v["value_cache"] = w.value_cache.to(dev)
    v["out"] = torch.empty_like(v["query"])

    def write():
        pa.pa_reshape_and_cache(v["key"], v["value"], v["key_cache"], v["value_cache"], v["slots"], stream=stream)

    def prefill(s=stream):
        pa.pa_prefill(v["out"], v["query"], v["key_cache"], v["value_cache"], v["tables"], v["ctx"], v["qstart"],
                      w.max_query_len, w.scale, stream=s)

    for _ in range(max(3, args.warmup)):
        write()
        prefill()
    torch.cuda.synchronize(dev)
    assert pa.pa_get_device_error(reset=True, stream=stream) == 0
    calls = args.config_calls
    sampler = ClockSampler(dev.index)
    with sampler:
        pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(calls)]
        for a, b in pairs:
            write()
            a.record(stream)
            prefill()
            b.record(stream)
        torch.cuda.synchronize(dev)
        ms = statistics.mean(a.elapsed_time(b) for a, b in pairs)
        graph_us = None
        try:
            per_graph, reps = 10, max(1, calls // 10)
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                for _ in range(per_graph):
                    prefill(None)
            graph.replay()
            torch.cuda.synchronize(dev)
            g0 = torch.cuda.Event(enable_timing=True)
            g1 = torch.cuda.Event(enable_timing=True)
            g0.record(stream)
            for _ in range(reps):
                graph.replay()
            g1.record(stream)
            torch.cuda.synchronize(dev)
            graph_us = g0.elapsed_time(g1) * 1e3 / (reps * per_graph)
            del graph
        except Exception as exc:
            print(f"graph timing unavailable: {exc}", file=sys.stderr)
    assert pa.pa_get_device_error(reset=True, stream=stream) == 0
    flops = prefill_flops(w)
    tflops = flops / (ms * 1e-3) / 1e12
    peak = peaks["bf16_tflops_sustained"]
    rec = {
        "workload": w.describe(),
        "calls": calls,
        "prefill_us_per_call": round(ms * 1e3, 3),
        "prefill_us_per_call_graph": None if graph_us is None else round(graph_us, 3),
        "flops": flops,
        "tflops": round(tflops, 2),
        "frac_of_sustained_bf16": round(tflops / peak, 4),
        "frac_graph": None if graph_us is None else round(flops / (graph_us * 1e-6) / 1e12 / peak, 4),
        "alg_bytes": prefill_bytes(w),
        "bytes_frac_of_measured_hbm": round(prefill_bytes(w) / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
        "ncu_traffic": NCU_PREFILL_TRAFFIC.get(name, {}).get("bytes_per_launch")
        if NCU_PREFILL_TRAFFIC.get(name, {}).get("source_hash") == source_hash() else None,
        "clocks": sampler.summary(),
    }
    del v
    torch.cuda.empty_cache()
    return rec


def run_prefill_gpu(args):
    """--workload chunked_prefill: one JSON line for the chunked-prefill step alone (1 GPU;
    under torchrun every rank runs its own replica and rank 0 reports its own)."""
    import torch
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local_rank)
    from paged_kv_cache_399_b200 import build as pa_build
    pa_build.build()
    dev = torch.device("cuda", local_rank)
    peaks = measured_peaks()
    args.config_calls = max(args.steps, 3)
    rec = measure_prefill(args.workload, args, dev, torch.cuda.current_stream(dev), peaks)
    if int(os.environ.get("RANK", "0")) == 0:
        print(json.dumps({
            "metric": "pa_prefill achieved TFLOP/s & fraction of the sustained bf16 tensor peak",
            "value": rec["tflops"], "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(rec["prefill_us_per_call"] / 1e3, 6), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": rec,
            "roofline": {"bound": "tensor", "achieved": rec["tflops"], "peak": peaks["bf16_tflops_sustained"],
                         "unit": "TFLOP/s", "frac": rec["frac_of_sustained_bf16"], "traffic": rec["ncu_traffic"],
                         "peak_source": peaks["source"] + " (sustained bf16)", "kernel": "prefill_tcm_kernel"},
            "gpu_launches": 2 * args.steps,
            "clocks": rec["clocks"],
        }), flush=True)


def run_context_parallel_gpu(args):
    """--context-parallel: one decode of the workload split over the job's GPUs (strong scaling).
    Rank r reads table entries rank_block_range(max_blocks, r, N) of every sequence
    (pa_decode_partial), the pieces are all-gathered (NCCL) and every rank merges them
    (pa_merge_partials). The whole decode's algorithmic bytes over the slowest rank's event
    time per call; rank 0 also times pa_decode alone and checks the merged output against it."""
    import torch
    import torch.distributed as dist

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    from paged_kv_cache_399_b200 import build as pa_build
    pa_build.build()
    from paged_kv_cache_399_b200 import pa, workloads
    from paged_kv_cache_399_b200.context_parallel import gather_partials, partial_pieces, rank_block_range

    w = workloads.make(args.workload, seed=rank_seed(args.workload, 0))  # the same decode on every rank
    if w.kv_dtype != "bf16" or w.shared_groups or w.window:
        raise SystemExit("--context-parallel takes a bf16 workload without sharing or window")
    dev = torch.device("cuda", local_rank)
    v = _device_inputs(w, dev)
    pa.pa_reshape_and_cache(v["key"], v["value"], v["key_cache"], v["value_cache"], v["slots"])
    B, QS, HQ, D = w.query.shape
    lo, hi = rank_block_range(w.max_blocks_per_seq, rank, world)
    S = partial_pieces(v["query"], v["key_cache"], w.max_blocks_per_seq, world)
    part_o = torch.empty((S, B, QS, HQ, D), dtype=torch.float32, device=dev)
    part_ml = torch.empty((S, B, QS, HQ, 2), dtype=torch.float32, device=dev)
    rec_o = torch.empty((B, QS, HQ, D), dtype=torch.float32, device=dev)
    rec_ml = torch.empty((B, QS, HQ, 2), dtype=torch.float32, device=dev)
    out = torch.empty_like(v["query"])

    def call():
        pa.pa_decode_partial(part_o, part_ml, v["query"], v["key_cache"], v["value_cache"], v["tables"], v["ctx"],
                             w.q_per_seq, w.scale, lo, hi)
        pa.pa_combine_partials(rec_o, rec_ml, part_o, part_ml)
        if world > 1:
            all_o, all_ml = gather_partials(rec_o, rec_ml)
        else:
            all_o, all_ml = rec_o.unsqueeze(0), rec_ml.unsqueeze(0)
        pa.pa_merge_partials(out, all_o, all_ml)

    def barrier():
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    sampler = ClockSampler(local_rank)
    with sampler:
        for _ in range(args.warmup):
            call()
        barrier()
        assert pa.pa_get_device_error(reset=True) == 0
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            call()
        e1.record()
        barrier()
        ms = reduce_over_ranks(e0.elapsed_time(e1), "max", dist if world > 1 else None, dev) / args.steps
    assert pa.pa_get_device_error(reset=True) == 0
    ref = torch.empty_like(out)
    plan = _plan_for(pa, w, args)
    ws_bytes = pa.pa_decode_workspace_size(plan, w.num_seqs, w.q_per_seq, w.num_q_heads, w.num_kv_heads,
                                           w.head_dim, w.max_blocks_per_seq)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev) if ws_bytes else None
    pa.pa_decode(ref, v["query"], v["key_cache"], v["value_cache"], v["tables"], v["ctx"], w.q_per_seq, w.scale,
                 plan=plan, workspace=ws)
    torch.cuda.synchronize(dev)
    diff = float((ref.float() - out.float()).abs().max())
    single_us = None
    if rank == 0:
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record()
        for _ in range(args.steps):
            pa.pa_decode(ref, v["query"], v["key_cache"], v["value_cache"], v["tables"], v["ctx"], w.q_per_seq,
                         w.scale, plan=plan, workspace=ws)
        f1.record()
        torch.cuda.synchronize(dev)
        single_us = f0.elapsed_time(f1) * 1e3 / args.steps
    dec_bytes = decode_bytes(w)
    gbs = dec_bytes / (ms * 1e-3) / 1e9
    peaks = measured_peaks()
    if rank == 0:
        print(json.dumps({
            "metric": "pa_decode of one batch split over the job's GPUs by table ranges (context parallelism): "
                      "achieved HBM GB/s of the whole decode",
            "value": round(gbs, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 6), "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {
                "workload": w.describe(),
                "step": "pa_decode_partial over this rank's table range + pa_combine_partials + all-gather (NCCL) "
                        "+ pa_merge_partials",
                "ranges": [rank_block_range(w.max_blocks_per_seq, r, world) for r in range(world)],
                "pieces_per_rank": S,
                "gather_bytes_per_rank": (rec_o.numel() + rec_ml.numel()) * 4,
                "decode_alg_bytes": dec_bytes,
                "frac_of_measured_hbm_per_gpu": round(gbs / world / peaks["hbm_gbs"], 4),
                "single_gpu_pa_decode_us": None if single_us is None else round(single_us, 3),
                "max_abs_diff_vs_pa_decode": diff,
                "parallelism": f"context parallel x{world} (one decode's blocks split across GPUs)",
            },
            "gpu_launches": 3 * args.steps,
            "clocks": sampler.summary(),
        }), flush=True)
    if world > 1:
        dist.destroy_process_group()


def run_gpu(args):
    import torch
    import torch.distributed as dist

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))

    from paged_kv_cache_399_b200 import build as pa_build
    pa_build.build()
    from paged_kv_cache_399_b200 import pa, workloads

    w = workloads.make(args.workload, seed=rank_seed(args.workload, rank))
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.current_stream(dev)
    v = _device_inputs(w, dev)
    query, key, value = v["query"], v["key"], v["value"]
    slots, tables, ctx = v["slots"], v["tables"], v["ctx"]
    key_cache, value_cache, out = v["key_cache"], v["value_cache"], v["out"]
    h_in, d_in, total = v["h_in"], v["d_in"], v["in_bytes"]
    plan = _plan_for(pa, w, args)
    ws_bytes = pa.pa_decode_workspace_size(plan, w.num_seqs, w.q_per_seq, w.num_q_heads,
                                           w.num_kv_heads, w.head_dim, w.max_blocks_per_seq)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev) if ws_bytes else None

    write, decode = _hot_path(pa, w, v, plan, ws, stream)

    def step():
        write()
        decode()

    def barrier():
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    def max_over_ranks(x: float) -> float:
        return reduce_over_ranks(x, "max", dist if world > 1 else None, dev)

    launches_per_step = 1 + decode_launches(plan)
    step_bytes = decode_bytes(w) + cache_write_bytes(w)
    dec_bytes = decode_bytes(w)

    sampler = ClockSampler(local_rank)
    with sampler:
        # warm-up once the clock sampler runs, right before the timed region: the GPU enters it
        # from work at its clocks, not from the sampler's start-up idle
        for _ in range(args.warmup):
            step()
        barrier()
        assert pa.pa_get_device_error(reset=True, stream=stream) == 0
        # (1) headline: K whole steps, events only around the region
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        barrier()
        ms_total = max_over_ranks(e0.elapsed_time(e1))

        # (2) per-kernel: events around each pa_decode launch of another K steps, and the
        # same calls graph-replayed (for the small configs the events mostly time the
        # Python call)
        decode_ms, _, _, graph_us, write_ms, paced_ms = _time_calls(pa, w, v, plan, ws, stream, args.steps,
                                                                   barrier)
        decode_ms = max_over_ranks(decode_ms)
        paced_ms = max_over_ranks(paced_ms)
        if graph_us is not None:
            graph_us = max_over_ranks(graph_us)

        # (3) end to end: every step's inputs come from pinned host memory and its output goes
        # back to it. Two input buffers and two outputs: one copy stream brings step k+1's inputs
        # and another takes step k-1's output while step k computes, ordered by events (a
        # step's compute waits for its inputs and for the copy-out of the output it reuses; an
        # input copy waits for the compute that last read its buffer).
        h_out = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        h2d = total
        d2h = h_out.numel() * h_out.element_size()
        e2e_steps = args.steps
        d_in2 = torch.empty_like(d_in)
        v2 = dict(v)
        for name in ("query", "key", "value", "slots", "tables", "ctx"):
            t = v[name]
            off = t.data_ptr() - d_in.data_ptr()
            v2[name] = d_in2[off:off + t.numel() * t.element_size()].view(t.dtype).view(t.shape)
        v2["out"] = torch.empty_like(out)
        write2, decode2 = _hot_path(pa, w, v2, plan, ws, stream)
        sets = [(d_in, write, decode, out), (d_in2, write2, decode2, v2["out"])]
        cs_in, cs_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        barrier()
        f0 = torch.cuda.Event(enable_timing=True)
        f1 = torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for k in range(e2e_steps):
            b = k & 1
            dbuf, wr, dc, o = sets[b]
            cs_in.wait_event(f0 if k < 2 else ev_done[b])
            with torch.cuda.stream(cs_in):
                dbuf.copy_(h_in, non_blocking=True)
            ev_in[b].record(cs_in)
            stream.wait_event(ev_in[b])
            if k >= 2:
                stream.wait_event(ev_out[b])
            wr()
            dc()
            ev_done[b].record(stream)
            cs_out.wait_event(ev_done[b])
            with torch.cuda.stream(cs_out):
                h_out.copy_(o, non_blocking=True)
            ev_out[b].record(cs_out)
        for b in range(min(2, e2e_steps)):
            stream.wait_event(ev_out[b])
        f1.record(stream)
        barrier()
        e2e_ms = max_over_ranks(f0.elapsed_time(f1))
    assert pa.pa_get_device_error(reset=True, stream=stream) == 0

    ms_per_step = ms_total / args.steps
    value_gbs = aggregate_throughput(step_bytes, args.steps, ms_total, world)
    e2e_gbs = aggregate_throughput(step_bytes, e2e_steps, e2e_ms, world)
    peaks = measured_peaks()
    achieved = dec_bytes / (decode_ms * 1e-3) / 1e9
    traffic = _ncu_traffic(args.workload)
    clocks = sampler.summary()

    per_config = None
    if world == 1 and not args.no_per_config:
        del v, ws
        torch.cuda.empty_cache()
        per_config = {}
        for name in PER_CONFIG:
            per_config[name] = measure_config(name, args, dev, stream, peaks)
        for name in PREFILL_CONFIG:
            per_config[name] = measure_prefill(name, args, dev, stream, peaks)

    if rank == 0:
        cpu = cpu_baseline(w, args) if (world == 1 and not args.no_cpu_baseline) else None
        line = {
            "metric": "pa_decode achieved HBM GB/s & % of B200 peak; us/call per config",
            "value": round(value_gbs, 2),
            "unit": "GB/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(ms_per_step, 6),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16" if w.kv_dtype == "bf16" else "bf16 queries, e4m3 KV codes, f16 MMA, fp32 accumulate",
            "data": "synthetic",
            "config": {
                "workload": w.describe(),
                "step": "pa_reshape_and_cache + pa_decode" if w.kv_dtype == "bf16"
                        else "pa_reshape_and_cache_fp8 + pa_decode_fp8",
                "alg_bytes_per_step": step_bytes,
                "decode_alg_bytes": dec_bytes,
                "decode_logical_bytes": decode_bytes(w, unique=False),
                "decode_us_per_call": round(decode_ms * 1e3, 3),
                "decode_us_per_call_host_paced": round(paced_ms * 1e3, 3),
                "decode_us_per_call_graph": None if graph_us is None else round(graph_us, 3),
                "cache_write_us_per_call": round(write_ms * 1e3, 3),
                "decode_gbs": round(achieved, 2),
                "decode_frac_of_measured_hbm": round(achieved / peaks["hbm_gbs"], 4),
                "decode_frac_of_spec_8tbs": round(achieved / 8000.0, 4),
                "step_frac_of_measured_hbm": round(value_gbs / world / peaks["hbm_gbs"], 4),
                "plan": plan.as_dict(),
                "l2": "no flush: each step reads more bytes than the 126 MB L2 holds"
                      if dec_bytes > 2 * 126e6 else
                      "no flush: the step's bytes are within twice the 126 MB L2, so later steps may "
                      "find part of them in L2",
                "parallelism": f"replicas x{world} (independent sequences per GPU, no collective)",
                "per_config": per_config,
            },
            "roofline": {
                "bound": "hbm",
                "achieved": round(achieved, 2),
                "peak": peaks["hbm_gbs"],
                "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4),
                "traffic": traffic,
                "peak_source": peaks["source"],
                "kernel": "pa_decode (its kernels on the launching stream)",
            },
            "e2e": {"value": round(e2e_gbs, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": e2e_steps},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks,
        }
        if cpu is not None:
            line["cpu_baseline"] = cpu
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def decode_launches(plan) -> int:
    """Kernel launches of one pa_decode call with this plan."""
    from paged_kv_cache_399_b200 import pa
    if plan.path == pa.PA_PATH_TCGEN05:
        return 2 + (1 if plan.share_cap > 1 else 0)      # [pre-pass], decode, merge
    if plan.schedule == pa.PA_SCHEDULE_PERSISTENT:
        return 2                                         # pre-pass, decode
    # grid: [sharing pre-pass], decode, [merge of split partials]
    return (1 if plan.share_cap else 0) + 1 + (1 if (plan.num_splits > 1 or plan.share_cap) else 0)


# ------------------------------------------------------------------ CPU oracle legs

def _oracle_step(orc, w, seqs):
    """One oracle step over the sequences `seqs` of w: cache write, then decode."""
    sub_slots = np.concatenate([w.slot_mapping[b * w.q_per_seq:(b + 1) * w.q_per_seq] for b in seqs])
    sub_key = w.key.view(w.num_seqs, w.q_per_seq, w.num_kv_heads, w.head_dim)[seqs].reshape(
        -1, w.num_kv_heads, w.head_dim)
    sub_val = w.value.view(w.num_seqs, w.q_per_seq, w.num_kv_heads, w.head_dim)[seqs].reshape(
        -1, w.num_kv_heads, w.head_dim)
    if w.kv_dtype == "fp8_e4m3":
        kc, vc = orc.reshape_and_cache_fp8(sub_key, sub_val, w.key_cache.numpy(), w.value_cache.numpy(),
                                           sub_slots, w.k_scale, w.v_scale)
        return orc.decode_fp8(w.query[seqs], kc, vc, w.block_tables[seqs], w.context_lens[seqs], w.q_per_seq,
                              w.scale, w.k_scale, w.v_scale, window=w.window)
    kc, vc = orc.reshape_and_cache(sub_key, sub_val, w.key_cache, w.value_cache, sub_slots)
    return orc.decode(w.query[seqs], kc, vc, w.block_tables[seqs], w.context_lens[seqs], w.q_per_seq,
                      w.scale, window=w.window)


def _sample_workload(w, seqs):
    import copy
    s = copy.copy(w)
    s.num_seqs = len(seqs)
    s.context_lens = w.context_lens[seqs]
    s.block_tables = w.block_tables[seqs]
    s.slot_mapping = np.concatenate([w.slot_mapping[b * w.q_per_seq:(b + 1) * w.q_per_seq] for b in seqs])
    return s


def cpu_baseline(w, args, target_s: float = 8.0):
    """The oracle, as it stands, on host cores over a bounded sample of the workload."""
    from oracle import Oracle
    orc = Oracle()
    seqs = list(range(min(w.num_seqs, args.cpu_sample_seqs)))
    sub = _sample_workload(w, seqs)
    sample_bytes = decode_bytes(sub) + cache_write_bytes(sub)
    t0 = time.perf_counter()
    reps = 0
    while True:
        _oracle_step(orc, w, seqs)
        reps += 1
        if time.perf_counter() - t0 >= target_s or reps >= 50:
            break
    dt = (time.perf_counter() - t0) / reps
    return {"value": round(sample_bytes / dt / 1e9, 4), "unit": "GB/s", "cores": orc.threads_used(),
            "kind": "oracle",
            "sample": f"{len(seqs)} of {w.num_seqs} sequences of {w.name} (cache write + decode, fp64), "
                      f"{reps} repetitions, {dt:.3f} s each"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from oracle import Oracle
    from paged_kv_cache_399_b200 import workloads
    w = workloads.make(args.workload, seed=rank_seed(args.workload, 0))
    orc = Oracle()
    seqs = list(range(min(w.num_seqs, args.ref_sample_seqs)))
    sub = _sample_workload(w, seqs)
    sample_bytes = decode_bytes(sub) + cache_write_bytes(sub)
    for _ in range(args.warmup):
        _oracle_step(orc, w, seqs)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _oracle_step(orc, w, seqs)
    dt = time.perf_counter() - t0
    value = sample_bytes * args.steps / dt / 1e9
    sample = f"{len(seqs)} of {w.num_seqs} sequences of {w.name} per step (cache write + decode, fp64)"
    line = {
        "impl": "reference",
        "metric": "pa_decode achieved HBM GB/s & % of B200 peak; us/call per config",
        "value": round(value, 4),
        "unit": "GB/s",
        "n_gpus": int(os.environ.get("WORLD_SIZE", "1")),
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(dt / args.steps * 1e3, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": w.describe(), "step": "oracle cache write + oracle decode"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": orc.threads_used(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_prefill_reference(args):
    """The oracle on the chunked-prefill workload: a bounded sample of each step (the rows of
    a few chunk tokens of every sequence, all heads), reported as TFLOP/s of that sample."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from oracle import Oracle
    from paged_kv_cache_399_b200 import workloads
    w = workloads.PREFILL_WORKLOADS[args.workload](seed=rank_seed(args.workload, 0))
    orc = Oracle()
    chunk = int(w.query_lens[0])
    toks = list(range(0, chunk, max(1, chunk // 8)))
    rows = [(b, i, h) for b in range(w.num_seqs) for i in toks for h in range(w.num_q_heads)]
    q = w.query.view(w.num_seqs, chunk, w.num_q_heads, w.head_dim)

    def step():
        kc, vc = orc.reshape_and_cache(w.key, w.value, w.key_cache, w.value_cache, w.slot_mapping)
        orc.decode_rows(rows, q, kc, vc, w.block_tables, w.context_lens, chunk, w.scale)
    flops = sum(4 * w.head_dim * (int(w.context_lens[b]) - chunk + i + 1) for b, i, _ in rows)
    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    value = flops * args.steps / dt / 1e12
    sample = f"{len(rows)} of {w.num_tokens * w.num_q_heads} query rows of {w.name} per step (fp64)"
    print(json.dumps({
        "impl": "reference", "metric": "pa_prefill achieved TFLOP/s & fraction of the sustained bf16 tensor peak",
        "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": int(os.environ.get("WORLD_SIZE", "1")),
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.describe(), "step": "oracle cache write + oracle rows"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": orc.threads_used(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


# ------------------------------------------------------------------ block copy

L2_BYTES = 126 * 1024 * 1024


def copy_bytes(w) -> int:
    """Algorithmic bytes of one pa_copy_blocks call: each copied block is read once and
    written once, in the key pool and in the value pool."""
    return 2 * 2 * w.block_bytes * w.num_pairs


def run_copy_gpu(args):
    """One step = one pa_copy_blocks call over the workload's pairs (the copies a fork
    needs before the step's cache write)."""
    import torch
    import torch.distributed as dist

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    from paged_kv_cache_399_b200 import build as pa_build
    pa_build.build()
    from paged_kv_cache_399_b200 import pa, workloads

    w = workloads.make_copy(args.workload, seed=rank_seed(args.workload, rank))
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.current_stream(dev)
    kc = w.key_cache.to(dev)
    vc = w.value_cache.to(dev)
    mapping = np.ascontiguousarray(w.mapping)
    nbytes = copy_bytes(w)
    launches = -(-w.num_pairs // 2048)
    # a step that moves less than twice L2 would find its blocks in L2 on the next step:
    # write a buffer larger than L2 between steps, outside the timed events
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev) if nbytes < 2 * L2_BYTES else None

    def barrier():
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    def max_over_ranks(x: float) -> float:
        return reduce_over_ranks(x, "max", dist if world > 1 else None, dev)

    def step():
        pa.pa_copy_blocks(kc, vc, mapping, stream=stream)

    for _ in range(args.warmup):
        step()
    barrier()
    sampler = ClockSampler(local_rank)
    with sampler:
        barrier()
        if flush is None:
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(args.steps):
                step()
            e1.record(stream)
            barrier()
            ms_total = e0.elapsed_time(e1)
        else:
            pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                     for _ in range(args.steps)]
            for a, b in pairs:
                flush.zero_()
                a.record(stream)
                step()
                b.record(stream)
            barrier()
            ms_total = sum(a.elapsed_time(b) for a, b in pairs)
        ms_total = max_over_ranks(ms_total)
        # end to end through the C ABI: the host mapping enters with the launches (its
        # checks and marshalling inside the timed region); the copies stay in the pools
        e2e_steps = max(1, args.steps // 4)
        barrier()
        f0 = torch.cuda.Event(enable_timing=True)
        f1 = torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(e2e_steps):
            step()
        f1.record(stream)
        barrier()
        e2e_ms = max_over_ranks(f0.elapsed_time(f1))
    clocks = sampler.summary()
    ms_per_step = ms_total / args.steps
    value_gbs = aggregate_throughput(nbytes, args.steps, ms_total, world)
    e2e_gbs = aggregate_throughput(nbytes, e2e_steps, e2e_ms, world)
    peaks = measured_peaks()
    # bytes of one launch over one launch's time (the launches of a step split the pairs
    # evenly, so this is the step's bytes over the step's time)
    achieved = nbytes / (ms_per_step * 1e-3) / 1e9
    traffic = None
    rec = NCU_COPY_TRAFFIC.get(args.workload)
    if rec and rec.get("source_hash") == source_hash(COPY_SOURCES):
        traffic = rec["bytes_per_launch"]
    if rank == 0:
        cpu = copy_cpu_baseline(w, args) if (world == 1 and not args.no_cpu_baseline) else None
        line = {
            "metric": "pa_copy_blocks GB/s (bytes read + written per copy-on-write step)",
            "value": round(value_gbs, 2),
            "unit": "GB/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(ms_per_step, 6),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16 bits (u16 copy)",
            "data": "synthetic",
            "config": {
                "workload": w.describe(),
                "step": "pa_copy_blocks",
                "alg_bytes_per_step": nbytes,
                "launches_per_step": launches,
                "us_per_call": round(ms_per_step * 1e3, 3),
                "l2": "flushed between steps (a 252 MB write outside the timed events)" if flush is not None
                      else "no flush: each step moves more bytes than twice the 126 MB L2",
                "parallelism": f"replicas x{world} (independent pools per GPU, no collective)",
            },
            "roofline": {
                "bound": "hbm",
                "achieved": round(achieved, 2),
                "peak": peaks["hbm_gbs"],
                "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4),
                "traffic": traffic,
                "peak_source": peaks["source"],
                "kernel": "copy_blocks_kernel (the measured peak is itself a copy: read + write bytes)",
            },
            "e2e": {"value": round(e2e_gbs, 2), "unit": "GB/s",
                    "h2d_bytes_per_step": int(mapping.nbytes), "d2h_bytes_per_step": 0,
                    "steps": e2e_steps,
                    "note": "the mapping is a host array carried by the launches; the result stays in the "
                            "device pools, where the next decode reads it"},
            "gpu_launches": launches * args.steps,
            "clocks": clocks,
        }
        if cpu is not None:
            line["cpu_baseline"] = cpu
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def _oracle_copy_arrays(w, pairs):
    from oracle import _u16
    kc = _u16(w.key_cache).copy()
    vc = _u16(w.value_cache).copy()
    m = np.ascontiguousarray(w.mapping[:pairs])
    return kc, vc, m


def _time_oracle_copy(orc, kc, vc, m, block_elems, min_s, max_reps=1000, fixed_reps=None):
    reps = 0
    t0 = time.perf_counter()
    while True:
        st = orc.lib.oracle_copy_blocks(kc.ctypes.data, vc.ctypes.data, kc.shape[0], block_elems,
                                        m.ctypes.data, m.shape[0])
        assert st == 0
        reps += 1
        if fixed_reps is not None:
            if reps >= fixed_reps:
                break
        elif time.perf_counter() - t0 >= min_s or reps >= max_reps:
            break
    return (time.perf_counter() - t0) / reps, reps


def copy_cpu_baseline(w, args, target_s: float = 8.0):
    """The oracle's copy, as it stands, on one host core over a bounded sample of pairs."""
    from oracle import Oracle
    orc = Oracle()
    pairs = min(w.num_pairs, 1024)
    kc, vc, m = _oracle_copy_arrays(w, pairs)
    block_elems = int(np.prod(kc.shape[1:]))
    dt, reps = _time_oracle_copy(orc, kc, vc, m, block_elems, target_s)
    sample_bytes = 2 * 2 * w.block_bytes * pairs
    return {"value": round(sample_bytes / dt / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"{pairs} of {w.num_pairs} pairs of {w.name} (element-wise copy), {reps} repetitions, "
                      f"{dt * 1e3:.2f} ms each"}


def run_copy_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from oracle import Oracle
    from paged_kv_cache_399_b200 import workloads
    w = workloads.make_copy(args.workload, seed=rank_seed(args.workload, 0))
    orc = Oracle()
    pairs = min(w.num_pairs, 256)
    kc, vc, m = _oracle_copy_arrays(w, pairs)
    block_elems = int(np.prod(kc.shape[1:]))
    _time_oracle_copy(orc, kc, vc, m, block_elems, 0.0, fixed_reps=args.warmup)
    dt, _ = _time_oracle_copy(orc, kc, vc, m, block_elems, 0.0, fixed_reps=args.steps)
    sample_bytes = 2 * 2 * w.block_bytes * pairs
    value = sample_bytes / dt / 1e9
    sample = f"{pairs} of {w.num_pairs} pairs of {w.name} per step (element-wise copy)"
    print(json.dumps({
        "impl": "reference",
        "metric": "pa_copy_blocks GB/s (bytes read + written per copy-on-write step)",
        "value": round(value, 4), "unit": "GB/s",
        "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "u16", "data": "synthetic",
        "config": {"workload": w.describe(), "step": "oracle block copy"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    choices=["tiny", "llama8b", "llama70b_long", "prefix_sharing", "spec_verify",
                             "sliding_window", "llama8b_fp8", "chunked_prefill", "cow_fork", "cow_bulk"],
                    help="decode workloads time cache write + decode; cow_fork / cow_bulk time the "
                         "copy-on-write block copy")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--schedule", choices=["auto", "grid", "persistent"], default="auto")
    ap.add_argument("--path", choices=["auto", "single", "tile", "tcgen05"], default="auto")
    ap.add_argument("--split-blocks", type=int, default=0, help="grid schedule split length (0 = heuristic)")
    ap.add_argument("--no-share-prefix", action="store_true",
                    help="do not ask pa_decode to read shared prefix blocks once per group")
    ap.add_argument("--no-per-config", action="store_true",
                    help="time only the chosen workload (the default also times every decode config)")
    ap.add_argument("--config-calls", type=int, default=200,
                    help="pa_decode calls timed per config in config.per_config")
    ap.add_argument("--cpu-sample-seqs", type=int, default=16)
    ap.add_argument("--ref-sample-seqs", type=int, default=4)
    ap.add_argument("--context-parallel", action="store_true",
                    help="split one decode of the workload over the job's GPUs by table ranges "
                         "(pa_decode_partial + all-gather + pa_merge_partials; strong scaling)")
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)  # at least 3 untimed warm-up steps
    copy = args.workload in ("cow_fork", "cow_bulk")
    prefill = args.workload in PREFILL_CONFIG
    if args.impl == "reference":
        (run_copy_reference if copy else run_prefill_reference if prefill else run_reference)(args)
    elif args.context_parallel:
        run_context_parallel_gpu(args)
    else:
        (run_copy_gpu if copy else run_prefill_gpu if prefill else run_gpu)(args)
    return 0


if __name__ == "__main__":
    sys.exit(main())
