"""Benchmark: emulated DCP MLA decode steps on B200, one JSON line on rank 0.

A step is the whole hot path for one batch: the N shard partial-attention
calls (``mla_decode_partial``, each a partial kernel plus its split combine)
and the LSE merge (``dcp_merge``).  The default workload is the
agentic-trace-shaped batch (64 requests, 64 heads, fp8 rows, lengths
lognormal with median 67,000 clipped to [4,096, 200,000], N = 8 shards): the
configuration the metric "KV-read GB/s and % of HBM peak at >= 64K context"
is quoted on.  ``value`` is KV bytes read per step / device time per step,
with the cache resident in HBM; the agentic cache (3.9 GB) is far larger than
L2, so no flush is needed between steps.  Workloads that read less than 4x
the L2 per step (``--workload tiny|dense|sparse``) are timed step by step
after a 256 MB write that evicts L2.  The same run adds secondary
measurements: every request at exactly 64K tokens, multi-query decode over
the same cache, and the cache write of one new token per request.

``--impl reference`` times the fp64 CPU oracle instead (bounded samples of
the same workload on the host cores), for the driver's reference arm.
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

METRIC = "MLA decode KV-read GB/s and % of HBM peak; decode steps/s at 64K context"
UNIT = "GB/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="agentic",
                    choices=["agentic", "dense", "million", "sparse", "tiny"])
    ap.add_argument("--kernel", default="auto", choices=["auto", "simt", "tc"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the secondary at-64K measurement")
    ap.add_argument("--shard-streams", type=int, default=None,
                    help="CUDA streams the N shard launches are spread over "
                         "(default N; 1 = serial)")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch (smaller cases for profiling)")
    return ap.parse_args()


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def max_over_ranks(values):
    """Element-wise max of a list of floats over all ranks (identity without a
    process group).  Every rank must call it, in the same order."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return list(values)
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor(list(values), dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def kv_bytes(prob) -> int:
    """KV bytes one step must read: every cached (or, sparse, every selected) row once."""
    from long_context_decode_mla_b200.workload import ROW_BYTES
    rb = ROW_BYTES[prob.kv_dtype]
    if prob.sparse_idx is None:
        return int(prob.seq_lens.long().sum()) * rb
    idx = prob.sparse_idx.long().cpu()
    lens = prob.seq_lens.long().cpu()[:, None]
    return int(((idx >= 0) & (idx < lens)).sum()) * rb


def shard_kv_bytes(prob, s) -> int:
    from long_context_decode_mla_b200.workload import ROW_BYTES
    rb = ROW_BYTES[prob.kv_dtype]
    N = prob.num_shards
    lens = prob.seq_lens.long().cpu()
    if prob.sparse_idx is None:
        n = ((lens - s - 1).clamp(min=-1) // N + 1).clamp(min=0)
        return int(n.sum()) * rb
    idx = prob.sparse_idx.long().cpu()
    ok = (idx >= 0) & (idx < lens[:, None]) & (idx % N == s)
    return int(ok.sum()) * rb


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# the translation unit of the partial kernel (whose DRAM traffic
# profiles/traffic.json records) and the headers it includes; other files are
# compiled separately and cannot change that kernel
PARTIAL_KERNEL_SOURCES = ("common.cuh", "kernels.h", "partial_tc.cu", "tc_ptx.cuh")


def _code_only(text: str) -> str:
    """C/C++ source without comments and with whitespace collapsed, so that
    edits to comments do not count as kernel changes."""
    import re
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_source_hash(read=None) -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "long_context_decode_mla_b200", "csrc")
    for name in PARTIAL_KERNEL_SOURCES:
        if read is None:
            with open(os.path.join(csrc, name), encoding="utf-8") as f:
                text = f.read()
        else:
            text = read(name)
        h.update(name.encode() + _code_only(text).encode())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str, kernel: str):
    """DRAM traffic per launch from a committed ncu summary, if it is current."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(f"{workload}/{kernel}")
    if not e or e.get("source_hash") != kernel_source_hash():
        return None
    return e.get("bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled in the background."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index, self.samples, self.proc = index, [], None
        self.t_on = self.t_off = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        threading.Thread(target=self._read, daemon=True).start()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), line.strip()))

    def mark(self, on: bool):
        if on:
            self.t_on = time.time()
        else:
            self.t_off = time.time()

    def stop(self):
        if self.proc:
            time.sleep(0.12)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = [s for t, s in self.samples if self.t_on and self.t_off and
                self.t_on <= t <= self.t_off + 0.06]
        window = "timed region"
        if not rows:
            rows = [s for _, s in self.samples]
            window = "whole run (timed region shorter than the sampling interval)"
        mhz, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            f = [x.strip() for x in r.split(",")]
            try:
                mhz.append(float(f[0]))
                mx = float(f[1])
            except (ValueError, IndexError):
                continue
            for name, v in zip(names, f[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(mhz), "window": window}


# ------------------------------------------------------------------ ours ----

def run_ours(args, rank, world, local):
    import torch
    import torch.distributed as dist

    from long_context_decode_mla_b200 import dcpmla, workload

    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", device_id=torch.device("cuda", local),
                                timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", local)
    # weak scaling: every rank decodes its own batch (distinct seed), no collectives
    cfg = dict(workload.CONFIGS[args.workload])
    over = {} if args.batch is None else {"batch": args.batch}
    prob = workload.make_problem(args.workload, device=dev, kv_device=dev,
                                 seed=cfg["seed"] + 1000 * rank, **over)
    N, B, H = prob.num_shards, prob.batch, prob.heads
    topk = 0 if prob.sparse_idx is None else prob.sparse_idx.shape[1]
    long_single = args.workload == "million"
    # the N shards are independent: each gets its own stream (a real DCP group
    # runs them on N GPUs), so one shard's ramp-up overlaps another's tail
    n_streams = N if args.shard_streams is None else max(1, min(N, args.shard_streams))
    streams = [torch.cuda.Stream(device=dev) for _ in range(n_streams)] if n_streams > 1 else None
    splits = max(1, dcpmla.device_sm_count() // N) if long_single else 0
    dec = dcpmla.DcpDecoder(B, H, N, topk=topk, num_splits=splits, device=dev,
                            impl=args.kernel, streams=streams)
    stream = torch.cuda.current_stream(dev)
    kvb = kv_bytes(prob)
    per_shard_kv = [shard_kv_bytes(prob, s) for s in range(N)]
    other_per_launch = B * H * 576 * 2 + B * H * 513 * 4

    # The whole step (and, for the roofline, the shard partials alone) is
    # captured once into a CUDA graph and replayed: the timed region then
    # measures the GPU, not Python launch overhead.
    step_graph = dec.capture(prob)
    partial_graph = dec.capture(prob, merge=False)

    # a step that reads less than 4x the L2 would partly hit in L2 on the next
    # step: flush it (write 256 MB) before every timed step, outside the events
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if kvb < 4 * L2_BYTES else None

    sampler = ClockSampler(local)
    sampler.start()
    for _ in range(max(3, args.warmup)):
        step_graph.replay()
    torch.cuda.synchronize(dev)
    assert dec.flags() == 0, "device flags set during warm-up"

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.mark(True)
    ms_step = timed_replays(step_graph, args.steps, stream, flush)
    sampler.mark(False)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    # the partial kernels alone (N shard launches + their split combines)
    ms_partials = timed_replays(partial_graph, args.steps, stream, flush)

    # end to end through the public API, host buffers in pinned memory
    h_q = prob.q.cpu().pin_memory()
    h_lens = prob.seq_lens.cpu().pin_memory()
    h_tables = prob.block_tables.cpu().pin_memory()
    h_idx = None if prob.sparse_idx is None else prob.sparse_idx.cpu().pin_memory()
    h_out = torch.empty_like(dec.out, device="cpu").pin_memory()
    h_lse = torch.empty_like(dec.out_lse, device="cpu").pin_memory()
    e_steps = max(3, args.steps // 4)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def e2e_step():
        prob.q.copy_(h_q, non_blocking=True)
        prob.seq_lens.copy_(h_lens, non_blocking=True)
        prob.block_tables.copy_(h_tables, non_blocking=True)
        if h_idx is not None:
            prob.sparse_idx.copy_(h_idx, non_blocking=True)
        step_graph.replay()
        h_out.copy_(dec.out, non_blocking=True)
        h_lse.copy_(dec.out_lse, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(e_steps):
        e2e_step()
    e1.record(stream)
    e1.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e_steps
    h2d = h_q.numel() * 2 + h_lens.numel() * 4 + h_tables.numel() * 4 + \
        (0 if h_idx is None else h_idx.numel() * 4)
    d2h = h_out.numel() * 4 + h_lse.numel() * 4
    assert dec.flags() == 0, "device flags set"
    sampler.stop()

    ms_step, e2e_ms, ms_partials = max_over_ranks([ms_step, e2e_ms, ms_partials])
    gpu_launches = args.steps * (N * (1 if (prob.sparse_idx is not None) else 2) + 1)
    peak, peak_kind = measured_peaks()
    result = None
    if rank == 0:
        value = world * kvb / (ms_step * 1e-3) / 1e9
        # algorithmic bytes of the N shard launches / their device time
        achieved = (kvb + N * other_per_launch) / (ms_partials * 1e-3) / 1e9
        traffic = recorded_traffic(args.workload, args.kernel)
        clocks = sampler.summary()
        result = {
            "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": round(ms_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if args.kernel != "simt" else "f32",
            "data": "synthetic (seeded; no public trace or checkpoint available)",
            "config": {
                "workload": describe(args.workload, prob), "global_batch": B * world,
                "heads": H, "shards": N, "kv_dtype": prob.kv_dtype,
                "seq_len_median": int(prob.seq_lens.float().median()),
                "kv_bytes_per_step_per_gpu": kvb, "kernel": args.kernel,
                "parallelism": f"{world} independent replicas, {N} DCP shards emulated per GPU "
                               f"on {n_streams} CUDA stream(s)",
                "l2": ("no flush: the KV read per step is larger than 4x the 126 MB L2"
                       if flush is None else
                       "256 MB written before every timed step (outside the timed events)"),
            },
            "steps_per_s": round(1e3 / ms_step, 2),
            "pct_hbm_peak_kv": round(100 * value / world / peak, 1),
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                         "unit": "GB/s", "frac": round(achieved / peak, 4),
                         "traffic": traffic, "peak_source": peak_kind,
                         "kernel": "mla_decode_partial (partial + split combine): the N shard "
                                   "launches of a step (one stream each, overlapping), algorithmic "
                                   "bytes / device time of that phase, CUDA-graph replay"},
            "ms_partials_per_step": round(ms_partials, 4),
            "e2e": {"value": round(world * kvb / (e2e_ms * 1e-3) / 1e9, 1), "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": round(e2e_ms, 4),
                    "note": "per step: q, lengths, block tables (and indices) host->device; "
                            "merged O and LSE device->host; the KV cache is resident state"},
            "gpu_launches": gpu_launches,
            "clocks": clocks,
        }
    # secondary measurements (same rank layout; every rank runs them, rank 0 reports)
    extras = {}
    if args.workload == "agentic" and not args.no_extras:
        extras["at_64k"] = time_other_workload("agentic64k", dev, rank, world, args, streams_for=N)
    if prob.sparse_idx is None and prob.heads % 4 == 0:
        extras["multi_query"] = time_multi_query(prob, dev, args, q_len=4)
    extras["kv_append"] = time_append(prob, dev, max(20, args.steps // 4))
    if H % N == 0:
        extras["merge_heads"] = time_merge_heads(dec, dev, max(20, args.steps // 4))
    if result is not None:
        result.update(extras)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return result, prob


L2_BYTES = 126 << 20


def timed_replays(graph, steps, stream, flush=None):
    """Mean device time (ms) of `steps` graph replays on `stream`.  With a
    flush buffer, each replay is timed alone after overwriting the buffer."""
    import torch
    if flush is None:
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(steps):
            graph.replay()
        t1.record(stream)
        t1.synchronize()
        return t0.elapsed_time(t1) / steps
    pairs = []
    for i in range(steps):
        flush.fill_(i & 0xFF)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        graph.replay()
        b.record(stream)
        pairs.append((a, b))
    pairs[-1][1].synchronize()
    return sum(a.elapsed_time(b) for a, b in pairs) / steps


def time_other_workload(name, dev, rank, world, args, streams_for):
    """Graph-replayed steps of another workload (for "steps/s at 64K context")."""
    import torch
    from long_context_decode_mla_b200 import dcpmla, workload
    cfg = dict(workload.CONFIGS[name])
    prob = workload.make_problem(name, device=dev, kv_device=dev, seed=cfg["seed"] + 1000 * rank)
    N = prob.num_shards
    streams = [torch.cuda.Stream(device=dev) for _ in range(N)]
    dec = dcpmla.DcpDecoder(prob.batch, prob.heads, N, device=dev, impl=args.kernel,
                            streams=streams)
    graph = dec.capture(prob)
    for _ in range(max(3, args.warmup)):
        graph.replay()
    torch.cuda.synchronize(dev)
    steps = max(20, args.steps // 4)
    stream = torch.cuda.current_stream(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        graph.replay()
    t1.record(stream)
    t1.synchronize()
    assert dec.flags() == 0, "device flags set"
    ms = max_over_ranks([t0.elapsed_time(t1) / steps])[0]
    kvb = kv_bytes(prob)
    desc = describe(name, prob)
    del graph, dec, prob
    torch.cuda.empty_cache()
    return {"workload": desc, "steps_per_s": round(world * 1e3 / ms, 2),
            "ms_per_step": round(ms, 4), "value": round(world * kvb / (ms * 1e-3) / 1e9, 1),
            "unit": UNIT, "steps": steps}


def time_multi_query(prob, dev, args, q_len):
    """The same cache and rows as the headline step, read as heads / q_len
    heads x q_len query tokens with causal limits (speculative verification):
    KV bytes per step are unchanged, query tokens per step are q_len x."""
    import torch
    from long_context_decode_mla_b200 import dcpmla
    B, N, H = prob.batch, prob.num_shards, prob.heads // q_len
    streams = [torch.cuda.Stream(device=dev) for _ in range(N)]
    dec = dcpmla.DcpDecoder(B, H, N, device=dev, impl=args.kernel, streams=streams, q_len=q_len)
    graph = dec.capture(prob)
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize(dev)
    steps = max(20, args.steps // 4)
    stream = torch.cuda.current_stream(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        graph.replay()
    t1.record(stream)
    t1.synchronize()
    assert dec.flags() == 0, "device flags set"
    ms = t0.elapsed_time(t1) / steps
    kvb = kv_bytes(prob)
    del graph, dec
    return {"heads": H, "q_len": q_len, "ms_per_step": round(ms, 4),
            "value": round(kvb / (ms * 1e-3) / 1e9, 1), "unit": UNIT,
            "query_tokens_per_s": round(B * q_len * 1e3 / ms, 1)}


def time_merge_heads(dec, dev, steps):
    """The cross-rank exchange of real multi-GPU DCP, emulated on one GPU: the
    step's N shard partials sit in N exchange buffers (one per rank), and each
    of the N ranks' dcp_merge_heads launches merges its H/N heads from all N
    buffers (graph-replayed, back to back on one stream).  On N GPUs each
    launch reads (N - 1) / N of its bytes over NVLink; here all are local."""
    import torch
    from long_context_decode_mla_b200 import dcp_group, dcpmla
    N, B, H = dec.partials.shape[0], dec.partials.shape[1], dec.partials.shape[2]
    lse_off, slot = dcp_group.slot_layout(B, H)
    bufs = [dcpmla.dcp_exchange_alloc(slot)[0] for _ in range(N)]
    try:
        for s, a in enumerate(bufs):
            dcp_group.device_view(a, (B, H, 512)).copy_(dec.partials[s])
            dcp_group.device_view(a + lse_off, (B, H)).copy_(dec.lses[s])
        lse_ptrs = [a + lse_off for a in bufs]
        slices = [dcp_group.head_slice(r, N, H) for r in range(N)]
        outs = [(torch.empty(B, hn, 512, device=dev), torch.empty(B, hn, device=dev))
                for _, hn in slices]

        def step(stream):
            for (h0, hn), (o, l) in zip(slices, outs):
                dcpmla.dcp_merge_heads(bufs, lse_ptrs, B, H, h0, hn, o, l, stream)

        side = torch.cuda.Stream(device=dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            step(side)
        torch.cuda.current_stream(dev).wait_stream(side)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            step(side)
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize(dev)
        merged = torch.cat([o for o, _ in outs], dim=1)
        assert torch.equal(merged, dec.out), "head-sliced merge differs from dcp_merge"
        stream = torch.cuda.current_stream(dev)
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(steps):
            graph.replay()
        t1.record(stream)
        t1.synchronize()
        us = t0.elapsed_time(t1) * 1e3 / steps / N
        del graph
    finally:
        torch.cuda.synchronize(dev)
        for a in bufs:
            dcpmla.dcp_exchange_free(a)
    per_rank = B * H * 513 * 4                  # its H/N heads from all N shards
    nvlink_gbs = 770.0                          # measured peer copy, GB/s per direction
    return {"ranks": N, "us_per_rank": round(us, 2), "bytes_per_rank": per_rank,
            "GBps_local": round(per_rank / (us * 1e-6) / 1e9, 1),
            "nvlink_bound_us_per_rank": round((N - 1) / N * per_rank / (nvlink_gbs * 1e9) * 1e6,
                                              2)}


def time_append(prob, dev, steps):
    """The DCP cache write of one new token per request on every shard
    (mla_kv_append x N, graph-replayed).  It rewrites each request's last
    existing token, so every write lands inside the block tables."""
    import torch
    from long_context_decode_mla_b200 import dcpmla
    B, N = prob.batch, prob.num_shards
    g = torch.Generator(device=dev).manual_seed(5)
    lat = torch.randn(B, 512, generator=g, device=dev).to(torch.bfloat16)
    rope = torch.randn(B, 64, generator=g, device=dev).to(torch.bfloat16)
    pos = (prob.seq_lens - 1).to(torch.int32).contiguous()
    req = torch.arange(B, dtype=torch.int32, device=dev)
    flags = torch.zeros(1, dtype=torch.int32, device=dev)

    def step(stream):
        for s in range(N):
            dcpmla.mla_kv_append(lat, rope, pos, req, prob.block_tables[s], s, N, prob.kv_cache,
                                 prob.kv_dtype, flags, stream)

    side = torch.cuda.Stream(device=dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        step(side)
    torch.cuda.current_stream(dev).wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        step(side)
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize(dev)
    stream = torch.cuda.current_stream(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        graph.replay()
    t1.record(stream)
    t1.synchronize()
    assert int(flags.item()) == 0, "append flags set"
    us = t0.elapsed_time(t1) / steps * 1e3
    from long_context_decode_mla_b200.workload import ROW_BYTES
    written = B * ROW_BYTES[prob.kv_dtype]
    return {"us_per_step": round(us, 2), "tokens_per_s": round(B / (us * 1e-6), 1),
            "launches_per_step": N, "bytes_written_per_step": written,
            "note": "one new token per request, written on its owner shard (N shard calls)"}


def describe(name, prob):
    lens = prob.seq_lens
    return (f"{name}: batch {prob.batch}, {prob.heads} heads, {prob.kv_dtype} rows, "
            f"lengths {int(lens.min())}..{int(lens.max())} (median {int(lens.float().median())}), "
            f"{prob.num_shards} round-robin shards + LSE merge")


# ------------------------------------------------------------------ oracle --

def oracle_sample_step(prob_np, b):
    import oracle
    return oracle.dcp_decode(prob_np["q"], prob_np["kv_cache"], prob_np["kv_dtype"],
                             prob_np["block_tables"], prob_np["seq_lens"],
                             prob_np["num_shards"], prob_np["softmax_scale"],
                             prob_np["sparse_idx"], prob_np["block_size"], [b])


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max((i.get("num_threads", 1) for i in info), default=1)
    except Exception:
        return 1


def cpu_sample_problem(workload_name, target_len):
    """One request of the workload's shape (same heads, row format, shards) on the CPU."""
    from long_context_decode_mla_b200 import workload
    cfg = workload.CONFIGS[workload_name]
    over = dict(batch=1, seq_len=[target_len])
    if cfg.get("topk"):
        over["topk"] = cfg["topk"]
    return workload.make_problem(workload_name, **over)


def time_oracle(workload_name, seconds_budget, sample_len=None):
    """Time the oracle on single-request samples until the budget is spent."""
    from long_context_decode_mla_b200 import workload
    cfg = workload.CONFIGS[workload_name]
    if sample_len is None:
        sample_len = 16384 if cfg["seq_len"] == "lognormal" else min(int(cfg["seq_len"]), 16384)
    prob = cpu_sample_problem(workload_name, sample_len)
    ni = prob.numpy_inputs()
    kvb = kv_bytes(prob)
    n, t0 = 0, time.perf_counter()
    while True:
        oracle_sample_step(ni, 0)
        n += 1
        el = time.perf_counter() - t0
        if el >= seconds_budget:
            break
    return {"value": round(n * kvb / el / 1e9, 4), "unit": UNIT, "cores": blas_threads(),
            "kind": "oracle",
            "sample": (f"{n} x one request of the {workload_name} workload "
                       f"(L={sample_len}, {prob.heads} heads, {prob.kv_dtype}, "
                       f"{prob.num_shards} shards + merge), {el:.1f} s of fp64 numpy")}, el / n


def run_reference(args, rank, world):
    if rank != 0:
        return None
    from long_context_decode_mla_b200 import workload
    cfg = workload.CONFIGS[args.workload]
    sample_len = 16384 if cfg["seq_len"] == "lognormal" else min(int(cfg["seq_len"]), 16384)
    prob = cpu_sample_problem(args.workload, sample_len)
    ni = prob.numpy_inputs()
    kvb = kv_bytes(prob)
    for _ in range(max(3, args.warmup)):
        oracle_sample_step(ni, 0)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_sample_step(ni, 0)
    el = time.perf_counter() - t0
    value = kvb * args.steps / el / 1e9
    cpu = {"value": round(value, 4), "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
           "sample": (f"each step: one request of the {args.workload} workload (L={sample_len}, "
                      f"{prob.heads} heads, {prob.kv_dtype}, {prob.num_shards} shards + merge)")}
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": max(3, args.warmup),
        "ms_per_step": round(1e3 * el / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": describe(args.workload, prob) + " (one-request CPU sample)"},
        "cpu_baseline": cpu,
        "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    rank, world, local = dist_env()
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    res, prob = run_ours(args, rank, world, local)
    if rank == 0:
        if not args.no_cpu_baseline:
            res["cpu_baseline"], _ = time_oracle(args.workload, args.cpu_seconds)
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
