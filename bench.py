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
    ap.add_argument("--kernel", default="auto", choices=["auto", "simt", "tc", "tc16"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the secondary at-64K measurement")
    ap.add_argument("--shard-streams", type=int, default=None,
                    help="CUDA streams the N shard launches are spread over "
                         "(default N; 1 = serial)")
    ap.add_argument("--splits", type=int, default=None,
                    help="CTAs each shard launch may use (0: all SMs; default: the "
                         "workload's own choice)")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch (smaller cases for profiling)")
    ap.add_argument("--million-layers", type=int, default=83,
                    help="resident layer caches of the million-token leg (83: the model)")
    ap.add_argument("--replicas", action="store_true",
                    help="with several GPUs: independent replicas of the emulated step "
                         "instead of the real DCP step across the GPUs")
    ap.add_argument("--dcp", action="store_true",
                    help="run the real DCP step (one shard per GPU, NCCL) even on one GPU")
    return ap.parse_args()


def shard_splits(name, N, args):
    """CTAs a shard launch may use.  The emulated step runs the N shard
    launches of a DCP group on one GPU at once, so each is sized for its
    share of the SMs (148 // N: one wave of about one CTA per SM for all N
    launches together), as each shard would own a whole GPU in the group.
    The real-DCP mode (one shard per GPU) uses every SM (splits 0)."""
    from long_context_decode_mla_b200 import dcpmla
    if args.splits is not None:
        return args.splits
    return max(1, dcpmla.device_sm_count() // N)


def launches_per_shard(kv_dtype, kernel, sparse, topk, batch, sms):
    """Kernel launches of one mla_decode_partial call.  Dense: the e4m3
    kernel (fp8 rows under the auto and tc choices) is preceded by its Q image
    kernel; the split combine follows.  Sparse on the tensor-core path: a
    pre-kernel localises the lists (and, for fp8 rows, builds the Q images in
    CTAs of its own), then the partial with whole requests per CTA (fp8), or
    the partial and the combine (bf16).  The
    fp16-operand and CUDA-core kernels select sparse rows in-kernel and need
    the combine only when a request's list spans several CTAs (lists longer
    than 2,048, or fewer requests than SMs)."""
    f8 = kv_dtype == "fp8" and kernel in ("auto", "tc")
    if sparse:
        if kernel in ("tc16", "simt"):
            parts = max(-(-topk // 2048), sms // max(1, batch))
            return 2 if parts > 1 else 1
        return 2 if f8 else 3
    return 3 if f8 else 2


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


# the translation unit of the fp8 partial kernel (whose DRAM traffic
# profiles/traffic.json records) and the headers it includes; other files are
# compiled separately and cannot change that kernel
PARTIAL_KERNEL_SOURCES = ("common.cuh", "kernels.h", "partial_f8.cu", "q_image.cuh",
                          "schedule.cuh", "tc_ptx.cuh")


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
                 "--format=csv,noheader,nounits", "-lms", "20"],
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
    # the N shards are independent: each gets its own stream (a real DCP group
    # runs them on N GPUs), so one shard's ramp-up overlaps another's tail
    n_streams = N if args.shard_streams is None else max(1, min(N, args.shard_streams))
    streams = [torch.cuda.Stream(device=dev) for _ in range(n_streams)] if n_streams > 1 else None
    splits = shard_splits(args.workload, N, args)
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
    st_step = replay_stats(step_graph, args.steps, stream, flush)
    sampler.mark(False)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    # the partial kernels alone (N shard launches + their split combines),
    # right after the steps, so that both run at the same clocks (a second of
    # load first would bring the power cap in)
    st_part = replay_stats(partial_graph, args.steps, stream, flush)
    # the same steps for about a second more (untimed), so that the clock
    # record under this load has enough samples even when K steps are short
    load = ClockSampler(local)
    load.samples = sampler.samples
    load.mark(True)
    t_end = time.time() + 1.0
    while time.time() < t_end:
        for _ in range(20):
            step_graph.replay()
        torch.cuda.synchronize(dev)
    load.mark(False)
    torch.cuda.synchronize(dev)
    ms_step, ms_partials = st_step["mean"], st_part["mean"]

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
    e2e_serial_ms = e0.elapsed_time(e1) / e_steps
    h2d = h_q.numel() * 2 + h_lens.numel() * 4 + h_tables.numel() * 4 + \
        (0 if h_idx is None else h_idx.numel() * 4)
    d2h = h_out.numel() * 4 + h_lse.numel() * 4
    assert dec.flags() == 0, "device flags set"

    # The same steps through dcpmla.HostPipeline: every step still copies its
    # inputs in and its results out, but step k + 1's inputs and step k - 1's
    # results cross PCIe while step k computes.  The timed region opens before
    # the first copy-in and closes after the last copy-out.
    pipe = dcpmla.HostPipeline(prob, topk=topk, num_splits=splits, impl=args.kernel,
                               streams=streams, compute_stream=stream)
    h_outs = [h_out, torch.empty_like(h_out).pin_memory()]
    h_lses = [h_lse, torch.empty_like(h_lse).pin_memory()]
    for i in range(2):
        pipe.submit(h_q, h_lens, h_tables, h_idx, h_outs[i % 2], h_lses[i % 2])
    pipe.join()
    torch.cuda.synchronize(dev)
    p_steps = max(3, args.steps)
    e0.record(stream)
    pipe.start_after(e0)
    for i in range(p_steps):
        pipe.submit(h_q, h_lens, h_tables, h_idx, h_outs[i % 2], h_lses[i % 2])
    pipe.join(stream)
    e1.record(stream)
    e1.synchronize()
    e2e_ms = e0.elapsed_time(e1) / p_steps
    assert pipe.flags() == 0, "device flags set"
    del pipe
    sampler.stop()

    ms_step, e2e_ms, ms_partials, e2e_serial_ms = max_over_ranks(
        [ms_step, e2e_ms, ms_partials, e2e_serial_ms])
    st_step = dict(zip(st_step, max_over_ranks(list(st_step.values()))))
    st_part = dict(zip(st_part, max_over_ranks(list(st_part.values()))))
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    per_shard = launches_per_shard(prob.kv_dtype, args.kernel, prob.sparse_idx is not None,
                                   topk, B, sms)
    gpu_launches = args.steps * (N * per_shard + 1)
    peak, peak_kind = measured_peaks()
    result = None
    if rank == 0:
        value = world * kvb / (ms_step * 1e-3) / 1e9
        # algorithmic bytes of the N shard launches / their device time
        achieved = (kvb + N * other_per_launch) / (ms_partials * 1e-3) / 1e9
        traffic = recorded_traffic(args.workload, args.kernel)
        clocks = sampler.summary()
        clocks["under_load_1s"] = load.summary()
        result = {
            "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": round(ms_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": dtype_label(prob.kv_dtype, args.kernel),
            "data": "synthetic (seeded; no public trace or checkpoint available)",
            "config": {
                "workload": describe(args.workload, prob), "global_batch": B * world,
                "heads": H, "shards": N, "kv_dtype": prob.kv_dtype,
                "seq_len_median": int(prob.seq_lens.float().median()),
                "kv_bytes_per_step_per_gpu": kvb, "kernel": args.kernel,
                "parallelism": f"{world} independent replicas, {N} DCP shards emulated per GPU "
                               f"on {n_streams} CUDA stream(s), each shard launch given "
                               f"{splits} CTAs (its share of the SMs)",
                "l2": ("no flush: the KV read per step is larger than 4x the 126 MB L2"
                       if flush is None else
                       "256 MB written before every timed step (outside the timed events)"),
            },
            "steps_per_s": round(1e3 / ms_step, 2),
            "pct_hbm_peak_kv": round(100 * value / world / peak, 1),
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                         "unit": "GB/s", "frac": round(achieved / peak, 4),
                         "traffic": traffic, "peak_source": peak_kind,
                         "kernel": "mla_decode_partial (Q image + partial + split combine): the N shard "
                                   "launches of a step (one stream each, overlapping), algorithmic "
                                   "bytes / device time of that phase, CUDA-graph replay"},
            "ms_partials_per_step": round(ms_partials, 4),
            "ms_step_stats": ms_summary(st_step),
            "ms_partials_stats": ms_summary(st_part),
            "e2e": {"value": round(world * kvb / (e2e_ms * 1e-3) / 1e9, 1), "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": round(e2e_ms, 4),
                    "serial_ms_per_step": round(e2e_serial_ms, 4),
                    "note": "dcpmla.HostPipeline from pinned host buffers: per step q, lengths, "
                            "block tables (and indices) host->device and merged O and LSE "
                            "device->host, overlapped with the neighbouring steps' compute; "
                            "serial_ms_per_step is the same step with copies and compute in "
                            "one stream; the KV cache is resident state"},
            "gpu_launches": gpu_launches,
            "clocks": clocks,
        }
    # secondary measurements (same rank layout; every rank runs them, rank 0 reports)
    extras = {}
    if args.workload == "agentic" and not args.no_extras:
        # every configuration, each timed as its own graph-replayed steps
        extras["at_64k"] = time_other_workload("agentic64k", dev, rank, world, args)
        legs = {"tiny": lambda: time_other_workload("tiny", dev, rank, world, args),
                "dense": lambda: time_other_workload("dense", dev, rank, world, args),
                "sparse": lambda: time_other_workload("sparse", dev, rank, world, args),
                "million": lambda: time_million_layers(dev, rank, world, args,
                                                       layers=args.million_layers)}
        extras["configs"] = {k: f() for k, f in legs.items()}
        extras["pcp_prefill"] = time_pcp_prefill(dev, args)
    if prob.sparse_idx is None and not args.no_extras:
        extras["multi_query"] = time_multi_query(prob, dev, args, q_len=4, world=world)
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


def replay_stats(graph, steps, stream, flush=None):
    """Device times (ms) of `steps` graph replays on `stream`, each between
    its own pair of CUDA events: mean, median, min and max.  Replays run back
    to back; with a flush buffer, each replay follows an overwrite of the
    buffer (outside its events)."""
    import torch
    pairs = []
    for i in range(steps):
        if flush is not None:
            flush.fill_(i & 0xFF)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        graph.replay()
        b.record(stream)
        pairs.append((a, b))
    pairs[-1][1].synchronize()
    t = [a.elapsed_time(b) for a, b in pairs]
    return {"mean": sum(t) / len(t), "median": statistics.median(t), "min": min(t),
            "max": max(t)}


def timed_replays(graph, steps, stream, flush=None):
    """Mean device time (ms) of `steps` graph replays (see replay_stats)."""
    return replay_stats(graph, steps, stream, flush)["mean"]


def ms_summary(st):
    return {k: round(v, 4) for k, v in st.items()}


def step_bytes(prob, kvb=None):
    """Algorithmic bytes of one emulated DCP step: the KV rows read once
    (sparse: the selected rows), and for each of the N shard launches its
    query (bf16), index list (sparse) and partial O + LSE (fp32) written,
    then the merge reading the N partials and writing the result."""
    B, H, N = prob.batch, prob.heads, prob.num_shards
    kvb = kv_bytes(prob) if kvb is None else kvb
    idx = 0 if prob.sparse_idx is None else prob.sparse_idx.numel() * 4
    per_launch = B * H * 576 * 2 + B * H * 513 * 4 + idx
    return kvb + N * per_launch + (N + 1) * B * H * 513 * 4


def leg(name, prob, stats, world, kvb=None, total=None, extra=None):
    """One secondary measurement: device-time statistics of graph-replayed
    steps, KV GB/s and total algorithmic GB/s (both whole job), and the
    fraction of the HBM peak."""
    peak, _ = measured_peaks()
    kvb = kv_bytes(prob) if kvb is None else kvb
    total = step_bytes(prob, kvb) if total is None else total
    ms = stats["mean"]
    d = {"workload": describe(name, prob), "ms_per_step": ms_summary(stats),
         "steps_per_s": round(world * 1e3 / ms, 2),
         "kv_GBps": round(world * kvb / (ms * 1e-3) / 1e9, 1),
         "total_GBps": round(world * total / (ms * 1e-3) / 1e9, 1),
         "frac": round(total / (ms * 1e-3) / 1e9 / peak, 4), "unit": UNIT,
         "kv_bytes_per_step": kvb, "total_bytes_per_step": total}
    if extra:
        d.update(extra)
    return d


def time_other_workload(name, dev, rank, world, args, streams_for=None):
    """Graph-replayed steps of another workload, each step timed alone (L2
    flushed first when the step reads less than 4x the L2)."""
    import torch
    from long_context_decode_mla_b200 import dcpmla, workload
    cfg = dict(workload.CONFIGS[name])
    prob = workload.make_problem(name, device=dev, kv_device=dev, seed=cfg["seed"] + 1000 * rank)
    N = prob.num_shards
    topk = 0 if prob.sparse_idx is None else prob.sparse_idx.shape[1]
    streams = [torch.cuda.Stream(device=dev) for _ in range(N)]
    splits = shard_splits(name, N, args)
    dec = dcpmla.DcpDecoder(prob.batch, prob.heads, N, topk=topk, num_splits=splits, device=dev,
                            impl=args.kernel, streams=streams)
    graph = dec.capture(prob)
    kvb = kv_bytes(prob)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if kvb < 4 * L2_BYTES else None
    for _ in range(max(3, args.warmup)):
        graph.replay()
    torch.cuda.synchronize(dev)
    steps = max(20, args.steps // 4)
    stream = torch.cuda.current_stream(dev)
    st = replay_stats(graph, steps, stream, flush)
    assert dec.flags() == 0, "device flags set"
    st = dict(zip(st, max_over_ranks(list(st.values()))))
    d = leg(name, prob, st, world, kvb,
            extra={"steps": steps, "ctas_per_shard_launch": splits,
                   "l2": "256 MB written before every step" if flush is not None else "no flush"})
    if prob.sparse_idx is not None:
        d["note"] = ("kv_GBps counts the selected rows read (each once); total_GBps adds the "
                     "queries, the index lists (read by every shard), partials and the merge")
    if name == "tiny":
        d["us_per_step"] = round(st["mean"] * 1e3, 2)
        d["note"] = ("1.2 MB per step: a latency figure (launches and one short pipeline), "
                     "not a bandwidth one")
    del graph, dec, prob, flush
    torch.cuda.empty_cache()
    return d


def time_million_layers(dev, rank, world, args, layers=83):
    """The million-token configuration as one model step: `layers` resident
    layer caches of the 1M-token request (about 53 GiB of fp8 rows), each
    layer one emulated DCP step over its own cache, all captured in one CUDA
    graph.  The caches are copies of one seeded layer in distinct memory
    (their contents do not change the work)."""
    import torch
    from long_context_decode_mla_b200 import dcpmla, workload
    cfg = dict(workload.CONFIGS["million"])
    prob = workload.make_problem("million", device=dev, kv_device=dev,
                                 seed=cfg["seed"] + 1000 * rank)
    N = prob.num_shards
    caches = [prob.kv_cache] + [prob.kv_cache.clone() for _ in range(layers - 1)]
    cache_bytes = sum(c.numel() for c in caches)
    streams = [torch.cuda.Stream(device=dev) for _ in range(N)]
    splits = max(1, dcpmla.device_sm_count() // N)
    dec = dcpmla.DcpDecoder(prob.batch, prob.heads, N, num_splits=splits, device=dev,
                            impl=args.kernel, streams=streams)
    views = [workload.DecodeProblem(prob.q, c, prob.kv_dtype, prob.block_tables, prob.seq_lens,
                                    N) for c in caches]
    side = torch.cuda.Stream(device=dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        dec.step(views[0], side)
    torch.cuda.current_stream(dev).wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        for v in views:
            dec.step(v, side)
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize(dev)
    steps = max(5, args.steps // 20)
    st = replay_stats(graph, steps, torch.cuda.current_stream(dev))
    assert dec.flags() == 0, "device flags set"
    st = dict(zip(st, max_over_ranks(list(st.values()))))
    kvb = layers * kv_bytes(prob)
    total = layers * step_bytes(prob)
    d = leg("million", prob, st, world, kvb, total,
            extra={"layers": layers, "resident_cache_GiB": round(cache_bytes / 2**30, 2),
                   "model_steps_per_s": round(world * 1e3 / st["mean"], 2), "steps": steps,
                   "note": f"one model step = {layers} layers x (N shard partials + merge) in one "
                           "CUDA graph; caches far larger than L2, no flush"})
    del graph, dec, views, caches, prob
    torch.cuda.empty_cache()
    return d


def time_multi_query(prob, dev, args, q_len, world=1):
    """Multi-query decode (speculative verification) over the headline cache
    at the models' head count: every request carries q_len query tokens of
    all its heads (q_len x 64 rows), causal at the cache end.  Rows beyond one
    64-row tile run as one pass per query over the cache, so each step reads
    the cache about q_len times: kv_GBps counts every pass's rows,
    cache_GBps the distinct cache once."""
    import torch
    from long_context_decode_mla_b200 import dcpmla, workload
    B, N, H = prob.batch, prob.num_shards, prob.heads
    q = workload.random_q(B, q_len * H, 9001).to(dev)
    mq = workload.DecodeProblem(q, prob.kv_cache, prob.kv_dtype, prob.block_tables,
                                prob.seq_lens, N)
    streams = [torch.cuda.Stream(device=dev) for _ in range(N)]
    dec = dcpmla.DcpDecoder(B, H, N, device=dev, impl=args.kernel, streams=streams, q_len=q_len)
    graph = dec.capture(mq)
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize(dev)
    steps = max(10, args.steps // 8)
    st = replay_stats(graph, steps, torch.cuda.current_stream(dev))
    assert dec.flags() == 0, "device flags set"
    st = dict(zip(st, max_over_ranks(list(st.values()))))
    from long_context_decode_mla_b200.workload import ROW_BYTES
    lens = prob.seq_lens.long().cpu()
    read = 0
    for k in range(q_len):
        Lk = (lens - (q_len - 1 - k)).clamp(min=0)
        read += int(Lk.sum()) * ROW_BYTES[prob.kv_dtype]
    kvb = kv_bytes(prob)
    total = read + N * (B * q_len * H * (576 * 2 + 513 * 4)) + (N + 1) * B * q_len * H * 513 * 4
    ms = st["mean"]
    d = leg("agentic", prob, st, world, read, total,
            extra={"heads": H, "q_len": q_len, "rows": q_len * H,
                   "cache_GBps": round(world * kvb / (ms * 1e-3) / 1e9, 1),
                   "query_tokens_per_s": round(world * B * q_len * 1e3 / ms, 1),
                   "passes_per_shard": q_len if q_len * H > 64 or prob.kv_dtype == "fp8" else 1,
                   "steps": steps})
    d["workload"] = (f"agentic cache, {H} heads x q_len {q_len} query tokens per request "
                     f"(causal), {N} shards + merge")
    del graph, dec, mq, q
    torch.cuda.empty_cache()
    return d


def time_pcp_prefill(dev, args, num_tokens=16384, pcp_size=8, num_shards=8, heads=64):
    """PCP prefill of one prompt on one GPU: the gather of its rows from the
    DCP-sharded cache and every rank's causal attention (the P ranks in turn;
    on a real PCP group each rank runs its share on its own GPU), graph-
    replayed.  Roofline: tensor.  Flops per prompt = sum over query tokens i
    of (i + 1) rows x heads x (576 + 512) x 2; the peak is fp8 dense taken as
    2x the measured bf16 GEMM rate, else 2x the recipe's 1.59 PFLOP/s."""
    import torch
    from long_context_decode_mla_b200 import dcpmla, workload
    prob = workload.make_problem("agentic", num_shards=num_shards, batch=1, heads=heads,
                                 seq_len=[num_tokens], device=dev, kv_device=dev, seed=2024)
    q = workload.random_q(num_tokens, heads, 2025).to(dev)
    pre = dcpmla.PcpPrefill(num_tokens, heads, pcp_size, "fp8", device=dev, impl=args.kernel)
    tables = prob.block_tables[:, 0].contiguous()

    def run(stream):
        pre.gather(prob.kv_cache, tables, stream)
        pre.attend(q, prob.softmax_scale, stream)

    side = torch.cuda.Stream(device=dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        run(side)
    torch.cuda.current_stream(dev).wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        run(side)
    for _ in range(2):
        graph.replay()
    torch.cuda.synchronize(dev)
    steps = max(3, args.steps // 10)
    st = replay_stats(graph, steps, torch.cuda.current_stream(dev))
    assert int(pre.flags.item()) == 0 and all(
        torch.isfinite(x).all() for x in pre.out_lse), "PCP prefill flags or non-finite LSE"
    flops = sum((i + 1) for i in range(num_tokens)) * heads * (576 + 512) * 2
    peak_bf16, kind = measured_tensor_peak()
    peak = 2 * peak_bf16
    ms = st["mean"]
    tflops = flops / (ms * 1e-3) / 1e12
    d = {"workload": f"one {num_tokens}-token prompt, {heads} heads, fp8 rows on {num_shards} "
                     f"DCP shards, PCP over {pcp_size} ranks (16 chunks for 8), gather + causal "
                     "attention of every rank", "ms_per_prompt": ms_summary(st),
         "prefill_tokens_per_s": round(num_tokens * 1e3 / ms, 1),
         "roofline": {"bound": "tensor", "achieved": round(tflops, 1), "unit": "TFLOP/s",
                      "peak": round(peak, 1), "frac": round(tflops / peak, 4),
                      "peak_source": f"fp8 = 2 x bf16 ({kind})"},
         "gathered_bytes": num_tokens * 656, "steps": steps}
    del graph, pre, prob, q
    torch.cuda.empty_cache()
    return d


def measured_tensor_peak():
    """Dense bf16 tensor peak (TFLOP/s) from MEASURED_PEAKS.json, else the fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        v = d.get("bf16_tflops")
        if v:
            return float(v), "measured"
    return 1590.0, "fallback"


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
    # an assumed link rate, not measured by this program (one GPU here): the
    # per-direction peer-copy figure this B200 pool documents for NVLink 5
    nvlink_gbs = 770.0
    return {"ranks": N, "us_per_rank": round(us, 2), "bytes_per_rank": per_rank,
            "GBps_local": round(per_rank / (us * 1e-6) / 1e9, 1),
            "nvlink_bound_us_per_rank": round((N - 1) / N * per_rank / (nvlink_gbs * 1e9) * 1e6,
                                              2),
            "nvlink_GBps_assumed": nvlink_gbs,
            "nvlink_note": "bound at an assumed 770 GB/s per direction (the pool's documented "
                           "peer copy), not a measurement of this run"}


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


def dtype_label(kv_dtype, kernel):
    """The arithmetic of the timed path, by cache format and kernel."""
    if kernel == "simt":
        return f"{kv_dtype} cache decoded to f32, f32 arithmetic"
    if kv_dtype == "fp8":
        return ("fp8 e4m3 cache codes x e4m3 two-term Q split on the tensor cores (exact "
                "products), fp32 accumulation; per-128 scales in fp32; P as two e4m3 terms")
    return "bf16 cache, fp16 MMA operands, fp32 accumulation"


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


def cpu_info():
    """Host cores this process may run on, the BLAS thread count and the CPU model."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        cores = len(os.sched_getaffinity(0))
    except AttributeError:
        cores = os.cpu_count() or 1
    return cores, blas_threads(), model


def config_slice(workload_name):
    """A declared slice of the workload for the CPU oracle: request 0 of the
    seeded configuration at its own length (same heads, row format, shards;
    for the sparse workload its index-list length), regenerated alone on the
    host."""
    from long_context_decode_mla_b200 import workload
    cfg = workload.CONFIGS[workload_name]
    if cfg["seq_len"] == "lognormal":
        L0 = int(workload.lognormal_lengths(cfg["batch"], cfg["seed"])[0])
    else:
        L0 = int(cfg["seq_len"])
    over = dict(batch=1, seq_len=[L0])
    if cfg.get("topk"):
        over["topk"] = cfg["topk"]
    prob = workload.make_problem(workload_name, **over)
    desc = (f"request 0 of the {workload_name} configuration (L={L0}, {prob.heads} heads, "
            f"{prob.kv_dtype} rows, {prob.num_shards} shards + merge"
            + (f", top-{cfg['topk']}" if cfg.get("topk") else "") + ")")
    return prob, desc


def time_oracle(workload_name, seconds_budget):
    """Time the oracle on the workload's declared slice until the budget is spent."""
    prob, desc = config_slice(workload_name)
    ni = prob.numpy_inputs()
    kvb = kv_bytes(prob)
    n, t0 = 0, time.perf_counter()
    while True:
        oracle_sample_step(ni, 0)
        n += 1
        el = time.perf_counter() - t0
        if el >= seconds_budget:
            break
    cores, threads, model = cpu_info()
    return {"value": round(n * kvb / el / 1e9, 4), "unit": UNIT, "cores": cores,
            "blas_threads": threads, "cpu_model": model, "kind": "oracle",
            "sample": f"{n} x {desc}, {el:.1f} s of fp64 numpy"}, el / n


def run_reference(args, rank, world):
    if rank != 0:
        return None
    prob, desc = config_slice(args.workload)
    ni = prob.numpy_inputs()
    kvb = kv_bytes(prob)
    for _ in range(max(3, args.warmup)):
        oracle_sample_step(ni, 0)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_sample_step(ni, 0)
    el = time.perf_counter() - t0
    value = kvb * args.steps / el / 1e9
    cores, threads, model = cpu_info()
    cpu = {"value": round(value, 4), "unit": UNIT, "cores": cores, "blas_threads": threads,
           "cpu_model": model, "kind": "oracle", "sample": f"each step: {desc}"}
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": max(3, args.warmup),
        "ms_per_step": round(1e3 * el / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": desc + " (CPU oracle)"},
        "cpu_baseline": cpu,
        "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


# ------------------------------------------------------------- real DCP ----

def run_dcp(args, rank, world, local):
    """The real DCP step across the GPUs of the job: one shard per rank
    (tokens t with t mod N == rank, N = the world size), NCCL query
    all-gather, the partial into the rank's exchange slot, a one-integer
    all-reduce, and the head-sliced merge that pulls the peers' partials over
    peer memory (DcpRankDecoder).  The batch is the workload's (the same on
    every rank), so the work per step is fixed as N grows: strong scaling.
    Steps are timed eagerly with CUDA events (NCCL is in the step), max over
    ranks; sampled requests are checked against the oracle at the end."""
    import datetime
    import numpy as np
    import torch
    import torch.distributed as dist

    from long_context_decode_mla_b200 import dcp_group, dcpmla, workload

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    # a one-process run (no launcher): a one-rank group on this host
    for k, v in (("RANK", "0"), ("WORLD_SIZE", "1"), ("MASTER_ADDR", "127.0.0.1"),
                 ("MASTER_PORT", "29511")):
        os.environ.setdefault(k, v)
    dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=120))
    over = {} if args.batch is None else {"batch": args.batch}
    prob = workload.make_problem(args.workload, num_shards=world, device=dev, kv_device=dev,
                                 **over)
    B, H = prob.batch, prob.heads
    if H % world:
        raise SystemExit(f"{H} heads do not split over {world} ranks")
    topk = 0 if prob.sparse_idx is None else prob.sparse_idx.shape[1]
    dec = dcp_group.DcpRankDecoder(B, H, topk=topk, impl=args.kernel)
    h0, hn = dec.head_begin, dec.head_count
    q_local = prob.q[:, h0:h0 + hn].contiguous()
    table = prob.block_tables[rank].contiguous()

    def step():
        return dec.step(q_local, prob.kv_cache, prob.kv_dtype, table, prob.seq_lens,
                        prob.softmax_scale, prob.sparse_idx)

    sampler = ClockSampler(local)
    sampler.start()
    try:
        for _ in range(max(3, args.warmup)):
            step()
        torch.cuda.synchronize(dev)
        dist.barrier()
        stream = torch.cuda.current_stream(dev)
        ev = []
        sampler.mark(True)
        for _ in range(args.steps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            step()
            b.record(stream)
            ev.append((a, b))
        ev[-1][1].synchronize()
        sampler.mark(False)
        t = [a.elapsed_time(b) for a, b in ev]
        st = {"mean": sum(t) / len(t), "median": statistics.median(t), "min": min(t),
              "max": max(t)}
        st = dict(zip(st, max_over_ranks(list(st.values()))))
        flags = dec.flags()
        # the merge alone, from the last step's slots (all complete)
        dist.barrier()
        parity = (dec.steps - 1) & 1
        slots = [dec.slot(r, parity) for r in range(world)]
        m0, m1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 20
        m0.record(stream)
        for _ in range(reps):
            dcpmla.dcp_merge_heads([x[0] for x in slots], [x[1] for x in slots], B, H, h0, hn,
                                   dec.out, dec.out_lse)
        m1.record(stream)
        m1.synchronize()
        merge_us = max_over_ranks([m0.elapsed_time(m1) * 1e3 / reps])[0]
        # results of every rank's heads on rank 0, for the oracle check
        outs = [torch.empty_like(dec.out) for _ in range(world)]
        lses = [torch.empty_like(dec.out_lse) for _ in range(world)]
        dist.all_gather(outs, dec.out)
        dist.all_gather(lses, dec.out_lse)
        torch.cuda.synchronize(dev)
        dist.barrier()
    finally:
        sampler.stop()
        dec.close()
    result = None
    if rank == 0:
        out = torch.cat(outs, dim=1).double().cpu().numpy()
        lse = torch.cat(lses, dim=1).double().cpu().numpy()
        import oracle
        ni = prob.to("cpu").numpy_inputs()
        ids = sorted({0, B // 2, B - 1})
        _, _, ro, rl = oracle.dcp_decode(ni["q"], ni["kv_cache"], ni["kv_dtype"],
                                         ni["block_tables"], ni["seq_lens"], world,
                                         ni["softmax_scale"], ni["sparse_idx"],
                                         ni["block_size"], ids)
        fin = np.isfinite(rl)
        eo = float(np.abs(out[ids] - ro).max() / max(np.abs(ro).max(), 1e-30))
        el = float(np.abs(lse[ids][fin] - rl[fin]).max()) if fin.any() else 0.0
        kvb = kv_bytes(prob)
        peak, peak_kind = measured_peaks()
        ms = st["mean"]
        result = {
            "metric": METRIC, "value": round(kvb / (ms * 1e-3) / 1e9, 1), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": max(3, args.warmup),
            "ms_per_step": round(ms, 4), "ms_step_stats": ms_summary(st),
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
            "dtype": dtype_label(prob.kv_dtype, args.kernel),
            "data": "synthetic (seeded; no public trace or checkpoint available)",
            "config": {"workload": describe(args.workload, prob) + " (the shards on the GPUs)",
                       "global_batch": B, "heads": H, "kv_dtype": prob.kv_dtype,
                       "parallelism": f"DCP over {world} GPU(s): NCCL query all-gather, "
                                      "one shard per rank, all-reduce tick, head-sliced "
                                      "merge over peer memory",
                       "l2": "no flush: the KV read per step is larger than 4x the 126 MB L2"},
            "pct_hbm_peak_kv": round(100 * kvb / (ms * 1e-3) / 1e9 / world / peak, 1),
            "nccl_ranks": world, "merge_us_per_rank": round(merge_us, 2),
            "flags": flags,
            "oracle_check": {"requests": ids, "max_dO_rel": eo, "max_dLSE": el},
            "gpu_launches": args.steps * 3,
            "clocks": sampler.summary(),
            "e2e": None,
            "note": "eager steps (NCCL collectives inside); e2e not measured in this mode",
        }
    dist.barrier()
    dist.destroy_process_group()
    return result


def main():
    args = parse()
    rank, world, local = dist_env()
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    if args.dcp or (world > 1 and not args.replicas):
        res = run_dcp(args, rank, world, local)
        if rank == 0:
            print(json.dumps(res), flush=True)
        return
    res, prob = run_ours(args, rank, world, local)
    if rank == 0:
        if not args.no_cpu_baseline:
            res["cpu_baseline"], _ = time_oracle(args.workload, args.cpu_seconds)
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
