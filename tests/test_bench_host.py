"""Host-side logic of the benchmark, on the CPU (no GPU is touched).

bench.py runs one process per GPU; every rank decodes its own batch (weak
scaling, no data-path collective) and the timings are reduced as the max over
ranks.  These tests run that reduction with two gloo ranks and check the
reference arm's rank behaviour; they also check the clock summary that decides
whether a run's clocks were valid (timed window, throttle reasons), the key
that ties the recorded DRAM traffic to the kernel source, and the KV byte
counts the GB/s figures divide by.
"""
import json
import os
import socket
import subprocess
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    vals = bench.max_over_ranks([1.0 + rank, 10.0 - rank, 0.5 * rank])
    out_q.put((rank, vals))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0] == res[1] == [2.0, 10.0, 0.5]


def test_max_over_ranks_without_group_is_identity():
    import bench
    assert bench.max_over_ranks([3.0, 4.0]) == [3.0, 4.0]


def _run_ref(rank):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank))
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                           "--steps", "1", "--warmup", "1", "--workload", "tiny"],
                          capture_output=True, text=True, env=env, timeout=600)


def test_reference_arm_prints_on_rank0_only():
    r1 = _run_ref(1)
    assert r1.returncode == 0 and r1.stdout.strip() == ""
    r0 = _run_ref(0)
    assert r0.returncode == 0
    line = json.loads(r0.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0


def test_ranks_draw_distinct_batches():
    from long_context_decode_mla_b200 import workload
    seed = workload.CONFIGS["tiny"]["seed"]
    a = workload.make_problem("tiny", seed=seed)
    b = workload.make_problem("tiny", seed=seed + 1000)
    assert not torch.equal(a.kv_cache, b.kv_cache)
    assert torch.equal(a.kv_cache, workload.make_problem("tiny", seed=seed).kv_cache)


def _sampler(samples, t_on, t_off):
    import bench
    s = bench.ClockSampler(0)
    s.samples, s.t_on, s.t_off = samples, t_on, t_off
    return s


def test_clock_summary_reads_the_timed_window_and_throttle_reasons():
    row = "{mhz}, 1965, 700.5, 0x{act:x}, {hw}, Not Active, Not Active, {pc}"
    samples = [
        (0.0, row.format(mhz=1005, act=0, hw="Not Active", pc="Not Active")),   # before: ignored
        (1.0, row.format(mhz=1900, act=4, hw="Not Active", pc="Active")),
        (1.1, row.format(mhz=1860, act=4, hw="Not Active", pc="Active")),
        (1.2, row.format(mhz=1965, act=0, hw="Not Active", pc="Not Active")),
        (1.3, "[N/A], [N/A], [N/A], [N/A], [N/A], [N/A], [N/A], [N/A]"),        # unparsable
        (9.0, row.format(mhz=300, act=8, hw="Active", pc="Not Active")),         # after: ignored
    ]
    s = _sampler(samples, 0.9, 1.35).summary()
    assert s["window"] == "timed region"
    assert s["samples"] == 3 and s["sm_mhz"] == 1900.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]
    # a throttle seen inside the window is reported by name
    s = _sampler(samples, 0.9, 9.5).summary()
    assert s["reasons"] == ["hw_slowdown", "sw_power_cap"]


def test_clock_summary_falls_back_to_the_whole_run_when_the_window_is_empty():
    samples = [(0.0, "1965, 1965, 500, 0x0, Not Active, Not Active, Not Active, Not Active")]
    s = _sampler(samples, 5.0, 5.01).summary()
    assert s["window"].startswith("whole run") and s["samples"] == 1
    assert _sampler([], None, None).summary()["sm_mhz"] is None


def test_traffic_key_ignores_comments_but_not_code():
    import bench
    csrc = os.path.join(ROOT, "long_context_decode_mla_b200", "csrc")

    def read(name, edit=None):
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            text = f.read()
        return edit(text) if edit and name == "partial_f8.cu" else text

    base = bench.kernel_source_hash(read)
    assert base == bench.kernel_source_hash()
    def recomment(t):
        return "// a new comment\n/* and a\n block */\n" + t.replace("\n", "  \n")

    commented = bench.kernel_source_hash(lambda n: read(n, recomment))
    assert commented == base
    changed = bench.kernel_source_hash(lambda n: read(n, lambda t: t + "\nstatic int x = 1;\n"))
    assert changed != base


def test_recorded_traffic_is_dropped_when_the_kernel_source_changes(monkeypatch):
    import bench
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        entry = json.load(f)["agentic/auto"]
    monkeypatch.setattr(bench, "kernel_source_hash", lambda read=None: entry["source_hash"])
    assert bench.recorded_traffic("agentic", "auto") == entry["bytes_per_launch"]
    monkeypatch.setattr(bench, "kernel_source_hash", lambda read=None: "0" * 16)
    assert bench.recorded_traffic("agentic", "auto") is None
    assert bench.recorded_traffic("no-such-workload", "auto") is None


def test_shard_kv_bytes_add_up_to_the_step():
    import bench
    from long_context_decode_mla_b200 import workload
    for name, over in (("tiny", {}), ("dense", dict(batch=3, seq_len=[700, 1, 0])),
                       ("sparse", dict(batch=2, seq_len=[5000, 100], topk=256))):
        for N in (1, 3, 8):
            p = workload.make_problem(name, num_shards=N, **over)
            assert sum(bench.shard_kv_bytes(p, s) for s in range(N)) == bench.kv_bytes(p)


def test_launches_per_shard_call():
    import bench
    sms = 148
    # dense: Q image + e4m3 partial + split combine for fp8 under auto/tc
    assert bench.launches_per_shard("fp8", "auto", False, 0, 64, sms) == 3
    assert bench.launches_per_shard("fp8", "tc", False, 0, 64, sms) == 3
    # dense bf16 rows, or the fp16-operand / CUDA-core kernels: partial + combine
    assert bench.launches_per_shard("bf16", "auto", False, 0, 32, sms) == 2
    assert bench.launches_per_shard("fp8", "tc16", False, 0, 64, sms) == 2
    assert bench.launches_per_shard("fp8", "simt", False, 0, 64, sms) == 2
    # sparse on the tensor-core path: lists with the Q images + partial (fp8),
    # or lists + partial + combine (bf16)
    assert bench.launches_per_shard("fp8", "auto", True, 2048, 128, sms) == 2
    assert bench.launches_per_shard("bf16", "auto", True, 2048, 128, sms) == 3
    # in-kernel selection: a combine only when a list spans several CTAs
    assert bench.launches_per_shard("fp8", "tc16", True, 2048, 128, sms) == 1
    assert bench.launches_per_shard("fp8", "simt", True, 4096, 128, sms) == 2
    assert bench.launches_per_shard("fp8", "tc16", True, 256, 16, sms) == 2


def test_shard_splits_is_the_sm_share(monkeypatch):
    import argparse
    import bench
    from long_context_decode_mla_b200 import dcpmla
    monkeypatch.setattr(dcpmla, "device_sm_count", lambda: 148)
    args = argparse.Namespace(splits=None)
    assert bench.shard_splits("agentic", 8, args) == 18
    assert bench.shard_splits("tiny", 2, args) == 74
    assert bench.shard_splits("million", 1, args) == 148
    args.splits = 37
    assert bench.shard_splits("sparse", 8, args) == 37
