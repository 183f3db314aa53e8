"""Host-side logic of the benchmark's multi-rank path, on CPU ranks (gloo).

bench.py runs one process per GPU; every rank decodes its own batch (weak
scaling, no data-path collective) and the timings are reduced as the max over
ranks.  These tests run that reduction with two gloo ranks on the CPU and
check the reference arm's rank behaviour; no GPU is touched.
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
