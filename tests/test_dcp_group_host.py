"""Host-side plumbing of real multi-GPU DCP decode (``dcp_group``), on CPU.

The query all-gather and the exchange of buffer handles run here with two and
three gloo ranks: the gathered heads must come out in rank order (gathered
head r * H/N + i is rank r's local head i, the order the per-rank merge
slices assume), and every rank must see every rank's handle at its rank's
index.  The head slices must tile the gathered heads exactly, and the
exchange slots must keep the LSEs 16-byte aligned behind the partials.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from long_context_decode_mla_b200 import dcp_group


def test_head_slices_tile_the_gathered_heads():
    for world in (1, 2, 4, 8):
        for heads in (8, 16, 64):
            if heads % world:
                continue
            covered = []
            for r in range(world):
                h0, hn = dcp_group.head_slice(r, world, heads)
                assert hn == heads // world
                covered += list(range(h0, h0 + hn))
            assert covered == list(range(heads))
    # the pages' geometry: 64 global heads, TP8 -> 8 local heads, DCP8 gathers 64
    assert dcp_group.head_slice(3, 8, 64) == (24, 8)


@pytest.mark.parametrize("args", [(0, 3, 64), (2, 2, 8), (-1, 2, 8), (0, 0, 8), (0, 2, 0)])
def test_head_slice_refuses_uneven_or_bad_groups(args):
    with pytest.raises(ValueError):
        dcp_group.head_slice(*args)


def test_slot_layout():
    for B, H in ((1, 8), (3, 64), (64, 64), (5, 7)):
        lse_off, size = dcp_group.slot_layout(B, H)
        assert lse_off == B * H * 512 * 4 and lse_off % 16 == 0
        assert size >= lse_off + B * H * 4 and size % dcp_group.SLOT_ALIGN == 0
        assert size - (lse_off + B * H * 4) < dcp_group.SLOT_ALIGN


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
    B, hn, D = 3, 2, 5
    # local head i of rank r carries the value 100 r + 10 i + b in every element
    q_local = torch.empty(B, hn, D)
    for b in range(B):
        for i in range(hn):
            q_local[b, i] = 100 * rank + 10 * i + b
    q = dcp_group.gather_query_heads(q_local)
    handles = dcp_group.exchange_handles(bytes([rank]) * 64)
    out_q.put((rank, q.tolist(), handles))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_query_gather_and_handle_exchange_with_gloo_ranks(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = dict((r, (g, h)) for r, g, h in (q.get(timeout=120) for _ in procs))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    B, hn = 3, 2
    for rank in range(world):
        gathered, handles = results[rank]
        assert handles == [bytes([r]) * 64 for r in range(world)]
        g = torch.tensor(gathered)
        assert g.shape == (B, world * hn, 5)
        for b in range(B):
            for h in range(world * hn):
                r, i = divmod(h, hn)
                assert bool((g[b, h] == 100 * r + 10 * i + b).all())


def _decoder_worker(rank, world, port, out_q):
    """One gloo rank running DcpRankDecoder with the library calls recorded
    instead of executed (no GPU here): the step's collectives are real."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from long_context_decode_mla_b200 import dcpmla
    log = []
    base = lambda r: 0x10000000 * (r + 1)                    # noqa: E731

    def alloc(nbytes):
        log.append(("alloc", nbytes))
        return base(rank), bytes([rank]) * dcpmla.IPC_HANDLE_BYTES

    def partial(q, kv, kvd, bt, lens, shard, nshards, idx, scale, o, l, ws, splits, impl, st, bs):
        log.append(("partial", shard, nshards, o.data_ptr(), l.data_ptr(), q.tolist()))

    def merge(parts, lses, B, H, h0, hn, out, out_lse):
        log.append(("merge", list(parts), list(lses), B, H, h0, hn))

    real_all_reduce = dist.all_reduce

    def all_reduce(t, group=None):
        log.append(("all_reduce",))
        return real_all_reduce(t, group=group)

    dcpmla.dcp_exchange_alloc = alloc
    dcpmla.dcp_exchange_open = lambda h: (log.append(("open", h[0])), base(h[0]))[1]
    dcpmla.dcp_exchange_close = lambda a: log.append(("close", a))
    dcpmla.dcp_exchange_free = lambda a: log.append(("free", a))
    dcpmla.mla_decode_partial = partial
    dcpmla.dcp_merge_heads = merge
    dcp_group.dist.all_reduce = all_reduce

    B, H = 2, 4 * world
    dec = dcp_group.DcpRankDecoder(B, H, topk=0, num_splits=4, device="cpu")
    for step in range(3):
        q_local = torch.full((B, H // world, 576), float(10 * step + rank), dtype=torch.bfloat16)
        dec.step(q_local, None, "fp8", None, None, 0.1)
    dec.close()
    out_q.put((rank, log, dcp_group.slot_layout(B, H)))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_rank_decoder_schedule_with_gloo_ranks(world):
    """Per rank: its own shard id, partials into alternating slots of its own
    buffer, the all-reduce strictly between its partial and its merge, a merge
    over every rank's slot of the same parity (rank order) for its own heads,
    queries gathered in rank order, and unmap -> all-reduce -> free at close."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_decoder_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = {r: (log, lay) for r, log, lay in (q.get(timeout=180) for _ in procs)}
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    B, H, hn = 2, 4 * world, 4
    base = lambda r: 0x10000000 * (r + 1)                    # noqa: E731
    for rank in range(world):
        log, (lse_off, slot) = results[rank]
        assert log[0] == ("alloc", 2 * slot)
        assert sorted(e[1] for e in log if e[0] == "open") == [r for r in range(world) if r != rank]
        steps = [e for e in log if e[0] in ("partial", "all_reduce", "merge")]
        body, tail = steps[:9], steps[9:]
        for k in range(3):
            part, red, mrg = body[3 * k:3 * k + 3]
            par = k & 1
            assert part[:5] == ("partial", rank, world, base(rank) + par * slot,
                                base(rank) + par * slot + lse_off)
            gathered = torch.tensor(part[5])
            for r in range(world):
                assert bool((gathered[:, r * hn:(r + 1) * hn] == 10 * k + r).all())
            assert red == ("all_reduce",)
            assert mrg == ("merge", [base(r) + par * slot for r in range(world)],
                           [base(r) + par * slot + lse_off for r in range(world)], B, H,
                           rank * hn, hn)
        assert tail == [("all_reduce",)]
        closes = [e for e in log if e[0] in ("close", "free")]
        assert closes[:-1] == [("close", base(r)) for r in range(world) if r != rank]
        assert closes[-1] == ("free", base(rank))
        assert log.index(("free", base(rank))) > len(log) - 2


def _failing_map_worker(rank, world, port, out_q):
    """Rank 1 cannot map a peer's buffer (a fake of the failing call returns
    an error code); every rank must unmap, free and raise, none may hang."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from long_context_decode_mla_b200 import dcpmla
    log = []
    base = lambda r: 0x10000000 * (r + 1)                    # noqa: E731

    def open_(h):
        if rank == 1:
            raise dcpmla.DcpMlaError(-5, "dcp_exchange_open")
        log.append(("open", h[0]))
        return base(h[0])

    dcpmla.lib = lambda: None                                # error text without the library
    dcpmla.error_string = lambda code: "CUDA runtime error"
    dcpmla.dcp_exchange_alloc = lambda n: (base(rank), bytes([rank]) * dcpmla.IPC_HANDLE_BYTES)
    dcpmla.dcp_exchange_open = open_
    dcpmla.dcp_exchange_close = lambda a: log.append(("close", a))
    dcpmla.dcp_exchange_free = lambda a: log.append(("free", a))
    try:
        dcp_group.DcpRankDecoder(2, 4 * world, num_splits=4, device="cpu")
        msg = None
    except RuntimeError as e:
        msg = str(e)
    out_q.put((rank, log, msg))
    dist.barrier()
    dist.destroy_process_group()


def test_a_failed_mapping_on_one_rank_fails_every_rank_cleanly():
    world = 3
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_failing_map_worker, args=(r, world, port, q))
             for r in range(world)]
    for p in procs:
        p.start()
    results = {r: (log, msg) for r, log, msg in (q.get(timeout=180) for _ in procs)}
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    base = lambda r: 0x10000000 * (r + 1)                    # noqa: E731
    for rank in range(world):
        log, msg = results[rank]
        assert msg is not None and "rank(s) [1]" in msg
        opened = [e[1] for e in log if e[0] == "open"]
        closed = [e[1] for e in log if e[0] == "close"]
        assert closed == [base(r) for r in opened]          # every mapping made is undone
        assert log[-1] == ("free", base(rank))               # and the own buffer is freed last
