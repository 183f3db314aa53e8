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
