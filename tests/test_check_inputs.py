"""The host-side debug validation of device contents (dcpmla.check_inputs)."""
import pytest
import torch

from long_context_decode_mla_b200 import dcpmla
from long_context_decode_mla_b200 import workload as wl


def _prob(name="tiny", **kw):
    return wl.make_problem(name, **kw)


def test_valid_problems_pass():
    for name, kw in [("tiny", {}), ("dense", dict(batch=3, seq_len=[700, 1, 0])),
                     ("sparse", dict(batch=2, seq_len=3000, topk=64))]:
        p = _prob(name, **kw)
        dcpmla.check_inputs(p.block_tables, p.seq_lens, p.kv_cache.shape[0], p.num_shards,
                            p.sparse_idx)


def test_bad_block_entry_is_reported_only_where_used():
    p = _prob("dense", num_shards=2, batch=2, seq_len=[200, 1])
    nb = p.kv_cache.shape[0]
    bt = p.block_tables.clone()
    bt[1, 1, -1] = nb + 5          # request 1 has one row: its last table entries are unused
    dcpmla.check_inputs(bt, p.seq_lens, nb, 2)
    bt[0, 0, 0] = nb
    with pytest.raises(ValueError, match=r"block_tables\[0\]\[0\]\[0\]"):
        dcpmla.check_inputs(bt, p.seq_lens, nb, 2)


def test_length_beyond_the_table_row_is_reported():
    p = _prob("tiny", num_shards=2)
    lens = p.seq_lens.clone()
    lens[0] = 10 ** 6
    with pytest.raises(ValueError, match="blocks, the table row has"):
        dcpmla.check_inputs(p.block_tables, lens, p.kv_cache.shape[0], 2)
    lens[0] = -3
    with pytest.raises(ValueError, match="negative"):
        dcpmla.check_inputs(p.block_tables, lens, p.kv_cache.shape[0], 2)


def test_sparse_indices_outside_the_request_are_reported():
    p = _prob("sparse", num_shards=2, batch=2, seq_len=3000, topk=16)
    idx = p.sparse_idx.clone()
    idx[1, 3] = -1                   # padding is fine
    dcpmla.check_inputs(p.block_tables, p.seq_lens, p.kv_cache.shape[0], 2, idx)
    idx[1, 4] = 3000
    with pytest.raises(ValueError, match=r"sparse_idx\[1\]\[4\]"):
        dcpmla.check_inputs(p.block_tables, p.seq_lens, p.kv_cache.shape[0], 2, idx)


def test_shape_errors():
    p = _prob("tiny", num_shards=2)
    with pytest.raises(ValueError):
        dcpmla.check_inputs(p.block_tables[0], p.seq_lens, p.kv_cache.shape[0], 2)
    with pytest.raises(ValueError):
        dcpmla.check_inputs(p.block_tables, torch.zeros(5, dtype=torch.int32),
                            p.kv_cache.shape[0], 2)
