"""Host-side checks of the C ABI: exported symbols and fail-closed argument checks.

None of these calls reaches a kernel launch: every case returns an error code
from the host-side checks, so they run without a GPU (and are harmless with
one).
"""
import ctypes
import json
import os
import re

import pytest

from long_context_decode_mla_b200 import dcpmla

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dcpmla.h")

OK, EINVAL, EUNSUP, EWS, EALIGN, ECUDA = 0, -1, -2, -3, -4, -5


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return set(re.findall(r"^\s*(?:const\s+)?\w+\**\s+\**(\w+)\s*\(", text, flags=re.M))


def test_header_declares_the_entry_points():
    names = _declared_functions()
    assert {"mla_decode_partial", "dcp_merge", "mla_decode_workspace_size",
            "dcpmla_error_string", "dcpmla_device_sm_count"} <= names


def test_library_exports_every_declared_symbol():
    L = dcpmla.lib()
    for name in _declared_functions():
        assert hasattr(L, name), name


def test_error_strings():
    for code in (OK, EINVAL, EUNSUP, EWS, EALIGN, ECUDA, -99):
        assert isinstance(dcpmla.error_string(code), str) and dcpmla.error_string(code)


def test_workspace_size_grows_with_splits_and_batch():
    a = dcpmla.mla_decode_workspace_size(64, 64, 148)
    b = dcpmla.mla_decode_workspace_size(64, 64, 296)
    c = dcpmla.mla_decode_workspace_size(128, 64, 148)
    assert 256 < a < b and a < c
    # (G + B) slots of H x 512 fp32 plus LSEs plus the 256-byte header
    assert a >= 256 + (148 + 64) * 64 * 513 * 4
    s = dcpmla.mla_decode_workspace_size(128, 64, 148, topk=2048)
    assert s >= 256 + 128 * 64 * 513 * 4


def test_workspace_size_rejects_bad_arguments():
    L = dcpmla.lib()
    n = ctypes.c_size_t(0)
    assert L.mla_decode_workspace_size(-1, 64, 1, 0, ctypes.byref(n)) == EINVAL
    assert L.mla_decode_workspace_size(1, 0, 1, 0, ctypes.byref(n)) == EINVAL
    # rows: 64 heads, or (query, head) pairs of a multi-query call, up to 64 x 64
    assert L.mla_decode_workspace_size(1, 64 * 64 + 1, 1, 0, ctypes.byref(n)) == EUNSUP
    assert L.mla_decode_workspace_size(1, 256, 1, 0, ctypes.byref(n)) == 0
    assert L.mla_decode_workspace_size(1, 8, 1, 0, None) == EINVAL


FAKE = 0x10000          # aligned, never dereferenced: every call below fails before launch


def _call(**kw):
    a = dict(q=FAKE, kv=FAKE, kv_dtype=0, num_blocks=16, block_size=64, bt=FAKE, bt_stride=4,
             lens=FAKE, batch=2, heads=8, shard=0, nshards=2, idx=None, topk=0, scale=0.07,
             out=FAKE, lse=FAKE, ws=FAKE, ws_bytes=0, splits=4, impl=0, stream=None)
    a.update(kw)
    return dcpmla.lib().mla_decode_partial(
        a["q"], a["kv"], a["kv_dtype"], a["num_blocks"], a["block_size"], a["bt"], a["bt_stride"],
        a["lens"], a["batch"], a["heads"], a["shard"], a["nshards"], a["idx"], a["topk"],
        a["scale"], a["out"], a["lse"], a["ws"], a["ws_bytes"], a["splits"], a["impl"],
        a["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(shard=2), EINVAL), (dict(shard=-1), EINVAL), (dict(nshards=0), EINVAL),
    (dict(batch=-1), EINVAL), (dict(heads=0), EINVAL), (dict(heads=65), EUNSUP),
    (dict(heads=128), EUNSUP), (dict(block_size=16), EUNSUP), (dict(block_size=0), EINVAL),
    (dict(kv_dtype=2), EINVAL), (dict(num_blocks=0), EINVAL), (dict(bt_stride=0), EINVAL),
    (dict(splits=-1), EINVAL), (dict(impl=7), EINVAL), (dict(scale=float("nan")), EINVAL),
    (dict(scale=float("inf")), EINVAL), (dict(idx=FAKE, topk=0), EINVAL),
    (dict(q=None), EINVAL), (dict(kv=None), EINVAL), (dict(bt=None), EINVAL),
    (dict(lens=None), EINVAL), (dict(out=None), EINVAL), (dict(lse=None), EINVAL),
    (dict(q=FAKE + 8), EALIGN), (dict(kv=FAKE + 4), EALIGN), (dict(out=FAKE + 4), EALIGN),
    (dict(ws=None), EWS), (dict(ws_bytes=1024), EWS),
])
def test_partial_fails_closed(kw, code):
    assert _call(**kw) == code


def test_empty_batch_is_a_no_op():
    assert _call(batch=0, q=None, kv=None, bt=None, lens=None, out=None, lse=None) == OK


def test_merge_fails_closed():
    L = dcpmla.lib()
    assert L.dcp_merge(FAKE, FAKE, 0, 1, 8, FAKE, None, None) == EINVAL
    assert L.dcp_merge(FAKE, FAKE, 2, -1, 8, FAKE, None, None) == EINVAL
    assert L.dcp_merge(FAKE, FAKE, 2, 1, 0, FAKE, None, None) == EINVAL
    assert L.dcp_merge(None, FAKE, 2, 1, 8, FAKE, None, None) == EINVAL
    assert L.dcp_merge(FAKE, FAKE, 2, 1, 8, None, None, None) == EINVAL
    assert L.dcp_merge(FAKE + 4, FAKE, 2, 1, 8, FAKE, None, None) == EALIGN
    assert L.dcp_merge(FAKE, FAKE, 2, 0, 8, FAKE, None, None) == OK


def test_head_envelope_matches_the_page_table():
    with open(os.path.join(ROOT, "tests", "golden", "head_envelope.json")) as f:
        g = json.load(f)
    for row in g["rows"]:
        assert row["local"] == g["global_heads"] // g["tp"]
        assert row["gathered"] == row["local"] * row["dcp"]
        assert dcpmla.padded_heads(row["local"]) == row["local_pad"]
        assert dcpmla.padded_heads(row["gathered"]) == row["gathered_pad"]


def test_noalloc_refuses_before_touching_the_device():
    """Refusals of mla_decode_partial_noalloc come from host checks alone."""
    L = dcpmla.lib()
    f = L.mla_decode_partial_noalloc
    vp, i32, i64, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float
    f.argtypes = [vp, vp, i32, i64, i32, vp, i32, vp, i32, i32, i32, i32, vp, i32, f32,
                  vp, vp, vp, i32, i32, vp]
    f.restype = i32

    def call(batch, heads, splits, topk=0, sparse=None):
        return f(None, None, 0, 1, 64, None, 1, None, batch, heads, 0, 1, sparse, topk, 1.0,
                 None, None, None, splits, 0, None)

    need = dcpmla.mla_decode_workspace_size(600, 64, 148)
    assert need > dcpmla.NOALLOC_SCRATCH_BYTES
    assert call(600, 64, 148) == EWS                 # beyond the built-in scratch
    assert call(4, 0, 148) == EINVAL                 # bad sizes fail before the size check
    assert call(-1, 64, 148) == EINVAL
    assert call(4, 65, 148) == EUNSUP


def test_noalloc_scratch_size_matches_header():
    text = open(HEADER).read()
    m = re.search(r"#define DCPMLA_NOALLOC_SCRATCH_BYTES \((\d+)u << (\d+)\)", text)
    assert m and int(m.group(1)) << int(m.group(2)) == dcpmla.NOALLOC_SCRATCH_BYTES


def _append_fn():
    L = dcpmla.lib()
    f = L.mla_kv_append
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    f.argtypes = [vp, vp, i32, vp, vp, vp, i32, i32, i32, i32, vp, i32, i64, i32, vp, vp]
    f.restype = i32
    return f


def test_kv_append_fails_closed_before_any_launch():
    f = _append_fn()
    A = 0x10000                       # 16-byte aligned fake pointers: never dereferenced
    base = dict(lat=A, rope=A, T=4, pos=A, req=A, bt=A, stride=2, B=1, s=0, N=2, cache=A,
                kvd=1, nb=8, bs=64)

    def call(**kw):
        a = dict(base, **kw)
        return f(a["lat"], a["rope"], a["T"], a["pos"], a["req"], a["bt"], a["stride"], a["B"],
                 a["s"], a["N"], a["cache"], a["kvd"], a["nb"], a["bs"], None, None)

    assert call(T=-1) == EINVAL
    assert call(s=2) == EINVAL and call(s=-1) == EINVAL and call(N=0) == EINVAL
    assert call(kvd=5) == EINVAL
    assert call(nb=0) == EINVAL and call(B=0) == EINVAL and call(stride=0) == EINVAL
    assert call(bs=32) == EUNSUP
    assert call(T=0) == OK                                   # nothing to write
    assert call(lat=None) == EINVAL and call(cache=None) == EINVAL and call(bt=None) == EINVAL
    assert call(lat=A + 8) == EALIGN and call(cache=A + 4) == EALIGN and call(rope=A + 2) == EALIGN


def test_multi_query_fails_closed_before_any_launch():
    L = dcpmla.lib()
    f = L.mla_decode_partial_multi
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    f32, sz = ctypes.c_float, ctypes.c_size_t
    f.argtypes = [vp, vp, i32, i64, i32, vp, i32, vp, i32, i32, i32, i32, i32, f32, vp, vp, vp, sz,
                  i32, i32, vp]
    f.restype = i32

    def call(heads=16, q_len=4, batch=2, shard=0, nshards=2, kvd=1, bs=64, impl=0, q=FAKE):
        return f(q, FAKE, kvd, 16, bs, FAKE, 4, FAKE, batch, heads, q_len, shard, nshards, 0.07,
                 FAKE, FAKE, FAKE, 0, 4, impl, None)

    assert call(q_len=0) == EINVAL and call(heads=0) == EINVAL
    # more than 64 rows run as passes over the cache: accepted, and then the
    # (empty) workspace is refused before anything is launched
    assert call(heads=16, q_len=5) == EWS and call(heads=64, q_len=4) == EWS
    assert call(heads=65) == EUNSUP and call(q_len=65) == EINVAL
    assert call(shard=2) == EINVAL and call(kvd=3) == EINVAL and call(bs=16) == EUNSUP
    assert call(q=FAKE + 2) == EALIGN
    assert call(batch=0) == OK                               # nothing to do


def test_merge_heads_fails_closed_before_any_launch():
    L = dcpmla.lib()
    P = ctypes.c_void_p * 2
    ok = P(FAKE, FAKE + 4096)

    def call(parts=ok, lses=ok, n=2, batch=1, heads=8, h0=0, hn=4, out=FAKE):
        return L.dcp_merge_heads(parts, lses, n, batch, heads, h0, hn, out, None, None)

    assert call(n=0) == EINVAL and call(n=dcpmla.MAX_MERGE_SHARDS + 1) == EINVAL
    assert call(heads=0) == EINVAL and call(batch=-1) == EINVAL
    assert call(h0=-1) == EINVAL and call(hn=0) == EINVAL and call(h0=5, hn=4) == EINVAL
    assert call(parts=None) == EINVAL and call(lses=None) == EINVAL and call(out=None) == EINVAL
    assert call(parts=P(FAKE, None)) == EINVAL and call(lses=P(None, FAKE)) == EINVAL
    assert call(parts=P(FAKE, FAKE + 4)) == EALIGN and call(out=FAKE + 8) == EALIGN
    assert call(batch=0, parts=None, lses=None, out=None) == OK      # nothing to do


def test_merge_heads_limits_match_header():
    text = open(HEADER).read()
    assert re.search(r"#define DCPMLA_MAX_MERGE_SHARDS (\d+)", text).group(1) == \
        str(dcpmla.MAX_MERGE_SHARDS)
    assert re.search(r"#define DCPMLA_IPC_HANDLE_BYTES (\d+)", text).group(1) == \
        str(dcpmla.IPC_HANDLE_BYTES)


def test_exchange_calls_refuse_null_arguments():
    L = dcpmla.lib()
    h = ctypes.create_string_buffer(dcpmla.IPC_HANDLE_BYTES)
    p = ctypes.c_void_p(0)
    assert L.dcp_exchange_alloc(0, ctypes.byref(p), h) == EINVAL
    assert L.dcp_exchange_alloc(1024, None, h) == EINVAL
    assert L.dcp_exchange_alloc(1024, ctypes.byref(p), None) == EINVAL
    assert L.dcp_exchange_open(None, ctypes.byref(p)) == EINVAL
    assert L.dcp_exchange_open(h, None) == EINVAL
    assert L.dcp_exchange_close(None) == EINVAL and L.dcp_exchange_free(None) == EINVAL
    with pytest.raises(ValueError):
        dcpmla.dcp_exchange_open(b"short")
