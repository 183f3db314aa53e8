"""The C ABI used from plain C: ``tests/c_abi/decode_from_c.c`` links only
libdcpmla.so and the CUDA runtime (no PyTorch, no Python) and runs one
emulated DCP step (every shard's ``mla_decode_partial``, then ``dcp_merge``).

The CPU test compiles and links it (the header is valid C99 and every symbol
it uses resolves); the GPU test runs it and checks its output file against
the CPU oracle."""
import os
import shutil
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "c_abi", "decode_from_c.c")
LIBDIR = os.path.join(ROOT, "long_context_decode_mla_b200")
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def _compile(tmp_path):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    if not os.path.exists(os.path.join(LIBDIR, "libdcpmla.so")):
        from long_context_decode_mla_b200 import build
        build.build()
    exe = str(tmp_path / "decode_from_c")
    cmd = [cc, "-O2", "-std=c99", "-Wall", "-Wextra", "-Werror",
           "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(CUDA, "include"), SRC, "-L", LIBDIR, "-ldcpmla",
           "-L", os.path.join(CUDA, "lib64"), "-lcudart", f"-Wl,-rpath,{LIBDIR}",
           f"-Wl,-rpath,{os.path.join(CUDA, 'lib64')}", "-o", exe]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return exe


def test_c_client_compiles_and_links(tmp_path):
    exe = _compile(tmp_path)
    assert os.path.exists(exe)


def _write_inputs(path, prob):
    ni = prob.numpy_inputs()
    B, H = ni["q"].shape[0], ni["q"].shape[1]
    N = ni["num_shards"]
    tables = np.ascontiguousarray(ni["block_tables"], dtype="<i4")
    kv = np.ascontiguousarray(ni["kv_cache"], dtype=np.uint8)
    kvd = 1 if ni["kv_dtype"] == "fp8" else 0
    with open(path, "wb") as f:
        f.write(np.array([B, H, N, tables.shape[2], kv.shape[0], kvd], dtype="<i4").tobytes())
        f.write(np.array([ni["softmax_scale"]], dtype="<f4").tobytes())
        f.write(np.ascontiguousarray(ni["seq_lens"], dtype="<i4").tobytes())
        f.write(tables.tobytes())
        f.write(np.ascontiguousarray(ni["q"], dtype="<u2").tobytes())
        f.write(kv.tobytes())
    return ni, B, H


@pytest.mark.gpu
@pytest.mark.parametrize("name,kv_dtype,over", [
    ("tiny", "bf16", {}),
    ("agentic", "fp8", dict(batch=3, seq_len=[5000, 64, 1])),
])
def test_c_client_matches_the_oracle(tmp_path, name, kv_dtype, over):
    import oracle
    from long_context_decode_mla_b200 import workload as wl
    exe = _compile(tmp_path)
    prob = wl.make_problem(name, num_shards=2, **over)
    ni, B, H = _write_inputs(tmp_path / "in.bin", prob)
    r = subprocess.run([exe, str(tmp_path / "in.bin"), str(tmp_path / "out.bin")],
                       capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    raw = np.fromfile(tmp_path / "out.bin", dtype="<f4")
    out = raw[:B * H * 512].reshape(B, H, 512).astype(np.float64)
    lse = raw[B * H * 512:].reshape(B, H).astype(np.float64)
    _, _, ref, ref_lse = oracle.dcp_decode(ni["q"], ni["kv_cache"], kv_dtype, ni["block_tables"],
                                           ni["seq_lens"], 2, ni["softmax_scale"])
    rel_o, abs_l = (2e-3, 1e-4) if kv_dtype == "bf16" else (2e-2, 5e-3)
    assert np.abs(out - ref).max() <= rel_o * np.abs(ref).max()
    fin = np.isfinite(ref_lse)
    assert np.array_equal(fin, np.isfinite(lse))
    assert np.abs(lse[fin] - ref_lse[fin]).max() <= abs_l
