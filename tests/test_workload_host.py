"""Host checks of the seeded input generators (no GPU)."""
import torch

from long_context_decode_mla_b200 import workload as wl


def test_device_id_coded_builder_matches_the_host_one():
    # the vectorised builder used by the full-size GPU tests places the same
    # rows through the same tables as the per-request host builder
    for kv in ("fp8", "bf16"):
        lens = [1, 7, 64, 65, 300, 1000]
        a = wl.id_coded_problem(lens, 3, kv, heads=4, seed=5)
        b = wl.id_coded_problem_device(lens, 3, kv, heads=4, seed=5, device="cpu")
        assert torch.equal(a.block_tables, b.block_tables)
        assert torch.equal(a.seq_lens, b.seq_lens)
        assert torch.equal(a.kv_cache, b.kv_cache)
