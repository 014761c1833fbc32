"""CPU tests of the benchmark's host-side accounting: the algorithmic bytes it divides
by (checked against the byte counts stated for the workloads), which decode kernel the
roofline names, and the rule that committed ncu traffic only counts for the kernel
sources it was captured from."""
import json
from types import SimpleNamespace

import pytest
import torch

import bench
from workloads import WORKLOADS, make_inputs


def _shape(lens, H, Hk, D, ps):
    """What the byte accounting reads of a workload: its lengths and shapes."""
    return SimpleNamespace(num_seqs=len(lens), num_heads=H, num_kv_heads=Hk, head_dim=D, page_size=ps,
                           seq_lens=torch.tensor(lens, dtype=torch.int32))


@pytest.mark.parametrize("shape,kv,qo", [
    (([17, 40], 4, 1, 64, 16), 14_592, 2_048),                  # tiny MQA; q+out 2x2x4x64x2
    (([8192] * 64, 96, 1, 128, 64), 268_435_456, 3_145_728),    # MQA batch; q+out 2x64x96x128x2
    (([131072] * 4, 64, 8, 128, 16), 2_147_483_648, 131_072),   # long context; q+out 2x4x64x128x2
])
def test_algorithmic_bytes_match_the_stated_workload_sizes(shape, kv, qo):
    inp = _shape(*shape)
    b = bench.algorithmic_bytes(inp, with_append=False)
    assert b["kv"] == kv
    pages = int(((inp.seq_lens.long() + inp.page_size - 1) // inp.page_size).sum())
    assert b["decode"] == kv + qo + pages * 4 + inp.num_seqs * 4
    assert b["append"] == 0 and b["step"] == b["decode"]


def test_the_generated_small_workload_has_the_stated_sizes():
    inp = make_inputs(1, poison=False)
    assert bench.algorithmic_bytes(inp, with_append=False)["kv"] == 14_592


def test_append_bytes_count_new_rows_and_indices():
    inp = _shape(list(range(1, 257)), 32, 8, 128, 16)
    b = bench.algorithmic_bytes(inp, with_append=True)
    B, Hk, D = inp.num_seqs, inp.num_kv_heads, inp.head_dim
    assert b["append"] == 2 * (B * Hk * D * 2) * 2 + 8 * B
    assert b["step"] == b["decode"] + b["append"]
    assert bench.algorithmic_bytes(inp, with_append=True, num_seqs=10)["kv"] == sum(range(1, 11)) * Hk * D * 4


def test_roofline_kernel_follows_the_group_size():
    class G:
        def __init__(self, h, hk):
            self.num_heads, self.num_kv_heads = h, hk
    assert bench.decode_kernel_for(G(32, 8)) == "decode_ws_kernel"
    assert bench.decode_kernel_for(G(16, 1)) == "decode_ws_kernel"
    assert bench.decode_kernel_for(G(17, 1)) == "decode_tc_kernel"
    assert bench.decode_kernel_for(G(96, 1)) == "decode_tc_kernel"
    for w in WORKLOADS.values():
        assert bench.decode_kernel_for(G(w.num_heads, w.num_kv_heads)) in bench.KERNEL_SOURCES


def test_profiled_traffic_counts_only_for_its_own_kernel_sources(tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    src.write_text("kernel v1")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setitem(bench.KERNEL_SOURCES, "decode_ws_kernel", ["k.cu"])
    sha = bench.kernel_source_sha("decode_ws_kernel")
    prof = tmp_path / "traffic.json"
    prof.write_text(json.dumps({"gqa_decode": {
        "kernel": "decode_ws_kernel<128>", "kernel_source_sha": sha,
        "dram_bytes_per_launch": 1000, "units_per_launch": 100}}))
    monkeypatch.setattr(bench, "PROFILE_TRAFFIC", str(prof))
    assert bench.profiled_traffic("gqa_decode", "decode_ws_kernel", 100) == 1000
    assert bench.profiled_traffic("gqa_decode", "decode_ws_kernel", 250) == 2500   # scaled by units
    assert bench.profiled_traffic("mqa_decode", "decode_ws_kernel", 100) is None    # no capture
    assert bench.profiled_traffic("gqa_decode", "decode_tc_kernel", 100) is None    # other kernel
    src.write_text("kernel v2")                                                      # source changed
    assert bench.kernel_source_sha("decode_ws_kernel") != sha
    assert bench.profiled_traffic("gqa_decode", "decode_ws_kernel", 100) is None


def test_measured_peak_is_the_copy_rate_or_the_fallback(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_peak() == (bench.FALLBACK_HBM_GBS, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6554.6}))
    assert bench.measured_peak() == (6554.6, "measured")


@pytest.mark.parametrize("index,shrink", [(4, 256), (5, 64), (2, 8)])
def test_shrunk_workload_keeps_shapes_and_divides_every_length(index, shrink):
    """The smaller case the profiler captures of a workload: same shapes, page size and
    seeded length recipe, every context length divided by N (rounded up)."""
    from workloads import WORKLOADS, _seq_lens_for, make_shrunk_inputs
    spec = WORKLOADS[index]
    small = make_shrunk_inputs(index, shrink, seed=1000 + index, poison=False)
    full = _seq_lens_for(spec, torch.Generator().manual_seed(1000 + index)).tolist()
    assert small.seq_lens.tolist() == [(L + shrink - 1) // shrink for L in full]
    assert (small.num_seqs, small.num_heads, small.num_kv_heads, small.head_dim, small.page_size) == (
        spec.num_seqs, spec.num_heads, spec.num_kv_heads, spec.head_dim, spec.page_size)
