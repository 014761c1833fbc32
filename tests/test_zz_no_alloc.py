"""GPU: the allocation-free decode entry point against the regular one.

gqa_paged_decode_attn_noalloc serves callers that cannot allocate device memory
(an engine that already owns nearly all of the GPU, a step loop that cannot take the
synchronisation of cudaMalloc, a plugin given no workspace).  It keeps its scratch
in a fixed array inside the library, shared by all calls, so these tests call it
twice in a row (with different shapes, so the second call finds the first call's
leftovers) and compare each result with gqa_paged_decode_attn on the same inputs,
within the parity tolerance of the other GPU tests.  This file is collected last.
"""
import ctypes

import pytest
import torch

import gqa_decode_attention_04_b200 as gq
from parity import assert_close, gpu_f64, host_arrays, oracle_out
from workloads import make_custom_inputs

pytestmark = pytest.mark.gpu


def _noalloc_c_abi(d, out):
    """Call the entry point through the C ABI (ctypes), exactly as a C caller would."""
    lib = gq.load_library()
    B, H, D = d.q.shape
    P, Hk, ps, _ = d.k_pages.shape
    return lib.gqa_paged_decode_attn_noalloc(
        d.q.data_ptr(), d.k_pages.data_ptr(), d.v_pages.data_ptr(), d.block_table.data_ptr(),
        d.seq_lens.data_ptr(), out.data_ptr(), B, H, Hk, D, ps, ctypes.c_float(d.scale),
        d.block_table.shape[1], P, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


CASES = [
    # (seq_lens, H, Hk, D, ps): long enough that segments span several CTAs, so the
    # split counters and partials in the shared array are exercised.
    ([3000, 17, 900, 1], 32, 8, 128, 16),   # token split (G = 4)
    ([700, 2500], 96, 1, 128, 64),          # tcgen05 kernel and split merge (MQA, G = 96)
    ([40, 33], 4, 1, 64, 16),               # head_dim 64, tiny
]


def test_noalloc_matches_regular_entry_point_on_consecutive_calls(cuda_device):
    gq.set_num_workers(0)
    for i, (lens, H, Hk, D, ps) in enumerate(CASES):
        inp = make_custom_inputs(lens, H, Hk, D, ps, seed=100 + i, extra_pages=2)
        d = inp.to(cuda_device)
        ref = gq.paged_decode_attn(d.q, d.k_pages, d.v_pages, d.block_table, d.seq_lens, scale=d.scale)
        gq.check_device_error()
        for rep in range(2):  # two calls in a row on the same array
            out = torch.full_like(ref, float("nan"))
            assert _noalloc_c_abi(d, out) == 0, gq.load_library().gqa_last_error_string()
            torch.cuda.synchronize()
            assert_close(gpu_f64(out), gpu_f64(ref), what=f"case {i} call {rep}")
        assert_close(gpu_f64(out), oracle_out(host_arrays(inp)), what=f"case {i} vs oracle")


def test_noalloc_with_many_split_workers(cuda_device):
    """Forced worker counts shrink to what the fixed array holds; results still agree."""
    inp = make_custom_inputs([5000, 3000], 16, 4, 128, 16, seed=7)
    d = inp.to(cuda_device)
    gq.set_num_workers(0)
    ref = gq.paged_decode_attn(d.q, d.k_pages, d.v_pages, d.block_table, d.seq_lens, scale=d.scale)
    try:
        for workers in (3, 700, 100000):
            gq.set_num_workers(workers)
            out = torch.empty_like(ref)
            gq.paged_decode_attn_noalloc(d.q, d.k_pages, d.v_pages, d.block_table, d.seq_lens, out,
                                         scale=d.scale)
            torch.cuda.synchronize()
            assert_close(gpu_f64(out), gpu_f64(ref), what=f"workers={workers}")
    finally:
        gq.set_num_workers(0)


def test_noalloc_fit_limit_caps_forced_workers(cuda_device):
    """With 128 query heads per kv head each worker's two partial slots take
    2 x 128 x (128 + 2) floats, so the fixed 16 MiB array holds about 125 workers; 1000
    forced workers (fewer than the 1250 blocks of work) must be cut to what fits, and the
    result must still agree with the regular entry point and the oracle."""
    lens = [40000, 40000]
    inp = make_custom_inputs(lens, 128, 1, 128, 64, seed=8, extra_pages=1)
    d = inp.to(cuda_device)
    per_worker = 2 * 128 * (128 + 2) * 4 + 512
    assert (16 << 20) // per_worker < 1000 <= sum((L + 63) // 64 for L in lens)
    try:
        gq.set_num_workers(1000)
        ref = gq.paged_decode_attn(d.q, d.k_pages, d.v_pages, d.block_table, d.seq_lens, scale=d.scale)
        gq.check_device_error()
        out = torch.full_like(ref, float("nan"))
        assert _noalloc_c_abi(d, out) == 0, gq.load_library().gqa_last_error_string()
        gq.check_device_error()
    finally:
        gq.set_num_workers(0)
    assert_close(gpu_f64(out), gpu_f64(ref), what="fit-limited workers vs regular")
    assert_close(gpu_f64(out), oracle_out(host_arrays(inp)), what="fit-limited workers vs oracle")


def test_noalloc_reports_device_errors(cuda_device):
    """A bad page id and a wait that runs out are reported by check_device_error through
    the fixed array's error word; a normal call afterwards is right again."""
    inp = make_custom_inputs([300, 90], 16, 4, 128, 16, seed=9)
    d = inp.to(cuda_device)
    out = torch.empty((2, 16, 128), dtype=torch.bfloat16, device=cuda_device)
    gq.check_device_error()  # nothing pending
    bt = d.block_table.clone()
    bt[0, 3] = 10 ** 6
    gq.paged_decode_attn_noalloc(d.q, d.k_pages, d.v_pages, bt, d.seq_lens, out, scale=d.scale)
    with pytest.raises(gq.GQAError) as ei:
        gq.check_device_error()
    assert ei.value.status == -4
    gq.check_device_error()  # the word was cleared by the read
    for H, Hk, ps in ((16, 4, 16),):  # the mma.sync kernel (the tcgen05 kernel's timeout path stays off GPUs)
        inp = make_custom_inputs([700, 90], H, Hk, 128, ps, seed=10 + H)
        d = inp.to(cuda_device)
        out = torch.empty((2, H, 128), dtype=torch.bfloat16, device=cuda_device)
        try:
            gq.set_num_workers(12)
            gq.set_wait_limit_ns(2_000_000, arm_without_copy=True)
            gq.paged_decode_attn_noalloc(d.q, d.k_pages, d.v_pages, d.block_table, d.seq_lens, out,
                                         scale=d.scale)
            with pytest.raises(gq.GQAError) as ei:
                gq.check_device_error()
            assert ei.value.status == -5
        finally:
            gq.set_wait_limit_ns(10 ** 9, False)
        try:
            gq.paged_decode_attn_noalloc(d.q, d.k_pages, d.v_pages, d.block_table, d.seq_lens, out,
                                         scale=d.scale)
            gq.check_device_error()
        finally:
            gq.set_num_workers(0)
        assert_close(gpu_f64(out), oracle_out(host_arrays(inp)), what=f"after timeout H={H}")


def test_noalloc_allocates_no_device_memory(cuda_device):
    """Free device memory is unchanged across a call with more segments and workers than
    any earlier call of this process (so a regular workspace would have had to grow)."""
    small = make_custom_inputs([100, 60], 32, 8, 128, 16, seed=11).to(cuda_device)
    big_lens = [64] * 2000  # 2000 sequences x 8 kv heads = 16000 segments
    big = make_custom_inputs(big_lens, 32, 8, 128, 16, seed=12, poison=False).to(cuda_device)
    out_s = torch.empty((2, 32, 128), dtype=torch.bfloat16, device=cuda_device)
    out_b = torch.empty((2000, 32, 128), dtype=torch.bfloat16, device=cuda_device)
    # first call on the device (the set-up) and module loading happen before measuring
    assert _noalloc_c_abi(small, out_s) == 0
    gq.check_device_error()
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    try:
        gq.set_num_workers(5000)
        for _ in range(2):
            assert _noalloc_c_abi(big, out_b) == 0, gq.load_library().gqa_last_error_string()
        gq.check_device_error()
        torch.cuda.synchronize()
    finally:
        gq.set_num_workers(0)
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, (free0, free1)


def test_noalloc_rejects_sizes_beyond_its_limit(cuda_device):
    # 4097 sequences x 4 kv heads = 16388 segments > 16384: refused before any launch
    lib = gq.load_library()
    p = ctypes.c_void_p(1 << 20)
    status = lib.gqa_paged_decode_attn_noalloc(p, p, p, p, p, p, 4097, 16, 4, 128, 16,
                                                ctypes.c_float(0.1), 4, 64, None)
    assert status == -2
    assert b"16384" in lib.gqa_last_error_string()
