"""GPU failure paths that fault nothing: device-side range checks and bounded waits.

Bad page ids and lengths are skipped by the kernels and reported through the
device error word.  The timeout path is exercised by arming the copy barriers
without issuing the copies, so every wait runs out after a short limit; the
kernel then returns and the host reads GQA_ERR_TIMEOUT.  No trap, assert or bad
address is involved.
"""
import numpy as np
import pytest
import torch

import gqa_decode_attention_04_b200 as gq
from parity import assert_close, gpu_f64, host_arrays, oracle_out
from workloads import make_custom_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _reset():
    gq.set_num_workers(0)
    gq.set_wait_limit_ns(10 ** 9, False)
    yield
    gq.set_wait_limit_ns(10 ** 9, False)
    gq.set_num_workers(0)


def test_bad_page_id_is_skipped_and_reported(cuda_device):
    inp = make_custom_inputs([100, 50], 8, 2, 128, 16, seed=21)
    bt = inp.block_table.clone()
    bt[0, 2] = -5
    d = inp.to(cuda_device)
    out = gq.paged_decode_attn(d.q, d.k_pages, d.v_pages, bt.to(cuda_device), d.seq_lens, scale=d.scale)
    with pytest.raises(gq.GQAError) as ei:
        gq.check_device_error()
    assert ei.value.status == -4
    assert torch.isfinite(out.float()).all()
    # the untouched sequence is still right
    want = oracle_out(host_arrays(inp))
    assert_close(gpu_f64(out)[1], want[1])


def test_seq_len_beyond_block_table_is_reported(cuda_device):
    inp = make_custom_inputs([40, 20], 4, 1, 64, 16, seed=22)
    sl = inp.seq_lens.clone()
    sl[1] = inp.max_blocks_per_seq * 16 + 1
    d = inp.to(cuda_device)
    gq.paged_decode_attn(d.q, d.k_pages, d.v_pages, d.block_table, sl.to(cuda_device), scale=d.scale)
    with pytest.raises(gq.GQAError) as ei:
        gq.check_device_error()
    assert ei.value.status == -4


def test_negative_seq_len_gives_zeros_and_is_reported(cuda_device):
    inp = make_custom_inputs([40, 20], 4, 1, 64, 16, seed=23)
    sl = inp.seq_lens.clone()
    sl[0] = -3
    d = inp.to(cuda_device)
    out = gq.paged_decode_attn(d.q, d.k_pages, d.v_pages, d.block_table, sl.to(cuda_device), scale=d.scale)
    with pytest.raises(gq.GQAError):
        gq.check_device_error()
    assert torch.count_nonzero(out[0]) == 0


def test_wait_timeout_returns_error_and_library_recovers(cuda_device):
    inp = make_custom_inputs([200, 64, 900], 8, 2, 128, 16, seed=24)
    d = inp.to(cuda_device)
    gq.set_num_workers(16)                          # several pieces per segment
    gq.set_wait_limit_ns(2_000_000, arm_without_copy=True)
    gq.paged_decode_attn(d.q, d.k_pages, d.v_pages, d.block_table, d.seq_lens, scale=d.scale)
    with pytest.raises(gq.GQAError) as ei:
        gq.check_device_error()
    assert ei.value.status == -5
    # normal operation afterwards: counters were reset, results match the oracle
    gq.set_wait_limit_ns(10 ** 9, False)
    out = gq.paged_decode_attn(d.q, d.k_pages, d.v_pages, d.block_table, d.seq_lens, scale=d.scale)
    gq.check_device_error()
    assert_close(gpu_f64(out), oracle_out(host_arrays(inp)))

