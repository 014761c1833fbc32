"""GPU: kv_append through the C ABI is bit-exact against the oracle scatter."""
import numpy as np
import pytest
import torch

import gqa_decode_attention_04_b200 as gq
import oracle
from workloads import bf16_bits, make_custom_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("Hk,D,ps", [(1, 64, 16), (8, 128, 16), (2, 128, 64), (4, 64, 32), (3, 8, 5)])
def test_append_bit_exact(cuda_device, Hk, D, ps):
    seq_lens = [1, 16, 17, 40, 100, 5]
    inp = make_custom_inputs(seq_lens, Hk, Hk, D, ps, seed=D + ps, append=True, extra_pages=3)
    d = inp.to(cuda_device)
    gq.kv_append(d.k_new, d.v_new, d.k_pages, d.v_pages, d.block_table, d.positions)
    gq.check_device_error()
    k2, v2 = oracle.kv_append(bf16_bits(inp.k_pages), bf16_bits(inp.v_pages), bf16_bits(inp.k_new),
                              bf16_bits(inp.v_new), inp.block_table.numpy(), inp.positions.numpy())
    assert np.array_equal(bf16_bits(d.k_pages), k2)
    assert np.array_equal(bf16_bits(d.v_pages), v2)


def test_append_random_positions_and_many_seqs(cuda_device):
    g = torch.Generator().manual_seed(5)
    B, Hk, D, ps, MB = 300, 8, 128, 16, 9
    P = B * MB
    perm = torch.randperm(P, generator=g).to(torch.int32)
    bt = perm.view(B, MB).contiguous()
    pos = torch.randint(0, MB * ps, (B,), generator=g, dtype=torch.int32)
    kp = torch.randn(P, Hk, ps, D, generator=g).to(torch.bfloat16)
    vp = torch.randn(P, Hk, ps, D, generator=g).to(torch.bfloat16)
    kn = torch.randn(B, Hk, D, generator=g).to(torch.bfloat16)
    vn = torch.randn(B, Hk, D, generator=g).to(torch.bfloat16)
    dk, dv = kp.to(cuda_device), vp.to(cuda_device)
    gq.kv_append(kn.to(cuda_device), vn.to(cuda_device), dk, dv, bt.to(cuda_device), pos.to(cuda_device))
    gq.check_device_error()
    k2, v2 = oracle.kv_append(bf16_bits(kp), bf16_bits(vp), bf16_bits(kn), bf16_bits(vn), bt.numpy(), pos.numpy())
    assert np.array_equal(bf16_bits(dk), k2)
    assert np.array_equal(bf16_bits(dv), v2)


def test_append_out_of_range_is_skipped_and_reported(cuda_device):
    inp = make_custom_inputs([10, 20, 30], 2, 2, 64, 16, seed=3, append=True, extra_pages=1)
    pos = inp.positions.clone()
    bt = inp.block_table.clone()
    pos[0] = inp.max_blocks_per_seq * 16     # past the block table
    bt[2, 1] = inp.num_pages + 7             # page id out of the pool
    d = inp.to(cuda_device)
    before_k = d.k_pages.clone()
    gq.kv_append(d.k_new, d.v_new, d.k_pages, d.v_pages, bt.to(cuda_device), pos.to(cuda_device))
    with pytest.raises(gq.GQAError) as ei:
        gq.check_device_error()
    assert ei.value.status == -4
    # sequence 1 was appended, 0 and 2 were not; the error word is now clear
    k2, _ = oracle.kv_append(bf16_bits(inp.k_pages), bf16_bits(inp.v_pages), bf16_bits(inp.k_new[1:2]),
                             bf16_bits(inp.v_new[1:2]), inp.block_table[1:2].numpy(), inp.positions[1:2].numpy())
    assert np.array_equal(bf16_bits(d.k_pages), k2)
    assert not torch.equal(before_k, d.k_pages)
    gq.check_device_error()
