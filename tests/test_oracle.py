"""CPU tests: the fp64 oracle against closed forms, a library routine, brute
force and structural invariants (see tests/oracle_pins.py for each fact's source)."""
import numpy as np
import pytest

import oracle_pins as P
from workloads import WORKLOADS, make_inputs, make_custom_inputs, bf16_bits
import oracle


@pytest.mark.parametrize("check", P.ALL_CHECKS, ids=lambda f: f.__name__)
def test_oracle_pin(check):
    check()


def test_workload1_oracle_matches_pure_python():
    """Workload 1 (tiny MQA) exactly as generated, against the pure-Python loops."""
    inp = make_inputs(1)
    args = (bf16_bits(inp.q), bf16_bits(inp.k_pages), bf16_bits(inp.v_pages),
            inp.block_table.numpy(), inp.seq_lens.numpy(), inp.scale)
    got = oracle.paged_decode_attention(*args)
    want = P._pure_python_attention(*args)
    assert np.all(np.isfinite(got))
    assert np.allclose(got, want, rtol=0, atol=1e-12)


def test_workload_recipes_shapes():
    inp = make_inputs(1)
    assert inp.seq_lens.tolist() == [17, 40]
    assert inp.num_pages == 8 and inp.max_blocks_per_seq == 3
    assert sorted(inp.block_table[inp.block_table >= 0].tolist()) == sorted(
        set(inp.block_table[inp.block_table >= 0].tolist()))
    assert abs(inp.scale - 0.125) < 1e-15
    inp2 = make_inputs(2, poison=False)
    L = inp2.seq_lens
    assert int(L.min()) >= 512 and int(L.max()) <= 4096
    need = int(((L + 15) // 16).sum())
    assert inp2.num_pages == int(np.ceil(1.25 * need))
    assert tuple(inp2.k_pages.shape) == (inp2.num_pages, 8, 16, 128)
    for idx, spec in WORKLOADS.items():
        assert spec.num_heads % spec.num_kv_heads == 0


def test_workload5_lengths_and_append_positions():
    # only the small pieces: lengths come from the CPU generator before any tensor
    inp = make_custom_inputs([1, 2, 17], 4, 2, 8, 16, append=True)
    assert inp.positions.tolist() == [0, 1, 16]
    import math
    import torch
    gen = torch.Generator().manual_seed(1005)
    u = torch.rand(256, generator=gen, dtype=torch.float64)
    lens = torch.round(torch.exp(u * math.log(32768.0))).clamp(1, 32768)
    assert lens.min() >= 1 and lens.max() <= 32768


def test_poisoned_slots_are_nan_and_unread():
    inp = make_custom_inputs([19, 3], 4, 2, 16, 16, extra_pages=2)
    kp = inp.k_pages.float()
    # last page of seq 0 holds 3 live tokens, slots 3.. are NaN
    last = int(inp.block_table[0, 1])
    assert kp[last, :, 3:, :].isnan().all() and not kp[last, :, :3, :].isnan().any()
    out = oracle.paged_decode_attention(bf16_bits(inp.q), bf16_bits(inp.k_pages),
                                        bf16_bits(inp.v_pages), inp.block_table.numpy(),
                                        inp.seq_lens.numpy(), inp.scale)
    assert np.all(np.isfinite(out))


def test_workload4_spikes_are_exact_powers_of_two():
    import torch
    inp = make_custom_inputs([400], 8, 1, 16, 16, spike_fraction=0.01, seed=3)
    base = make_custom_inputs([400], 8, 1, 16, 16, spike_fraction=0.0, seed=3)
    a = inp.k_pages.float()
    b = base.k_pages.float()
    live = ~b.isnan()
    ratio = a[live] / torch.where(b[live] == 0, torch.ones_like(b[live]), b[live])
    changed = (a[live] != b[live])
    assert torch.all((ratio[changed] == 4.0))
    # 1% of 400 positions = 4 tokens x 16 dims changed (zeros excepted)
    assert int(changed.sum()) <= 4 * 16
