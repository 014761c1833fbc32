"""Several query tokens per sequence on the GPU (gqa_paged_multi_query_attn,
gqa_kv_append_multi, gqa_multi_query_step) against the oracle: query token i of sequence
b attends to positions 0 .. seq_lens[b] - q_len + i.  Cases cover every kernel shape the
q_len x group rows select (mma.sync for up to 16 rows, tcgen05 for 17..128), both head
dims, page sizes 16..64, windows that end inside a sub-chunk, a block or a page, empty
windows (seq_len < q_len), forced split counts (pieces merged across CTAs) and poisoned
unused slots."""
import numpy as np
import pytest
import torch

import gqa_decode_attention_04_b200 as gq
import oracle
from parity import assert_close, gpu_f64
from workloads import bf16_bits, make_custom_inputs

pytestmark = pytest.mark.gpu


def _case(lens, Q, H, Hk, D, ps, seed):
    inp = make_custom_inputs(lens, H, Hk, D, ps, seed=seed, extra_pages=2)
    gen = torch.Generator().manual_seed(seed + 99)
    q = torch.randn(len(lens), Q, H, D, generator=gen).to(torch.bfloat16)
    return inp, q


def _oracle(inp, q):
    return oracle.paged_multi_query_attention(bf16_bits(q), bf16_bits(inp.k_pages), bf16_bits(inp.v_pages),
                                              inp.block_table.numpy(), inp.seq_lens.numpy(), inp.scale)


CASES = [
    # lens, q_len, H, Hk, D, ps           rows per kv head (kernel)
    ([5, 37, 64, 130, 1, 16], 4, 8, 2, 128, 16),    # 16: mma.sync, two n-tiles
    ([200, 17, 3, 66], 2, 4, 1, 64, 16),            # 8: mma.sync, one n-tile, D = 64
    ([77, 300, 4], 5, 4, 4, 128, 16),               # MHA: 5 rows, mma.sync
    ([300, 65, 48, 7], 8, 4, 1, 128, 32),           # 32: tcgen05
    ([150, 90, 2], 3, 24, 4, 128, 16),              # 18: tcgen05
    ([1000, 20], 2, 16, 1, 128, 64),                # 32, page size 64
    ([129, 63, 64, 65], 7, 4, 1, 64, 16),           # 28, D = 64: windows around block edges
    ([700, 130, 9], 16, 8, 1, 128, 16),             # 128 rows: a full tcgen05 tile
    ([513, 64, 3], 4, 96, 4, 128, 64),              # 96 rows (4 tokens x 24 heads)
    ([260, 31], 6, 16, 2, 64, 32),                  # 48 rows, D = 64
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"L{len(c[0])}_Q{c[1]}_H{c[2]}_Hk{c[3]}_D{c[4]}_ps{c[5]}")
def test_multi_query_parity(cuda_device, case):
    lens, Q, H, Hk, D, ps = case
    inp, q = _case(lens, Q, H, Hk, D, ps, seed=len(lens) * 31 + Q)
    d = inp.to(cuda_device)
    out = gq.paged_multi_query_attn(q.to(cuda_device), d.k_pages, d.v_pages, d.block_table, d.seq_lens,
                                    scale=inp.scale)
    gq.check_device_error()
    assert_close(gpu_f64(out), _oracle(inp, q), what=str(case))


@pytest.mark.parametrize("rows", [8, 16, 64])
@pytest.mark.parametrize("workers", [1, 3, 57, 400])
def test_multi_query_forced_splits(cuda_device, workers, rows):
    """8 rows per kv head run on the one-n-tile mma.sync kernel, whose CTAs finish a cut
    final piece by merging the segment's other pieces directly; 16 on two n-tiles; 64 on
    tcgen05 with the merge kernel."""
    lens, Q, H, Hk, D, ps = [900, 333, 64, 2], rows // 4, 8, 2, 128, 16
    inp, q = _case(lens, Q, H, Hk, D, ps, seed=5)
    d = inp.to(cuda_device)
    try:
        gq.set_num_workers(workers)
        out = gq.paged_multi_query_attn(q.to(cuda_device), d.k_pages, d.v_pages, d.block_table, d.seq_lens,
                                        scale=inp.scale)
        gq.check_device_error()
    finally:
        gq.set_num_workers(0)
    assert_close(gpu_f64(out), _oracle(inp, q), what=f"workers={workers}")


def test_single_query_token_equals_the_decode(cuda_device):
    inp, q = _case([40, 700, 3], 1, 8, 2, 128, 16, seed=9)
    d = inp.to(cuda_device)
    a = gq.paged_multi_query_attn(q.to(cuda_device), d.k_pages, d.v_pages, d.block_table, d.seq_lens,
                                  scale=inp.scale)
    b = gq.paged_decode_attn(q[:, 0].contiguous().to(cuda_device), d.k_pages, d.v_pages, d.block_table,
                             d.seq_lens, scale=inp.scale)
    gq.check_device_error()
    assert torch.equal(a[:, 0], b)


def test_newest_token_equals_a_decode_over_the_whole_sequence(cuda_device):
    """The last query token sees every token: the same numbers as a one-token decode
    within the tolerance, and the first sees q_len - 1 fewer."""
    Q = 4
    inp, q = _case([90, 513, 16], Q, 8, 2, 128, 16, seed=12)
    d = inp.to(cuda_device)
    out = gq.paged_multi_query_attn(q.to(cuda_device), d.k_pages, d.v_pages, d.block_table, d.seq_lens,
                                    scale=inp.scale)
    last = gq.paged_decode_attn(q[:, Q - 1].contiguous().to(cuda_device), d.k_pages, d.v_pages,
                                d.block_table, d.seq_lens, scale=inp.scale)
    first = gq.paged_decode_attn(q[:, 0].contiguous().to(cuda_device), d.k_pages, d.v_pages, d.block_table,
                                 (d.seq_lens - (Q - 1)).contiguous(), scale=inp.scale)
    gq.check_device_error()
    assert_close(gpu_f64(out[:, Q - 1]), gpu_f64(last), max_abs=1e-2, mean_abs=1e-3, what="newest")
    assert_close(gpu_f64(out[:, 0]), gpu_f64(first), max_abs=1e-2, mean_abs=1e-3, what="oldest")


def test_kv_append_multi_is_bit_exact(cuda_device):
    Q = 3
    inp = make_custom_inputs([20, 6, 33], 4, 2, 128, 16, seed=14, extra_pages=3)
    gen = torch.Generator().manual_seed(15)
    kn = torch.randn(3, Q, 2, 128, generator=gen).to(torch.bfloat16)
    vn = torch.randn(3, Q, 2, 128, generator=gen).to(torch.bfloat16)
    pos = (inp.seq_lens - Q).to(torch.int32)
    d = inp.to(cuda_device)
    gq.kv_append_multi(kn.to(cuda_device), vn.to(cuda_device), d.k_pages, d.v_pages, d.block_table,
                       pos.to(cuda_device))
    gq.check_device_error()
    k2, v2 = oracle.kv_append_multi(bf16_bits(inp.k_pages), bf16_bits(inp.v_pages), bf16_bits(kn),
                                    bf16_bits(vn), inp.block_table.numpy(), pos.numpy())
    assert np.array_equal(bf16_bits(d.k_pages), k2) and np.array_equal(bf16_bits(d.v_pages), v2)


@pytest.mark.parametrize("Q,H,Hk", [(4, 8, 2), (8, 4, 1), (2, 32, 2), (16, 8, 1)])
def test_multi_query_step_equals_append_then_attend(cuda_device, Q, H, Hk):
    lens = [70, 300, 5, 129]
    inp = make_custom_inputs(lens, H, Hk, 128, 16, seed=17 + Q, extra_pages=2)
    gen = torch.Generator().manual_seed(18 + Q)
    B = len(lens)
    q = torch.randn(B, Q, H, 128, generator=gen).to(torch.bfloat16)
    kn = torch.randn(B, Q, Hk, 128, generator=gen).to(torch.bfloat16)
    vn = torch.randn(B, Q, Hk, 128, generator=gen).to(torch.bfloat16)
    pos = (inp.seq_lens - Q).clamp(min=0).to(torch.int32)
    d = inp.to(cuda_device)
    out = gq.multi_query_step(q.to(cuda_device), kn.to(cuda_device), vn.to(cuda_device), d.k_pages,
                              d.v_pages, d.block_table, pos.to(cuda_device), d.seq_lens, scale=inp.scale)
    gq.check_device_error()
    k2, v2 = oracle.kv_append_multi(bf16_bits(inp.k_pages), bf16_bits(inp.v_pages), bf16_bits(kn),
                                    bf16_bits(vn), inp.block_table.numpy(), pos.numpy())
    assert np.array_equal(bf16_bits(d.k_pages), k2) and np.array_equal(bf16_bits(d.v_pages), v2)
    want = oracle.paged_multi_query_attention(bf16_bits(q), k2, v2, inp.block_table.numpy(),
                                              inp.seq_lens.numpy(), inp.scale)
    assert_close(gpu_f64(out), want, what=f"Q={Q} H={H} Hk={Hk}")


def test_too_many_rows_is_refused_and_launches_nothing(cuda_device):
    inp, q = _case([40], 33, 4, 1, 128, 16, seed=3)
    d = inp.to(cuda_device)
    n0 = gq.launch_count()
    with pytest.raises(gq.GQAError) as e:
        gq.paged_multi_query_attn(q.to(cuda_device), d.k_pages, d.v_pages, d.block_table, d.seq_lens)
    assert e.value.status == -2 and gq.launch_count() == n0


@pytest.mark.parametrize("Q,H,Hk", [(4, 8, 2), (8, 32, 8)])
def test_multi_query_step_replays_in_a_cuda_graph(cuda_device, Q, H, Hk):
    """After a first call the multi-token step is captured once and replayed with new
    buffer contents: new draft rows, positions and lengths advanced by q_len each time
    (rows per kv head: 16 on the mma.sync kernel, 32 on the tcgen05 kernel)."""
    D, ps = 128, 16
    lens0 = [200, 27, 70]
    B = len(lens0)
    inp = make_custom_inputs(lens0, H, Hk, D, ps, seed=40 + Q, extra_pages=12, max_blocks_per_seq=24)
    d = inp.to(cuda_device)
    gen = torch.Generator().manual_seed(41 + Q)
    q = torch.randn(B, Q, H, D, generator=gen).to(torch.bfloat16).to(cuda_device)
    kn = torch.empty(B, Q, Hk, D, dtype=torch.bfloat16, device=cuda_device)
    vn = torch.empty_like(kn)
    pos = torch.empty(B, dtype=torch.int32, device=cuda_device)
    lens = torch.empty(B, dtype=torch.int32, device=cuda_device)
    out = torch.empty(B, Q, H, D, dtype=torch.bfloat16, device=cuda_device)
    # each sequence's block-table row gets the pages its four steps of q_len tokens need
    steps = 4
    bt = torch.full((B, 24), -1, dtype=torch.int32)
    used = set(int(x) for x in inp.block_table.flatten().tolist() if x >= 0)
    free = [p for p in range(inp.num_pages) if p not in used]
    for b in range(B):
        row = [int(x) for x in inp.block_table[b].tolist() if x >= 0]
        need = -(-(lens0[b] + steps * Q) // ps) - len(row)
        assert need <= len(free)
        row += free[:need]
        free = free[need:]
        bt[b, :len(row)] = torch.tensor(row, dtype=torch.int32)
    bt_d = bt.to(cuda_device)
    h_k, h_v = bf16_bits(inp.k_pages), bf16_bits(inp.v_pages)
    cur = torch.tensor(lens0, dtype=torch.int32)
    s = torch.cuda.Stream(cuda_device)
    graph = None
    for step in range(steps):
        new_k = torch.randn(B, Q, Hk, D, generator=gen).to(torch.bfloat16)
        new_v = torch.randn(B, Q, Hk, D, generator=gen).to(torch.bfloat16)
        hpos = cur.clone()
        cur = cur + Q
        kn.copy_(new_k)
        vn.copy_(new_v)
        pos.copy_(hpos)
        lens.copy_(cur)
        if step == 0:  # first call, then capture
            with torch.cuda.stream(s):
                gq.multi_query_step(q, kn, vn, d.k_pages, d.v_pages, bt_d, pos, lens, out=out, scale=d.scale)
            s.synchronize()
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=s):
                gq.multi_query_step(q, kn, vn, d.k_pages, d.v_pages, bt_d, pos, lens, out=out, scale=d.scale)
            # capture records the launch only; the first call's effect is what the state holds
        else:
            graph.replay()
        torch.cuda.synchronize()
        gq.check_device_error()
        h_k, h_v = oracle.kv_append_multi(h_k, h_v, bf16_bits(new_k), bf16_bits(new_v), bt.numpy(), hpos.numpy())
        want = oracle.paged_multi_query_attention(bf16_bits(q), h_k, h_v, bt.numpy(), cur.numpy(), d.scale)
        assert np.array_equal(bf16_bits(d.k_pages), h_k), f"step {step}"
        assert_close(gpu_f64(out), want, what=f"step {step}")
    del graph
