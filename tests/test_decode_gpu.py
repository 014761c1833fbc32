"""GPU parity: paged_decode_attn through the C ABI against the fp64 oracle."""
import numpy as np
import pytest
import torch

import gqa_decode_attention_04_b200 as gq
import oracle
from parity import assert_close, gpu_f64, host_arrays, oracle_out, oracle_rows
from workloads import bf16_bits, make_custom_inputs, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _default_workers():
    gq.set_num_workers(0)
    yield
    gq.set_num_workers(0)


def _run(inp, dev):
    d = inp.to(dev)
    out = gq.paged_decode_attn(d.q, d.k_pages, d.v_pages, d.block_table, d.seq_lens, scale=d.scale)
    gq.check_device_error()
    return d, out


# (seq_lens, H, Hk, D, ps): several chunks and pages per sequence, ragged tails,
# every group size the kernels specialise on, both head dims, all page-size classes.
SMALL_CASES = [
    ([17, 40], 4, 1, 64, 16),                      # workload-1 shapes
    ([1, 15, 16, 17, 31, 33, 100], 8, 2, 128, 16),  # G=4
    ([300, 1, 77], 32, 8, 128, 16),                # G=4, longer
    ([129, 64, 65], 16, 2, 128, 32),               # G=8, ps=32
    ([250, 7], 12, 1, 128, 64),                    # G=12 (16-row tile)
    ([90, 200], 16, 1, 64, 128),                   # G=16, D=64, ps=128
    ([40, 160], 32, 1, 128, 64),                   # G=32: two head tiles
    ([70], 96, 1, 128, 64),                        # G=96 (MQA, workload-3 shape)
    ([5, 0, 33], 8, 8, 128, 16),                   # MHA (G=1) and an empty sequence
    ([1000, 3, 500, 2048], 8, 1, 64, 16),          # D=64 long
    ([700, 47, 96], 16, 4, 128, 48),               # G=4, ps=48: blocks straddle pages
    ([1300, 81], 8, 1, 64, 80),                    # G=8, D=64, ps=80
    ([2000, 239, 240, 241], 12, 2, 128, 240),      # G=6, ps=240 (two 16-head windows of pages)
]


@pytest.mark.parametrize("case", SMALL_CASES, ids=lambda c: f"L{len(c[0])}_H{c[1]}_Hk{c[2]}_D{c[3]}_ps{c[4]}")
def test_small_parity(cuda_device, case):
    seq_lens, H, Hk, D, ps = case
    inp = make_custom_inputs(seq_lens, H, Hk, D, ps, seed=(sum(seq_lens) * 31 + H * 7 + D + ps) % 10007, extra_pages=3)
    d, out = _run(inp, cuda_device)
    assert_close(gpu_f64(out), oracle_out(host_arrays(inp)), what=str(case))
    # an empty sequence gives exact zeros
    for b, L in enumerate(seq_lens):
        if L == 0:
            assert torch.count_nonzero(out[b]) == 0


@pytest.mark.parametrize("workers", [1, 2, 3, 7, 64, 1000, 5000])
def test_forced_split_counts(cuda_device, workers):
    """Any number of split workers (1 .. more than chunks) gives the oracle's answer."""
    inp = make_custom_inputs([700, 33, 1, 2000, 129], 16, 4, 128, 16, seed=11)
    gq.set_num_workers(workers)
    d, out = _run(inp, cuda_device)
    assert_close(gpu_f64(out), oracle_out(host_arrays(inp)), what=f"workers={workers}")


@pytest.mark.parametrize("workers", [1, 5, 999])
def test_long_mqa_sequence_any_split(cuda_device, workers):
    """One 3000-token sequence of an MQA group of 8 on the mma.sync kernel, cut into 1,
    5 or up to 999 pieces (one per 64-token block), against the oracle."""
    inp = make_custom_inputs([3000, 17], 8, 1, 128, 16, seed=12)
    gq.set_num_workers(workers)
    d, out = _run(inp, cuda_device)
    assert_close(gpu_f64(out), oracle_out(host_arrays(inp)), what=f"workers={workers}")


def test_single_token_context_returns_v_exactly(cuda_device):
    inp = make_custom_inputs([1, 1, 1, 1], 16, 4, 128, 16, seed=13)
    d, out = _run(inp, cuda_device)
    G = 4
    for b in range(4):
        page = int(inp.block_table[b, 0])
        for h in range(16):
            assert torch.equal(out[b, h].cpu(), inp.v_pages[page, h // G, 0].cpu()), (b, h)


def test_identical_v_rows_return_that_row(cuda_device):
    inp = make_custom_inputs([333], 8, 2, 128, 16, seed=14)
    row = torch.randn(128).to(torch.bfloat16)
    vp = inp.v_pages.clone()
    live = ~vp.float().isnan()
    vp[live.all(dim=-1)] = row
    inp.v_pages = vp
    d, out = _run(inp, cuda_device)
    err = (out.float().cpu() - row.float()).abs().max().item()
    assert err <= 2e-2


def test_identity_and_shuffled_block_tables_agree(cuda_device):
    """The same token data through an identity and a shuffled block table."""
    seq_lens = [150, 47, 16]
    inp = make_custom_inputs(seq_lens, 8, 2, 128, 16, seed=15, poison=False)
    # rebuild the pool so pages are laid out in identity order
    bt = inp.block_table
    npg = [(L + 15) // 16 for L in seq_lens]
    order = torch.cat([bt[b, :n] for b, n in enumerate(npg)]).long()
    ident = inp.to("cpu")
    ident.k_pages = inp.k_pages[order].contiguous()
    ident.v_pages = inp.v_pages[order].contiguous()
    ident.num_pages = len(order)
    nbt = torch.full_like(bt, -1)
    off = 0
    for b, n in enumerate(npg):
        nbt[b, :n] = torch.arange(off, off + n, dtype=torch.int32)
        off += n
    ident.block_table = nbt
    _, o1 = _run(inp, cuda_device)
    _, o2 = _run(ident, cuda_device)
    assert torch.equal(o1, o2)


@pytest.mark.parametrize("layout", ["v_pool_below_k_pool", "one_pool_for_both"])
@pytest.mark.parametrize("heads", [(8, 2, 128), (16, 1, 64)], ids=["G4_D128", "G16_D64"])
def test_pool_placement(cuda_device, layout, heads):
    """Where the two pools lie in memory does not change the result: V below K in one
    buffer, and one pool passed as both K and V (attention over V = K)."""
    H, Hk, D = heads
    inp = make_custom_inputs([150, 47, 16, 300], H, Hk, D, 16, seed=21)
    d = inp.to(cuda_device)
    if layout == "v_pool_below_k_pool":
        both = torch.stack([d.v_pages, d.k_pages])
        kp, vp = both[1], both[0]
        assert vp.data_ptr() < kp.data_ptr()
    else:
        kp = vp = d.k_pages
        inp.v_pages = inp.k_pages
    out = gq.paged_decode_attn(d.q, kp, vp, d.block_table, d.seq_lens, scale=d.scale)
    gq.check_device_error()
    assert_close(gpu_f64(out), oracle_out(host_arrays(inp)), what=layout)


def test_nan_in_unread_slots_does_not_leak(cuda_device):
    inp = make_custom_inputs([17, 31, 2], 8, 2, 128, 16, seed=16, extra_pages=5)
    assert inp.k_pages.float().isnan().any()
    _, out = _run(inp, cuda_device)
    assert torch.isfinite(out.float()).all()


def test_large_scale_peaked_softmax(cuda_device):
    inp = make_custom_inputs([2000, 517], 16, 2, 128, 16, seed=17, spike_fraction=0.01, scale=0.5)
    _, out = _run(inp, cuda_device)
    assert_close(gpu_f64(out), oracle_out(host_arrays(inp)), what="peaked")


@pytest.mark.parametrize("heads", [(16, 2), (96, 1)], ids=["gqa", "mqa"])
@pytest.mark.parametrize("scale", [0.0, -0.3], ids=["zero", "negative"])
def test_zero_and_negative_scale(cuda_device, heads, scale):
    """Any finite scale: 0 gives the plain mean of V over each sequence; a negative scale
    favours the smallest scores.  Poisoned slots past each length must stay masked."""
    H, Hk = heads
    inp = make_custom_inputs([300, 45, 130], H, Hk, 128, 16, seed=19, extra_pages=3, scale=scale)
    _, out = _run(inp, cuda_device)
    assert_close(gpu_f64(out), oracle_out(host_arrays(inp)), what=f"scale={scale}")


@pytest.mark.parametrize("heads", [(8, 2), (96, 1)], ids=["gqa", "mqa"])
def test_out_only_8_byte_aligned(cuda_device, heads):
    """out may start on any 8-byte boundary (here 8 bytes past a 16-byte one)."""
    H, Hk = heads
    inp = make_custom_inputs([260, 70], H, Hk, 128, 16, seed=20)
    d = inp.to(cuda_device)
    n = 2 * H * 128
    buf = torch.full((n + 8,), float("nan"), dtype=torch.bfloat16, device=cuda_device)
    out = buf[4:4 + n].view(2, H, 128)
    assert out.data_ptr() % 16 == 8
    gq.paged_decode_attn(d.q, d.k_pages, d.v_pages, d.block_table, d.seq_lens, out=out, scale=d.scale)
    torch.cuda.synchronize()
    assert_close(gpu_f64(out), oracle_out(host_arrays(inp)), what="misaligned out")
    assert torch.isnan(buf[:4].float()).all() and torch.isnan(buf[4 + n:].float()).all()


def test_out_buffer_is_written_in_place(cuda_device):
    inp = make_custom_inputs([40, 9], 4, 1, 64, 16, seed=18)
    d = inp.to(cuda_device)
    out = torch.full((2, 4, 64), float("nan"), dtype=torch.bfloat16, device=cuda_device)
    r = gq.paged_decode_attn(d.q, d.k_pages, d.v_pages, d.block_table, d.seq_lens, out=out, scale=d.scale)
    assert r.data_ptr() == out.data_ptr()
    assert_close(gpu_f64(out), oracle_out(host_arrays(inp)))


# ------------------------------------------------------------------ full-size workloads

def _sample_rows(inp, n_seq=6, seed=0):
    rng = np.random.default_rng(seed)
    B, H = inp.num_seqs, inp.num_heads
    L = inp.seq_lens.cpu().numpy()
    seqs = {int(np.argmax(L)), int(np.argmin(L))}
    seqs |= set(int(b) for b in rng.choice(B, size=min(n_seq, B), replace=False))
    return [(b, h) for b in sorted(seqs) for h in range(H)]


@pytest.mark.slow
@pytest.mark.parametrize("index", [1, 2, 3])
def test_workload_full_parity(cuda_device, index):
    """Workloads 1-3 at full size, every output row, default launch configuration."""
    inp = make_inputs(index)
    d, out = _run(inp, cuda_device)
    mx, mean = assert_close(gpu_f64(out), oracle_out(host_arrays(inp)), what=inp.name)
    print(f"{inp.name}: max abs {mx:.2e} mean abs {mean:.2e}")


@pytest.mark.slow
def test_workload4_long_context_sampled(cuda_device):
    """131072-token contexts with a peaked softmax: every head of sampled sequences."""
    inp = make_inputs(4)
    d, out = _run(inp, cuda_device)
    rows = [(b, h) for b in range(4) for h in range(0, 64, 3)]
    got = gpu_f64(out)[[r[0] for r in rows], [r[1] for r in rows]]
    assert_close(got, oracle_rows(host_arrays(inp), rows), what="long_context")


@pytest.mark.slow
def test_workload5_append_then_attend(cuda_device):
    """Continuous batch: kv_append of each sequence's new token, then decode attention."""
    inp = make_inputs(5)
    d = inp.to(cuda_device)
    gq.kv_append(d.k_new, d.v_new, d.k_pages, d.v_pages, d.block_table, d.positions)
    out = gq.paged_decode_attn(d.q, d.k_pages, d.v_pages, d.block_table, d.seq_lens, scale=d.scale)
    gq.check_device_error()
    h = host_arrays(inp)
    k2, v2 = oracle.kv_append(h["k"], h["v"], bf16_bits(inp.k_new), bf16_bits(inp.v_new),
                              h["bt"], inp.positions.numpy())
    # the scatter is bit-exact over the whole pool (NaN patterns included)
    assert np.array_equal(bf16_bits(d.k_pages), k2)
    assert np.array_equal(bf16_bits(d.v_pages), v2)
    h["k"], h["v"] = k2, v2
    rows = _sample_rows(inp, n_seq=10)
    got = gpu_f64(out)[[r[0] for r in rows], [r[1] for r in rows]]
    assert_close(got, oracle_rows(h, rows), what="continuous_batch")


# ------------------------------------------------------------------ fused decode step

@pytest.mark.parametrize("case", [([1, 17, 300, 64, 2000], 32, 8, 128, 16),
                                  ([40, 9], 4, 1, 64, 16),
                                  ([700, 129], 96, 1, 128, 64)],
                         ids=["gqa", "tiny_mqa", "mqa"])
def test_decode_step_equals_append_then_attend(cuda_device, case):
    seq_lens, H, Hk, D, ps = case
    inp = make_custom_inputs(seq_lens, H, Hk, D, ps, seed=31, append=True, extra_pages=2)
    d = inp.to(cuda_device)
    out = gq.decode_step(d.q, d.k_new, d.v_new, d.k_pages, d.v_pages, d.block_table, d.positions,
                         d.seq_lens, scale=d.scale)
    gq.check_device_error()
    h = host_arrays(inp)
    k2, v2 = oracle.kv_append(h["k"], h["v"], bf16_bits(inp.k_new), bf16_bits(inp.v_new),
                              h["bt"], inp.positions.numpy())
    assert np.array_equal(bf16_bits(d.k_pages), k2)
    assert np.array_equal(bf16_bits(d.v_pages), v2)
    h["k"], h["v"] = k2, v2
    assert_close(gpu_f64(out), oracle_out(h), what=str(case))


def test_consecutive_steps_rewrite_what_the_previous_decode_read(cuda_device):
    """Back-to-back steps append different rows at the same positions: each decode must
    see its own step's rows, never a later or earlier step's."""
    inp = make_custom_inputs([500, 33, 1], 16, 4, 128, 16, seed=32, append=True)
    d = inp.to(cuda_device)
    g = torch.Generator().manual_seed(5)
    outs, rows = [], []
    for step in range(4):
        kn = torch.randn(d.k_new.shape, generator=g).to(torch.bfloat16)
        vn = torch.randn(d.v_new.shape, generator=g).to(torch.bfloat16) * (step + 1)
        rows.append((kn, vn))
        outs.append(gq.decode_step(d.q, kn.to(cuda_device), vn.to(cuda_device), d.k_pages, d.v_pages,
                                   d.block_table, d.positions, d.seq_lens, scale=d.scale))
    gq.check_device_error()
    h = host_arrays(inp)
    for step, (kn, vn) in enumerate(rows):
        k2, v2 = oracle.kv_append(h["k"], h["v"], bf16_bits(kn), bf16_bits(vn), h["bt"], inp.positions.numpy())
        assert_close(gpu_f64(outs[step]), oracle_out(dict(h, k=k2, v=v2)), what=f"step {step}")


def _append_then_attend_reference(inp, positions, kn, vn):
    h = host_arrays(inp)
    k2, v2 = oracle.kv_append(h["k"], h["v"], bf16_bits(kn), bf16_bits(vn), h["bt"], positions.numpy())
    return k2, v2, oracle_out(dict(h, k=k2, v=v2))


@pytest.mark.parametrize("heads", [(16, 4), (96, 1), (200, 1)], ids=["gqa", "mqa", "two_head_tiles"])
def test_decode_step_positions_outside_attended_range(cuda_device, heads):
    """A row appended beyond seq_lens[b] is written to the pool but not attended; one at
    seq_lens[b] - 1 is attended (the one-launch step writes both kinds)."""
    H, Hk = heads
    # No slot is reserved for the append here (append=False), so attended slots all hold data.
    inp = make_custom_inputs([300, 70, 129], H, Hk, 64, 16, seed=33, extra_pages=6)
    g = torch.Generator().manual_seed(33)
    kn = torch.randn((3, Hk, 64), generator=g).to(torch.bfloat16)
    vn = torch.randn((3, Hk, 64), generator=g).to(torch.bfloat16)
    # 303 and 140 lie past the attended lengths but inside each sequence's last page
    positions = torch.tensor([303, 69, 140], dtype=torch.int32)
    d = inp.to(cuda_device)
    out = gq.decode_step(d.q, kn.to(cuda_device), vn.to(cuda_device), d.k_pages, d.v_pages, d.block_table,
                         positions.to(cuda_device), d.seq_lens, scale=d.scale)
    gq.check_device_error()
    k2, v2, want = _append_then_attend_reference(inp, positions, kn, vn)
    assert np.array_equal(bf16_bits(d.k_pages), k2)
    assert np.array_equal(bf16_bits(d.v_pages), v2)
    assert_close(gpu_f64(out), want, what=str(heads))


@pytest.mark.parametrize("workers", [1, 3, 57, 400])
@pytest.mark.parametrize("heads", [(16, 2), (200, 1)], ids=["gqa", "two_head_tiles"])
def test_decode_step_under_forced_splits(cuda_device, heads, workers):
    """The block holding the appended row may sit anywhere in a CTA's range (first, last,
    alone); with two head tiles two CTAs write the same row before reading it."""
    H, Hk = heads
    inp = make_custom_inputs([1100, 513, 64, 1], H, Hk, 128, 16, seed=34 + workers, append=True)
    d = inp.to(cuda_device)
    gq.set_num_workers(workers)
    try:
        out = gq.decode_step(d.q, d.k_new, d.v_new, d.k_pages, d.v_pages, d.block_table, d.positions,
                             d.seq_lens, scale=d.scale)
        gq.check_device_error()
    finally:
        gq.set_num_workers(0)
    k2, v2, want = _append_then_attend_reference(inp, inp.positions, inp.k_new, inp.v_new)
    assert np.array_equal(bf16_bits(d.k_pages), k2)
    assert np.array_equal(bf16_bits(d.v_pages), v2)
    assert_close(gpu_f64(out), want, what=f"workers={workers}")


def test_decode_step_bad_position_skips_row_and_reports(cuda_device):
    inp = make_custom_inputs([200, 40], 8, 2, 128, 16, seed=35, append=True, max_blocks_per_seq=16)
    positions = inp.positions.clone()
    positions[1] = 16 * 16 + 3  # beyond max_blocks_per_seq * page_size
    d = inp.to(cuda_device)
    gq.decode_step(d.q, d.k_new, d.v_new, d.k_pages, d.v_pages, d.block_table, positions.to(cuda_device),
                   d.seq_lens, scale=d.scale)
    with pytest.raises(gq.GQAError) as ei:
        gq.check_device_error()
    assert ei.value.status == -4
    # only sequence 0's row is appended; every other byte of the pools is unchanged
    h = host_arrays(inp)
    k2, v2 = oracle.kv_append(h["k"], h["v"], bf16_bits(inp.k_new[:1]), bf16_bits(inp.v_new[:1]), h["bt"][:1],
                              positions[:1].numpy())
    assert np.array_equal(bf16_bits(d.k_pages), k2)
    assert np.array_equal(bf16_bits(d.v_pages), v2)


def test_decode_step_replays_in_a_cuda_graph(cuda_device):
    """After a first call, the step is captured once and replayed with new buffer contents
    (new rows, positions and lengths advanced by one each step)."""
    B, H, Hk, D, ps = 3, 32, 8, 128, 16
    # lengths leave room in each sequence's last page for three more appended tokens
    inp = make_custom_inputs([200, 27, 70], H, Hk, D, ps, seed=36, append=True, extra_pages=8,
                             max_blocks_per_seq=24)
    d = inp.to(cuda_device)
    out = torch.empty((B, H, D), dtype=torch.bfloat16, device=cuda_device)
    kn = d.k_new.clone()
    vn = d.v_new.clone()
    pos = d.positions.clone()
    lens = d.seq_lens.clone()
    s = torch.cuda.Stream(cuda_device)
    with torch.cuda.stream(s):
        gq.decode_step(d.q, kn, vn, d.k_pages, d.v_pages, d.block_table, pos, lens, out=out, scale=d.scale)
    s.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        gq.decode_step(d.q, kn, vn, d.k_pages, d.v_pages, d.block_table, pos, lens, out=out, scale=d.scale)
    g = torch.Generator().manual_seed(7)
    h = host_arrays(inp)
    h["k"], h["v"] = oracle.kv_append(h["k"], h["v"], bf16_bits(inp.k_new), bf16_bits(inp.v_new), h["bt"],
                                     inp.positions.numpy())
    assert_close(gpu_f64(out), oracle_out(h), what="first call")
    hpos = inp.positions.clone()
    hlens = inp.seq_lens.clone()
    for step in range(3):
        hpos += 1
        hlens += 1
        new_k = torch.randn((B, Hk, D), generator=g).to(torch.bfloat16)
        new_v = torch.randn((B, Hk, D), generator=g).to(torch.bfloat16)
        kn.copy_(new_k)
        vn.copy_(new_v)
        pos.copy_(hpos)
        lens.copy_(hlens)
        graph.replay()
        torch.cuda.synchronize()
        gq.check_device_error()
        h["k"], h["v"] = oracle.kv_append(h["k"], h["v"], bf16_bits(new_k), bf16_bits(new_v), h["bt"],
                                         hpos.numpy())
        h["sl"] = hlens.numpy()
        assert_close(gpu_f64(out), oracle_out(h), what=f"replay {step}")
    del graph


# ------------------------------------------------------------------ large groups (tcgen05 path)

TC_CASES = [
    ([70], 96, 1, 128, 64),                   # MQA, one partial block
    ([1000, 63, 129], 96, 1, 128, 64),        # MQA, several blocks, ragged tails
    ([500, 17], 64, 1, 64, 16),               # head_dim 64, page 16 (16-row copies)
    ([300, 1, 65], 128, 2, 128, 32),          # G = 64 per kv head, page 32
    ([200, 33], 128, 1, 128, 128),            # G = 128 (full tile), page 128
    ([150], 200, 1, 64, 16),                  # G = 200: two head tiles per kv head
    ([257, 2, 31], 48, 1, 128, 16),           # G = 48 (tile partly padding)
    ([400, 5], 64, 1, 64, 64),                # head_dim 64, page 64 (one box per block)
    ([700, 90], 96, 1, 128, 256),             # page 256: four blocks per page
    ([2100, 700, 3], 64, 1, 128, 16),         # block-table rows spanning several windows
    ([1500, 47], 96, 1, 128, 48),             # page 48: blocks straddle pages (16-row copies)
    ([900, 130], 64, 1, 128, 80),             # page 80
    ([1100, 96], 40, 1, 64, 96),              # page 96 (32-row copies), head_dim 64
    ([800, 193], 72, 1, 128, 192),            # page 192: 64-row copies, three blocks per page
    ([600, 33, 2], 17, 1, 128, 16),           # G = 17: smallest group on tcgen05
    ([450, 129], 48, 2, 64, 32),              # G = 24, head_dim 64
    ([1000, 64, 7], 128, 4, 128, 16),         # G = 32, four kv heads
]


@pytest.mark.parametrize("case", TC_CASES, ids=lambda c: f"L{len(c[0])}_H{c[1]}_Hk{c[2]}_D{c[3]}_ps{c[4]}")
def test_large_group_parity(cuda_device, case):
    seq_lens, H, Hk, D, ps = case
    inp = make_custom_inputs(seq_lens, H, Hk, D, ps, seed=sum(seq_lens) + H, extra_pages=2)
    d, out = _run(inp, cuda_device)
    assert_close(gpu_f64(out), oracle_out(host_arrays(inp)), what=str(case))


@pytest.mark.parametrize("workers", [1, 2, 5, 40, 500])
def test_large_group_forced_splits(cuda_device, workers):
    """Pieces of one MQA segment spread over many CTAs and merged by log-sum-exp."""
    inp = make_custom_inputs([3000, 640], 96, 1, 128, 64, seed=44, spike_fraction=0.01)
    gq.set_num_workers(workers)
    d, out = _run(inp, cuda_device)
    assert_close(gpu_f64(out), oracle_out(host_arrays(inp)), what=f"workers={workers}")


@pytest.mark.parametrize("workers", [1, 2, 3])
def test_large_group_many_short_pieces_in_one_cta(cuda_device, workers):
    """Many one-block sequences in a row inside one CTA's range on the tcgen05 kernel: the
    query tile is reloaded for every piece, by the two producers in turns, and each load
    must wait for the previous piece's S MMAs."""
    lens = [64, 1, 5, 64, 3, 130, 1, 1, 1, 200, 2, 64, 1, 9]
    inp = make_custom_inputs(lens, 96, 1, 128, 64, seed=45, extra_pages=2)
    gq.set_num_workers(workers)
    d, out = _run(inp, cuda_device)
    assert_close(gpu_f64(out), oracle_out(host_arrays(inp)), what=f"workers={workers}")


@pytest.mark.parametrize("heads", [(8, 2), (96, 1)], ids=["mma_sync", "tcgen05"])
@pytest.mark.parametrize("workers", [0, 5])
def test_every_sequence_empty_gives_zeros(cuda_device, heads, workers):
    """No block of work at all: every CTA returns after zeroing its share of the empty
    sequences' rows (out starts as NaN, so a row left unwritten fails)."""
    H, Hk = heads
    inp = make_custom_inputs([0, 0, 0], H, Hk, 128, 16, seed=31, extra_pages=2)
    d = inp.to(cuda_device)
    out = torch.full((3, H, 128), float("nan"), dtype=torch.bfloat16, device=cuda_device)
    gq.set_num_workers(workers)
    gq.paged_decode_attn(d.q, d.k_pages, d.v_pages, d.block_table, d.seq_lens, out=out, scale=d.scale)
    gq.check_device_error()
    assert torch.count_nonzero(out) == 0
