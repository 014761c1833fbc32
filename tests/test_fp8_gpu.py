"""GPU parity of the 8-bit (e4m3) K/V cache through the C ABI against the oracle.

Writing (the whole-pool quantiser and the append) must be bit-exact: each code is the
oracle's encode of the fp32 quotient x / scale.  The decode over the coded pools is
compared with the oracle's attention over the cached values code * scale, at the same
tolerance as the bf16 cache (max abs 2e-2, mean abs 2e-3): the kernel widens codes to
fp16 exactly, rounds P to fp16 instead of bf16 and accumulates in fp32, so its rounding
steps are those of the bf16 kernel or finer.
"""
import numpy as np
import pytest
import torch

import gqa_decode_attention_04_b200 as gq
import oracle
from parity import assert_close, gpu_f64
from workloads import bf16_bits, make_custom_inputs, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _default_workers():
    gq.set_num_workers(0)
    yield
    gq.set_num_workers(0)


def _scales(pages: torch.Tensor) -> torch.Tensor:
    """One scale per kv head: the largest finite magnitude over the pool / 448."""
    a = torch.nan_to_num(pages.float(), nan=0.0, posinf=0.0, neginf=0.0).abs().amax(dim=(0, 2, 3))
    return (a / 448.0).clamp(min=1e-20).to(torch.float32).contiguous()


def _coded(d):
    """e4m3 pools of a device workload (quantised on the GPU) and their scales."""
    ks, vs = _scales(d.k_pages), _scales(d.v_pages)
    kc = torch.empty(d.k_pages.shape, dtype=torch.uint8, device=d.k_pages.device)
    vc = torch.empty_like(kc)
    gq.quantize_pages_fp8(d.k_pages, kc, ks)
    gq.quantize_pages_fp8(d.v_pages, vc, vs)
    return kc, vc, ks, vs


def _assert_codes(got: np.ndarray, src_bits: np.ndarray, scales: np.ndarray, what=""):
    """Codes equal the oracle's encode wherever the source is finite; NaN stays NaN."""
    want = oracle.quantize_bf16_pages(src_bits, scales)
    x = oracle.bf16_bits_to_f64(src_bits)
    fin = np.isfinite(x)
    bad = np.nonzero((got != want) & fin)
    assert bad[0].size == 0, f"{what}: {bad[0].size} codes differ, first at {tuple(a[0] for a in bad)}"
    assert np.all((got[~fin] & 0x7F) == 0x7F), f"{what}: a NaN source gave a non-NaN code"


def _oracle_fp8(q_bits, kc, vc, ks, vs, bt, sl, scale):
    return oracle.paged_decode_attention_fp8(q_bits, kc, vc, ks, vs, bt, sl, scale)


def test_quantize_pool_is_bit_exact(cuda_device):
    inp = make_custom_inputs([100, 37, 260], 8, 4, 128, 16, seed=51, extra_pages=3)
    d = inp.to(cuda_device)
    # kv heads of different magnitudes, and one scale small enough that values saturate
    mags = torch.tensor([1.0, 30.0, 1e-3, 5.0], device=cuda_device).view(1, 4, 1, 1)
    d.k_pages = (d.k_pages.float() * mags).to(torch.bfloat16)
    ks = _scales(d.k_pages)
    ks[3] = ks[3] / 8  # every value of kv head 3 above 56 * scale saturates
    kc = torch.empty(d.k_pages.shape, dtype=torch.uint8, device=cuda_device)
    gq.quantize_pages_fp8(d.k_pages, kc, ks)
    torch.cuda.synchronize()
    got = kc.cpu().numpy()
    _assert_codes(got, bf16_bits(d.k_pages), ks.cpu().numpy(), "pool")
    assert np.any((got[:, 3] & 0x7F) == 0x7E)  # saturated codes exist


@pytest.mark.parametrize("D", [64, 128])
def test_kv_append_fp8_is_bit_exact(cuda_device, D):
    inp = make_custom_inputs([1, 15, 16, 17, 300], 8, 2, D, 16, seed=52 + D, append=True, extra_pages=2)
    d = inp.to(cuda_device)
    kc, vc, ks, vs = _coded(d)
    k0, v0 = kc.cpu().numpy(), vc.cpu().numpy()
    gq.kv_append_fp8(d.k_new, d.v_new, kc, vc, ks, vs, d.block_table, d.positions)
    gq.check_device_error()
    k2, v2 = oracle.kv_append_fp8(k0, v0, bf16_bits(inp.k_new), bf16_bits(inp.v_new), ks.cpu().numpy(),
                                  vs.cpu().numpy(), inp.block_table.numpy(), inp.positions.numpy())
    assert np.array_equal(kc.cpu().numpy(), k2)
    assert np.array_equal(vc.cpu().numpy(), v2)


# (seq_lens, H, Hk, D, ps): several chunks and pages per sequence, ragged tails, group
# sizes 1 to 16 (9 to 16 take two 8-head segments), both head dims, page sizes 16 to 256.
SMALL_CASES = [
    ([17, 40], 4, 1, 64, 16),                      # workload-1 shapes
    ([1, 15, 16, 17, 31, 33, 100], 8, 2, 128, 16),  # G = 4
    ([300, 1, 77], 32, 8, 128, 16),                # G = 4, longer
    ([129, 64, 65], 16, 2, 128, 32),               # G = 8, ps = 32
    ([250, 7], 12, 1, 128, 64),                    # G = 12: two segments
    ([90, 200], 16, 1, 64, 128),                   # G = 16, D = 64, ps = 128
    ([5, 0, 33], 8, 8, 128, 16),                   # MHA (G = 1) and an empty sequence
    ([1000, 3, 500, 2048], 8, 1, 64, 16),          # D = 64 long
    ([700, 90], 8, 1, 128, 256),                   # ps = 256
    ([700, 47, 96], 16, 4, 128, 48),               # G = 4, ps = 48: blocks straddle pages
    ([1300, 81], 8, 1, 64, 80),                    # G = 8, D = 64, ps = 80
    # more than 16 query heads per kv head: the tcgen05 kernel with its converter warps
    ([70], 96, 1, 128, 64),                        # MQA, one partial block
    ([1000, 63, 129], 96, 1, 128, 64),             # MQA, several blocks, ragged tails
    ([500, 17], 64, 1, 64, 16),                    # D = 64, 16-row copies
    ([300, 1, 65], 128, 2, 128, 32),               # 64 per kv head, ps = 32
    ([200, 33], 128, 1, 128, 128),                 # full 128-row tile, ps = 128
    ([150], 200, 1, 64, 16),                       # two head tiles per kv head
    ([1500, 47], 96, 1, 128, 48),                  # ps = 48: blocks straddle pages
    ([800, 193], 72, 1, 128, 192),                 # ps = 192
    ([600, 33, 2], 17, 1, 128, 16),                # 17: the smallest group on tcgen05
    ([1000, 64, 7], 128, 4, 128, 16),              # 32 per kv head, four kv heads
]


@pytest.mark.parametrize("case", SMALL_CASES, ids=lambda c: f"L{len(c[0])}_H{c[1]}_Hk{c[2]}_D{c[3]}_ps{c[4]}")
def test_fp8_decode_parity(cuda_device, case):
    seq_lens, H, Hk, D, ps = case
    inp = make_custom_inputs(seq_lens, H, Hk, D, ps, seed=(sum(seq_lens) * 17 + H + D + ps) % 9973, extra_pages=3)
    d = inp.to(cuda_device)
    kc, vc, ks, vs = _coded(d)
    out = gq.paged_decode_attn_fp8(d.q, kc, vc, ks, vs, d.block_table, d.seq_lens, scale=d.scale)
    gq.check_device_error()
    kcn, vcn = kc.cpu().numpy(), vc.cpu().numpy()
    _assert_codes(kcn, bf16_bits(inp.k_pages), ks.cpu().numpy(), "K")
    want = _oracle_fp8(bf16_bits(inp.q), kcn, vcn, ks.cpu().numpy(), vs.cpu().numpy(), inp.block_table.numpy(),
                       inp.seq_lens.numpy(), inp.scale)
    assert_close(gpu_f64(out), want, what=str(case))
    for b, L in enumerate(seq_lens):
        if L == 0:
            assert torch.count_nonzero(out[b]) == 0


@pytest.mark.parametrize("heads", [(16, 4), (96, 1)], ids=["gqa", "mqa"])
@pytest.mark.parametrize("workers", [1, 3, 64, 1000])
def test_fp8_forced_splits(cuda_device, workers, heads):
    H, Hk = heads
    inp = make_custom_inputs([700, 33, 1, 2000, 129], H, Hk, 128, 16, seed=53, spike_fraction=0.01)
    d = inp.to(cuda_device)
    kc, vc, ks, vs = _coded(d)
    gq.set_num_workers(workers)
    out = gq.paged_decode_attn_fp8(d.q, kc, vc, ks, vs, d.block_table, d.seq_lens, scale=d.scale)
    gq.check_device_error()
    want = _oracle_fp8(bf16_bits(inp.q), kc.cpu().numpy(), vc.cpu().numpy(), ks.cpu().numpy(), vs.cpu().numpy(),
                       inp.block_table.numpy(), inp.seq_lens.numpy(), inp.scale)
    assert_close(gpu_f64(out), want, what=f"workers={workers}")


@pytest.mark.parametrize("workers", [1, 3])
def test_fp8_many_short_pieces_in_one_cta(cuda_device, workers):
    """One-block sequences in a row inside one CTA's range on the tcgen05 kernel: each
    piece's query tile is copied, converted to fp16 by the converter warp of its first
    block (the two take blocks in turns) and released after its S MMAs."""
    lens = [64, 1, 5, 64, 3, 130, 1, 1, 1, 200, 2, 64, 1, 9]
    inp = make_custom_inputs(lens, 96, 1, 128, 64, seed=57, extra_pages=2)
    d = inp.to(cuda_device)
    kc, vc, ks, vs = _coded(d)
    gq.set_num_workers(workers)
    out = gq.paged_decode_attn_fp8(d.q, kc, vc, ks, vs, d.block_table, d.seq_lens, scale=d.scale)
    gq.check_device_error()
    want = _oracle_fp8(bf16_bits(inp.q), kc.cpu().numpy(), vc.cpu().numpy(), ks.cpu().numpy(), vs.cpu().numpy(),
                       inp.block_table.numpy(), inp.seq_lens.numpy(), inp.scale)
    assert_close(gpu_f64(out), want, what=f"workers={workers}")


@pytest.mark.parametrize("layout", ["v_pool_below_k_pool", "one_pool_for_both"])
def test_fp8_pool_placement(cuda_device, layout):
    """Where the two code pools lie in memory does not change the result."""
    inp = make_custom_inputs([150, 47, 16, 300], 8, 2, 128, 16, seed=22)
    d = inp.to(cuda_device)
    kc, vc, ks, vs = _coded(d)
    if layout == "v_pool_below_k_pool":
        both = torch.stack([vc, kc])
        kp, vp = both[1], both[0]
        assert vp.data_ptr() < kp.data_ptr()
    else:
        kp = vp = kc
        vs = ks
    out = gq.paged_decode_attn_fp8(d.q, kp, vp, ks, vs, d.block_table, d.seq_lens, scale=d.scale)
    gq.check_device_error()
    kcn = kc.cpu().numpy()
    vcn = kcn if layout == "one_pool_for_both" else vc.cpu().numpy()
    want = _oracle_fp8(bf16_bits(inp.q), kcn, vcn, ks.cpu().numpy(), vs.cpu().numpy(), inp.block_table.numpy(),
                       inp.seq_lens.numpy(), inp.scale)
    assert_close(gpu_f64(out), want, what=layout)


def test_fp8_single_token_and_uniform_scores(cuda_device):
    """One cached token returns its V value; a zero scale averages V over the context."""
    inp = make_custom_inputs([1, 1, 300], 8, 2, 128, 16, seed=54)
    d = inp.to(cuda_device)
    kc, vc, ks, vs = _coded(d)
    for scale in (d.scale, 0.0):
        out = gq.paged_decode_attn_fp8(d.q, kc, vc, ks, vs, d.block_table, d.seq_lens, scale=scale)
        gq.check_device_error()
        want = _oracle_fp8(bf16_bits(inp.q), kc.cpu().numpy(), vc.cpu().numpy(), ks.cpu().numpy(), vs.cpu().numpy(),
                           inp.block_table.numpy(), inp.seq_lens.numpy(), scale)
        assert_close(gpu_f64(out), want, what=f"scale={scale}")
    # sequences 0 and 1 hold one token: out = its cached V value, up to the fp32 product
    # with the scale and the final bf16 rounding (half a bf16 step, 2^-9 relative)
    out = gq.paged_decode_attn_fp8(d.q, kc, vc, ks, vs, d.block_table, d.seq_lens, scale=d.scale)
    torch.cuda.synchronize()
    o = gpu_f64(out)
    vcn, vsn = vc.cpu().numpy(), vs.cpu().numpy()
    for b in range(2):
        page = int(inp.block_table[b, 0])
        v = oracle.e4m3_bits_to_f64(vcn[page, :, 0, :]) * vsn[:, None]  # [Hk, D]
        for h in range(8):
            assert np.all(np.abs(o[b, h] - v[h // 4]) <= 2.0 ** -8 * np.abs(v[h // 4]) + 1e-30), (b, h)


@pytest.mark.parametrize("case", [([1, 17, 300, 64, 2000], 32, 8, 128, 16), ([40, 9], 4, 1, 64, 16),
                                  ([700, 129], 96, 1, 128, 64)],
                         ids=["gqa", "tiny_mqa", "mqa"])
def test_fp8_decode_step(cuda_device, case):
    seq_lens, H, Hk, D, ps = case
    inp = make_custom_inputs(seq_lens, H, Hk, D, ps, seed=55, append=True, extra_pages=2)
    d = inp.to(cuda_device)
    kc, vc, ks, vs = _coded(d)
    k0, v0 = kc.cpu().numpy(), vc.cpu().numpy()
    out = gq.decode_step_fp8(d.q, d.k_new, d.v_new, kc, vc, ks, vs, d.block_table, d.positions, d.seq_lens,
                             scale=d.scale)
    gq.check_device_error()
    ksn, vsn = ks.cpu().numpy(), vs.cpu().numpy()
    k2, v2 = oracle.kv_append_fp8(k0, v0, bf16_bits(inp.k_new), bf16_bits(inp.v_new), ksn, vsn,
                                  inp.block_table.numpy(), inp.positions.numpy())
    assert np.array_equal(kc.cpu().numpy(), k2) and np.array_equal(vc.cpu().numpy(), v2)
    want = _oracle_fp8(bf16_bits(inp.q), k2, v2, ksn, vsn, inp.block_table.numpy(), inp.seq_lens.numpy(), inp.scale)
    assert_close(gpu_f64(out), want, what=str(case))


def test_fp8_rejects_missing_scales(cuda_device):
    inp = make_custom_inputs([40], 32, 1, 128, 16, seed=56)
    d = inp.to(cuda_device)
    kc, vc, ks, vs = _coded(d)
    lib = gq.load_library()
    st = lib.gqa_paged_decode_attn_fp8(d.q.data_ptr(), kc.data_ptr(), vc.data_ptr(), None, vs.data_ptr(),
                                       d.block_table.data_ptr(), d.seq_lens.data_ptr(), d.q.data_ptr(), 1, 32, 1,
                                       128, 16, 0.1, d.block_table.shape[1], inp.num_pages, None)
    assert st == -1


# ------------------------------------------------------------------ full-size workloads

def _sample_rows(inp, n_seq=6, seed=0):
    rng = np.random.default_rng(seed)
    B, H = inp.num_seqs, inp.num_heads
    L = inp.seq_lens.cpu().numpy()
    seqs = {int(np.argmax(L)), int(np.argmin(L))}
    seqs |= set(int(b) for b in rng.choice(B, size=min(n_seq, B), replace=False))
    return [(b, h) for b in sorted(seqs) for h in range(0, H, max(1, H // 16))]


def _sampled_codes_check(kc_dev, src_dev, scales_dev, n=1 << 20, seed=0):
    """Bit-exactness of a full-size quantised pool on n sampled elements."""
    g = torch.Generator(device=src_dev.device).manual_seed(seed)
    idx = torch.randint(0, src_dev.numel(), (n,), generator=g, device=src_dev.device)
    kvh = (idx // (src_dev.shape[2] * src_dev.shape[3])) % src_dev.shape[1]
    src = bf16_bits(src_dev.reshape(-1)[idx])
    got = kc_dev.reshape(-1)[idx].cpu().numpy()
    s = scales_dev[kvh].cpu().numpy().astype(np.float32)
    want = oracle.encode_fp32_quotient(oracle.bf16_bits_to_f64(src), s)
    fin = np.isfinite(oracle.bf16_bits_to_f64(src))
    assert np.array_equal(got[fin], want[fin])


@pytest.mark.slow
@pytest.mark.parametrize("index", [1, 2, 3, 4, 5])
def test_fp8_workload_parity(cuda_device, index):
    """Every workload over an e4m3 copy of its cache: workload 5 appends its new rows
    with the quantising append first; rows of 1 and 2 in full, sampled rows of 3, 4 and 5."""
    inp = make_inputs(index, device=cuda_device)
    kc, vc, ks, vs = _coded(inp)
    _sampled_codes_check(kc, inp.k_pages, ks, seed=index)
    _sampled_codes_check(vc, inp.v_pages, vs, seed=index + 10)
    if inp.has_append:
        gq.kv_append_fp8(inp.k_new, inp.v_new, kc, vc, ks, vs, inp.block_table, inp.positions)
    out = gq.paged_decode_attn_fp8(inp.q, kc, vc, ks, vs, inp.block_table, inp.seq_lens, scale=inp.scale)
    gq.check_device_error()
    q = bf16_bits(inp.q)
    kcn, vcn = kc.cpu().numpy(), vc.cpu().numpy()
    ksn, vsn = ks.cpu().numpy(), vs.cpu().numpy()
    bt, sl = inp.block_table.cpu().numpy(), inp.seq_lens.cpu().numpy()
    if inp.has_append:  # the appended slots hold the oracle's codes of the new rows
        pos = inp.positions.cpu().numpy()
        ps = inp.page_size
        for b in range(0, inp.num_seqs, 7):
            page, slot = bt[b][pos[b] // ps], pos[b] % ps
            want = oracle.encode_fp32_quotient(oracle.bf16_bits_to_f64(bf16_bits(inp.k_new[b])), ksn[:, None])
            assert np.array_equal(kcn[page, :, slot, :], want)
    if index in (1, 2):
        want = oracle.paged_decode_attention_fp8(q, kcn, vcn, ksn, vsn, bt, sl, inp.scale)
        mx, mean = assert_close(gpu_f64(out), want, what=inp.name)
    else:
        rows = _sample_rows(inp, n_seq=4 if index == 4 else 10)
        got = gpu_f64(out)[[r[0] for r in rows], [r[1] for r in rows]]
        want = oracle.paged_decode_attention_fp8_rows(q, kcn, vcn, ksn, vsn, bt, sl, inp.scale, rows)
        mx, mean = assert_close(got, want, what=inp.name)
    print(f"{inp.name} fp8: max abs {mx:.2e} mean abs {mean:.2e}")


@pytest.mark.parametrize("heads", [(8, 2), (96, 1)], ids=["mma_sync", "tcgen05"])
def test_fp8_every_sequence_empty_gives_zeros(cuda_device, heads):
    """No block of work at all over an e4m3 cache: the output rows are exact zeros."""
    H, Hk = heads
    inp = make_custom_inputs([0, 0, 0], H, Hk, 128, 16, seed=32, extra_pages=2)
    d = inp.to(cuda_device)
    kc, vc, ks, vs = _coded(d)
    out = torch.full((3, H, 128), float("nan"), dtype=torch.bfloat16, device=cuda_device)
    gq.paged_decode_attn_fp8(d.q, kc, vc, ks, vs, d.block_table, d.seq_lens, out=out, scale=d.scale)
    gq.check_device_error()
    assert torch.count_nonzero(out) == 0
