"""Checks that pin the fp64 oracle to facts outside itself.

Each check raises AssertionError on failure.  They look the oracle's functions
up through the module object at call time, so tests/test_oracle_mutants.py can
swap in a deliberately wrong function and confirm some check rejects it.

Sources of the facts (by page and section):
  * "TensorRT对Multi-Query Attention的专项优化支持": MHA has per-head K_i, V_i; MQA
    shares one K, V across all query heads (so MQA == MHA whose K/V heads are
    all copies of the shared one); the KV cache shrinks from h*d_k*s to d_k*s;
    the cache is paged.
  * tiny-llm "优化" page: GQA (num_kv_heads != num_heads); KV bytes
    2 x layers x kv_heads x head_dim x seq_len x 2 B; paged KV by block table
    with scatter/gather, diffed token by token against a contiguous cache;
    FlashDecoding for long contexts.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

import oracle.fp8_cache as F8
import oracle.paged_attention as PA

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "closed_forms.json")


def golden():
    with open(GOLDEN) as f:
        return json.load(f)


def _rand_bits(rng, shape, scale=1.0):
    return PA.f64_to_bf16_bits(rng.standard_normal(shape) * scale)


def _random_paged(rng, seq_lens, H, Hk, D, ps, extra_pages=2, scale=1.0):
    """Random contiguous per-sequence K/V, then scattered into a shuffled pool.

    Returns (q, k_pages, v_pages, block_table, contiguous K list, contiguous V list).
    The scatter here is written independently of the oracle's gather.
    """
    B = len(seq_lens)
    npg = [(L + ps - 1) // ps for L in seq_lens]
    P = sum(npg) + extra_pages
    MB = max(1, max(npg))
    perm = rng.permutation(P)
    bt = np.full((B, MB), -1, dtype=np.int64)
    off = 0
    for b, n in enumerate(npg):
        bt[b, :n] = perm[off:off + n]
        off += n
    q = _rand_bits(rng, (B, H, D))
    kp = np.full((P, Hk, ps, D), 0x7FC0, dtype=np.uint16)  # NaN everywhere unused
    vp = np.full((P, Hk, ps, D), 0x7FC0, dtype=np.uint16)
    Kc, Vc = [], []
    for b, L in enumerate(seq_lens):
        K = _rand_bits(rng, (Hk, L, D), scale)
        V = _rand_bits(rng, (Hk, L, D))
        Kc.append(K)
        Vc.append(V)
        for j in range(npg[b]):
            n = min(ps, L - j * ps)
            kp[bt[b, j], :, :n, :] = K[:, j * ps:j * ps + n, :]
            vp[bt[b, j], :, :n, :] = V[:, j * ps:j * ps + n, :]
    return q, kp, vp, bt, Kc, Vc


def _sdpa_reference(q_bits, Kc, Vc, H, Hk, scale):
    """torch scaled_dot_product_attention (CPU, float64) on contiguous K/V.

    K/V heads are expanded to query heads with repeat_interleave (query head h
    reads kv head h // G).  Empty contexts give zeros.
    """
    B, _, D = q_bits.shape
    G = H // Hk
    out = np.zeros((B, H, D))
    for b in range(B):
        L = Kc[b].shape[1]
        if L == 0:
            continue
        qt = torch.from_numpy(PA.bf16_bits_to_f64(q_bits[b])).reshape(1, H, 1, D)
        Kt = torch.from_numpy(PA.bf16_bits_to_f64(Kc[b])).repeat_interleave(G, dim=0)[None]
        Vt = torch.from_numpy(PA.bf16_bits_to_f64(Vc[b])).repeat_interleave(G, dim=0)[None]
        o = torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt, scale=scale)
        out[b] = o[0, :, 0, :].numpy()
    return out


# --------------------------------------------------------------------------- checks

def check_bf16_decode():
    """bf16 -> fp64 decoding on known bit patterns and against torch's cast."""
    bits = np.array([0x3F80, 0xC000, 0x0000, 0x8000, 0x3F81, 0x7F80, 0x0001, 0x4049],
                    dtype=np.uint16)
    want = [1.0, -2.0, 0.0, -0.0, 1.0 + 2.0 ** -7, math.inf, 2.0 ** -133, 3.140625]
    got = PA.bf16_bits_to_f64(bits)
    assert np.array_equal(got, np.array(want)), got
    x = np.random.default_rng(0).standard_normal(1000) * 100
    tb = torch.from_numpy(x).to(torch.bfloat16)
    assert np.array_equal(PA.f64_to_bf16_bits(x), tb.view(torch.int16).numpy().view(np.uint16))
    assert np.array_equal(PA.bf16_bits_to_f64(PA.f64_to_bf16_bits(x)), tb.to(torch.float64).numpy())


def check_closed_form_three_tokens():
    g = golden()["three_token_softmax"]
    q = PA.f64_to_bf16_bits(np.array(g["q"]))
    K = PA.bf16_bits_to_f64(PA.f64_to_bf16_bits(np.array(g["K"])))
    V = PA.bf16_bits_to_f64(PA.f64_to_bf16_bits(np.array(g["V"])))
    out = PA.attend_one_query(PA.bf16_bits_to_f64(q), K, V, g["scale"])
    assert np.allclose(out, g["expected_out"], rtol=0, atol=1e-13), out


def check_closed_form_paged():
    """The golden three tokens, stored through a reversed block table, single and MQA heads."""
    g = golden()["three_token_softmax"]
    p = golden()["paged_three_token"]
    ps, P = p["page_size"], p["num_pages"]
    K = PA.f64_to_bf16_bits(np.array(g["K"]))
    V = PA.f64_to_bf16_bits(np.array(g["V"]))
    kp = np.full((P, 1, ps, 2), 0x7FC0, dtype=np.uint16)
    vp = np.full((P, 1, ps, 2), 0x7FC0, dtype=np.uint16)
    bt = np.array([p["block_table"]])
    for t in range(3):
        kp[bt[0, t // ps], 0, t % ps] = K[t]
        vp[bt[0, t // ps], 0, t % ps] = V[t]
    # Three query heads sharing the single kv head (MQA): e0 -> golden answer,
    # 0 -> mean of V rows, -e0 -> weights 1/7, 2/7, 4/7.
    q = PA.f64_to_bf16_bits(np.array([[[1.0, 0.0], [0.0, 0.0], [-1.0, 0.0]]]))
    out = PA.paged_decode_attention(q, kp, vp, bt, np.array([3]), g["scale"])
    Vf = PA.bf16_bits_to_f64(V)
    assert np.allclose(out[0, 0], p["expected_out"], atol=1e-13), out
    assert np.allclose(out[0, 1], Vf.mean(axis=0), atol=1e-13), out
    assert np.allclose(out[0, 2], (Vf[0] + 2 * Vf[1] + 4 * Vf[2]) / 7, atol=1e-13), out


def check_single_token_returns_v():
    rng = np.random.default_rng(1)
    q, kp, vp, bt, Kc, Vc = _random_paged(rng, [1, 1, 1], 8, 2, 64, 16)
    out = PA.paged_decode_attention(q, kp, vp, bt, np.array([1, 1, 1]), 0.125)
    for b in range(3):
        for h in range(8):
            assert np.array_equal(out[b, h], PA.bf16_bits_to_f64(Vc[b][h // 4, 0])), (b, h)


def check_identical_v_rows():
    rng = np.random.default_rng(2)
    L = 37
    q, kp, vp, bt, Kc, Vc = _random_paged(rng, [L], 4, 1, 32, 16)
    row = _rand_bits(rng, (32,))
    for j in range((L + 15) // 16):
        n = min(16, L - 16 * j)
        vp[bt[0, j], 0, :n, :] = row
    out = PA.paged_decode_attention(q, kp, vp, bt, np.array([L]), 0.3)
    for h in range(4):
        assert np.allclose(out[0, h], PA.bf16_bits_to_f64(row), rtol=0, atol=1e-13)


def check_zero_query_gives_mean():
    rng = np.random.default_rng(3)
    L = 50
    q, kp, vp, bt, Kc, Vc = _random_paged(rng, [L], 2, 2, 16, 16)
    q[:] = 0
    out = PA.paged_decode_attention(q, kp, vp, bt, np.array([L]), 1.0)
    for h in range(2):
        assert np.allclose(out[0, h], PA.bf16_bits_to_f64(Vc[0][h]).mean(axis=0), atol=1e-14)


def _pure_python_attention(q_bits, kp, vp, bt, seq_lens, scale):
    """Triple loop, no numpy arithmetic: math.exp and float sums only."""
    B, H, D = q_bits.shape
    Hk, ps = kp.shape[1], kp.shape[2]
    G = H // Hk
    f = lambda bits: float(PA.bf16_bits_to_f64(np.uint16(bits)))  # noqa: E731
    out = [[[0.0] * D for _ in range(H)] for _ in range(B)]
    for b in range(B):
        L = int(seq_lens[b])
        for h in range(H):
            kvh = h // G
            qv = [f(q_bits[b, h, d]) for d in range(D)]
            scores = []
            for t in range(L):
                pg, sl = int(bt[b][t // ps]), t % ps
                scores.append(scale * sum(qv[d] * f(kp[pg, kvh, sl, d]) for d in range(D)))
            if L == 0:
                continue
            mx = max(scores)
            w = [math.exp(s - mx) for s in scores]
            tot = sum(w)
            for d in range(D):
                acc = 0.0
                for t in range(L):
                    pg, sl = int(bt[b][t // ps]), t % ps
                    acc += w[t] * f(vp[pg, kvh, sl, d])
                out[b][h][d] = acc / tot
    return np.array(out)


def check_brute_force_tiny():
    """Workload-1 shapes (MQA, D=64) and a small GQA case against pure Python."""
    rng = np.random.default_rng(4)
    for seq_lens, H, Hk, D, ps in [([17, 40], 4, 1, 16, 16), ([5, 0, 9], 6, 3, 8, 4)]:
        q, kp, vp, bt, Kc, Vc = _random_paged(rng, seq_lens, H, Hk, D, ps)
        sl = np.array(seq_lens)
        got = PA.paged_decode_attention(q, kp, vp, bt, sl, 1.0 / math.sqrt(D))
        want = _pure_python_attention(q, kp, vp, bt, sl, 1.0 / math.sqrt(D))
        assert np.allclose(got, want, rtol=0, atol=1e-12), np.abs(got - want).max()


def check_against_sdpa():
    """Paged oracle == torch SDPA (float64) on the contiguous K/V it was scattered from."""
    rng = np.random.default_rng(5)
    cases = [([17, 40], 4, 1, 64, 16, 0.125),
             ([3, 100, 33, 64], 8, 2, 32, 16, 0.2),
             ([70, 1, 129], 12, 4, 16, 32, 0.5),
             ([200], 96, 1, 8, 64, 0.35),
             ([31, 0, 16], 8, 8, 8, 16, 1.0)]
    for seq_lens, H, Hk, D, ps, scale in cases:
        q, kp, vp, bt, Kc, Vc = _random_paged(rng, seq_lens, H, Hk, D, ps)
        got = PA.paged_decode_attention(q, kp, vp, bt, np.array(seq_lens), scale)
        want = _sdpa_reference(q, Kc, Vc, H, Hk, scale)
        assert np.allclose(got, want, rtol=0, atol=1e-12), (seq_lens, np.abs(got - want).max())


def check_mqa_equals_mha_replicated():
    """MQA (one shared K/V head) equals MHA whose per-head K/V are copies of it."""
    rng = np.random.default_rng(6)
    H = 6
    q, kp, vp, bt, Kc, Vc = _random_paged(rng, [23, 48], H, 1, 16, 8)
    sl = np.array([23, 48])
    mqa = PA.paged_decode_attention(q, kp, vp, bt, sl, 0.25)
    mha = PA.paged_decode_attention(q, np.repeat(kp, H, axis=1), np.repeat(vp, H, axis=1),
                                    bt, sl, 0.25)
    assert np.array_equal(mqa, mha)
    # GQA with G=1 on the replicated cache also equals MHA per head.
    assert mqa.shape == (2, H, 16)


def check_page_permutation_invariance():
    """Relabelling pages (moving their data and the block table together) changes nothing."""
    rng = np.random.default_rng(7)
    sl = np.array([45, 16, 3])
    q, kp, vp, bt, Kc, Vc = _random_paged(rng, list(sl), 4, 2, 16, 16, extra_pages=3)
    base = PA.paged_decode_attention(q, kp, vp, bt, sl, 0.3)
    P = kp.shape[0]
    sigma = rng.permutation(P)  # new page id of old page p is sigma[p]
    kp2 = np.empty_like(kp)
    vp2 = np.empty_like(vp)
    kp2[sigma] = kp
    vp2[sigma] = vp
    bt2 = np.where(bt >= 0, sigma[np.maximum(bt, 0)], -1)
    perm_out = PA.paged_decode_attention(q, kp2, vp2, bt2, sl, 0.3)
    assert np.array_equal(base, perm_out)


def check_large_scores_stay_finite():
    """Scores near 1e3 (overflow for a naive exp) give the one-hot closed form."""
    K = np.zeros((4, 2))
    K[2, 0] = 1.0
    V = np.arange(8, dtype=np.float64).reshape(4, 2)
    out = PA.attend_one_query(np.array([1.0, 0.0]), K, V, 2000.0)
    assert np.all(np.isfinite(out))
    assert np.allclose(out, V[2], atol=1e-12)


def check_zero_length_context():
    rng = np.random.default_rng(8)
    q, kp, vp, bt, Kc, Vc = _random_paged(rng, [0, 5], 4, 2, 8, 16)
    out = PA.paged_decode_attention(q, kp, vp, bt, np.array([0, 5]), 0.5)
    assert np.array_equal(out[0], np.zeros((4, 8)))
    assert np.all(np.isfinite(out[1]))


def check_unused_slots_never_read():
    """NaN in unused pages and tail slots does not reach the output (the scatter
    in _random_paged leaves them NaN)."""
    rng = np.random.default_rng(9)
    sl = np.array([19, 1, 32])
    q, kp, vp, bt, Kc, Vc = _random_paged(rng, list(sl), 4, 2, 8, 16, extra_pages=4)
    out = PA.paged_decode_attention(q, kp, vp, bt, sl, 0.5)
    assert np.all(np.isfinite(out))


def check_rows_subset_matches_full():
    rng = np.random.default_rng(10)
    sl = np.array([30, 7, 64])
    q, kp, vp, bt, Kc, Vc = _random_paged(rng, list(sl), 8, 2, 16, 16)
    full = PA.paged_decode_attention(q, kp, vp, bt, sl, 0.4)
    rows = [(2, 7), (0, 0), (1, 3), (2, 0)]
    sub = PA.paged_decode_attention_rows(q, kp, vp, bt, sl, 0.4, rows)
    for i, (b, h) in enumerate(rows):
        assert np.array_equal(sub[i], full[b, h])


def check_kv_append():
    """After the scatter, the gather at positions[b] returns k_new[b] bit for bit;
    every other byte of both pools is unchanged."""
    rng = np.random.default_rng(11)
    sl = [5, 16, 33, 1]
    Hk, D, ps = 2, 8, 16
    q, kp, vp, bt, Kc, Vc = _random_paged(rng, sl, 4, Hk, D, ps, extra_pages=2)
    pos = np.array([4, 15, 32, 0])
    kn = _rand_bits(rng, (4, Hk, D))
    vn = _rand_bits(rng, (4, Hk, D))
    k2, v2 = PA.kv_append(kp, vp, kn, vn, bt, pos)
    changed_k = np.zeros(kp.shape[:3], dtype=bool)
    for b in range(4):
        for kvh in range(Hk):
            gk = PA.gather_sequence_kv(k2, bt[b], kvh, pos[b] + 1, ps)
            gv = PA.gather_sequence_kv(v2, bt[b], kvh, pos[b] + 1, ps)
            assert np.array_equal(gk[pos[b]], PA.bf16_bits_to_f64(kn[b, kvh]))
            assert np.array_equal(gv[pos[b]], PA.bf16_bits_to_f64(vn[b, kvh]))
        changed_k[bt[b, pos[b] // ps], :, pos[b] % ps] = True
    assert np.array_equal(k2[~changed_k], kp[~changed_k])
    assert np.array_equal(v2[~changed_k], vp[~changed_k])
    # inputs untouched
    assert not np.shares_memory(k2, kp)


def check_kv_cache_bytes():
    g = golden()
    for c in g["kv_cache_bytes"]["cases"]:
        assert PA.kv_cache_bytes(c["num_layers"], c["num_kv_heads"], c["head_dim"],
                                 c["seq_len"], c["batch"]) == c["bytes"], c
    # Bytes the gather touches equal the formula (one layer, bf16).
    rng = np.random.default_rng(12)
    sl = [37, 5]
    Hk, D, ps = 2, 8, 16
    q, kp, vp, bt, Kc, Vc = _random_paged(rng, sl, 4, Hk, D, ps)
    touched = 0
    for b, L in enumerate(sl):
        slots = {(int(bt[b][t // ps]), t % ps) for t in range(L)}
        touched += 2 * len(slots) * Hk * D * 2
    assert touched == sum(PA.kv_cache_bytes(1, Hk, D, L) for L in sl)
    r = g["mqa_cache_ratio"]
    assert PA.kv_cache_bytes(1, r["num_heads"], 128, 1000) // PA.kv_cache_bytes(1, 1, 128, 1000) == r["ratio"]


def check_lse_merge():
    """Splitting the context anywhere and merging (o_i, lse_i) gives the full result."""
    rng = np.random.default_rng(13)
    L, D = 97, 16
    qv = rng.standard_normal(D)
    K = rng.standard_normal((L, D)) * 3
    V = rng.standard_normal((L, D))
    full = PA.attend_one_query(qv, K, V, 0.7)
    for cuts in ([97], [1, 96], [50, 47], [10, 10, 10, 67], [1] * 97):
        pieces, s = [], 0
        for n in cuts:
            pieces.append(PA.partial_softmax_piece(qv, K[s:s + n], V[s:s + n], 0.7))
            s += n
        assert np.allclose(PA.merge_partial_pieces(pieces), full, atol=1e-13), cuts
    # The lse of the whole context is log(sum exp(s)) directly.
    _, lse = PA.partial_softmax_piece(qv, K, V, 0.7)
    s = 0.7 * (K @ qv)
    assert abs(lse - math.log(np.sum(np.exp(s)))) < 1e-11


def _random_multi(rng, seq_lens, Q, H, Hk, D, ps):
    """A paged cache as _random_paged plus a [B, Q, H, D] block of query tokens."""
    _, kp, vp, bt, Kc, Vc = _random_paged(rng, seq_lens, H, Hk, D, ps)
    return _rand_bits(rng, (len(seq_lens), Q, H, D)), kp, vp, bt, Kc, Vc


def check_multi_query_against_sdpa_causal():
    """Several query tokens per sequence against torch scaled_dot_product_attention
    (CPU, float64) with an explicit boolean mask: query token i (the token at position
    L - Q + i) may read key j iff j <= L - Q + i."""
    rng = np.random.default_rng(21)
    for sl, Q, H, Hk, D, ps in (([9, 40, 17], 4, 8, 2, 16, 16), ([33, 5], 3, 6, 1, 8, 4),
                                ([64, 7], 7, 4, 4, 32, 16)):
        q, kp, vp, bt, Kc, Vc = _random_multi(rng, sl, Q, H, Hk, D, ps)
        scale = 0.3
        got = PA.paged_multi_query_attention(q, kp, vp, bt, np.array(sl), scale)
        G = H // Hk
        for b, L in enumerate(sl):
            qt = torch.from_numpy(PA.bf16_bits_to_f64(q[b])).permute(1, 0, 2)[None]   # [1, H, Q, D]
            Kt = torch.from_numpy(PA.bf16_bits_to_f64(Kc[b])).repeat_interleave(G, dim=0)[None]
            Vt = torch.from_numpy(PA.bf16_bits_to_f64(Vc[b])).repeat_interleave(G, dim=0)[None]
            allowed = torch.arange(L)[None, :] <= (L - Q + torch.arange(Q))[:, None]
            ok = allowed.any(dim=1)
            o = torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt, attn_mask=allowed, scale=scale)
            want = o[0].permute(1, 0, 2).numpy()                                    # [Q, H, D]
            assert np.allclose(got[b][ok.numpy()], want[ok.numpy()], rtol=0, atol=1e-12), (sl, Q, b)
            assert np.all(got[b][~ok.numpy()] == 0.0)                                # empty windows


def check_multi_query_single_token_and_newest():
    """q_len = 1 is the decode; the newest query token sees the whole sequence, the
    oldest sees all but the q_len - 1 tokens after it."""
    rng = np.random.default_rng(22)
    sl, H, Hk, D, ps = [30, 3, 17], 4, 2, 16, 8
    q, kp, vp, bt, Kc, Vc = _random_multi(rng, sl, 1, H, Hk, D, ps)
    one = PA.paged_multi_query_attention(q, kp, vp, bt, np.array(sl), 0.5)[:, 0]
    assert np.array_equal(one, PA.paged_decode_attention(q[:, 0], kp, vp, bt, np.array(sl), 0.5))
    Q = 3
    q, kp, vp, bt, Kc, Vc = _random_multi(rng, sl, Q, H, Hk, D, ps)
    got = PA.paged_multi_query_attention(q, kp, vp, bt, np.array(sl), 0.5)
    assert np.array_equal(got[:, Q - 1], PA.paged_decode_attention(q[:, Q - 1], kp, vp, bt, np.array(sl), 0.5))
    shorter = np.maximum(np.array(sl) - (Q - 1), 0)
    assert np.array_equal(got[:, 0], PA.paged_decode_attention(q[:, 0], kp, vp, bt, shorter, 0.5))
    assert PA.multi_query_window(3, 3, 0) == 1 and PA.multi_query_window(2, 4, 0) == 0
    assert PA.multi_query_window(2, 4, 3) == 2 and PA.multi_query_window(0, 1, 0) == 0


def check_kv_append_multi():
    """Row i of sequence b lands at position positions[b] + i bit for bit (gathered
    back through the block table); every other byte is unchanged; q_len = 1 is kv_append."""
    rng = np.random.default_rng(23)
    sl = [20, 6, 33]
    Hk, D, ps, Q = 2, 8, 4, 3
    _, kp, vp, bt, Kc, Vc = _random_paged(rng, sl, 4, Hk, D, ps, extra_pages=2)
    pos = np.array([17, 3, 30])
    kn = _rand_bits(rng, (3, Q, Hk, D))
    vn = _rand_bits(rng, (3, Q, Hk, D))
    k2, v2 = PA.kv_append_multi(kp, vp, kn, vn, bt, pos)
    changed = np.zeros(kp.shape[:3], dtype=bool)
    for b in range(3):
        for kvh in range(Hk):
            gk = PA.gather_sequence_kv(k2, bt[b], kvh, pos[b] + Q, ps)
            gv = PA.gather_sequence_kv(v2, bt[b], kvh, pos[b] + Q, ps)
            for i in range(Q):
                assert np.array_equal(gk[pos[b] + i], PA.bf16_bits_to_f64(kn[b, i, kvh]))
                assert np.array_equal(gv[pos[b] + i], PA.bf16_bits_to_f64(vn[b, i, kvh]))
        for i in range(Q):
            t = pos[b] + i
            changed[bt[b, t // ps], :, t % ps] = True
    assert np.array_equal(k2[~changed], kp[~changed]) and np.array_equal(v2[~changed], vp[~changed])
    k1, v1 = PA.kv_append_multi(kp, vp, kn[:, :1], vn[:, :1], bt, pos)
    k0, v0 = PA.kv_append(kp, vp, kn[:, 0], vn[:, 0], bt, pos)
    assert np.array_equal(k1, k0) and np.array_equal(v1, v0)


# ------------------------------------------------------------- FP8 (e4m3) K/V cache

def check_e4m3_decode_matches_torch():
    """All 256 e4m3 codes decode to torch.float8_e4m3fn's values (a library routine);
    S.1111.111 is NaN, the largest value 448, the smallest subnormal 2^-9."""
    codes = np.arange(256, dtype=np.uint8)
    ours = F8.e4m3_bits_to_f64(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(ours[ok], ref[ok])
    assert np.nanmax(ours) == 448.0 and ours[1] == 2.0 ** -9 and np.isnan(ours[0x7F]) and np.isnan(ours[0xFF])


def check_e4m3_encode_rounding_and_saturation():
    """Nearest code with ties to the even mantissa, every finite code round-trips, values
    up to the overflow midpoint match torch's cast, larger ones saturate to 448."""
    codes = np.arange(256, dtype=np.uint8)
    vals = F8.e4m3_bits_to_f64(codes)
    fin = codes[~np.isnan(vals)]
    assert np.array_equal(F8.f64_to_e4m3_bits(F8.e4m3_bits_to_f64(fin)), fin)
    pos = np.sort(np.unique(vals[(vals > 0) & ~np.isnan(vals)]))
    for a, b in zip(pos[:-1], pos[1:]):
        mid = (a + b) / 2
        ca, cb = F8.f64_to_e4m3_bits([a, b])
        want = ca if (ca & 1) == 0 else cb      # the even mantissa wins a tie
        assert F8.f64_to_e4m3_bits([mid])[0] == want, (a, b)
        assert F8.f64_to_e4m3_bits([-mid])[0] == (want | 0x80)
    rng = np.random.default_rng(24)
    x = np.concatenate([rng.standard_normal(4000) * 40, rng.uniform(-463.9, 463.9, 2000),
                        rng.standard_normal(1000) * 2.0 ** -7])
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(F8.f64_to_e4m3_bits(x), ref)
    big = np.array([464.0, 500.0, 1e30, -464.0, -7e4])
    assert list(F8.f64_to_e4m3_bits(big)) == [0x7E, 0x7E, 0x7E, 0xFE, 0xFE]


def check_fp8_cache_attention_on_exact_values():
    """K/V on the e4m3 grid times power-of-two scales (exact in bf16): attention over the
    coded cache equals the bf16 oracle over the same values; scales differ per kv head
    and between K and V."""
    rng = np.random.default_rng(25)
    sl = [33, 7, 64]
    H, Hk, D, ps = 8, 2, 16, 16
    q, kp, vp, bt, _, _ = _random_paged(rng, sl, H, Hk, D, ps)
    ks = np.array([0.5, 2.0 ** -3])
    vs = np.array([4.0, 1.0])
    grid = F8.e4m3_bits_to_f64(np.arange(0, 0x7E, dtype=np.uint8))
    grid = np.concatenate([grid, -grid])
    kval = rng.choice(grid, size=kp.shape) * ks[None, :, None, None]
    vval = rng.choice(grid, size=vp.shape) * vs[None, :, None, None]
    kc, vc = F8.quantize_pages(kval, ks), F8.quantize_pages(vval, vs)
    assert np.array_equal(F8.dequantize_pages(kc, ks), kval)
    got = F8.paged_decode_attention_fp8(q, kc, vc, ks, vs, bt, np.array(sl), 0.3)
    kb, vb = PA.f64_to_bf16_bits(kval), PA.f64_to_bf16_bits(vval)
    assert np.array_equal(PA.bf16_bits_to_f64(kb), kval)
    want = PA.paged_decode_attention(q, kb, vb, bt, np.array(sl), 0.3)
    assert np.allclose(got, want, rtol=0, atol=1e-12)


def check_fp8_quantization_error_bound():
    """Writing a value costs at most half a step: relative 2^-4 in the normal range
    (3 mantissa bits), absolute 2^-10 * scale below the smallest normal."""
    rng = np.random.default_rng(26)
    s = np.array([0.25, 3.0])
    x = rng.standard_normal((4, 2, 16, 8)) * np.array([20.0, 300.0])[None, :, None, None]
    y = F8.dequantize_pages(F8.quantize_pages(x, s), s)
    r = np.abs(x) / s[None, :, None, None]
    normal = (r >= 2.0 ** -6) & (r <= 448.0)
    assert np.all(np.abs(y - x)[normal] <= 2.0 ** -4 * np.abs(x)[normal] + 1e-300)
    sub = r < 2.0 ** -6
    assert np.all(np.abs(y - x)[sub] <= 2.0 ** -10 * np.broadcast_to(s[None, :, None, None], x.shape)[sub])


def check_fp8_encode_of_the_fp32_quotient():
    """Writing bf16 values into the coded cache: the code of x / scale is decided on the
    IEEE fp32 quotient.  torch's fp32 division followed by its float8_e4m3fn cast (a
    library routine) gives the same codes below the overflow midpoint; 41 / fp32(6.56)
    is exactly 6.25 in fp32, a tie that goes to the even code 0x4C, while the fp64
    quotient lies just above the tie (code 0x4D); NaN gives a NaN code."""
    rng = np.random.default_rng(27)
    x = PA.bf16_bits_to_f64(_rand_bits(rng, 6000, scale=30.0))
    sc = rng.uniform(0.01, 4.0, 6000).astype(np.float32)
    got = F8.encode_fp32_quotient(x, sc)
    qt = torch.from_numpy(x.astype(np.float32)) / torch.from_numpy(sc)
    ok = qt.abs() < 464.0
    ref = qt[ok].to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got[ok.numpy()], ref)
    sat = (~ok).numpy()
    assert np.all((got[sat] & 0x7F) == 0x7E) and np.array_equal(got[sat] >> 7, (x[sat] < 0).astype(np.uint8))
    s656 = np.float32(6.56)
    assert F8.encode_fp32_quotient([41.0], s656)[0] == 0x4C
    assert F8.f64_to_e4m3_bits([41.0 / float(s656)])[0] == 0x4D
    c = F8.encode_fp32_quotient([np.nan, -0.0, 0.0], np.float32(1.0))
    assert (c[0] & 0x7F) == 0x7F and c[1] == 0x80 and c[2] == 0x00


def check_fp8_quantize_bf16_pool_per_kv_head():
    """A whole bf16 pool becomes codes with its own kv head's scale: every element's code
    is the fp32-quotient encode with scales[kvh] (kv heads on axis 1 of [P, Hk, ps, D]),
    and decoding gives the value back within half a step."""
    rng = np.random.default_rng(28)
    P_, Hk, ps, D = 5, 3, 16, 8
    mags = np.array([0.05, 1.0, 40.0])
    bits = PA.f64_to_bf16_bits(rng.standard_normal((P_, Hk, ps, D)) * mags[None, :, None, None])
    x = PA.bf16_bits_to_f64(bits)
    scales = (np.abs(x).max(axis=(0, 2, 3)) / 448.0).astype(np.float32)
    codes = F8.quantize_bf16_pages(bits, scales)
    assert codes.shape == bits.shape and codes.dtype == np.uint8
    for kvh in range(Hk):
        want = F8.encode_fp32_quotient(x[:, kvh], np.float32(scales[kvh]))
        assert np.array_equal(codes[:, kvh], want)
    y = F8.dequantize_pages(codes, scales.astype(np.float64))
    r = np.abs(x) / scales.astype(np.float64)[None, :, None, None]
    normal = r >= 2.0 ** -6
    assert np.all(np.abs(y - x)[normal] <= 2.0 ** -4 * np.abs(x)[normal] * (1 + 2.0 ** -20))
    assert np.abs(F8.e4m3_bits_to_f64(codes)).max() == 448.0  # the largest magnitude maps to the top code


def check_kv_append_fp8():
    """The coded append writes exactly the target slot of every sequence -- K with the K
    scales, V with the V scales -- and leaves every other byte of both pools unchanged."""
    rng = np.random.default_rng(29)
    B, Hk, D, ps, P_ = 3, 2, 8, 16, 7
    kc = rng.integers(0, 256, (P_, Hk, ps, D), dtype=np.uint8)
    vc = rng.integers(0, 256, (P_, Hk, ps, D), dtype=np.uint8)
    bt = np.array([[4, 1, -1], [0, -1, -1], [6, 2, 5]])
    pos = np.array([17, 3, 40])
    kn = _rand_bits(rng, (B, Hk, D), scale=3.0)
    vn = _rand_bits(rng, (B, Hk, D), scale=0.2)
    ks = np.array([0.05, 0.5], dtype=np.float32)     # no appended value saturates
    vs = np.array([0.004, 0.03], dtype=np.float32)
    k2, v2 = F8.kv_append_fp8(kc, vc, kn, vn, ks, vs, bt, pos)
    touched = np.zeros(kc.shape, dtype=bool)
    for b in range(B):
        page, slot = bt[b][pos[b] // ps], pos[b] % ps
        touched[page, :, slot, :] = True
        for kvh in range(Hk):
            assert np.array_equal(k2[page, kvh, slot], F8.encode_fp32_quotient(PA.bf16_bits_to_f64(kn[b, kvh]), ks[kvh]))
            assert np.array_equal(v2[page, kvh, slot], F8.encode_fp32_quotient(PA.bf16_bits_to_f64(vn[b, kvh]), vs[kvh]))
    assert np.array_equal(k2[~touched], kc[~touched]) and np.array_equal(v2[~touched], vc[~touched])
    # the appended rows read back within half a step of the bf16 values
    for b in range(B):
        page, slot = bt[b][pos[b] // ps], pos[b] % ps
        y = F8.e4m3_bits_to_f64(k2[page, :, slot, :]) * ks[:, None]
        xk = PA.bf16_bits_to_f64(kn[b])
        assert np.all(np.abs(y - xk) <= 2.0 ** -4 * np.abs(xk) * (1 + 2.0 ** -20) + 2.0 ** -10 * ks[:, None])


def check_fp8_rows_match_full():
    """The row-subset attention over a coded cache equals the full one on those rows."""
    rng = np.random.default_rng(30)
    sl = [40, 3, 70]
    H, Hk, D, ps = 6, 2, 8, 16
    q, kp, vp, bt, _, _ = _random_paged(rng, sl, H, Hk, D, ps)
    ks = np.array([0.01, 0.02], dtype=np.float32)
    vs = np.array([0.005, 0.04], dtype=np.float32)
    kc = F8.quantize_bf16_pages(kp, ks)
    vc = F8.quantize_bf16_pages(vp, vs)
    full = F8.paged_decode_attention_fp8(q, kc, vc, ks, vs, bt, np.array(sl), 0.4)
    rows = [(0, 5), (2, 0), (1, 3), (2, 4)]
    got = F8.paged_decode_attention_fp8_rows(q, kc, vc, ks, vs, bt, np.array(sl), 0.4, rows)
    assert np.allclose(got, np.stack([full[b, h] for b, h in rows]), rtol=0, atol=1e-13)


ALL_CHECKS = [
    check_bf16_decode,
    check_closed_form_three_tokens,
    check_closed_form_paged,
    check_single_token_returns_v,
    check_identical_v_rows,
    check_zero_query_gives_mean,
    check_brute_force_tiny,
    check_against_sdpa,
    check_mqa_equals_mha_replicated,
    check_page_permutation_invariance,
    check_large_scores_stay_finite,
    check_zero_length_context,
    check_unused_slots_never_read,
    check_rows_subset_matches_full,
    check_kv_append,
    check_kv_cache_bytes,
    check_lse_merge,
    check_multi_query_against_sdpa_causal,
    check_multi_query_single_token_and_newest,
    check_kv_append_multi,
    check_e4m3_decode_matches_torch,
    check_e4m3_encode_rounding_and_saturation,
    check_fp8_cache_attention_on_exact_values,
    check_fp8_quantization_error_bound,
    check_fp8_encode_of_the_fp32_quotient,
    check_fp8_quantize_bf16_pool_per_kv_head,
    check_kv_append_fp8,
    check_fp8_rows_match_full,
]
