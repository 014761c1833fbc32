"""Oracle: plain, slow, obviously correct fp64 CPU decode attention over a paged KV cache.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module; it
exists so the CUDA kernels can be checked against the plain definition.  It
shares no code with the CUDA path: it receives raw bf16 bit patterns (uint16
numpy arrays), decodes them exactly to fp64, gathers each sequence's K/V rows
through the block table one token at a time, and evaluates softmax attention
directly from its definition.

What the method computes (sources, by page and section):
  * "TensorRT对Multi-Query Attention的专项优化支持" -- decoding one new token
    re-reads every cached Key/Value row of its sequence; MHA keeps one K/V
    projection per head (Q_i = X W_Q^i, K_i = X W_K^i, V_i = X W_V^i) while
    MQA shares one K = X W_K, V = X W_V across all query heads, shrinking the
    cache from h*d_k*s to d_k*s; the cache is kept in fixed-length pages
    ("Page-Based管理机制").  The plugin computes QK^T and AV (softmax attention).
  * tiny-llm "优化" page, section 3 -- GQA: num_kv_heads may differ from
    num_heads.  Section 2 -- per-sequence KV bytes are
    2 x num_layers x num_kv_heads x head_dim x max_seq_len x 2 bytes.
    Planned-optimisation table -- paged KV "strategy 1": a block table with
    scatter (append) / gather (attention), checked token by token against a
    contiguous cache; FlashDecoding is named for long-context decode.

Readings where the pages are silent (each is restated in the design notes):
  * head -> kv-head map: contiguous groups, kvh = h // (num_heads // num_kv_heads).
  * token t of sequence b lives in page block_table[b][t // page_size], slot
    t % page_size of kv head kvh: k_pages[page, kvh, slot, :].
  * a decode query sees all seq_len tokens (no causal or window mask).
  * seq_len == 0 yields an all-zero output row.
  * the split-KV combine (FlashDecoding) is not spelled out on the pages; the
    oracle states the plain log-sum-exp merge of softmax pieces.
  * several query tokens per sequence (the MQA plugin's entry point carries a
    query length, seq_q, beside seq_kv): they are the sequence's q_len newest
    tokens, and each attends to itself and every token before it, as the
    same tokens would one step at a time (speculative verification, chunked
    prefill over the cache).

Every function is pinned by tests in tests/test_oracle.py against closed forms,
a library routine (torch scaled_dot_product_attention in float64), brute-force
pure-Python loops and structural invariants.
"""
from __future__ import annotations

import math
from typing import Iterable, List, Sequence, Tuple

import numpy as np

__all__ = [
    "bf16_bits_to_f64",
    "f64_to_bf16_bits",
    "kv_head_of",
    "gather_sequence_kv",
    "attend_one_query",
    "paged_decode_attention",
    "paged_decode_attention_rows",
    "kv_append",
    "multi_query_window",
    "paged_multi_query_attention",
    "kv_append_multi",
    "partial_softmax_piece",
    "merge_partial_pieces",
    "kv_cache_bytes",
]


def bf16_bits_to_f64(bits) -> np.ndarray:
    """Exact value of bf16 bit patterns: bf16 is the top half of an IEEE fp32."""
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def f64_to_bf16_bits(x) -> np.ndarray:
    """Round fp64 values to bf16 (via fp32, round-to-nearest-even), return bits.

    Used only by tests that build inputs from chosen real values.
    """
    f = np.asarray(x, dtype=np.float64).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    is_nan = np.isnan(f)
    rounding_bias = ((u >> np.uint64(16)) & np.uint64(1)) + np.uint64(0x7FFF)
    r = ((u + rounding_bias) >> np.uint64(16)).astype(np.uint16)
    r = np.where(is_nan, np.uint16(0x7FC0), r)
    return r.astype(np.uint16)


def kv_head_of(h: int, num_heads: int, num_kv_heads: int) -> int:
    """KV head read by query head h: contiguous groups of num_heads/num_kv_heads."""
    if num_heads % num_kv_heads != 0:
        raise ValueError("num_heads must be a multiple of num_kv_heads")
    return h // (num_heads // num_kv_heads)


def gather_sequence_kv(pages_bits, block_table_row, kv_head: int, seq_len: int,
                       page_size: int) -> np.ndarray:
    """Rows [seq_len, head_dim] (fp64) of one kv head of one sequence.

    Token t is read from page block_table_row[t // page_size], slot
    t % page_size -- the gather half of the block-table scheme.
    """
    t = np.arange(seq_len, dtype=np.int64)
    page = np.asarray(block_table_row, dtype=np.int64)[t // page_size]
    slot = t % page_size
    return bf16_bits_to_f64(pages_bits[page, kv_head, slot, :])


def attend_one_query(q_row: np.ndarray, K: np.ndarray, V: np.ndarray,
                     scale: float) -> np.ndarray:
    """softmax(scale * K q) weighted sum of V rows, in fp64.

    The largest score is subtracted before exponentiation (an exact identity of
    softmax that keeps exp() finite).  An empty context gives zeros.
    """
    if K.shape[0] == 0:
        return np.zeros(V.shape[-1], dtype=np.float64)
    s = scale * (K @ q_row)
    w = np.exp(s - s.max())
    return (w @ V) / w.sum()


def paged_decode_attention(q_bits, k_pages_bits, v_pages_bits, block_table,
                           seq_lens, scale: float) -> np.ndarray:
    """Decode attention for every (sequence, query head): out [B, H, D] fp64.

    q_bits [B, H, D] uint16, k/v_pages_bits [P, Hk, ps, D] uint16,
    block_table [B, MB] int, seq_lens [B] int.
    """
    B, H, D = q_bits.shape
    Hk, ps = k_pages_bits.shape[1], k_pages_bits.shape[2]
    out = np.zeros((B, H, D), dtype=np.float64)
    q = bf16_bits_to_f64(q_bits)
    for b in range(B):
        L = int(seq_lens[b])
        for kvh in range(Hk):
            K = gather_sequence_kv(k_pages_bits, block_table[b], kvh, L, ps)
            V = gather_sequence_kv(v_pages_bits, block_table[b], kvh, L, ps)
            for h in range(H):
                if kv_head_of(h, H, Hk) == kvh:
                    out[b, h] = attend_one_query(q[b, h], K, V, scale)
    return out


def paged_decode_attention_rows(q_bits, k_pages_bits, v_pages_bits, block_table,
                                seq_lens, scale: float,
                                rows: Iterable[Tuple[int, int]]) -> np.ndarray:
    """Same definition, evaluated only for the listed (b, h) pairs: [len(rows), D]."""
    H = q_bits.shape[1]
    Hk, ps = k_pages_bits.shape[1], k_pages_bits.shape[2]
    rows = list(rows)
    out = np.zeros((len(rows), q_bits.shape[2]), dtype=np.float64)
    cache = {}
    for i, (b, h) in enumerate(rows):
        kvh = kv_head_of(h, H, Hk)
        key = (b, kvh)
        if key not in cache:
            L = int(seq_lens[b])
            cache.clear()
            cache[key] = (gather_sequence_kv(k_pages_bits, block_table[b], kvh, L, ps),
                          gather_sequence_kv(v_pages_bits, block_table[b], kvh, L, ps))
        K, V = cache[key]
        out[i] = attend_one_query(bf16_bits_to_f64(q_bits[b, h]), K, V, scale)
    return out


def kv_append(k_pages_bits, v_pages_bits, k_new_bits, v_new_bits, block_table,
              positions) -> Tuple[np.ndarray, np.ndarray]:
    """Scatter each sequence's new K/V row into its page slot; returns new pools.

    For every sequence b and kv head kvh, the row at token position
    positions[b] -- page block_table[b][pos // page_size], slot
    pos % page_size -- becomes k_new[b, kvh] (resp. v_new).  Bits are copied
    unchanged; every other byte of the pools is left as it was.
    """
    k = np.array(k_pages_bits, copy=True)
    v = np.array(v_pages_bits, copy=True)
    ps = k.shape[2]
    for b in range(k_new_bits.shape[0]):
        pos = int(positions[b])
        page = int(block_table[b][pos // ps])
        slot = pos % ps
        k[page, :, slot, :] = k_new_bits[b]
        v[page, :, slot, :] = v_new_bits[b]
    return k, v


def multi_query_window(seq_len: int, q_len: int, i: int) -> int:
    """Tokens that query token i of q_len sees when the sequence holds seq_len tokens
    (the q_len newest included): positions 0 .. seq_len - q_len + i, none if that is
    negative."""
    return max(0, min(seq_len, seq_len - q_len + 1 + i))


def paged_multi_query_attention(q_bits, k_pages_bits, v_pages_bits, block_table,
                                seq_lens, scale: float) -> np.ndarray:
    """Attention of q_len query tokens per sequence over the paged cache: [B, Q, H, D].

    q_bits [B, Q, H, D] uint16.  Query token i of sequence b is the token at
    position seq_lens[b] - Q + i; it attends to the first multi_query_window(...)
    tokens of its sequence.  With Q = 1 this is paged_decode_attention.
    """
    B, Q, H, D = q_bits.shape
    Hk, ps = k_pages_bits.shape[1], k_pages_bits.shape[2]
    out = np.zeros((B, Q, H, D), dtype=np.float64)
    q = bf16_bits_to_f64(q_bits)
    for b in range(B):
        L = int(seq_lens[b])
        for kvh in range(Hk):
            K = gather_sequence_kv(k_pages_bits, block_table[b], kvh, L, ps)
            V = gather_sequence_kv(v_pages_bits, block_table[b], kvh, L, ps)
            for i in range(Q):
                n = multi_query_window(L, Q, i)
                for h in range(H):
                    if kv_head_of(h, H, Hk) == kvh:
                        out[b, i, h] = attend_one_query(q[b, i, h], K[:n], V[:n], scale)
    return out


def kv_append_multi(k_pages_bits, v_pages_bits, k_new_bits, v_new_bits, block_table,
                    positions) -> Tuple[np.ndarray, np.ndarray]:
    """q_len new rows per sequence: k_new [B, Q, Hk, D]; row i of sequence b goes to
    token position positions[b] + i (same page/slot rule as kv_append)."""
    k = np.array(k_pages_bits, copy=True)
    v = np.array(v_pages_bits, copy=True)
    ps = k.shape[2]
    for b in range(k_new_bits.shape[0]):
        for i in range(k_new_bits.shape[1]):
            pos = int(positions[b]) + i
            page = int(block_table[b][pos // ps])
            k[page, :, pos % ps, :] = k_new_bits[b, i]
            v[page, :, pos % ps, :] = v_new_bits[b, i]
    return k, v


def partial_softmax_piece(q_row: np.ndarray, K: np.ndarray, V: np.ndarray,
                          scale: float) -> Tuple[np.ndarray, float]:
    """Attention over one contiguous piece of the context, with its log-sum-exp.

    Returns (o, lse): o is the piece's own normalised softmax average of V and
    lse = log(sum_t exp(s_t)) over the piece's scores s_t = scale * <q, K_t>.
    """
    s = scale * (K @ q_row)
    m = s.max()
    w = np.exp(s - m)
    return (w @ V) / w.sum(), float(m + math.log(w.sum()))


def merge_partial_pieces(pieces: Sequence[Tuple[np.ndarray, float]]) -> np.ndarray:
    """Combine per-piece (o_i, lse_i) into the attention over their union.

    Each piece's normaliser is exp(lse_i); the full softmax weights piece i by
    exp(lse_i) / sum_j exp(lse_j).  The largest lse is subtracted first.
    """
    lse = np.array([p[1] for p in pieces], dtype=np.float64)
    M = lse.max()
    w = np.exp(lse - M)
    acc = sum(wi * p[0] for wi, p in zip(w, pieces))
    return acc / w.sum()


def kv_cache_bytes(num_layers: int, num_kv_heads: int, head_dim: int,
                   seq_len: int, batch: int = 1, bytes_per_elem: int = 2) -> int:
    """KV-cache bytes: 2 (K and V) x layers x kv heads x head_dim x seq_len x batch x elem."""
    return 2 * num_layers * num_kv_heads * head_dim * seq_len * batch * bytes_per_elem
