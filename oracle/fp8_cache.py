"""Oracle: an FP8 (e4m3) K/V cache -- exact decode and encode, and decode attention over it.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module.  It is the
plain statement of what a decode over an 8-bit cache computes, written before any kernel
for it, so that kernels can be checked against it.

What the pages say (by page and section):
  * "TensorRT对Multi-Query Attention的专项优化支持": in 8-bit mode Q, K and V are calibrated
    separately (per-tensor scaling), because one scale shared by K and V loses precision
    to their different dynamic ranges.
  * TensorRT-LLM hands-on guide (precision section): FP16/BF16 as the baseline, INT8 or
    FP8 for more throughput where precision holds.
  * recsys page (feature table): FP8 quantisation for its attention.
Readings where the pages are silent (restated in the design notes):
  * the 8-bit format is e4m3 in its finite form: 1 sign, 4 exponent (bias 7) and 3
    mantissa bits; exponent 0 holds the subnormals m/8 * 2^-6; there are no infinities
    and S.1111.111 is NaN, so the largest value is 1.75 * 2^8 = 448;
  * K and V each carry one float scale per kv head (a per-tensor scale is the case of
    equal scales); a cached value is decode(code) * scale;
  * writing a value x stores the code nearest to x / scale, ties to the even code, and
    magnitudes beyond the format saturate to +-448 (not NaN);
  * when bf16 values are written into the cache (kv_append, or converting a whole bf16
    pool), the quotient x / scale is formed in IEEE fp32 (round to nearest even) and the
    code is the one nearest to that fp32 quotient: a quantised code is an integer decided
    by floating point, so the oracle takes that decision in the precision the kernels
    use.  A NaN input gives a NaN code.
"""
from __future__ import annotations

import math

import numpy as np

from .paged_attention import attend_one_query, bf16_bits_to_f64, kv_head_of

__all__ = [
    "E4M3_MAX",
    "e4m3_bits_to_f64",
    "f64_to_e4m3_bits",
    "quantize_pages",
    "dequantize_pages",
    "paged_decode_attention_fp8",
    "paged_decode_attention_fp8_rows",
    "encode_fp32_quotient",
    "quantize_bf16_pages",
    "kv_append_fp8",
]

E4M3_MAX = 448.0


def e4m3_bits_to_f64(bits) -> np.ndarray:
    """Exact value of e4m3 codes (uint8): sign, 4-bit exponent with bias 7, 3-bit mantissa."""
    b = np.asarray(bits, dtype=np.uint8).astype(np.int64)
    sign = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = b & 0x7
    normal = sign * (1.0 + m / 8.0) * np.exp2(e - 7.0)
    sub = sign * (m / 8.0) * 2.0 ** -6
    out = np.where(e == 0, sub, normal)
    return np.where((e == 15) & (m == 7), np.nan, out)


def _encode_one(x: float) -> int:
    if math.isnan(x):
        return 0x7F
    s = 0x80 if math.copysign(1.0, x) < 0 else 0
    a = abs(x)
    if a >= 464.0:  # at or beyond the midpoint above 448: saturate
        return s | 0x7E
    if a < 2.0 ** -6:  # subnormal range: steps of 2^-9 (m = 8 is the smallest normal)
        m = int(np.rint(a / 2.0 ** -9))
        return s | m
    f, E = math.frexp(a)  # a = f * 2^E, f in [0.5, 1)
    e = E - 1
    m = int(np.rint((2.0 * f - 1.0) * 8.0))  # mantissa to 3 bits, half to even
    if m == 8:
        e, m = e + 1, 0
    return s | ((e + 7) << 3) | m


def f64_to_e4m3_bits(x) -> np.ndarray:
    """Nearest e4m3 code to each value (ties to the even code), saturating to +-448."""
    a = np.asarray(x, dtype=np.float64)
    return np.vectorize(_encode_one, otypes=[np.uint8])(a) if a.size else a.astype(np.uint8)


def quantize_pages(pages_f64, scales) -> np.ndarray:
    """Codes of a page pool [P, Hk, ps, D] with one scale per kv head: code(x / scale)."""
    p = np.asarray(pages_f64, dtype=np.float64)
    return f64_to_e4m3_bits(p / np.asarray(scales, dtype=np.float64)[None, :, None, None])


def dequantize_pages(codes, scales) -> np.ndarray:
    """Values of a coded pool: decode(code) * scale of the row's kv head."""
    return e4m3_bits_to_f64(codes) * np.asarray(scales, dtype=np.float64)[None, :, None, None]


def paged_decode_attention_fp8(q_bits, k_codes, v_codes, k_scales, v_scales, block_table,
                               seq_lens, scale: float) -> np.ndarray:
    """Decode attention [B, H, D] over an e4m3 cache: the plain attention of each query head
    over its sequence's cached values decode(code) * scale (q in bf16 bits)."""
    B, H, D = q_bits.shape
    Hk, ps = k_codes.shape[1], k_codes.shape[2]
    K = dequantize_pages(k_codes, k_scales)
    V = dequantize_pages(v_codes, v_scales)
    q = bf16_bits_to_f64(q_bits)
    out = np.zeros((B, H, D), dtype=np.float64)
    for b in range(B):
        L = int(seq_lens[b])
        t = np.arange(L, dtype=np.int64)
        page = np.asarray(block_table[b], dtype=np.int64)[t // ps]
        slot = t % ps
        for h in range(H):
            kvh = kv_head_of(h, H, Hk)
            out[b, h] = attend_one_query(q[b, h], K[page, kvh, slot, :], V[page, kvh, slot, :], scale)
    return out


def paged_decode_attention_fp8_rows(q_bits, k_codes, v_codes, k_scales, v_scales, block_table,
                                    seq_lens, scale: float, rows) -> np.ndarray:
    """The same attention for selected (b, h) rows only, decoding just the codes those rows
    read (full-size pools hold billions of codes).  Returns [len(rows), D]."""
    Hk, ps = k_codes.shape[1], k_codes.shape[2]
    H = q_bits.shape[1]
    q = bf16_bits_to_f64(q_bits)
    out = np.zeros((len(rows), q_bits.shape[2]), dtype=np.float64)
    for i, (b, h) in enumerate(rows):
        L = int(seq_lens[b])
        t = np.arange(L, dtype=np.int64)
        page = np.asarray(block_table[b], dtype=np.int64)[t // ps]
        slot = t % ps
        kvh = kv_head_of(h, H, Hk)
        K = e4m3_bits_to_f64(k_codes[page, kvh, slot, :]) * float(k_scales[kvh])
        V = e4m3_bits_to_f64(v_codes[page, kvh, slot, :]) * float(v_scales[kvh])
        out[i] = attend_one_query(q[b, h], K, V, scale)
    return out


def encode_fp32_quotient(x, scale) -> np.ndarray:
    """Codes of x / scale: the quotient in IEEE fp32 (x and scale as fp32, round to nearest
    even), then the e4m3 code nearest to that fp32 value (f64_to_e4m3_bits)."""
    quotient = np.asarray(x, dtype=np.float32) / np.asarray(scale, dtype=np.float32)
    return f64_to_e4m3_bits(quotient.astype(np.float64))


def quantize_bf16_pages(pages_bits, scales) -> np.ndarray:
    """Codes of a bf16 pool [P, Hk, ps, D] (raw bits) with one fp32 scale per kv head:
    element [p, kvh, t, d] becomes encode_fp32_quotient(x, scales[kvh])."""
    x = bf16_bits_to_f64(pages_bits)
    s = np.asarray(scales, dtype=np.float32)[None, :, None, None]
    return encode_fp32_quotient(x, np.broadcast_to(s, x.shape))


def kv_append_fp8(k_codes, v_codes, k_new_bits, v_new_bits, k_scales, v_scales, block_table,
                  positions):
    """kv_append into a coded cache: the slot of position positions[b] of sequence b takes
    the codes of k_new[b, kvh, :] / k_scales[kvh] (V likewise with v_scales); every other
    byte is unchanged.  k_new, v_new [B, Hk, D] are bf16 bits; returns new (K, V) pools."""
    kc = np.array(k_codes, dtype=np.uint8, copy=True)
    vc = np.array(v_codes, dtype=np.uint8, copy=True)
    ps = kc.shape[2]
    ks = np.asarray(k_scales, dtype=np.float32)[:, None]
    vs = np.asarray(v_scales, dtype=np.float32)[:, None]
    for b in range(len(positions)):
        pos = int(positions[b])
        page = int(block_table[b][pos // ps])
        slot = pos % ps
        kc[page, :, slot, :] = encode_fp32_quotient(bf16_bits_to_f64(k_new_bits[b]), np.broadcast_to(ks, kc.shape[1:2] + kc.shape[3:]))
        vc[page, :, slot, :] = encode_fp32_quotient(bf16_bits_to_f64(v_new_bits[b]), np.broadcast_to(vs, vc.shape[1:2] + vc.shape[3:]))
    return kc, vc
