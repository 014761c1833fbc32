"""Plant plausible mistakes in the oracle (on the CPU) and check a pin rejects each.

Each mutant replaces one oracle function through the module object; the pins
in tests/oracle_pins.py then run against the mutated oracle.  A mutant that no
pin catches would mean the pins cannot see that class of mistake.
"""
import numpy as np
import pytest

import oracle.fp8_cache as F8
import oracle.paged_attention as PA
import oracle_pins as P


def _kv_head_modulo(h, num_heads, num_kv_heads):
    return h % num_kv_heads                      # wrong head -> kv-head map


def _gather_swapped(pages_bits, bt_row, kv_head, seq_len, page_size):
    t = np.arange(seq_len)
    page = np.asarray(bt_row)[np.minimum(t % page_size, len(bt_row) - 1)]
    slot = np.minimum(t // page_size, page_size - 1)  # page/slot indices swapped
    return PA.bf16_bits_to_f64(pages_bits[page, kv_head, slot, :])


def _gather_off_by_one(pages_bits, bt_row, kv_head, seq_len, page_size):
    n = max(seq_len - 1, 0)                     # drops the newest token
    t = np.arange(n)
    page = np.asarray(bt_row)[t // page_size]
    return PA.bf16_bits_to_f64(pages_bits[page, kv_head, t % page_size, :])


def _attend_no_scale(q_row, K, V, scale):
    if K.shape[0] == 0:
        return np.zeros(V.shape[-1])
    s = K @ q_row                               # scale dropped
    w = np.exp(s - s.max())
    return (w @ V) / w.sum()


def _attend_no_max(q_row, K, V, scale):
    if K.shape[0] == 0:
        return np.zeros(V.shape[-1])
    with np.errstate(over="ignore", invalid="ignore"):
        w = np.exp(scale * (K @ q_row))         # max not subtracted
        return (w @ V) / w.sum()


def _attend_transposed(q_row, K, V, scale):
    if K.shape[0] == 0:
        return np.zeros(V.shape[-1])
    s = scale * (K @ q_row)
    w = np.exp(s - s.max())
    w = w / w.sum()
    if V.shape[0] == V.shape[1]:
        return V @ w                            # transposed operand
    return (w @ V)[::-1].copy()                 # reversed output dims


def _attend_sign(q_row, K, V, scale):
    if K.shape[0] == 0:
        return np.zeros(V.shape[-1])
    s = -scale * (K @ q_row)                    # wrong sign on the scores
    w = np.exp(s - s.max())
    return (w @ V) / w.sum()


def _merge_no_weights(pieces):
    return sum(p[0] for p in pieces) / len(pieces)  # ignores the lse weights


def _append_wrong_slot(kp, vp, kn, vn, bt, positions):
    k = np.array(kp, copy=True)
    v = np.array(vp, copy=True)
    ps = k.shape[2]
    for b in range(kn.shape[0]):
        pos = int(positions[b]) + 1               # off by one slot
        pg = int(bt[b][min(pos // ps, bt.shape[1] - 1)])
        k[pg, :, pos % ps, :] = kn[b]
        v[pg, :, pos % ps, :] = vn[b]
    return k, v


def _cache_bytes_single(num_layers, num_kv_heads, head_dim, seq_len, batch=1, bytes_per_elem=2):
    return num_layers * num_kv_heads * head_dim * seq_len * batch * bytes_per_elem  # K only


def _window_excludes_self(seq_len, q_len, i):
    return max(0, min(seq_len, seq_len - q_len + i))   # a query token misses itself


def _window_sees_drafts(seq_len, q_len, i):
    return seq_len                                  # no causal limit among new tokens


def _append_multi_reversed(kp, vp, kn, vn, bt, positions):
    return PA.kv_append(kp, vp, kn[:, -1], vn[:, -1], bt, positions) if kn.shape[1] == 1 else \
        _append_multi_rows_reversed(kp, vp, kn, vn, bt, positions)


def _append_multi_rows_reversed(kp, vp, kn, vn, bt, positions):
    k = np.array(kp, copy=True)
    v = np.array(vp, copy=True)
    ps = k.shape[2]
    Q = kn.shape[1]
    for b in range(kn.shape[0]):
        for i in range(Q):
            pos = int(positions[b]) + i
            pg = int(bt[b][pos // ps])
            k[pg, :, pos % ps, :] = kn[b, Q - 1 - i]   # rows in reverse order
            v[pg, :, pos % ps, :] = vn[b, Q - 1 - i]
    return k, v


def _e4m3_bias8(bits):
    b = np.asarray(bits, dtype=np.uint8).astype(np.int64)
    sign = np.where(b & 0x80, -1.0, 1.0)
    e, m = (b >> 3) & 0xF, b & 0x7
    out = np.where(e == 0, sign * (m / 8.0) * 2.0 ** -7, sign * (1.0 + m / 8.0) * np.exp2(e - 8.0))
    return np.where((e == 15) & (m == 7), np.nan, out)   # exponent bias 8 instead of 7


def _e4m3_truncating(x):
    a = np.asarray(x, dtype=np.float64)
    codes = np.arange(0x7F, dtype=np.uint8)
    vals = F8.e4m3_bits_to_f64(codes)
    out = np.zeros(a.shape, dtype=np.uint8)
    for i, v in np.ndenumerate(a):
        mag = min(abs(v), 448.0)
        c = codes[np.searchsorted(vals, mag, side="right") - 1]   # rounds toward zero
        out[i] = c | (0x80 if v < 0 else 0)
    return out


def _fp8_attention_swapped_scales(q, kc, vc, ks, vs, bt, sl, scale):
    return _ORIG_FP8_ATTN(q, kc, vc, vs, ks, bt, sl, scale)       # K and V scales swapped


_ORIG_FP8_ATTN = F8.paged_decode_attention_fp8

def _encode_fp64_quotient(x, scale):
    return F8.f64_to_e4m3_bits(np.asarray(x, dtype=np.float64) /
                               np.asarray(scale, dtype=np.float32).astype(np.float64))  # fp64 quotient


_ORIG_QUANT = F8.quantize_bf16_pages


def _quantize_scale_by_page(pages_bits, scales):
    s = np.asarray(scales, dtype=np.float32)
    P_ = pages_bits.shape[0]
    per_page = np.resize(s, P_)[:, None, None, None]          # scale indexed by page, not kv head
    x = PA.bf16_bits_to_f64(pages_bits)
    return F8.encode_fp32_quotient(x, np.broadcast_to(per_page, x.shape))


_ORIG_APPEND8 = F8.kv_append_fp8


def _append_fp8_swapped_scales(kc, vc, kn, vn, ks, vs, bt, pos):
    return _ORIG_APPEND8(kc, vc, kn, vn, vs, ks, bt, pos)       # K and V scales swapped


def _append_fp8_next_slot(kc, vc, kn, vn, ks, vs, bt, pos):
    return _ORIG_APPEND8(kc, vc, kn, vn, ks, vs, bt, np.asarray(pos) + 1)  # one slot late


MUTANTS = [
    ("kv_head_of", _kv_head_modulo),
    ("gather_sequence_kv", _gather_swapped),
    ("gather_sequence_kv", _gather_off_by_one),
    ("attend_one_query", _attend_no_scale),
    ("attend_one_query", _attend_no_max),
    ("attend_one_query", _attend_transposed),
    ("attend_one_query", _attend_sign),
    ("merge_partial_pieces", _merge_no_weights),
    ("kv_append", _append_wrong_slot),
    ("kv_cache_bytes", _cache_bytes_single),
    ("multi_query_window", _window_excludes_self),
    ("multi_query_window", _window_sees_drafts),
    ("kv_append_multi", _append_multi_reversed),
    ("F8:e4m3_bits_to_f64", _e4m3_bias8),
    ("F8:f64_to_e4m3_bits", _e4m3_truncating),
    ("F8:paged_decode_attention_fp8", _fp8_attention_swapped_scales),
    ("F8:encode_fp32_quotient", _encode_fp64_quotient),
    ("F8:quantize_bf16_pages", _quantize_scale_by_page),
    ("F8:kv_append_fp8", _append_fp8_swapped_scales),
    ("F8:kv_append_fp8", _append_fp8_next_slot),
]


@pytest.mark.parametrize("name,fn", MUTANTS, ids=[f.__name__ for _, f in MUTANTS])
def test_mutant_is_caught(monkeypatch, name, fn):
    if name.startswith("F8:"):
        monkeypatch.setattr(F8, name[3:], fn)
    else:
        monkeypatch.setattr(PA, name, fn)
    caught = []
    for check in P.ALL_CHECKS:
        try:
            with np.errstate(all="ignore"):
                check()
        except (AssertionError, IndexError, ValueError, FloatingPointError):
            caught.append(check.__name__)
    assert caught, f"no pin rejects mutant {fn.__name__} of {name}"
