"""Paged GQA/MQA decode attention for B200 (sm_100a): Python binding of libgqa_decode.so.

The binding only marshals arguments: every step of the computation runs in the
library's CUDA kernels (see include/gqa_decode.h).  PyTorch supplies device
memory and the current stream.  There is no CPU fallback: if the shared library
is missing or the tensors are not on a CUDA device, the calls raise.

    kv_append(k_new, v_new, k_pages, v_pages, block_table, positions)
    paged_decode_attn(q, k_pages, v_pages, block_table, seq_lens, out=None, scale=None)
    Pager(num_pages, page_size, max_seqs, max_blocks_per_seq)   host page bookkeeping
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

__all__ = [
    "GQAError",
    "library_path",
    "load_library",
    "kv_append",
    "paged_decode_attn",
    "decode_step",
    "paged_decode_attn_noalloc",
    "quantize_pages_fp8",
    "kv_append_fp8",
    "paged_decode_attn_fp8",
    "decode_step_fp8",
    "kv_append_multi",
    "paged_multi_query_attn",
    "multi_query_step",
    "check_device_error",
    "kv_cache_bytes",
    "set_num_workers",
    "set_wait_limit_ns",
    "launch_count",
    "Pager",
    "EXPORTED_SYMBOLS",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_NAME = "libgqa_decode.so"

GQA_OK = 0
STATUS_NAMES = {0: "GQA_OK", -1: "GQA_ERR_INVALID_ARG", -2: "GQA_ERR_UNSUPPORTED",
                -3: "GQA_ERR_CUDA", -4: "GQA_ERR_DEVICE_BOUNDS", -5: "GQA_ERR_TIMEOUT",
                -6: "GQA_ERR_OUT_OF_PAGES"}

# Every extern "C" entry point declared in include/*.h.
EXPORTED_SYMBOLS = (
    "gqa_kv_append",
    "gqa_paged_decode_attn",
    "gqa_decode_step",
    "gqa_paged_decode_attn_noalloc",
    "gqa_kv_quantize_fp8",
    "gqa_kv_append_fp8",
    "gqa_paged_decode_attn_fp8",
    "gqa_decode_step_fp8",
    "gqa_kv_append_multi",
    "gqa_paged_multi_query_attn",
    "gqa_multi_query_step",
    "gqa_check_device_error",
    "gqa_last_error_string",
    "gqa_kv_cache_bytes",
    "gqa_set_num_workers",
    "gqa_set_wait_limit_ns",
    "gqa_launch_count",
    "gqa_abi_version",
    # include/gqa_pager.h
    "gqa_pager_create",
    "gqa_pager_destroy",
    "gqa_pager_extend",
    "gqa_pager_step",
    "gqa_pager_truncate",
    "gqa_pager_gather",
    "gqa_pager_free_pages",
    "gqa_pager_seq_len",
)


class GQAError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


def library_path() -> str:
    """The in-tree library; GQA_DECODE_LIB may name another build of the same ABI."""
    return os.environ.get("GQA_DECODE_LIB") or os.path.join(_HERE, _LIB_NAME)


_lib = None


def load_library() -> ctypes.CDLL:
    """Load the in-tree shared library (built by gqa_decode_attention_04_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if not os.path.exists(path):
        raise ImportError(
            f"{path} not found: build it with `python -m gqa_decode_attention_04_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i32, f32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_int64
    lib.gqa_kv_append.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp]
    lib.gqa_kv_append.restype = i32
    lib.gqa_paged_decode_attn.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, f32,
                                          i32, i32, vp]
    lib.gqa_paged_decode_attn.restype = i32
    lib.gqa_decode_step.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32,
                                    f32, i32, i32, vp]
    lib.gqa_decode_step.restype = i32
    lib.gqa_paged_decode_attn_noalloc.argtypes = lib.gqa_paged_decode_attn.argtypes
    lib.gqa_paged_decode_attn_noalloc.restype = i32
    lib.gqa_kv_quantize_fp8.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp]
    lib.gqa_kv_quantize_fp8.restype = i32
    lib.gqa_kv_append_fp8.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp]
    lib.gqa_kv_append_fp8.restype = i32
    lib.gqa_paged_decode_attn_fp8.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, f32,
                                              i32, i32, vp]
    lib.gqa_paged_decode_attn_fp8.restype = i32
    lib.gqa_decode_step_fp8.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, f32,
                                        i32, i32, vp]
    lib.gqa_decode_step_fp8.restype = i32
    lib.gqa_kv_append_multi.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, vp]
    lib.gqa_kv_append_multi.restype = i32
    lib.gqa_paged_multi_query_attn.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, f32,
                                               i32, i32, vp]
    lib.gqa_paged_multi_query_attn.restype = i32
    lib.gqa_multi_query_step.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32,
                                         f32, i32, i32, vp]
    lib.gqa_multi_query_step.restype = i32
    lib.gqa_check_device_error.argtypes = [vp]
    lib.gqa_check_device_error.restype = i32
    lib.gqa_last_error_string.argtypes = []
    lib.gqa_last_error_string.restype = ctypes.c_char_p
    lib.gqa_kv_cache_bytes.argtypes = [i32, i32, i32, i64]
    lib.gqa_kv_cache_bytes.restype = ctypes.c_size_t
    lib.gqa_set_num_workers.argtypes = [i32]
    lib.gqa_set_num_workers.restype = i32
    lib.gqa_set_wait_limit_ns.argtypes = [i64, i32]
    lib.gqa_set_wait_limit_ns.restype = i32
    lib.gqa_launch_count.argtypes = []
    lib.gqa_launch_count.restype = ctypes.c_uint64
    lib.gqa_abi_version.argtypes = []
    lib.gqa_abi_version.restype = i32
    lib.gqa_pager_create.argtypes = [i32, i32, i32, i32, ctypes.POINTER(vp)]
    lib.gqa_pager_create.restype = i32
    lib.gqa_pager_destroy.argtypes = [vp]
    lib.gqa_pager_destroy.restype = None
    lib.gqa_pager_extend.argtypes = [vp, i32, i32]
    lib.gqa_pager_extend.restype = i32
    lib.gqa_pager_step.argtypes = [vp, vp, i32, vp, vp]
    lib.gqa_pager_step.restype = i32
    lib.gqa_pager_truncate.argtypes = [vp, i32, i32]
    lib.gqa_pager_truncate.restype = i32
    lib.gqa_pager_gather.argtypes = [vp, vp, i32, vp, vp]
    lib.gqa_pager_gather.restype = i32
    lib.gqa_pager_free_pages.argtypes = [vp]
    lib.gqa_pager_free_pages.restype = i32
    lib.gqa_pager_seq_len.argtypes = [vp, i32]
    lib.gqa_pager_seq_len.restype = i32
    _lib = lib
    return lib


def _check(status: int) -> None:
    if status != GQA_OK:
        msg = load_library().gqa_last_error_string().decode(errors="replace")
        raise GQAError(status, msg)


def _stream_ptr(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _need(t: torch.Tensor, name: str, dtype, device) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor (no CPU path exists)")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def kv_append(k_new, v_new, k_pages, v_pages, block_table, positions, stream=None) -> None:
    """Write k_new/v_new [B, Hk, D] into the pages at positions[b] (bit-exact scatter)."""
    dev = k_pages.device
    for t, n, dt in ((k_new, "k_new", torch.bfloat16), (v_new, "v_new", torch.bfloat16),
                     (k_pages, "k_pages", torch.bfloat16), (v_pages, "v_pages", torch.bfloat16),
                     (block_table, "block_table", torch.int32), (positions, "positions", torch.int32)):
        _need(t, n, dt, dev)
    P, Hk, ps, D = k_pages.shape
    if tuple(v_pages.shape) != (P, Hk, ps, D):
        raise ValueError("v_pages shape differs from k_pages")
    B = k_new.shape[0]
    if tuple(k_new.shape) != (B, Hk, D) or tuple(v_new.shape) != (B, Hk, D):
        raise ValueError("k_new / v_new must be [num_seqs, num_kv_heads, head_dim]")
    if block_table.dim() != 2 or block_table.shape[0] != B or tuple(positions.shape) != (B,):
        raise ValueError("block_table must be [num_seqs, max_blocks], positions [num_seqs]")
    lib = load_library()
    with torch.cuda.device(dev):
        _check(lib.gqa_kv_append(k_new.data_ptr(), v_new.data_ptr(), k_pages.data_ptr(),
                                 v_pages.data_ptr(), block_table.data_ptr(), positions.data_ptr(),
                                 B, Hk, D, ps, block_table.shape[1], P, _stream_ptr(stream)))


def paged_decode_attn(q, k_pages, v_pages, block_table, seq_lens, out: Optional[torch.Tensor] = None,
                      scale: Optional[float] = None, stream=None) -> torch.Tensor:
    """out[b, h] = softmax(scale * q[b, h] . K_b^T) V_b over the paged cache (bf16 out)."""
    dev = q.device
    for t, n, dt in ((q, "q", torch.bfloat16), (k_pages, "k_pages", torch.bfloat16),
                     (v_pages, "v_pages", torch.bfloat16), (block_table, "block_table", torch.int32),
                     (seq_lens, "seq_lens", torch.int32)):
        _need(t, n, dt, dev)
    B, H, D = q.shape
    P, Hk, ps, D2 = k_pages.shape
    if D2 != D or tuple(v_pages.shape) != (P, Hk, ps, D):
        raise ValueError("page pools must be [num_pages, num_kv_heads, page_size, head_dim]")
    if block_table.dim() != 2 or block_table.shape[0] != B or tuple(seq_lens.shape) != (B,):
        raise ValueError("block_table must be [num_seqs, max_blocks], seq_lens [num_seqs]")
    if out is None:
        out = torch.empty((B, H, D), dtype=torch.bfloat16, device=dev)
    else:
        _need(out, "out", torch.bfloat16, dev)
        if tuple(out.shape) != (B, H, D):
            raise ValueError("out must be [num_seqs, num_heads, head_dim]")
    if scale is None:
        scale = 1.0 / (D ** 0.5)
    lib = load_library()
    with torch.cuda.device(dev):
        _check(lib.gqa_paged_decode_attn(q.data_ptr(), k_pages.data_ptr(), v_pages.data_ptr(),
                                         block_table.data_ptr(), seq_lens.data_ptr(), out.data_ptr(),
                                         B, H, Hk, D, ps, float(scale), block_table.shape[1], P,
                                         _stream_ptr(stream)))
    return out


def decode_step(q, k_new, v_new, k_pages, v_pages, block_table, positions, seq_lens,
                out: Optional[torch.Tensor] = None, scale: Optional[float] = None,
                stream=None) -> torch.Tensor:
    """One decode step: append k_new/v_new at positions, then attend over seq_lens tokens."""
    dev = q.device
    for t, n, dt in ((q, "q", torch.bfloat16), (k_new, "k_new", torch.bfloat16),
                     (v_new, "v_new", torch.bfloat16), (k_pages, "k_pages", torch.bfloat16),
                     (v_pages, "v_pages", torch.bfloat16), (block_table, "block_table", torch.int32),
                     (positions, "positions", torch.int32), (seq_lens, "seq_lens", torch.int32)):
        _need(t, n, dt, dev)
    B, H, D = q.shape
    P, Hk, ps, D2 = k_pages.shape
    if D2 != D or tuple(v_pages.shape) != (P, Hk, ps, D):
        raise ValueError("page pools must be [num_pages, num_kv_heads, page_size, head_dim]")
    if tuple(k_new.shape) != (B, Hk, D) or tuple(v_new.shape) != (B, Hk, D):
        raise ValueError("k_new / v_new must be [num_seqs, num_kv_heads, head_dim]")
    if (block_table.dim() != 2 or block_table.shape[0] != B or tuple(seq_lens.shape) != (B,)
            or tuple(positions.shape) != (B,)):
        raise ValueError("block_table must be [num_seqs, max_blocks]; seq_lens, positions [num_seqs]")
    if out is None:
        out = torch.empty((B, H, D), dtype=torch.bfloat16, device=dev)
    else:
        _need(out, "out", torch.bfloat16, dev)
        if tuple(out.shape) != (B, H, D):
            raise ValueError("out must be [num_seqs, num_heads, head_dim]")
    if scale is None:
        scale = 1.0 / (D ** 0.5)
    lib = load_library()
    with torch.cuda.device(dev):
        _check(lib.gqa_decode_step(q.data_ptr(), k_new.data_ptr(), v_new.data_ptr(), k_pages.data_ptr(),
                                   v_pages.data_ptr(), block_table.data_ptr(), positions.data_ptr(),
                                   seq_lens.data_ptr(), out.data_ptr(), B, H, Hk, D, ps, float(scale),
                                   block_table.shape[1], P, _stream_ptr(stream)))
    return out


def _multi_shapes(q, k_pages, v_pages, block_table, seq_lens):
    B, Q, H, D = q.shape
    P, Hk, ps, D2 = k_pages.shape
    if D2 != D or tuple(v_pages.shape) != (P, Hk, ps, D):
        raise ValueError("page pools must be [num_pages, num_kv_heads, page_size, head_dim]")
    if block_table.dim() != 2 or block_table.shape[0] != B or tuple(seq_lens.shape) != (B,):
        raise ValueError("block_table must be [num_seqs, max_blocks], seq_lens [num_seqs]")
    return B, Q, H, D, P, Hk, ps


def _multi_out(out, shape, dev):
    if out is None:
        return torch.empty(shape, dtype=torch.bfloat16, device=dev)
    _need(out, "out", torch.bfloat16, dev)
    if tuple(out.shape) != tuple(shape):
        raise ValueError(f"out must be {list(shape)}")
    return out


def kv_append_multi(k_new, v_new, k_pages, v_pages, block_table, positions, stream=None) -> None:
    """Write k_new/v_new [B, Q, Hk, D]: row i of sequence b to position positions[b] + i."""
    dev = k_pages.device
    for t, n, dt in ((k_new, "k_new", torch.bfloat16), (v_new, "v_new", torch.bfloat16),
                     (k_pages, "k_pages", torch.bfloat16), (v_pages, "v_pages", torch.bfloat16),
                     (block_table, "block_table", torch.int32), (positions, "positions", torch.int32)):
        _need(t, n, dt, dev)
    P, Hk, ps, D = k_pages.shape
    if tuple(v_pages.shape) != (P, Hk, ps, D):
        raise ValueError("v_pages shape differs from k_pages")
    if k_new.dim() != 4:
        raise ValueError("k_new / v_new must be [num_seqs, q_len, num_kv_heads, head_dim]")
    B, Q = k_new.shape[0], k_new.shape[1]
    if tuple(k_new.shape) != (B, Q, Hk, D) or tuple(v_new.shape) != (B, Q, Hk, D):
        raise ValueError("k_new / v_new must be [num_seqs, q_len, num_kv_heads, head_dim]")
    if block_table.dim() != 2 or block_table.shape[0] != B or tuple(positions.shape) != (B,):
        raise ValueError("block_table must be [num_seqs, max_blocks], positions [num_seqs]")
    lib = load_library()
    with torch.cuda.device(dev):
        _check(lib.gqa_kv_append_multi(k_new.data_ptr(), v_new.data_ptr(), k_pages.data_ptr(),
                                       v_pages.data_ptr(), block_table.data_ptr(), positions.data_ptr(),
                                       B, Q, Hk, D, ps, block_table.shape[1], P, _stream_ptr(stream)))


def paged_multi_query_attn(q, k_pages, v_pages, block_table, seq_lens, out: Optional[torch.Tensor] = None,
                           scale: Optional[float] = None, stream=None) -> torch.Tensor:
    """q [B, Q, H, D]: query token i of sequence b (position seq_lens[b] - Q + i) attends to
    positions 0 .. seq_lens[b] - Q + i; out [B, Q, H, D] bf16."""
    dev = q.device
    for t, n, dt in ((q, "q", torch.bfloat16), (k_pages, "k_pages", torch.bfloat16),
                     (v_pages, "v_pages", torch.bfloat16), (block_table, "block_table", torch.int32),
                     (seq_lens, "seq_lens", torch.int32)):
        _need(t, n, dt, dev)
    if q.dim() != 4:
        raise ValueError("q must be [num_seqs, q_len, num_heads, head_dim]")
    B, Q, H, D, P, Hk, ps = _multi_shapes(q, k_pages, v_pages, block_table, seq_lens)
    out = _multi_out(out, (B, Q, H, D), dev)
    if scale is None:
        scale = 1.0 / (D ** 0.5)
    lib = load_library()
    with torch.cuda.device(dev):
        _check(lib.gqa_paged_multi_query_attn(q.data_ptr(), k_pages.data_ptr(), v_pages.data_ptr(),
                                              block_table.data_ptr(), seq_lens.data_ptr(), out.data_ptr(),
                                              B, Q, H, Hk, D, ps, float(scale), block_table.shape[1], P,
                                              _stream_ptr(stream)))
    return out


def multi_query_step(q, k_new, v_new, k_pages, v_pages, block_table, positions, seq_lens,
                     out: Optional[torch.Tensor] = None, scale: Optional[float] = None,
                     stream=None) -> torch.Tensor:
    """kv_append_multi of k_new/v_new [B, Q, Hk, D] at positions, then paged_multi_query_attn."""
    dev = q.device
    for t, n, dt in ((q, "q", torch.bfloat16), (k_new, "k_new", torch.bfloat16),
                     (v_new, "v_new", torch.bfloat16), (k_pages, "k_pages", torch.bfloat16),
                     (v_pages, "v_pages", torch.bfloat16), (block_table, "block_table", torch.int32),
                     (positions, "positions", torch.int32), (seq_lens, "seq_lens", torch.int32)):
        _need(t, n, dt, dev)
    if q.dim() != 4:
        raise ValueError("q must be [num_seqs, q_len, num_heads, head_dim]")
    B, Q, H, D, P, Hk, ps = _multi_shapes(q, k_pages, v_pages, block_table, seq_lens)
    if tuple(k_new.shape) != (B, Q, Hk, D) or tuple(v_new.shape) != (B, Q, Hk, D):
        raise ValueError("k_new / v_new must be [num_seqs, q_len, num_kv_heads, head_dim]")
    if tuple(positions.shape) != (B,):
        raise ValueError("positions must be [num_seqs]")
    out = _multi_out(out, (B, Q, H, D), dev)
    if scale is None:
        scale = 1.0 / (D ** 0.5)
    lib = load_library()
    with torch.cuda.device(dev):
        _check(lib.gqa_multi_query_step(q.data_ptr(), k_new.data_ptr(), v_new.data_ptr(), k_pages.data_ptr(),
                                        v_pages.data_ptr(), block_table.data_ptr(), positions.data_ptr(),
                                        seq_lens.data_ptr(), out.data_ptr(), B, Q, H, Hk, D, ps, float(scale),
                                        block_table.shape[1], P, _stream_ptr(stream)))
    return out


def paged_decode_attn_noalloc(q, k_pages, v_pages, block_table, seq_lens, out: torch.Tensor,
                              scale: Optional[float] = None, stream=None) -> torch.Tensor:
    """paged_decode_attn without any device allocation, for callers that cannot allocate
    (their engine owns all device memory, or allocation's synchronisation is too costly).

    Scratch is a fixed array inside the library, shared by every call: calls that
    overlap on the GPU race, and the first call on a device should come before any
    stream capture.  `out` must be given.  Device-side errors (range, timeout) are
    reported by check_device_error, which reads the array's error word.
    """
    dev = q.device
    for t, n, dt in ((q, "q", torch.bfloat16), (k_pages, "k_pages", torch.bfloat16),
                     (v_pages, "v_pages", torch.bfloat16), (block_table, "block_table", torch.int32),
                     (seq_lens, "seq_lens", torch.int32), (out, "out", torch.bfloat16)):
        _need(t, n, dt, dev)
    B, H, D = q.shape
    P, Hk, ps, D2 = k_pages.shape
    if D2 != D or tuple(v_pages.shape) != (P, Hk, ps, D) or tuple(out.shape) != (B, H, D):
        raise ValueError("shapes must match paged_decode_attn's")
    if block_table.dim() != 2 or block_table.shape[0] != B or tuple(seq_lens.shape) != (B,):
        raise ValueError("block_table must be [num_seqs, max_blocks], seq_lens [num_seqs]")
    if scale is None:
        scale = 1.0 / (D ** 0.5)
    lib = load_library()
    with torch.cuda.device(dev):
        _check(lib.gqa_paged_decode_attn_noalloc(
            q.data_ptr(), k_pages.data_ptr(), v_pages.data_ptr(), block_table.data_ptr(),
            seq_lens.data_ptr(), out.data_ptr(), B, H, Hk, D, ps, float(scale),
            block_table.shape[1], P, _stream_ptr(stream)))
    return out


def _pools_fp8(k_pages, v_pages, k_scales, v_scales, dev):
    for t, n, dt in ((k_pages, "k_pages", torch.uint8), (v_pages, "v_pages", torch.uint8),
                     (k_scales, "k_scales", torch.float32), (v_scales, "v_scales", torch.float32)):
        _need(t, n, dt, dev)
    if k_pages.dim() != 4 or tuple(v_pages.shape) != tuple(k_pages.shape):
        raise ValueError("e4m3 pools must both be [num_pages, num_kv_heads, page_size, head_dim] uint8")
    P, Hk, ps, D = k_pages.shape
    if tuple(k_scales.shape) != (Hk,) or tuple(v_scales.shape) != (Hk,):
        raise ValueError("k_scales / v_scales must be [num_kv_heads] float32")
    return P, Hk, ps, D


def quantize_pages_fp8(src, dst, scales, stream=None) -> torch.Tensor:
    """e4m3 codes of a bf16 pool: dst[p, kvh] = code of src[p, kvh] / scales[kvh]."""
    dev = src.device
    _need(src, "src", torch.bfloat16, dev)
    _need(dst, "dst", torch.uint8, dev)
    _need(scales, "scales", torch.float32, dev)
    if src.dim() != 4 or tuple(dst.shape) != tuple(src.shape):
        raise ValueError("src and dst must both be [num_pages, num_kv_heads, page_size, head_dim]")
    P, Hk, ps, D = src.shape
    if tuple(scales.shape) != (Hk,):
        raise ValueError("scales must be [num_kv_heads] float32")
    with torch.cuda.device(dev):
        _check(load_library().gqa_kv_quantize_fp8(src.data_ptr(), dst.data_ptr(), scales.data_ptr(), P, Hk, ps, D,
                                                  _stream_ptr(stream)))
    return dst


def kv_append_fp8(k_new, v_new, k_pages, v_pages, k_scales, v_scales, block_table, positions,
                  stream=None) -> None:
    """Write k_new/v_new [B, Hk, D] (bf16) into the e4m3 pools at positions[b]."""
    dev = k_pages.device
    P, Hk, ps, D = _pools_fp8(k_pages, v_pages, k_scales, v_scales, dev)
    for t, n, dt in ((k_new, "k_new", torch.bfloat16), (v_new, "v_new", torch.bfloat16),
                     (block_table, "block_table", torch.int32), (positions, "positions", torch.int32)):
        _need(t, n, dt, dev)
    B = k_new.shape[0]
    if tuple(k_new.shape) != (B, Hk, D) or tuple(v_new.shape) != (B, Hk, D):
        raise ValueError("k_new / v_new must be [num_seqs, num_kv_heads, head_dim]")
    if block_table.dim() != 2 or block_table.shape[0] != B or tuple(positions.shape) != (B,):
        raise ValueError("block_table must be [num_seqs, max_blocks], positions [num_seqs]")
    with torch.cuda.device(dev):
        _check(load_library().gqa_kv_append_fp8(
            k_new.data_ptr(), v_new.data_ptr(), k_pages.data_ptr(), v_pages.data_ptr(), k_scales.data_ptr(),
            v_scales.data_ptr(), block_table.data_ptr(), positions.data_ptr(), B, Hk, D, ps, block_table.shape[1], P,
            _stream_ptr(stream)))


def paged_decode_attn_fp8(q, k_pages, v_pages, k_scales, v_scales, block_table, seq_lens,
                          out: Optional[torch.Tensor] = None, scale: Optional[float] = None,
                          stream=None) -> torch.Tensor:
    """paged_decode_attn over e4m3 pools (cached value = code * scale of its kv head)."""
    dev = q.device
    _need(q, "q", torch.bfloat16, dev)
    P, Hk, ps, D = _pools_fp8(k_pages, v_pages, k_scales, v_scales, dev)
    _need(block_table, "block_table", torch.int32, dev)
    _need(seq_lens, "seq_lens", torch.int32, dev)
    B, H, D2 = q.shape
    if D2 != D:
        raise ValueError("q's head_dim differs from the pools'")
    if block_table.dim() != 2 or block_table.shape[0] != B or tuple(seq_lens.shape) != (B,):
        raise ValueError("block_table must be [num_seqs, max_blocks], seq_lens [num_seqs]")
    out = _multi_out(out, (B, H, D), dev)
    if scale is None:
        scale = 1.0 / (D ** 0.5)
    with torch.cuda.device(dev):
        _check(load_library().gqa_paged_decode_attn_fp8(
            q.data_ptr(), k_pages.data_ptr(), v_pages.data_ptr(), k_scales.data_ptr(), v_scales.data_ptr(),
            block_table.data_ptr(), seq_lens.data_ptr(), out.data_ptr(), B, H, Hk, D, ps, float(scale),
            block_table.shape[1], P, _stream_ptr(stream)))
    return out


def decode_step_fp8(q, k_new, v_new, k_pages, v_pages, k_scales, v_scales, block_table, positions, seq_lens,
                    out: Optional[torch.Tensor] = None, scale: Optional[float] = None,
                    stream=None) -> torch.Tensor:
    """kv_append_fp8 of k_new/v_new at positions, then paged_decode_attn_fp8 (one call)."""
    dev = q.device
    _need(q, "q", torch.bfloat16, dev)
    P, Hk, ps, D = _pools_fp8(k_pages, v_pages, k_scales, v_scales, dev)
    for t, n, dt in ((k_new, "k_new", torch.bfloat16), (v_new, "v_new", torch.bfloat16),
                     (block_table, "block_table", torch.int32), (positions, "positions", torch.int32),
                     (seq_lens, "seq_lens", torch.int32)):
        _need(t, n, dt, dev)
    B, H, D2 = q.shape
    if D2 != D or tuple(k_new.shape) != (B, Hk, D) or tuple(v_new.shape) != (B, Hk, D):
        raise ValueError("q [B, H, D], k_new / v_new [B, Hk, D] must match the pools")
    if (block_table.dim() != 2 or block_table.shape[0] != B or tuple(seq_lens.shape) != (B,)
            or tuple(positions.shape) != (B,)):
        raise ValueError("block_table must be [num_seqs, max_blocks]; seq_lens, positions [num_seqs]")
    out = _multi_out(out, (B, H, D), dev)
    if scale is None:
        scale = 1.0 / (D ** 0.5)
    with torch.cuda.device(dev):
        _check(load_library().gqa_decode_step_fp8(
            q.data_ptr(), k_new.data_ptr(), v_new.data_ptr(), k_pages.data_ptr(), v_pages.data_ptr(),
            k_scales.data_ptr(), v_scales.data_ptr(), block_table.data_ptr(), positions.data_ptr(),
            seq_lens.data_ptr(), out.data_ptr(), B, H, Hk, D, ps, float(scale), block_table.shape[1], P,
            _stream_ptr(stream)))
    return out


def check_device_error(stream=None) -> None:
    """Synchronise the stream; raise GQAError if a kernel flagged a device-side error."""
    _check(load_library().gqa_check_device_error(_stream_ptr(stream)))


def kv_cache_bytes(num_layers: int, num_kv_heads: int, head_dim: int, seq_len: int) -> int:
    return int(load_library().gqa_kv_cache_bytes(num_layers, num_kv_heads, head_dim, seq_len))


def set_num_workers(n: int) -> None:
    _check(load_library().gqa_set_num_workers(int(n)))


def set_wait_limit_ns(limit_ns: int, arm_without_copy: bool = False) -> None:
    _check(load_library().gqa_set_wait_limit_ns(int(limit_ns), 1 if arm_without_copy else 0))


def launch_count() -> int:
    return int(load_library().gqa_launch_count())


def _host_i32(x, name: str) -> torch.Tensor:
    t = torch.as_tensor(x, dtype=torch.int32)
    if t.device.type != "cpu":
        raise ValueError(f"{name} must be on the host")
    return t.contiguous().reshape(-1)


class Pager:
    """Host page bookkeeping for one preallocated page pool (include/gqa_pager.h).

    Slots own pool pages in token order; `gather` gives the block table and lengths of a
    batch of slots (host int32 tensors, ready to copy to the device), `step` grows every
    listed slot by one token and returns the new tokens' positions and the new lengths.
    Every call is all-or-nothing and raises GQAError (GQA_ERR_OUT_OF_PAGES when the free
    list is too short).  Host-only and not thread-safe.
    """

    def __init__(self, num_pages: int, page_size: int, max_seqs: int, max_blocks_per_seq: int):
        self._lib = load_library()
        h = ctypes.c_void_p()
        _check(self._lib.gqa_pager_create(int(num_pages), int(page_size), int(max_seqs),
                                          int(max_blocks_per_seq), ctypes.byref(h)))
        self._h = h
        self.num_pages, self.page_size = int(num_pages), int(page_size)
        self.max_seqs, self.max_blocks_per_seq = int(max_seqs), int(max_blocks_per_seq)

    def close(self) -> None:
        if getattr(self, "_h", None) is not None and self._h.value:
            self._lib.gqa_pager_destroy(self._h)
        self._h = None

    def __del__(self):
        self.close()

    def _handle(self):
        if self._h is None:
            raise ValueError("pager is closed")
        return self._h

    def extend(self, seq: int, n_tokens: int) -> None:
        _check(self._lib.gqa_pager_extend(self._handle(), int(seq), int(n_tokens)))

    def step(self, seqs):
        s = _host_i32(seqs, "seqs")
        pos = torch.empty(s.numel(), dtype=torch.int32)
        lens = torch.empty(s.numel(), dtype=torch.int32)
        _check(self._lib.gqa_pager_step(self._handle(), s.data_ptr(), s.numel(), pos.data_ptr(), lens.data_ptr()))
        return pos, lens

    def truncate(self, seq: int, new_len: int) -> None:
        _check(self._lib.gqa_pager_truncate(self._handle(), int(seq), int(new_len)))

    def release(self, seq: int) -> None:
        self.truncate(seq, 0)

    def gather(self, seqs):
        s = _host_i32(seqs, "seqs")
        bt = torch.empty(s.numel(), self.max_blocks_per_seq, dtype=torch.int32)
        lens = torch.empty(s.numel(), dtype=torch.int32)
        _check(self._lib.gqa_pager_gather(self._handle(), s.data_ptr(), s.numel(), bt.data_ptr(), lens.data_ptr()))
        return bt, lens

    @property
    def free_pages(self) -> int:
        return int(self._lib.gqa_pager_free_pages(self._handle()))

    def seq_len(self, seq: int) -> int:
        n = int(self._lib.gqa_pager_seq_len(self._handle(), int(seq)))
        if n < 0:
            raise ValueError(f"slot {seq} out of range")
        return n
