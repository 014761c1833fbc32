"""Plain fp64 CPU oracle for paged GQA/MQA decode attention (test infrastructure).

Only the tests, the package's smoke check and the benchmark's CPU-baseline leg
may import this package.  The product path never calls it.
"""
from .paged_attention import (  # noqa: F401
    bf16_bits_to_f64,
    f64_to_bf16_bits,
    kv_head_of,
    gather_sequence_kv,
    attend_one_query,
    paged_decode_attention,
    paged_decode_attention_rows,
    kv_append,
    multi_query_window,
    paged_multi_query_attention,
    kv_append_multi,
    partial_softmax_piece,
    merge_partial_pieces,
    kv_cache_bytes,
)
from .fp8_cache import (  # noqa: F401
    E4M3_MAX,
    e4m3_bits_to_f64,
    f64_to_e4m3_bits,
    quantize_pages,
    dequantize_pages,
    paged_decode_attention_fp8,
    paged_decode_attention_fp8_rows,
    encode_fp32_quotient,
    quantize_bf16_pages,
    kv_append_fp8,
)
