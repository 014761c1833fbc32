"""CPU tests of the C-ABI library: it loads, exports every declared entry point, and
rejects bad arguments on the host before touching a GPU."""
import ctypes
import glob
import json
import os
import re

import pytest

import gqa_decode_attention_04_b200 as gq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = sorted(glob.glob(os.path.join(ROOT, "include", "*.h")))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(gq.library_path()):
        from gqa_decode_attention_04_b200 import build
        build.build()
    return gq.load_library()


def _declared_functions():
    text = "".join(open(h).read() for h in HEADERS)
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gqa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_binding_symbols():
    assert _declared_functions() == sorted(gq.EXPORTED_SYMBOLS)


def test_library_exports_every_declared_symbol(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), name
    # the names are C symbols (extern "C"), not C++-mangled
    out = os.popen(f"nm -D --defined-only {gq.library_path()}").read()
    for name in _declared_functions():
        assert re.search(rf"\bT {name}$", out, flags=re.M), name


def test_abi_version(lib):
    assert lib.gqa_abi_version() == 1


def test_kv_cache_bytes_formula(lib):
    g = json.load(open(os.path.join(ROOT, "tests", "golden", "closed_forms.json")))
    for c in g["kv_cache_bytes"]["cases"]:
        per_seq = gq.kv_cache_bytes(c["num_layers"], c["num_kv_heads"], c["head_dim"], c["seq_len"])
        assert per_seq * c["batch"] == c["bytes"]
    assert gq.kv_cache_bytes(-1, 8, 128, 10) == 0


def _decode(lib, B=2, H=4, Hk=1, D=64, ps=16, MB=4, P=8, scale=0.125, ptr=1 << 20):
    p = ctypes.c_void_p(ptr)
    return lib.gqa_paged_decode_attn(p, p, p, p, p, p, B, H, Hk, D, ps, ctypes.c_float(scale),
                                     MB, P, None)


@pytest.mark.parametrize("kw,status", [
    (dict(H=6, Hk=4), -1),          # num_heads not a multiple of num_kv_heads
    (dict(B=-1), -1),
    (dict(D=96), -2),               # head_dim not built
    (dict(ps=8), -2),               # page size not a multiple of 16
    (dict(ps=48 * 16), -2),
    (dict(scale=float("inf")), -1),
    (dict(MB=0), -1),
    (dict(ptr=0), -1),              # null pointers
    (dict(ptr=(1 << 20) + 2), -1),  # misaligned pool
    (dict(B=0), 0),                 # nothing to do, nothing launched
])
def test_decode_host_validation(lib, kw, status):
    assert _decode(lib, **kw) == status
    if status != 0:
        assert len(lib.gqa_last_error_string()) > 0


def test_kv_append_host_validation(lib):
    p = ctypes.c_void_p(1 << 20)
    # head_dim not a multiple of 8
    assert lib.gqa_kv_append(p, p, p, p, p, p, 2, 1, 12, 16, 4, 8, None) == -2
    assert lib.gqa_kv_append(p, p, p, p, p, p, -1, 1, 64, 16, 4, 8, None) == -1
    assert lib.gqa_kv_append(None, p, p, p, p, p, 2, 1, 64, 16, 4, 8, None) == -1
    assert lib.gqa_kv_append(p, p, p, p, p, p, 0, 1, 64, 16, 4, 8, None) == 0


def test_tuning_knob_validation(lib):
    assert lib.gqa_set_num_workers(-3) == -1
    assert lib.gqa_set_num_workers(0) == 0
    assert lib.gqa_set_wait_limit_ns(0, 0) == -1
    assert lib.gqa_set_wait_limit_ns(10 ** 9, 0) == 0


def test_binding_refuses_cpu_tensors():
    import torch
    q = torch.zeros(1, 4, 64, dtype=torch.bfloat16)
    kp = torch.zeros(2, 1, 16, 64, dtype=torch.bfloat16)
    bt = torch.zeros(1, 1, dtype=torch.int32)
    sl = torch.ones(1, dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA"):
        gq.paged_decode_attn(q, kp, kp, bt, sl)


def _multi(lib, B=2, Q=2, H=4, Hk=1, D=64, ps=16, MB=4, P=8, ptr=1 << 20):
    p = ctypes.c_void_p(ptr)
    return lib.gqa_paged_multi_query_attn(p, p, p, p, p, p, B, Q, H, Hk, D, ps, ctypes.c_float(0.125),
                                          MB, P, None)


@pytest.mark.parametrize("kw,status", [
    (dict(Q=0), -1),                # no query token
    (dict(Q=33, H=4, Hk=1), -2),    # 33 x 4 rows per kv head > 128
    (dict(Q=3, H=96, Hk=2), -2),    # 3 x 48 > 128
    (dict(B=0, Q=32, H=4, Hk=1), 0),  # 128 rows: accepted, nothing to do
])
def test_multi_query_host_validation(lib, kw, status):
    assert _multi(lib, **kw) == status
    if status != 0:
        assert len(lib.gqa_last_error_string()) > 0


def test_kv_append_multi_host_validation(lib):
    p = ctypes.c_void_p(1 << 20)
    assert lib.gqa_kv_append_multi(p, p, p, p, p, p, 2, 0, 1, 64, 16, 4, 8, None) == -1
    assert lib.gqa_kv_append_multi(p, p, p, p, p, p, 0, 3, 1, 64, 16, 4, 8, None) == 0
