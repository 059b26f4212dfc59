"""The C-ABI library loads, exports every entry point include/gqa.h declares, and validates
its arguments on the host (no GPU needed: every call here fails before any CUDA work)."""
import ctypes
import os
import re

import pytest

import grouped_query_attention_gqa_b200 as G
from grouped_query_attention_gqa_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gqa.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return G.load()


def declared():
    txt = open(HEADER).read()
    return re.findall(r"GQA_API\s+[\w\s\*]+?\b(gqa_\w+)\s*\(", txt)


def codes():
    txt = open(HEADER).read()
    return {m[0]: int(m[1]) for m in re.findall(r"#define (GQA_\w+) \(?(-?\d+)\)?", txt)}


def test_header_declares_the_entry_points():
    names = set(declared())
    for n in ["gqa_prefill", "gqa_decode", "gqa_decode_paged", "gqa_qkv_rope", "gqa_prefill_rotated",
              "gqa_out_proj", "gqa_qkv_append", "gqa_set_decode_self_in_cache", "gqa_set_decode_cache_rotated",
              "gqa_set_stream", "gqa_last_error",
              "gqa_release",
              "gqa_strerror", "gqa_abi_version", "gqa_set_timing_events"]:
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared():
        assert hasattr(lib, name), f"{name} declared in gqa.h but not exported"


def test_version_and_strerror(lib):
    assert lib.gqa_abi_version() == 2
    c = codes()
    for k, v in c.items():
        if k.startswith("GQA_ERR_"):
            assert G.strerror(v) != "unknown error code"
    assert G.strerror(12345) == "unknown error code"


F = ctypes.c_float(1.0e6)
P16 = ctypes.c_void_p(256)


@pytest.mark.parametrize("args,code", [
    ((P16, P16, P16, P16, -1, 16, 28, 4, 128, F), "GQA_ERR_DIMS"),
    ((P16, P16, P16, P16, 1, -3, 28, 4, 128, F), "GQA_ERR_DIMS"),
    ((P16, P16, P16, P16, 1, 16, 28, 5, 128, F), "GQA_ERR_DIMS"),
    ((P16, P16, P16, P16, 1, 16, 0, 4, 128, F), "GQA_ERR_DIMS"),
    ((P16, P16, P16, P16, 1, 16, 28, 0, 128, F), "GQA_ERR_DIMS"),
    ((P16, P16, P16, P16, 1, 16, 28, 4, 96, F), "GQA_ERR_HEAD_DIM"),
    ((P16, P16, P16, P16, 1, 16, 28, 4, 128, ctypes.c_float(0.0)), "GQA_ERR_THETA"),
    ((P16, P16, P16, P16, 1, 16, 28, 4, 128, ctypes.c_float(float("inf"))), "GQA_ERR_THETA"),
    ((P16, P16, P16, P16, 1, 16, 28, 4, 128, ctypes.c_float(float("nan"))), "GQA_ERR_THETA"),
    ((None, P16, P16, P16, 1, 16, 28, 4, 128, F), "GQA_ERR_NULL"),
    ((P16, P16, P16, None, 1, 16, 28, 4, 128, F), "GQA_ERR_NULL"),
    ((P16, P16, ctypes.c_void_p(264), P16, 1, 16, 28, 4, 128, F), "GQA_ERR_ALIGN"),
    ((None, None, None, None, 0, 16, 28, 4, 128, F), "GQA_OK"),      # empty batch: no-op
    ((None, None, None, None, 2, 0, 28, 4, 128, F), "GQA_OK"),       # empty sequence: no-op
])
def test_prefill_validation(lib, args, code):
    assert lib.gqa_prefill(*args) == codes()[code]


@pytest.mark.parametrize("args,code", [
    ((P16, P16, P16, P16, P16, -1, 28, 4, 128, F), "GQA_ERR_DIMS"),
    ((P16, P16, P16, P16, P16, 4, 28, 3, 128, F), "GQA_ERR_DIMS"),
    ((P16, P16, P16, P16, P16, 4, 28, 4, 32, F), "GQA_ERR_HEAD_DIM"),
    ((P16, P16, P16, P16, P16, 4, 28, 4, 64, ctypes.c_float(-1.0)), "GQA_ERR_THETA"),
    ((P16, P16, P16, None, P16, 4, 28, 4, 128, F), "GQA_ERR_NULL"),
    ((P16, None, P16, P16, P16, 4, 28, 4, 128, F), "GQA_ERR_NULL"),
    ((ctypes.c_void_p(260), P16, P16, P16, P16, 4, 28, 4, 128, F), "GQA_ERR_ALIGN"),
    ((None, None, None, None, None, 0, 28, 4, 128, F), "GQA_OK"),
])
def test_decode_validation(lib, args, code):
    assert lib.gqa_decode(*args) == codes()[code]


def paged_args(q=P16, kp=P16, vp=P16, bt=P16, s=P16, out=P16, B=4, h_q=28, h_kv=4, d=128, page=16, npages=64,
               maxp=8, theta=F):
    return (q, kp, vp, bt, s, out, B, h_q, h_kv, d, page, npages, maxp, theta)


@pytest.mark.parametrize("args,code", [
    (paged_args(B=-1), "GQA_ERR_DIMS"),
    (paged_args(page=0), "GQA_ERR_DIMS"),
    (paged_args(page=-16), "GQA_ERR_DIMS"),
    (paged_args(npages=0), "GQA_ERR_DIMS"),
    (paged_args(maxp=0), "GQA_ERR_DIMS"),
    (paged_args(npages=1 << 30, page=1 << 12), "GQA_ERR_DIMS"),      # storage rows beyond 2^40
    (paged_args(h_kv=3), "GQA_ERR_DIMS"),
    (paged_args(d=80), "GQA_ERR_HEAD_DIM"),
    (paged_args(theta=ctypes.c_float(0.0)), "GQA_ERR_THETA"),
    (paged_args(bt=None), "GQA_ERR_NULL"),
    (paged_args(kp=None), "GQA_ERR_NULL"),
    (paged_args(s=None), "GQA_ERR_NULL"),
    (paged_args(vp=ctypes.c_void_p(264)), "GQA_ERR_ALIGN"),
    (paged_args(q=None, kp=None, vp=None, bt=None, s=None, out=None, B=0), "GQA_OK"),
])
def test_decode_paged_validation(lib, args, code):
    assert lib.gqa_decode_paged(*args) == codes()[code]


def qkv_args(x=P16, w=P16, b=None, qr=P16, kr=P16, k=P16, v=P16, B=1, L=16, dm=256, h_q=28, h_kv=4, d=128, theta=F):
    return (x, w, b, qr, kr, k, v, B, L, dm, h_q, h_kv, d, theta)


@pytest.mark.parametrize("args,code", [
    (qkv_args(B=-1), "GQA_ERR_DIMS"),
    (qkv_args(dm=0), "GQA_ERR_DIMS"),
    (qkv_args(dm=100), "GQA_ERR_DIMS"),          # not a multiple of 8
    (qkv_args(h_kv=3), "GQA_ERR_DIMS"),
    (qkv_args(d=96), "GQA_ERR_HEAD_DIM"),
    (qkv_args(theta=ctypes.c_float(-2.0)), "GQA_ERR_THETA"),
    (qkv_args(x=None), "GQA_ERR_NULL"),
    (qkv_args(v=None), "GQA_ERR_NULL"),
    (qkv_args(b=ctypes.c_void_p(264)), "GQA_ERR_ALIGN"),
    (qkv_args(kr=ctypes.c_void_p(8)), "GQA_ERR_ALIGN"),
    (qkv_args(x=None, w=None, qr=None, kr=None, k=None, v=None, L=0), "GQA_OK"),
])
def test_qkv_rope_validation(lib, args, code):
    assert lib.gqa_qkv_rope(*args) == codes()[code]


@pytest.mark.parametrize("args,code", [
    ((P16, P16, P16, P16, -1, 16, 28, 4, 128), "GQA_ERR_DIMS"),
    ((P16, P16, P16, P16, 1, 16, 28, 4, 80), "GQA_ERR_HEAD_DIM"),
    ((P16, None, P16, P16, 1, 16, 28, 4, 128), "GQA_ERR_NULL"),
    ((P16, P16, P16, ctypes.c_void_p(4), 1, 16, 28, 4, 128), "GQA_ERR_ALIGN"),
    ((None, None, None, None, 0, 16, 28, 4, 128), "GQA_OK"),
])
def test_prefill_rotated_validation(lib, args, code):
    assert lib.gqa_prefill_rotated(*args) == codes()[code]


@pytest.mark.parametrize("args,code", [
    ((P16, P16, None, P16, -1, 256, 256), "GQA_ERR_DIMS"),
    ((P16, P16, None, P16, 16, 100, 256), "GQA_ERR_DIMS"),     # d_in not a multiple of 8
    ((P16, P16, None, P16, 16, 256, 200), "GQA_ERR_DIMS"),     # d_model not a multiple of 128
    ((None, P16, None, P16, 16, 256, 256), "GQA_ERR_NULL"),
    ((P16, P16, ctypes.c_void_p(24), P16, 16, 256, 256), "GQA_ERR_ALIGN"),
    ((None, None, None, None, 0, 256, 256), "GQA_OK"),
])
def test_out_proj_validation(lib, args, code):
    assert lib.gqa_out_proj(*args) == codes()[code]


@pytest.mark.parametrize("factor,orig,code", [
    (0.5, 32768, "GQA_ERR_DIMS"), (float("nan"), 32768, "GQA_ERR_DIMS"), (float("inf"), 32768, "GQA_ERR_DIMS"),
    (4.0, 0, "GQA_ERR_DIMS"), (4.0, 32768, "GQA_OK"), (1.0, 0, "GQA_OK"),
])
def test_set_rope_scaling_validation(lib, factor, orig, code):
    assert lib.gqa_set_rope_scaling(ctypes.c_float(factor), orig) == codes()[code]
    lib.gqa_set_rope_scaling(ctypes.c_float(1.0), 0)


def test_set_stream_accepts_null(lib):
    assert lib.gqa_set_stream(None) == 0


def append_args(x=P16, w=P16, b=None, s=P16, q=P16, kp=P16, vp=P16, bt=P16, B=2, dm=256, h_q=28, h_kv=4, d=128,
                page=16, npages=8, maxp=4, theta=1.0e6):
    return (x, w, b, s, q, kp, vp, bt, B, dm, h_q, h_kv, d, page, npages, maxp, ctypes.c_float(theta))


@pytest.mark.parametrize("args,code", [
    (append_args(B=-1), "GQA_ERR_DIMS"),
    (append_args(dm=0), "GQA_ERR_DIMS"),
    (append_args(dm=100), "GQA_ERR_DIMS"),          # not a multiple of 8
    (append_args(page=0), "GQA_ERR_DIMS"),
    (append_args(npages=0), "GQA_ERR_DIMS"),
    (append_args(maxp=0), "GQA_ERR_DIMS"),
    (append_args(npages=1 << 30, page=1 << 12), "GQA_ERR_DIMS"),      # storage rows beyond 2^40
    (append_args(h_kv=3), "GQA_ERR_DIMS"),
    (append_args(d=96), "GQA_ERR_HEAD_DIM"),
    (append_args(theta=0.0), "GQA_ERR_THETA"),
    (append_args(theta=float("nan")), "GQA_ERR_THETA"),
    (append_args(x=None), "GQA_ERR_NULL"),
    (append_args(s=None), "GQA_ERR_NULL"),
    (append_args(bt=None), "GQA_ERR_NULL"),
    (append_args(kp=None), "GQA_ERR_NULL"),
    (append_args(b=ctypes.c_void_p(264)), "GQA_ERR_ALIGN"),
    (append_args(vp=ctypes.c_void_p(8)), "GQA_ERR_ALIGN"),
    (append_args(x=None, w=None, s=None, q=None, kp=None, vp=None, bt=None, B=0), "GQA_OK"),
])
def test_qkv_append_validation(lib, args, code):
    assert lib.gqa_qkv_append(*args) == codes()[code]


@pytest.mark.parametrize("on,code", [(0, "GQA_OK"), (1, "GQA_OK"), (2, "GQA_ERR_DIMS"), (-1, "GQA_ERR_DIMS")])
def test_set_decode_self_in_cache_validation(lib, on, code):
    assert lib.gqa_set_decode_self_in_cache(on) == codes()[code]
    lib.gqa_set_decode_self_in_cache(0)


@pytest.mark.parametrize("on,code", [(0, "GQA_OK"), (1, "GQA_OK"), (2, "GQA_ERR_DIMS"), (-1, "GQA_ERR_DIMS")])
def test_set_decode_cache_rotated_validation(lib, on, code):
    assert lib.gqa_set_decode_cache_rotated(on) == codes()[code]
    lib.gqa_set_decode_cache_rotated(0)
