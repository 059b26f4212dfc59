"""gqa_decode_noalloc: the decode step for callers that cannot let the library allocate.

Some callers own all device memory themselves -- a serving process that reserves nearly all of HBM
for its KV cache and weights at start-up, where a cudaMalloc from inside a library would fail or
fragment that reservation -- or run on a latency-critical path that cannot pay for cudaMalloc /
cudaFree, which may synchronise the whole device.  gqa_decode_noalloc keeps its scratch in a fixed
device array instead of allocating.  These tests call it through the C ABI and check:
  * on two calls in a row (the second reuses the scratch the first one left behind), that it gives
    the same result as gqa_decode and matches the fp64 oracle;
  * a g = 16 shape, whose combine step merges two blocks of 8 query heads, run after a call of
    another shape;
  * that a call of a new shape leaves the device's free memory unchanged (it allocates nothing);
  * the documented size limit, exactly: the largest B the header's formula allows runs, B + 1 is
    refused with GQA_ERR_TOO_LARGE and launches nothing.

This file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import gqa_inputs as gi
from oracle import gqa_ref as R
from tests.parity_util import assert_close

pytestmark = pytest.mark.gpu

GQA_ERR_TOO_LARGE = -9
FIXED_SCRATCH_BYTES = 16 << 20


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from grouped_query_attention_gqa_b200 import build
    build.build()
    import grouped_query_attention_gqa_b200 as G
    lib = G.load()
    vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.gqa_decode_noalloc.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f]
    lib.gqa_decode_noalloc.restype = i
    return lib


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _decode_both(lib, w, seqlens):
    """Run gqa_decode and gqa_decode_noalloc on the same inputs; return both outputs (host, fp32) and
    the oracle's."""
    dev = torch.device("cuda")
    s_h, q_h, kc_h, vc_h = gi.decode_inputs(w, seqlens=seqlens)
    s, q, kc, vc = (x.to(dev) for x in (s_h, q_h, kc_h, vc_h))
    ref = torch.empty_like(q)
    got = torch.full_like(q, float("nan"))
    lib.gqa_set_stream(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    args = (w.B, w.h_q, w.h_kv, w.d, ctypes.c_float(w.theta))
    assert lib.gqa_decode(_p(q), _p(kc), _p(vc), _p(s), _p(ref), *args) == 0
    assert lib.gqa_decode_noalloc(_p(q), _p(kc), _p(vc), _p(s), _p(got), *args) == 0
    assert lib.gqa_last_error() == 0
    oracle = R.decode_ref(q_h, kc_h, vc_h, s_h, w.theta)
    return got.float().cpu().numpy(), ref.float().cpu().numpy(), oracle


def test_noalloc_matches_decode_on_two_calls_in_a_row(lib):
    # First call: the Qwen2-7B head shape with a mix of short and long caches.
    w1 = gi.small("decode", B=4, max_len=4099, h_q=28, h_kv=4, d=128, seed=31)
    got1, ref1, or1 = _decode_both(lib, w1, [1, 17, 300, 4099])
    assert_close(got1, ref1, "first gqa_decode_noalloc call vs gqa_decode")
    assert_close(got1, or1, "first gqa_decode_noalloc call vs the oracle")
    # Second call, different shape and more sequences: it must not depend on what the first left.
    w2 = gi.small("decode", B=9, max_len=900, h_q=14, h_kv=2, d=64, seed=32)
    got2, ref2, or2 = _decode_both(lib, w2, [900, 3, 64, 65, 1, 250, 17, 512, 16])
    assert_close(got2, ref2, "second gqa_decode_noalloc call vs gqa_decode")
    assert_close(got2, or2, "second gqa_decode_noalloc call vs the oracle")
    assert np.all(np.isfinite(got2))


def test_noalloc_two_head_blocks_after_another_shape_and_no_allocation(lib):
    dev = torch.device("cuda")
    # A call of another shape first: it leaves its partials in the fixed array.
    w1 = gi.small("decode", B=5, max_len=3000, h_q=28, h_kv=4, d=128, seed=33)
    _decode_both(lib, w1, [3000, 1, 129, 2048, 77])
    # g = 16: two blocks of 8 query heads per KV group, merged by the combine step.
    w2 = gi.small("decode", B=6, max_len=2500, h_q=32, h_kv=2, d=128, seed=34)
    lens = [2500, 5, 1024, 1, 333, 1700]
    s_h, q_h, kc_h, vc_h = gi.decode_inputs(w2, seqlens=lens)
    s, q, kc, vc = (x.to(dev) for x in (s_h, q_h, kc_h, vc_h))
    got = torch.full_like(q, float("nan"))
    lib.gqa_set_stream(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info()
    rc = lib.gqa_decode_noalloc(_p(q), _p(kc), _p(vc), _p(s), _p(got), w2.B, w2.h_q, w2.h_kv, w2.d,
                                ctypes.c_float(w2.theta))
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    assert rc == 0
    assert lib.gqa_last_error() == 0
    assert free_after == free_before, f"device free memory changed by {free_before - free_after} bytes"
    ref = R.decode_ref(q_h, kc_h, vc_h, s_h, w2.theta)
    assert_close(got.float().cpu().numpy(), ref, "g = 16 gqa_decode_noalloc vs the oracle")


def _max_batch(num_sms, h_q, h_kv, d):
    """The largest B whose scratch fits the fixed array, by the formula stated in include/gqa.h."""
    g = h_q // h_kv
    groups = h_kv * -(-g // 8)
    P = 4 * -(-3 * num_sms // groups)
    part = (16 + 8 * d) * 4

    def need(B):
        return -(-8 * (B + 1) // 256) * 256 + (P + B) * groups * part

    B = 1
    while need(B + 1) <= FIXED_SCRATCH_BYTES:
        B += 1
    return B


def test_noalloc_size_limit_is_the_documented_formula(lib):
    dev = torch.device("cuda")
    h_q, h_kv, d = 28, 4, 128
    bmax = _max_batch(torch.cuda.get_device_properties(dev).multi_processor_count, h_q, h_kv, d)
    if torch.cuda.get_device_properties(dev).multi_processor_count == 148:
        assert bmax == 563   # the figure the header quotes for a 148-SM B200
    s = torch.ones(bmax + 1, dtype=torch.int32, device=dev)
    q = torch.randn(bmax + 1, h_q, d, device=dev).to(torch.bfloat16)
    kc = torch.randn(bmax + 1, h_kv, d, device=dev).to(torch.bfloat16)
    vc = torch.randn(bmax + 1, h_kv, d, device=dev).to(torch.bfloat16)
    lib.gqa_set_stream(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    # B = bmax fits: every sequence has one cached row, so its output is that row's value v_0
    out = torch.zeros(bmax, h_q, d, dtype=torch.bfloat16, device=dev)
    rc = lib.gqa_decode_noalloc(_p(q), _p(kc), _p(vc), _p(s), _p(out), bmax, h_q, h_kv, d, ctypes.c_float(1e6))
    assert rc == 0
    assert lib.gqa_last_error() == 0
    expect = vc[:bmax].repeat_interleave(h_q // h_kv, dim=1)
    assert torch.equal(out, expect)
    # B = bmax + 1 does not: refused, nothing launched
    out1 = torch.zeros(bmax + 1, h_q, d, dtype=torch.bfloat16, device=dev)
    rc = lib.gqa_decode_noalloc(_p(q), _p(kc), _p(vc), _p(s), _p(out1), bmax + 1, h_q, h_kv, d,
                                ctypes.c_float(1e6))
    assert rc == GQA_ERR_TOO_LARGE
    assert "fixed" in lib.gqa_strerror(rc).decode()
    torch.cuda.synchronize()
    assert torch.count_nonzero(out1).item() == 0


def test_noalloc_refuses_problems_far_beyond_its_fixed_scratch(lib):
    dev = torch.device("cuda")
    B = 4096   # (444 + 4096) slots x 4 groups x 4160 B of partials: far beyond 16 MiB
    q = torch.zeros(B, 28, 128, dtype=torch.bfloat16, device=dev)
    kc = torch.zeros(B, 4, 128, dtype=torch.bfloat16, device=dev)
    s = torch.ones(B, dtype=torch.int32, device=dev)
    out = torch.zeros_like(q)
    rc = lib.gqa_decode_noalloc(_p(q), _p(kc), _p(kc), _p(s), _p(out), B, 28, 4, 128, ctypes.c_float(1e6))
    assert rc == GQA_ERR_TOO_LARGE
    assert torch.count_nonzero(out).item() == 0   # nothing was launched


def test_noalloc_over_a_cache_that_keeps_keys_after_rope(lib):
    """With gqa_set_decode_cache_rotated(1) the no-allocation decode reads the keys as already rotated at
    their positions, like gqa_decode: the two agree bit for bit and match the oracle's k_rotated decode."""
    dev = torch.device("cuda")
    w = gi.small("decode", B=5, max_len=2100, h_q=28, h_kv=4, d=128, seed=35)
    lens = [2100, 1, 640, 17, 1000]
    s_h, q_h, kc_h, vc_h = gi.decode_inputs(w, seqlens=lens)
    off = R.packed_offsets(lens)
    krot_h = torch.from_numpy(np.concatenate([R.rope(R.as_f64(kc_h[off[b]:off[b + 1]]), np.arange(lens[b]), w.theta)
                                              for b in range(w.B)])).to(torch.bfloat16)
    s, q, krot, vc = (x.to(dev) for x in (s_h, q_h, krot_h, vc_h))
    ref = torch.empty_like(q)
    got = torch.full_like(q, float("nan"))
    lib.gqa_set_stream(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    args = (w.B, w.h_q, w.h_kv, w.d, ctypes.c_float(w.theta))
    assert lib.gqa_set_decode_cache_rotated(1) == 0
    try:
        assert lib.gqa_decode(_p(q), _p(krot), _p(vc), _p(s), _p(ref), *args) == 0
        assert lib.gqa_decode_noalloc(_p(q), _p(krot), _p(vc), _p(s), _p(got), *args) == 0
        torch.cuda.synchronize()
    finally:
        lib.gqa_set_decode_cache_rotated(0)
    assert lib.gqa_last_error() == 0
    assert torch.equal(got, ref)
    oracle = R.decode_ref(q_h, krot_h, vc_h, s_h, w.theta, k_rotated=True)
    assert_close(got.float().cpu().numpy(), oracle, "gqa_decode_noalloc over a rotated cache vs the oracle")
