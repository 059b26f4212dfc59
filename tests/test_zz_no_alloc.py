"""gqa_decode_noalloc: the decode step for callers that cannot let the library allocate.

Some callers own all device memory themselves -- a serving process that reserves nearly all of HBM
for its KV cache and weights at start-up, where a cudaMalloc from inside a library would fail or
fragment that reservation -- or run on a latency-critical path that cannot pay for cudaMalloc /
cudaFree, which may synchronise the whole device.  gqa_decode_noalloc keeps its scratch in a fixed
device array instead of allocating.  These tests call it through the C ABI and check that it gives
the same result as gqa_decode, on two calls in a row (the second call reuses the scratch the first
one left behind), and that a problem too large for the fixed array is refused cleanly.

This file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import gqa_inputs as gi
from tests.parity_util import assert_close

pytestmark = pytest.mark.gpu

GQA_ERR_TOO_LARGE = -9


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
    """Run gqa_decode and gqa_decode_noalloc on the same inputs; return both outputs (host, fp32)."""
    dev = torch.device("cuda")
    s, q, kc, vc = (x.to(dev) for x in gi.decode_inputs(w, seqlens=seqlens))
    ref = torch.empty_like(q)
    got = torch.full_like(q, float("nan"))
    lib.gqa_set_stream(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    args = (w.B, w.h_q, w.h_kv, w.d, ctypes.c_float(w.theta))
    assert lib.gqa_decode(_p(q), _p(kc), _p(vc), _p(s), _p(ref), *args) == 0
    assert lib.gqa_decode_noalloc(_p(q), _p(kc), _p(vc), _p(s), _p(got), *args) == 0
    assert lib.gqa_last_error() == 0
    return got.float().cpu().numpy(), ref.float().cpu().numpy()


def test_noalloc_matches_decode_on_two_calls_in_a_row(lib):
    # First call: the Qwen2-7B head shape with a mix of short and long caches.
    w1 = gi.small("decode", B=4, max_len=4099, h_q=28, h_kv=4, d=128, seed=31)
    got1, ref1 = _decode_both(lib, w1, [1, 17, 300, 4099])
    assert_close(got1, ref1, "first gqa_decode_noalloc call")
    # Second call, different shape and more sequences: it must not depend on what the first left.
    w2 = gi.small("decode", B=9, max_len=900, h_q=14, h_kv=2, d=64, seed=32)
    got2, ref2 = _decode_both(lib, w2, [900, 3, 64, 65, 1, 250, 17, 512, 16])
    assert_close(got2, ref2, "second gqa_decode_noalloc call")
    assert np.all(np.isfinite(got2))


def test_noalloc_refuses_problems_beyond_its_fixed_scratch(lib):
    dev = torch.device("cuda")
    B = 4096   # (296 + 4096) slots x 4 groups x 4160 B of partials: far beyond 16 MiB
    q = torch.zeros(B, 28, 128, dtype=torch.bfloat16, device=dev)
    kc = torch.zeros(B, 4, 128, dtype=torch.bfloat16, device=dev)
    s = torch.ones(B, dtype=torch.int32, device=dev)
    out = torch.zeros_like(q)
    rc = lib.gqa_decode_noalloc(_p(q), _p(kc), _p(kc), _p(s), _p(out), B, 28, 4, 128, ctypes.c_float(1e6))
    assert rc == GQA_ERR_TOO_LARGE
    assert "fixed" in lib.gqa_strerror(rc).decode()
    assert torch.count_nonzero(out).item() == 0   # nothing was launched
