"""GPU decode step (libgqa through its C ABI) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import gqa_inputs as gi
from oracle import gqa_ref as R
from tests.parity_util import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def G():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from grouped_query_attention_gqa_b200 import build
    build.build()
    import grouped_query_attention_gqa_b200 as G
    return G


def run(G, seqlens, q, kc, vc, theta):
    dev = torch.device("cuda")
    out = G.decode(q.to(dev), kc.to(dev), vc.to(dev), seqlens.to(dev), theta=theta)
    err = G.last_error()
    return out.float().cpu().numpy(), err


CASES = [
    # (seqlens, h_q, h_kv, d)
    ([1, 17, 300], 28, 4, 128),
    ([15, 16, 17, 32, 33], 14, 2, 64),
    ([1000, 1, 4099], 28, 4, 128),
    ([200, 70], 16, 1, 128),      # MQA, g = 16: two head blocks
    ([64, 3], 8, 8, 128),         # MHA, g = 1
    ([5000], 64, 8, 128),         # 72B shape, one long sequence split over many warps
]


@pytest.mark.parametrize("seqlens,h_q,h_kv,d", CASES)
def test_decode_small_full_output(G, seqlens, h_q, h_kv, d):
    w = gi.small("decode", B=len(seqlens), max_len=max(seqlens), h_q=h_q, h_kv=h_kv, d=d,
                 seed=sum(seqlens) + h_q)
    s, q, kc, vc = gi.decode_inputs(w, seqlens=seqlens)
    got, err = run(G, s, q, kc, vc, w.theta)
    assert err == 0
    ref = R.decode_ref(q, kc, vc, s, w.theta)
    assert_close(got, ref, f"decode {seqlens} h_q={h_q} h_kv={h_kv} d={d}")


def test_decode_many_short_sequences(G):
    """More sequences than warps' slices and rows shorter than a block: empty slices, many pieces."""
    rng = np.random.default_rng(3)
    seqlens = rng.integers(1, 40, 700).tolist()
    w = gi.small("decode", B=700, max_len=40, h_q=28, h_kv=4, d=128, seed=21)
    s, q, kc, vc = gi.decode_inputs(w, seqlens=seqlens)
    got, err = run(G, s, q, kc, vc, w.theta)
    assert err == 0
    assert_close(got, R.decode_ref(q, kc, vc, s, w.theta), "700 short sequences")


def test_decode_length_one_is_v0_exactly(G):
    w = gi.small("decode", B=4, max_len=1, h_q=28, h_kv=4, d=128, seed=2)
    s, q, kc, vc = gi.decode_inputs(w, seqlens=[1, 1, 1, 1])
    got, err = run(G, s, q, kc, vc, w.theta)
    assert err == 0
    vv = vc.float().numpy()
    for b in range(4):
        for t in range(28):
            assert np.array_equal(got[b, t], vv[b, t // 7])


def test_decode_nonpositive_length_zeroes_row_and_flags(G):
    seqlens = [9, 0, 12]
    w = gi.small("decode", B=3, max_len=12, h_q=8, h_kv=2, d=64, seed=4)
    s, q, kc, vc = gi.decode_inputs(w, seqlens=seqlens)
    got, err = run(G, s, q, kc, vc, w.theta)
    assert err & G.DEVERR_SEQLEN
    assert np.all(got[1] == 0.0)
    ref = R.decode_ref(q, kc, vc, s, w.theta, batch_rows=[0, 2])
    assert_close(got[[0, 2]], ref, "rows around the empty sequence")
    assert G.last_error() == 0   # reading the word clears it


def test_decode_full_size_sampled_sequences(G):
    """The full Qwen2-7B decode workload (B=64, lengths U[1, 32768]); the oracle checks a sample."""
    w = gi.BY_NAME["qwen2-7b-decode-B64"]
    s, q, kc, vc = gi.decode_inputs(w)
    got, err = run(G, s, q, kc, vc, w.theta)
    assert err == 0
    lens = s.numpy()
    pick = sorted({int(np.argmin(lens)), int(np.argmax(lens)), 0, w.B - 1, 17, 42})
    ref = R.decode_ref(q, kc, vc, s, w.theta, batch_rows=pick)
    assert_close(got[pick], ref, "qwen2-7b decode B=64 sampled")
