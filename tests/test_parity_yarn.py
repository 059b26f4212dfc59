"""YaRN-scaled RoPE on the GPU (gqa_set_rope_scaling, then the prefill, decode and projection entry points)
against the oracle with the same Yarn spec.  The window and factor are chosen so that positions run past
the original window and every regime of the ramp (kept, interpolated, in between) occurs."""
import numpy as np
import pytest
import torch

import gqa_inputs as gi
from oracle import gqa_ref as R
from tests.parity_util import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture()
def G():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from grouped_query_attention_gqa_b200 import build
    build.build()
    import grouped_query_attention_gqa_b200 as G
    yield G
    G.set_rope_scaling(1.0)


@pytest.mark.parametrize("L,d,factor,orig", [(1500, 128, 4.0, 1024), (700, 64, 8.0, 256)])
def test_prefill_with_yarn(G, L, d, factor, orig):
    w = gi.small("prefill", B=1, L=L, h_q=28 if d == 128 else 14, h_kv=4 if d == 128 else 2, d=d, seed=L + d)
    q, k, v = gi.prefill_inputs(w)
    G.set_rope_scaling(factor, orig)
    got = G.prefill(q.cuda(), k.cuda(), v.cuda(), theta=w.theta).float().cpu().numpy()
    assert G.last_error() == 0
    spec = R.Yarn(w.theta, factor, orig)
    assert_close(got, R.prefill_ref(q, k, v, spec), f"prefill YaRN s={factor} orig={orig}")
    # and it is not the unscaled result
    G.set_rope_scaling(1.0)
    plain = G.prefill(q.cuda(), k.cuda(), v.cuda(), theta=w.theta).float().cpu().numpy()
    assert np.abs(plain - got).max() > 5e-2


def test_decode_packed_and_paged_with_yarn(G):
    seqlens = [1, 300, 2500, 4099]
    w = gi.small("decode", B=4, max_len=4099, h_q=28, h_kv=4, d=128, seed=41)
    s, q, kp, vp, table, _, kc, vc = gi.decode_paged_inputs(w, 16, seqlens=seqlens)
    G.set_rope_scaling(4.0, 1024)
    dev = torch.device("cuda")
    got = G.decode(q.to(dev), kc.to(dev), vc.to(dev), s.to(dev), theta=w.theta)
    paged = G.decode_paged(q.to(dev), kp.to(dev), vp.to(dev), table.to(dev), s.to(dev), theta=w.theta)
    assert G.last_error() == 0
    ref = R.decode_ref(q, kc, vc, s, R.Yarn(w.theta, 4.0, 1024))
    assert_close(got.float().cpu().numpy(), ref, "decode YaRN")
    assert torch.equal(got, paged)


def test_qkv_projection_and_rotated_attention_with_yarn(G):
    B, L, h_q, h_kv, d, dm = 1, 900, 28, 4, 128, 256
    w = gi.small("prefill", B=B, L=L, h_q=h_q, h_kv=h_kv, d=d, seed=43)
    x, wq, b = gi.qkv_inputs(w, d_model=dm)
    G.set_rope_scaling(4.0, 512)
    dev = torch.device("cuda")
    qr, kr, k, v = G.qkv_rope(x.to(dev), wq.to(dev), b.to(dev), h_q, h_kv, theta=w.theta)
    out = G.prefill_rotated(qr, kr, v).float().cpu().numpy()
    assert G.last_error() == 0
    spec = R.Yarn(w.theta, 4.0, 512)
    ref_q = R.qkv_rope_ref(x, wq, b, h_q, h_kv, d, spec)
    got_q = [t.float().cpu().numpy() for t in (qr, kr, k, v)]
    for name, g_, r_ in zip(("qr", "kr", "k", "v"), got_q, ref_q):
        excess = np.abs(g_ - r_) - 2.0 ** -8 * np.abs(r_)
        assert float(excess.max()) <= 2e-3, name
    # attention on the rotated rows: scores of Q' K'^T (which carry the temperature) through the definition
    g = h_q // h_kv
    qrr, krr, vv = ref_q[0][0], ref_q[1][0], ref_q[3][0]
    ref = np.empty((L, h_q, d))
    for t in range(h_q):
        ref[:, t] = R.causal_weights(qrr[t], np.arange(L), krr[t // g]) @ vv[:, t // g]
    assert_close(out[0], ref, "rotated attention with YaRN")


def test_factor_one_is_bitwise_the_plain_path(G):
    w = gi.small("prefill", B=1, L=333, h_q=28, h_kv=4, d=128, seed=44)
    q, k, v = (t.cuda() for t in gi.prefill_inputs(w))
    a = G.prefill(q, k, v, theta=w.theta)
    G.set_rope_scaling(1.0, 12345)
    b = G.prefill(q, k, v, theta=w.theta)
    assert torch.equal(a, b)
