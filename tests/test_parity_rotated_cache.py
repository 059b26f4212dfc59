"""GPU decode over caches that keep their keys after RoPE (gqa_set_decode_cache_rotated(1)), through the C
ABI, against the fp64 oracle (``decode_ref`` / ``decode_paged_ref`` with ``k_rotated=True``,
``qkv_append_ref`` with ``rotate_k=True``).

The rotated cache the GPU reads is the oracle's fp64 rope(k) at each row's position, rounded to bf16; the
oracle decodes that same bf16 cache, so the comparison covers the decode's own arithmetic.  Tolerances: the
attention tolerance (max 2e-2, mean 2e-3) for decode outputs; one bf16 rounding of an fp32 sum (2^-8 |ref|
+ 2e-3) for the appended rows; bit-identity where two GPU routes compute the same rounded values.
"""
import numpy as np
import pytest
import torch

import gqa_inputs as gi
from oracle import gqa_ref as R
from tests.parity_util import assert_close

pytestmark = pytest.mark.gpu

REL, ABS = 2.0 ** -8, 2e-3


@pytest.fixture(scope="module")
def G():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from grouped_query_attention_gqa_b200 import build
    build.build()
    import grouped_query_attention_gqa_b200 as G
    yield G
    G.set_decode_cache_rotated(False)
    G.set_decode_self_in_cache(False)
    G.set_rope_scaling(1.0)


def rotate_cache(kc, seqlens, theta):
    """The packed cache [N, h_kv, d] with each row rotated at its position in its sequence (oracle RoPE,
    fp64), rounded to bf16."""
    k = R.as_f64(kc)
    off = R.packed_offsets(seqlens)
    rows = [R.rope(k[off[b]:off[b + 1]], np.arange(int(seqlens[b])), theta) for b in range(len(seqlens))]
    return torch.from_numpy(np.concatenate(rows)).to(torch.bfloat16)


CASES = [
    # (seqlens, h_q, h_kv, d)
    ([1, 17, 300], 28, 4, 128),
    ([15, 16, 17, 32, 33], 14, 2, 64),
    ([1000, 1, 4099], 28, 4, 128),
    ([200, 70], 16, 1, 128),      # MQA, g = 16: two head blocks
    ([5000], 64, 8, 128),         # 72B shape, one long sequence split over many warps
]


@pytest.mark.parametrize("seqlens,h_q,h_kv,d", CASES)
def test_rotated_cache_decode_matches_the_oracle(G, seqlens, h_q, h_kv, d):
    w = gi.small("decode", B=len(seqlens), max_len=max(seqlens), h_q=h_q, h_kv=h_kv, d=d, seed=300 + d)
    s, q, kc, vc = gi.decode_inputs(w, seqlens=seqlens)
    krot = rotate_cache(kc, s.numpy(), w.theta)
    dev = torch.device("cuda")
    G.set_decode_cache_rotated(True)
    try:
        out = G.decode(q.to(dev), krot.to(dev), vc.to(dev), s.to(dev), theta=w.theta)
    finally:
        G.set_decode_cache_rotated(False)
    assert G.last_error() == 0
    ref = R.decode_ref(q, krot, vc, s.numpy(), w.theta, k_rotated=True)
    assert_close(out.float().cpu().numpy(), ref, "rotated cache")
    # the same keys kept raw and rotated on load give the same decode, within the tolerance of both
    raw = G.decode(q.to(dev), kc.to(dev), vc.to(dev), s.to(dev), theta=w.theta)
    assert_close(raw.float().cpu().numpy(), ref, "raw cache against the rotated-cache oracle")


def test_rotated_paged_cache_is_bit_identical_to_rotated_packed(G):
    w = gi.BY_NAME["qwen2-7b-decode-B64"]
    s, q, kp, vp, table, npages, kc, vc = gi.decode_paged_inputs(w, 16)
    krot = rotate_cache(kc, s.numpy(), w.theta)
    _, _, store_row = gi.paged_layout(s, 16, w.seed + 7919, 3)
    kp_rot = kp.reshape(-1, w.h_kv, w.d).clone()
    kp_rot[store_row] = krot
    kp_rot = kp_rot.reshape(kp.shape)
    dev = torch.device("cuda")
    G.set_decode_cache_rotated(True)
    try:
        packed = G.decode(q.to(dev), krot.to(dev), vc.to(dev), s.to(dev), theta=w.theta)
        paged = G.decode_paged(q.to(dev), kp_rot.to(dev), vp.to(dev), table.to(dev), s.to(dev), theta=w.theta)
    finally:
        G.set_decode_cache_rotated(False)
    assert G.last_error() == 0
    assert torch.equal(paged, packed)
    rows = [0, int(np.argmax(s.numpy())), int(np.argmin(s.numpy())), 33]
    ref = R.decode_ref(q, krot, vc, s.numpy(), w.theta, batch_rows=rows, k_rotated=True)
    assert_close(packed[rows].float().cpu().numpy(), ref, "Qwen2-7B B=64, sampled sequences")


def test_rotated_cache_under_yarn(G):
    w = gi.small("decode", B=3, max_len=3000, h_q=28, h_kv=4, d=128, seed=321)
    s, q, kc, vc = gi.decode_inputs(w, seqlens=[40, 1500, 3000])
    spec = R.Yarn(w.theta, 4.0, 1024)
    krot = rotate_cache(kc, s.numpy(), spec)
    dev = torch.device("cuda")
    G.set_rope_scaling(4.0, 1024)
    G.set_decode_cache_rotated(True)
    try:
        out = G.decode(q.to(dev), krot.to(dev), vc.to(dev), s.to(dev), theta=w.theta)
    finally:
        G.set_decode_cache_rotated(False)
        G.set_rope_scaling(1.0)
    assert G.last_error() == 0
    ref = R.decode_ref(q, krot, vc, s.numpy(), spec, k_rotated=True)
    assert_close(out.float().cpu().numpy(), ref, "rotated cache, YaRN")


def assert_rounded(got, ref, what):
    excess = np.abs(np.asarray(got, dtype=np.float64) - ref) - REL * np.abs(ref)
    worst = float(excess.max())
    assert worst <= ABS, f"{what}: |got - ref| exceeds 2^-8 |ref| by {worst:.3e} (allowed {ABS})"


def test_rotated_append_then_decode_loop(G):
    """Three decode steps with a cache that keeps keys after RoPE: the append writes each new key rotated
    at its position, the decode uses every cached key as loaded; the oracle runs the same loop."""
    B, dm, h_q, h_kv, d, page = 6, 512, 28, 4, 128, 16
    lens = [1, 15, 16, 100, 511, 2000]
    w = gi.small("decode", B=B, max_len=max(lens) + 3, h_q=h_q, h_kv=h_kv, d=d, seed=401)
    s0, _, kp, vp, table, npages, _, _ = gi.decode_paged_inputs(w, page, seqlens=[n + 3 for n in lens])
    pw = gi.small("prefill", B=B, L=1, h_q=h_q, h_kv=h_kv, d=d, seed=402)
    _, wq, b = gi.qkv_inputs(pw, d_model=dm)
    dev = torch.device("cuda")
    kp_o, vp_o = R.as_f64(kp), R.as_f64(vp)   # random keys, read as keys already rotated
    kpg, vpg, tg = kp.to(dev), vp.to(dev), table.to(dev)
    gen = torch.Generator().manual_seed(403)
    G.set_decode_self_in_cache(True)
    G.set_decode_cache_rotated(True)
    try:
        for step in range(3):
            x = torch.randn(B, dm, generator=gen).to(torch.bfloat16)
            cur = torch.tensor([n + step for n in lens], dtype=torch.int32)
            q_o, kp_o, vp_o = R.qkv_append_ref(x, wq, b, h_q, h_kv, d, cur.numpy(), kp_o, vp_o, table.numpy(),
                                               rotate_k=True, theta=1.0e6)
            ref = R.decode_paged_ref(q_o, kp_o, vp_o, table.numpy(), (cur + 1).numpy(), 1.0e6, include_self=True,
                                     k_rotated=True)
            q = G.qkv_append(x.to(dev), wq.to(dev), b.to(dev), h_q, h_kv, cur.to(dev), kpg, vpg, tg, theta=1.0e6)
            out = G.decode_paged(q, kpg, vpg, tg, (cur + 1).to(dev))
            assert G.last_error() == 0
            for i, n in enumerate(cur.tolist()):
                pg, sl = int(table[i, n // page]), n % page
                assert_rounded(kpg[pg, sl].float().cpu().numpy(), kp_o[pg, sl], f"step {step}: rotated key row {i}")
            assert_close(out.float().cpu().numpy(), ref, f"decode step {step}")
    finally:
        G.set_decode_cache_rotated(False)
        G.set_decode_self_in_cache(False)


def test_qkv_rope_k_output_holds_the_rotated_keys(G):
    """With the rotated cache in effect the projection's token-major k output is the rotated K: the same
    rounded values as its head-major kr output, bit for bit."""
    w = gi.small("prefill", B=2, L=300, h_q=14, h_kv=2, d=64, seed=404)
    x, wq, b = gi.qkv_inputs(w, d_model=256)
    dev = torch.device("cuda")
    G.set_decode_cache_rotated(True)
    try:
        qr, kr, k, v = G.qkv_rope(x.to(dev), wq.to(dev), b.to(dev), w.h_q, w.h_kv, theta=w.theta)
    finally:
        G.set_decode_cache_rotated(False)
    assert G.last_error() == 0
    assert torch.equal(k, kr.permute(0, 2, 1, 3))
    qr0, kr0, k0, v0 = G.qkv_rope(x.to(dev), wq.to(dev), b.to(dev), w.h_q, w.h_kv, theta=w.theta)
    assert torch.equal(kr0, kr) and torch.equal(qr0, qr) and torch.equal(v0, v)
    assert not torch.equal(k0, k)


@pytest.mark.parametrize("page", [1, 5])
def test_rotated_paged_cache_small_pages(G, page):
    """Pages shorter than a 16-row block (the per-row table lookup of the paged decode) over a rotated
    cache: bit-identical to the rotated packed decode and within tolerance of the oracle."""
    w = gi.small("decode", B=4, max_len=700, h_q=28, h_kv=4, d=128, seed=410 + page)
    lens = [700, 1, 33, 250]
    s, q, kp, vp, table, npages, kc, vc = gi.decode_paged_inputs(w, page, seqlens=lens)
    krot = rotate_cache(kc, s.numpy(), w.theta)
    _, _, store_row = gi.paged_layout(s, page, w.seed + 7919, 3)
    kp_rot = kp.reshape(-1, w.h_kv, w.d).clone()
    kp_rot[store_row] = krot
    kp_rot = kp_rot.reshape(kp.shape)
    dev = torch.device("cuda")
    G.set_decode_cache_rotated(True)
    try:
        packed = G.decode(q.to(dev), krot.to(dev), vc.to(dev), s.to(dev), theta=w.theta)
        paged = G.decode_paged(q.to(dev), kp_rot.to(dev), vp.to(dev), table.to(dev), s.to(dev), theta=w.theta)
    finally:
        G.set_decode_cache_rotated(False)
    assert G.last_error() == 0
    assert torch.equal(paged, packed)
    ref = R.decode_ref(q, krot, vc, s.numpy(), w.theta, k_rotated=True)
    assert_close(paged.float().cpu().numpy(), ref, f"rotated cache, {page}-row pages")
