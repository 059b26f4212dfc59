"""GPU fused QKV projection + bias + RoPE (gqa_qkv_rope) and attention on its rotated outputs
(gqa_prefill_rotated), through the C ABI, against the fp64 oracle.

Tolerance of the projection, from its arithmetic: each output element is an fp32 sum over d_model
products of bf16 values (plus the bias, then the rotation, in fp32), rounded once to bf16.  Rounding to
nearest bf16 is off by at most 2^-9 |y|; the fp32 accumulation and rotation differ from the fp64
definition by far less than 2e-3 at these scales (|y| ~ 1).  The check is |got - ref| <= 2^-8 |ref| +
2e-3 element by element.  The attention on top of it uses the attention tolerance."""
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
    return G


def assert_rounded(got, ref, what):
    got = np.asarray(got, dtype=np.float64)
    excess = np.abs(got - ref) - REL * np.abs(ref)
    worst = float(excess.max())
    assert worst <= ABS, f"{what}: |got - ref| exceeds 2^-8 |ref| by {worst:.3e} (allowed {ABS})"


def run_qkv(G, w, dm, bias=True):
    x, wq, b = gi.qkv_inputs(w, d_model=dm, bias=bias)
    dev = torch.device("cuda")
    outs = G.qkv_rope(x.to(dev), wq.to(dev), None if b is None else b.to(dev), w.h_q, w.h_kv, theta=w.theta)
    assert G.last_error() == 0
    return x, wq, b, [o.float().cpu().numpy() for o in outs]


CASES = [
    # (B, L, d_model, h_q, h_kv, d, bias)
    (1, 200, 256, 4, 2, 128, True),      # 2 token tiles (the second ragged), 4 column tiles
    (2, 130, 512, 14, 2, 64, True),      # d = 64, 4.5 column tiles, ragged token tiles across sequences
    (1, 64, 72, 2, 1, 128, False),       # d_model not a multiple of the 64-wide K block, no bias
    (3, 97, 896, 14, 2, 64, True),       # Qwen2-0.5B hidden size and heads
    (1, 300, 1024, 8, 8, 128, True),     # MHA (h_q = h_kv)
    (1, 1152, 256, 28, 4, 128, True),    # 162 tiles: one whole wave of 148 CTAs and 14 more
    (4, 1024, 512, 14, 2, 64, True),     # d = 64, 160 tiles over 4 sequences
]


@pytest.mark.parametrize("B,L,dm,h_q,h_kv,d,bias", CASES)
def test_qkv_rope_small_full_output(G, B, L, dm, h_q, h_kv, d, bias):
    w = gi.small("prefill", B=B, L=L, h_q=h_q, h_kv=h_kv, d=d, seed=B * 1000 + L + dm)
    x, wq, b, got = run_qkv(G, w, dm, bias)
    ref = R.qkv_rope_ref(x, wq, b, h_q, h_kv, d, w.theta)
    for name, g_, r_ in zip(("qr", "kr", "k", "v"), got, ref):
        assert g_.shape == r_.shape, name
        assert_rounded(g_, r_, f"{name} B={B} L={L} d_model={dm} heads={h_q}/{h_kv} d={d}")


def test_qkv_rope_full_size_sampled_rows(G):
    """Qwen2-7B projection at the prefill workload's size (L=4096, d_model=3584, 28/4 heads): every
    output of a sample of token rows, including the first and last tiles."""
    w = gi.BY_NAME["qwen2-7b-prefill-L4096"]
    x, wq, b, got = run_qkv(G, w, 3584)
    rows = sorted({0, 1, 127, 128, 129, 2047, 2500, 4095, 4094, 3968})
    ref = R.qkv_rope_ref(x[:, rows], wq, b, w.h_q, w.h_kv, w.d, w.theta, positions=rows)
    qr, kr, k, v = got
    assert_rounded(qr[:, :, rows], ref[0], "qr sampled rows")
    assert_rounded(kr[:, :, rows], ref[1], "kr sampled rows")
    assert_rounded(k[:, rows], ref[2], "k sampled rows")
    assert_rounded(v[:, rows], ref[3], "v sampled rows")


@pytest.mark.parametrize("B,L,h_q,h_kv,d", [(1, 333, 28, 4, 128), (2, 200, 14, 2, 64)])
def test_prefill_rotated_matches_the_attention_oracle(G, B, L, h_q, h_kv, d):
    """Attention on the GPU's own rotated projection outputs: the oracle rotates them back by -position
    (exact in fp64) and runs the prefill definition on the raw Q and K."""
    dm = 256
    w = gi.small("prefill", B=B, L=L, h_q=h_q, h_kv=h_kv, d=d, seed=L + d)
    x, wq, b = gi.qkv_inputs(w, d_model=dm)
    dev = torch.device("cuda")
    qr, kr, k, v = G.qkv_rope(x.to(dev), wq.to(dev), b.to(dev), h_q, h_kv, theta=w.theta)
    out = G.prefill_rotated(qr, kr, v)
    assert G.last_error() == 0
    pos = np.arange(L)
    qrh, krh = qr.float().cpu().numpy(), kr.float().cpu().numpy()
    q_raw = np.stack([R.rope(qrh[bb].transpose(1, 0, 2), -pos, w.theta) for bb in range(B)])
    k_raw = np.stack([R.rope(krh[bb].transpose(1, 0, 2), -pos, w.theta) for bb in range(B)])
    ref = R.prefill_ref(q_raw, k_raw, v.float().cpu().numpy(), w.theta)
    assert_close(out.float().cpu().numpy(), ref, f"prefill_rotated B={B} L={L} d={d}")
    # and the cache rows written by the projection are the un-rotated K the rotated K' came from: k and K'
    # are two independent bf16 roundings (each within 2^-9 of the row's norm; the rotation keeps norms), so
    # row by row ||k - rotate_back(K')|| <= 2^-8 ||k|| (+ slack for the fp32 rotation).
    kh = k.float().cpu().numpy()
    diff = np.linalg.norm(kh - k_raw, axis=-1)
    assert np.all(diff <= 2.0 ** -8 * np.linalg.norm(k_raw, axis=-1) + 1e-3), float((diff / np.linalg.norm(k_raw, axis=-1)).max())


def test_qkv_then_attention_matches_gqa_prefill_on_the_raw_projection(G):
    """Two routes to the same attention output: projection -> rotated attention, and the raw projection
    (K from the kernel, Q rotated back) -> gqa_prefill, which rotates in its own prep pass."""
    w = gi.small("prefill", B=1, L=500, h_q=28, h_kv=4, d=128, seed=99)
    x, wq, b = gi.qkv_inputs(w, d_model=512)
    dev = torch.device("cuda")
    qr, kr, k, v = G.qkv_rope(x.to(dev), wq.to(dev), b.to(dev), w.h_q, w.h_kv, theta=w.theta)
    out1 = G.prefill_rotated(qr, kr, v).float().cpu().numpy()
    pos = np.arange(500)
    q_raw = R.rope(qr[0].float().cpu().numpy().transpose(1, 0, 2), -pos, w.theta)[None]
    out2 = G.prefill(torch.from_numpy(np.ascontiguousarray(q_raw)).to(torch.bfloat16).to(dev), k, v, theta=w.theta)
    assert G.last_error() == 0
    assert_close(out1, out2.float().cpu().numpy(), "rotated route vs prep route")


# ---------------------------------------------------------------- output projection + residual
@pytest.mark.parametrize("T,d_in,dm,resid,inplace", [
    (200, 256, 256, True, False),    # 2 token tiles, the second ragged
    (130, 512, 896, True, True),     # 3.5 column tiles (Qwen2-0.5B hidden size), updated in place
    (64, 72, 128, False, False),     # d_in not a multiple of the 64-wide K block, no residual
    (4736, 512, 1024, True, False),  # 37 x 4 tiles: exactly one full wave of 148 CTAs
    (1280, 512, 4096, True, True),   # 160 tiles: one whole wave and 12 more, in place
    # The last wave's 12 tiles split into 64-column units, with an odd number (9) of K blocks per unit
    (1280, 576, 4096, True, False),
    # 150 tiles, the last two split; the last tile is half past d_model (two of its units store nothing);
    # a ragged K block (200 = 3 x 64 + 8)
    (1280, 200, 3712, True, True),
])
def test_out_proj_small_full_output(G, T, d_in, dm, resid, inplace):
    rng = torch.Generator().manual_seed(T + d_in + dm)
    attn = torch.randn(T, d_in, generator=rng).to(torch.bfloat16)
    w_o = (torch.randn(dm, d_in, generator=rng) / d_in ** 0.5).to(torch.bfloat16)
    res = torch.randn(T, dm, generator=rng).to(torch.bfloat16) if resid else None
    dev = torch.device("cuda")
    res_d = res.to(dev) if resid else None
    got = G.out_proj(attn.to(dev), w_o.to(dev), res_d, out=res_d if inplace else None)
    assert G.last_error() == 0
    assert_rounded(got.float().cpu().numpy(), R.out_proj_ref(attn, w_o, res), f"out_proj T={T} {d_in}->{dm}")


def test_out_proj_full_size_sampled_rows(G):
    w = gi.BY_NAME["qwen2-7b-prefill-L4096"]
    attn, w_o, res = gi.out_proj_inputs(w)
    got = G.out_proj(attn.cuda(), w_o.cuda(), res.cuda()).float().cpu().numpy()
    rows = [0, 1, 127, 128, 2047, 4094, 4095]
    assert_rounded(got[rows], R.out_proj_ref(attn[rows], w_o, res[rows]), "out_proj Qwen2-7B sampled rows")


def test_attention_sublayer_end_to_end(G):
    """Steps 1-6 of the single-layer data flow on the GPU (projection + RoPE, attention on the rotated
    inputs, W_O + residual) against the oracles chained the same way."""
    B, L, h_q, h_kv, d, dm = 1, 300, 28, 4, 128, 512
    w = gi.small("prefill", B=B, L=L, h_q=h_q, h_kv=h_kv, d=d, seed=77)
    x, wq, b = gi.qkv_inputs(w, d_model=dm)
    rng = torch.Generator().manual_seed(78)
    w_o = (torch.randn(dm, h_q * d, generator=rng) / (h_q * d) ** 0.5).to(torch.bfloat16)
    x_in = torch.randn(B * L, dm, generator=rng).to(torch.bfloat16)
    dev = torch.device("cuda")
    qr, kr, k, v = G.qkv_rope(x.to(dev), wq.to(dev), b.to(dev), h_q, h_kv, theta=w.theta)
    heads = G.prefill_rotated(qr, kr, v)
    y = G.out_proj(heads, w_o.to(dev), x_in.to(dev)).float().cpu().numpy()
    assert G.last_error() == 0
    qr_r, kr_r, k_r, v_r = R.qkv_rope_ref(x, wq, b, h_q, h_kv, d, w.theta)
    pos = np.arange(L)
    q_raw = R.rope(qr_r[0].transpose(1, 0, 2), -pos, w.theta)[None]
    heads_r = R.prefill_ref(q_raw, k_r, v_r, w.theta)
    ref = R.out_proj_ref(heads_r.reshape(B * L, h_q * d), w_o, x_in)
    assert_close(y, ref, "attention sub-layer end to end")
