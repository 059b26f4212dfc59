"""GPU decode-step projection with cache append (gqa_qkv_append) and the decode with the query's own row in
the cache (gqa_set_decode_self_in_cache), through the C ABI, against the fp64 oracle (``qkv_append_ref``,
``decode_paged_ref(include_self=True)``).

Tolerances: the projected q and the appended K, V rows are one bf16 rounding of an fp32 sum, so
|got - ref| <= 2^-8 |ref| + 2e-3 element by element (as for gqa_qkv_rope); every page slot the append
does not own must be bit-identical to what it held before.  The decode outputs use the attention
tolerance (max 2e-2, mean 2e-3); the oracle decodes its own fp64 cache, the GPU its bf16 one.
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
    G.set_decode_self_in_cache(False)


def assert_rounded(got, ref, what):
    excess = np.abs(np.asarray(got, dtype=np.float64) - ref) - REL * np.abs(ref)
    worst = float(excess.max())
    assert worst <= ABS, f"{what}: |got - ref| exceeds 2^-8 |ref| by {worst:.3e} (allowed {ABS})"


def append_case(B, dm, h_q, h_kv, d, page, lens, seed):
    """Hidden states and weights of one decode step plus a paged cache holding `lens` rows per sequence
    (with room for at least one more), all seeded."""
    w = gi.small("decode", B=B, max_len=max(lens) + 1, h_q=h_q, h_kv=h_kv, d=d, seed=seed)
    s, q0, kp, vp, table, npages, _, _ = gi.decode_paged_inputs(w, page, seqlens=[n + 1 for n in lens])
    pw = gi.small("prefill", B=B, L=1, h_q=h_q, h_kv=h_kv, d=d, seed=seed + 1)
    x, wq, b = gi.qkv_inputs(pw, d_model=dm)
    return x.reshape(B, dm), wq, b, torch.tensor(lens, dtype=torch.int32), kp, vp, table, npages


CASES = [
    # (B, d_model, h_q, h_kv, d, page, lengths before the append)
    (5, 256, 28, 4, 128, 16, [0, 15, 16, 33, 300]),      # page boundaries, an empty sequence
    (3, 128, 14, 2, 64, 5, [4, 5, 11]),                   # d = 64, odd page size
    (130, 512, 8, 2, 128, 16, list(range(0, 1300, 10))),  # two token tiles (the second ragged)
    (4, 896, 14, 2, 64, 1, [0, 1, 2, 77]),                # one row per page, Qwen2-0.5B hidden size
]


@pytest.mark.parametrize("B,dm,h_q,h_kv,d,page,lens", CASES)
def test_append_matches_the_oracle_and_touches_nothing_else(G, B, dm, h_q, h_kv, d, page, lens):
    x, wq, b, s, kp, vp, table, npages = append_case(B, dm, h_q, h_kv, d, page, lens, seed=40 + B)
    q_ref, kp_ref, vp_ref = R.qkv_append_ref(x, wq, b, h_q, h_kv, d, s.numpy(), kp, vp, table.numpy())
    dev = torch.device("cuda")
    kpg, vpg = kp.to(dev), vp.to(dev)
    q = G.qkv_append(x.to(dev), wq.to(dev), b.to(dev), h_q, h_kv, s.to(dev), kpg, vpg, table.to(dev))
    assert G.last_error() == 0
    assert_rounded(q.float().cpu().numpy(), q_ref, "q")
    owned = np.zeros(kp.shape[:2], dtype=bool)
    for i, n in enumerate(lens):
        owned[int(table[i, n // page]), n % page] = True
    k_got, v_got = kpg.cpu(), vpg.cpu()
    assert torch.equal(k_got[~torch.from_numpy(owned)], kp[~torch.from_numpy(owned)])
    assert torch.equal(v_got[~torch.from_numpy(owned)], vp[~torch.from_numpy(owned)])
    assert_rounded(k_got.float().numpy()[owned], kp_ref[owned], "appended K rows")
    assert_rounded(v_got.float().numpy()[owned], vp_ref[owned], "appended V rows")


def test_append_then_decode_loop(G):
    """Three decode steps of the Qwen2-7B head shape: append each new token, decode it with its own row in
    the cache, grow the lengths; the oracle runs the same loop on its own fp64 cache."""
    B, dm, h_q, h_kv, d, page = 6, 512, 28, 4, 128, 16
    lens = [1, 15, 16, 100, 511, 2000]
    dev = torch.device("cuda")
    _, wq, b, s, kp, vp, table, npages = append_case(B, dm, h_q, h_kv, d, page, [n + 2 for n in lens], seed=77)
    kp_o, vp_o = R.as_f64(kp), R.as_f64(vp)
    kpg, vpg, tg = kp.to(dev), vp.to(dev), table.to(dev)
    gen = torch.Generator().manual_seed(78)
    G.set_decode_self_in_cache(True)
    try:
        for step in range(3):
            x = torch.randn(B, dm, generator=gen).to(torch.bfloat16)
            cur = torch.tensor([n + step for n in lens], dtype=torch.int32)
            q_o, kp_o, vp_o = R.qkv_append_ref(x, wq, b, h_q, h_kv, d, cur.numpy(), kp_o, vp_o, table.numpy())
            ref = R.decode_paged_ref(q_o, kp_o, vp_o, table.numpy(), (cur + 1).numpy(), 1.0e6, include_self=True)
            q = G.qkv_append(x.to(dev), wq.to(dev), b.to(dev), h_q, h_kv, cur.to(dev), kpg, vpg, tg)
            out = G.decode_paged(q, kpg, vpg, tg, (cur + 1).to(dev))
            assert G.last_error() == 0
            assert_close(out.float().cpu().numpy(), ref, f"decode step {step}")
    finally:
        G.set_decode_self_in_cache(False)


def test_self_in_cache_length_one_is_v0_and_default_is_restored(G):
    dev = torch.device("cuda")
    w = gi.small("decode", B=3, max_len=40, h_q=28, h_kv=4, d=128, seed=81)
    s, q, kc, vc = (t.to(dev) for t in gi.decode_inputs(w, seqlens=[1, 1, 40]))
    G.set_decode_self_in_cache(True)
    try:
        out = G.decode(q, kc, vc, s)
    finally:
        G.set_decode_self_in_cache(False)
    assert G.last_error() == 0
    # a one-row cache holding the query's own row: the output is that row's value, exactly
    assert torch.equal(out[0], vc[0].repeat_interleave(7, dim=0))
    assert torch.equal(out[1], vc[1].repeat_interleave(7, dim=0))
    ref = R.decode_ref(q.cpu(), kc.cpu(), vc.cpu(), s.cpu(), w.theta, include_self=True)
    assert_close(out.float().cpu().numpy(), ref, "self in cache")
    # and the default (query after the cache) is back
    out0 = G.decode(q, kc, vc, s)
    ref0 = R.decode_ref(q.cpu(), kc.cpu(), vc.cpu(), s.cpu(), w.theta)
    assert_close(out0.float().cpu().numpy(), ref0, "default position")


def test_append_bad_table_entry_writes_no_row_and_flags(G):
    B, dm, h_q, h_kv, d, page = 3, 256, 14, 2, 64, 16
    x, wq, b, s, kp, vp, table, npages = append_case(B, dm, h_q, h_kv, d, page, [3, 20, 40], seed=90)
    bad = table.clone()
    bad[1, 20 // page] = -1                 # sequence 1's slot: no valid page
    dev = torch.device("cuda")
    kpg, vpg = kp.to(dev), vp.to(dev)
    q = G.qkv_append(x.to(dev), wq.to(dev), b.to(dev), h_q, h_kv, s.to(dev), kpg, vpg, bad.to(dev))
    assert G.last_error() & G.DEVERR_PAGE
    q_ref, kp_ref, vp_ref = R.qkv_append_ref(x, wq, b, h_q, h_kv, d, s.numpy(), kp, vp, table.numpy())
    assert_rounded(q.float().cpu().numpy(), q_ref, "q is still written")
    # sequence 1 wrote nothing; sequences 0 and 2 did
    k_got = kpg.cpu()
    assert torch.equal(k_got[int(table[1, 1]), 20 % page], kp[int(table[1, 1]), 20 % page])
    for i, n in ((0, 3), (2, 40)):
        pg, sl = int(table[i, n // page]), n % page
        assert_rounded(k_got[pg, sl].float().numpy(), kp_ref[pg, sl], f"sequence {i}")
