"""Pins of the oracle's decode-step projection and cache append, ``qkv_append_ref`` (page "Qwen2
architecture introduction", aicoding.csdn.net, §4.1.3 steps 1-2 and its closing paragraph: each decode
step appends the current token's K and V to the cache of the h_kv groups; page "从 Qwen 1 到 Qwen 2",
nxmr.cn, §2.4: that cache kept in pages), and of ``decode_paged_ref(include_self=True)``, the decode in
which the cache already holds the query's own row.

What fixes them, none of it a restatement of the function under test:
  * a pure-Python brute force (dot-product loops, slot arithmetic by hand) on a tiny case;
  * position 0: RoPE is the identity there, so the projection oracle ``qkv_rope_ref`` at position 0 must
    give the same q, k, v;
  * the whole loop: appending the tokens of a sequence one by one and decoding each with its own row in
    the cache reproduces, row by row, the causal prefill of the same sequence;
  * planted mistakes (wrong slot, wrong page, bias dropped, keys cached rotated) are caught.
"""
import numpy as np

import gqa_inputs as gi
from oracle import gqa_ref as R

THETA = 1.0e6


def _case(B=3, d_model=24, h_q=4, h_kv=2, d=8, page_size=4, seed=11):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((B, d_model))
    n = (h_q + 2 * h_kv) * d
    w = rng.standard_normal((n, d_model)) / np.sqrt(d_model)
    bias = 0.1 * rng.standard_normal(n)
    seqlens = np.array([0, 5, 9][:B])
    num_pages = 12
    kp = rng.standard_normal((num_pages, page_size, h_kv, d))
    vp = rng.standard_normal((num_pages, page_size, h_kv, d))
    table = np.array([[7, 1, 3], [2, 9, 0], [11, 4, 6]][:B])
    return x, w, bias, seqlens, kp, vp, table


def test_append_brute_force():
    x, w, bias, seqlens, kp, vp, table = _case()
    h_q, h_kv, d, ps = 4, 2, 8, 4
    q, kp2, vp2 = R.qkv_append_ref(x, w, bias, h_q, h_kv, d, seqlens, kp, vp, table)
    B, dm = x.shape
    for b in range(B):
        y = [sum(float(x[b, i]) * float(w[c, i]) for i in range(dm)) + float(bias[c]) for c in range(w.shape[0])]
        for t in range(h_q):
            for e in range(d):
                assert abs(q[b, t, e] - y[t * d + e]) < 1e-12
        pos = int(seqlens[b])
        page, slot = int(table[b][pos // ps]), pos % ps
        for u in range(h_kv):
            for e in range(d):
                assert abs(kp2[page, slot, u, e] - y[(h_q + u) * d + e]) < 1e-12
                assert abs(vp2[page, slot, u, e] - y[(h_q + h_kv + u) * d + e]) < 1e-12
    # every other slot is untouched, and the inputs are not modified
    written = {(int(table[b][int(seqlens[b]) // ps]), int(seqlens[b]) % ps) for b in range(B)}
    for pg in range(kp.shape[0]):
        for sl in range(ps):
            if (pg, sl) not in written:
                assert np.array_equal(kp2[pg, sl], kp[pg, sl]) and np.array_equal(vp2[pg, sl], vp[pg, sl])
    assert not np.array_equal(kp2, kp)


def test_append_agrees_with_the_projection_oracle_at_position_zero():
    x, w, bias, _, kp, vp, table = _case()
    h_q, h_kv, d = 4, 2, 8
    q, kp2, vp2 = R.qkv_append_ref(x, w, bias, h_q, h_kv, d, [0, 0, 0], kp, vp, table)
    qr, kr, k, v = R.qkv_rope_ref(x[:, None, :], w, bias, h_q, h_kv, d, THETA, positions=[0])
    np.testing.assert_allclose(q, qr[:, :, 0, :], rtol=0, atol=1e-12)   # RoPE at 0 is the identity
    for b in range(3):
        np.testing.assert_allclose(kp2[table[b][0], 0], k[b, 0], rtol=0, atol=1e-12)
        np.testing.assert_allclose(vp2[table[b][0], 0], v[b, 0], rtol=0, atol=1e-12)


def _loop_matches_prefill(append_fn, decode_fn):
    """Append the L tokens of B sequences one by one into pages, decoding each token with its own row in
    the cache; compare with the causal prefill of the whole sequences (raw q, k, v from the same
    projection)."""
    rng = np.random.default_rng(3)
    B, L, dm, h_q, h_kv, d, ps = 2, 7, 16, 4, 2, 8, 3
    X = rng.standard_normal((B, L, dm))
    n = (h_q + 2 * h_kv) * d
    W = rng.standard_normal((n, dm)) / np.sqrt(dm)
    bias = 0.1 * rng.standard_normal(n)
    Y = X @ W.T + bias
    Q = Y[..., :h_q * d].reshape(B, L, h_q, d)
    K = Y[..., h_q * d:(h_q + h_kv) * d].reshape(B, L, h_kv, d)
    V = Y[..., (h_q + h_kv) * d:].reshape(B, L, h_kv, d)
    ref = R.prefill_ref(Q, K, V, THETA)
    npg = -(-L // ps)
    table = np.array([[2 * i + b for i in range(npg)] for b in range(B)])[:, ::-1].copy()   # scattered
    kp = rng.standard_normal((B * npg, ps, h_kv, d))
    vp = rng.standard_normal((B * npg, ps, h_kv, d))
    worst = 0.0
    for t in range(L):
        q, kp, vp = append_fn(X[:, t], W, bias, h_q, h_kv, d, [t] * B, kp, vp, table)
        out = decode_fn(q, kp, vp, table, [t + 1] * B, THETA)
        worst = max(worst, float(np.abs(out - ref[:, t]).max()))
    return worst


def test_append_then_decode_with_self_is_the_causal_prefill():
    worst = _loop_matches_prefill(R.qkv_append_ref,
                                  lambda *a: R.decode_paged_ref(*a, include_self=True))
    assert worst < 1e-12, worst


def test_append_pins_catch_planted_mistakes():
    def slot_off_by_one(x, w, bias, h_q, h_kv, d, seqlens, kp, vp, table):
        return R.qkv_append_ref(x, w, bias, h_q, h_kv, d, [s + 1 for s in seqlens], kp, vp, table)

    def no_bias(x, w, bias, *rest):
        return R.qkv_append_ref(x, w, None, *rest)

    def keys_cached_rotated(x, w, bias, h_q, h_kv, d, seqlens, kp, vp, table):
        q, kp2, vp2 = R.qkv_append_ref(x, w, bias, h_q, h_kv, d, seqlens, kp, vp, table)
        ps = kp.shape[1]
        for b, pos in enumerate(seqlens):
            pg, sl = table[b][pos // ps], pos % ps
            kp2[pg, sl] = R.rope(kp2[pg, sl][None], [pos], THETA)[0]
        return q, kp2, vp2

    def page_by_remainder(x, w, bias, h_q, h_kv, d, seqlens, kp, vp, table):
        t2 = np.array(table)
        ps = kp.shape[1]
        for b, pos in enumerate(seqlens):   # a page index taken from the slot instead of the quotient
            t2[b, pos // ps] = table[b][(pos % ps) % t2.shape[1]]
        return R.qkv_append_ref(x, w, bias, h_q, h_kv, d, seqlens, kp, vp, t2)

    dec = lambda *a: R.decode_paged_ref(*a, include_self=True)
    for bad in (slot_off_by_one, no_bias, keys_cached_rotated, page_by_remainder):
        assert _loop_matches_prefill(bad, dec) > 1e-6, bad.__name__
    # and the decode must include the query's own row
    assert _loop_matches_prefill(R.qkv_append_ref, lambda *a: R.decode_paged_ref(*a, include_self=False)
                                 if a[4][0] > 1 else R.decode_paged_ref(*a, include_self=True)) > 1e-6


def test_paged_include_self_matches_packed_include_self():
    w = gi.small("decode", B=4, max_len=40, h_q=6, h_kv=2, d=8, seed=21)
    s, q, kp, vp, table, _, kc, vc = gi.decode_paged_inputs(w, 5)
    a = R.decode_paged_ref(q.float().numpy(), kp.float().numpy(), vp.float().numpy(), table.numpy(), s, w.theta,
                           include_self=True)
    b = R.decode_ref(q, kc, vc, s, w.theta, include_self=True)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)
