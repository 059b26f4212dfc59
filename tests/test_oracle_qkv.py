"""Pins of the fused QKV projection oracle (aicoding.csdn.net page, §4.1.3 steps 1-3: projections with
bias, split into h_q / h_kv heads, RoPE on Q and K).  The projection is pinned by a brute-force dot
product loop, the rotation by the pinned RoPE restatement, the whole by its consistency with the pinned
prefill oracle, and planted mistakes must fail."""
import numpy as np
import pytest

import gqa_inputs as gi
from oracle import gqa_ref as R
from tests.test_oracle_pins import _bf_rope_row

THETA = 10.0   # a small base so every pair rotates visibly at these positions


def _case(B=2, L=5, h_q=4, h_kv=2, d=8, dm=12, seed=3):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((B, L, dm))
    w = rng.standard_normal(((h_q + 2 * h_kv) * d, dm))
    b = rng.standard_normal(((h_q + 2 * h_kv) * d,))
    return x, w, b, h_q, h_kv, d


def _brute(x, w, b, h_q, h_kv, d, theta):
    B, L, dm = x.shape
    n = w.shape[0]
    y = [[[sum(x[bb, l, kk] * w[c, kk] for kk in range(dm)) + (b[c] if b is not None else 0.0)
           for c in range(n)] for l in range(L)] for bb in range(B)]
    qr = np.zeros((B, h_q, L, d)); kr = np.zeros((B, h_kv, L, d))
    k = np.zeros((B, L, h_kv, d)); v = np.zeros((B, L, h_kv, d))
    for bb in range(B):
        for l in range(L):
            row = y[bb][l]
            for t in range(h_q):
                qr[bb, t, l] = _bf_rope_row(row[t * d:(t + 1) * d], l, theta)
            for u in range(h_kv):
                kraw = row[(h_q + u) * d:(h_q + u + 1) * d]
                k[bb, l, u] = kraw
                kr[bb, u, l] = _bf_rope_row(kraw, l, theta)
                v[bb, l, u] = row[(h_q + h_kv + u) * d:(h_q + h_kv + u + 1) * d]
    return qr, kr, k, v


def _pins_pass(fn):
    try:
        for args in [_case(), _case(B=1, L=3, h_q=3, h_kv=3, d=4, dm=5, seed=4), _case(h_q=6, h_kv=1, seed=5)]:
            x, w, b, h_q, h_kv, d = args
            got = fn(x, w, b, h_q, h_kv, d, THETA)
            ref = _brute(x, w, b, h_q, h_kv, d, THETA)
            for g_, r_ in zip(got, ref):
                if g_.shape != r_.shape or not np.allclose(g_, r_, atol=1e-10):
                    return False
        return True
    except Exception:
        return False


def test_qkv_ref_matches_brute_force():
    assert _pins_pass(R.qkv_rope_ref)


def test_zero_input_gives_the_bias_and_no_bias_gives_zero():
    x, w, b, h_q, h_kv, d = _case()
    x[:] = 0.0
    qr, kr, k, v = R.qkv_rope_ref(x, w, b, h_q, h_kv, d, THETA)
    assert np.allclose(v[0, 3, 1], b[(h_q + h_kv + 1) * d:(h_q + h_kv + 2) * d], atol=0)
    assert np.allclose(k[1, 0, 0], b[h_q * d:(h_q + 1) * d], atol=0)
    assert np.allclose(qr[0, 2, 0], b[2 * d:3 * d], atol=0)   # position 0: no rotation
    for a in R.qkv_rope_ref(x, w, None, h_q, h_kv, d, THETA):
        assert np.all(a == 0.0)


def test_qkv_then_prefill_oracle_consistency():
    """Attention on the oracle's Q', K' (rotated here) equals the prefill oracle on the raw Q, K it implies:
    rotating back by -position recovers the raw projection."""
    x, w, b, h_q, h_kv, d = _case(B=1, L=6, h_q=4, h_kv=2, d=8, dm=10, seed=7)
    qr, kr, k, v = R.qkv_rope_ref(x, w, b, h_q, h_kv, d, THETA)
    pos = np.arange(6)
    q_raw = R.rope(qr[0].transpose(1, 0, 2), -pos, THETA)[None]     # [1, L, h_q, d]
    k_raw = R.rope(kr[0].transpose(1, 0, 2), -pos, THETA)[None]
    np.testing.assert_allclose(k_raw, k, atol=1e-12)
    out = R.prefill_ref(q_raw, k, v, THETA)
    g = h_q // h_kv
    for t in range(h_q):
        s = qr[0, t] @ kr[0, t // g].T / np.sqrt(d)
        s = np.where(np.arange(6)[None, :] > np.arange(6)[:, None], -np.inf, s)
        a = np.exp(s - s.max(1, keepdims=True)); a /= a.sum(1, keepdims=True)
        np.testing.assert_allclose(out[0, :, t], a @ v[0, :, t // g], atol=1e-12)


def _mut_swap_kv(x, w, b, h_q, h_kv, d, theta):
    qr, kr, k, v = R.qkv_rope_ref(x, w, b, h_q, h_kv, d, theta)
    return qr, kr, v, k


def _mut_no_bias(x, w, b, h_q, h_kv, d, theta):
    return R.qkv_rope_ref(x, w, None, h_q, h_kv, d, theta)


def _mut_head_interleave(x, w, b, h_q, h_kv, d, theta):
    """Heads taken as interleaved columns (column c of head t at c * h + t) instead of contiguous blocks."""
    n = w.shape[0]
    perm = np.arange(n)
    qcols = np.arange(h_q * d).reshape(d, h_q).T.reshape(-1)
    perm[:h_q * d] = qcols
    return R.qkv_rope_ref(x, w[perm], None if b is None else b[perm], h_q, h_kv, d, theta)


def _mut_no_rope_on_k(x, w, b, h_q, h_kv, d, theta):
    qr, kr, k, v = R.qkv_rope_ref(x, w, b, h_q, h_kv, d, theta)
    return qr, k.transpose(0, 2, 1, 3), k, v


@pytest.mark.parametrize("fn", [_mut_swap_kv, _mut_no_bias, _mut_head_interleave, _mut_no_rope_on_k])
def test_qkv_pins_catch_planted_mistakes(fn):
    assert not _pins_pass(fn), fn.__name__


def test_qkv_inputs_shapes_scales_and_determinism():
    w = gi.small("prefill", B=1, L=64, h_q=4, h_kv=2, d=64, seed=2)
    x, wq, b = gi.qkv_inputs(w, d_model=256)
    x2, wq2, b2 = gi.qkv_inputs(w, d_model=256)
    assert x.shape == (1, 64, 256) and wq.shape == (8 * 64, 256) and b.shape == (8 * 64,)
    assert bool((x == x2).all()) and bool((wq == wq2).all()) and bool((b == b2).all())
    assert 0.8 < float(wq.float().std()) * 16 < 1.2   # std 1/sqrt(d_model)
    assert gi.qkv_inputs(w, d_model=256, bias=False)[2] is None


def test_explicit_positions_match_the_full_sequence():
    x, w, b, h_q, h_kv, d = _case(B=1, L=9, seed=8)
    full = R.qkv_rope_ref(x, w, b, h_q, h_kv, d, THETA)
    rows = [0, 4, 8]
    part = R.qkv_rope_ref(x[:, rows], w, b, h_q, h_kv, d, THETA, positions=rows)
    np.testing.assert_allclose(part[0], full[0][:, :, rows], atol=1e-12)
    np.testing.assert_allclose(part[1], full[1][:, :, rows], atol=1e-12)
    np.testing.assert_allclose(part[2], full[2][:, rows], atol=1e-12)
    np.testing.assert_allclose(part[3], full[3][:, rows], atol=1e-12)


# ---------------------------------------------------------------- output projection + residual
def _brute_out(attn, w_o, res):
    T, k = attn.shape
    n = w_o.shape[0]
    return np.array([[sum(attn[t, kk] * w_o[c, kk] for kk in range(k)) + (res[t, c] if res is not None else 0.0)
                      for c in range(n)] for t in range(T)])


def _out_pins_pass(fn):
    try:
        rng = np.random.default_rng(21)
        for T, k, n in [(5, 8, 6), (3, 12, 4)]:
            attn, w_o, res = rng.standard_normal((T, k)), rng.standard_normal((n, k)), rng.standard_normal((T, n))
            for r_ in (res, None):
                if not np.allclose(fn(attn, w_o, r_), _brute_out(attn, w_o, r_), atol=1e-12):
                    return False
        return True
    except Exception:
        return False


def test_out_proj_ref_matches_brute_force():
    assert _out_pins_pass(R.out_proj_ref)


def test_out_proj_of_the_attention_output_is_concat_times_w_o():
    """The prefill output [B, L, h_q, d] viewed as rows is the Concat of step 5: head t occupies columns
    t*d .. t*d + d - 1, so projecting it equals summing per-head products with the column blocks of W_O."""
    rng = np.random.default_rng(5)
    B, L, h_q, h_kv, d, dm = 1, 6, 4, 2, 8, 10
    q, k, v = (rng.standard_normal((B, L, h, d)) for h in (h_q, h_kv, h_kv))
    heads = R.prefill_ref(q, k, v, THETA)
    w_o = rng.standard_normal((dm, h_q * d))
    got = R.out_proj_ref(heads.reshape(B * L, h_q * d), w_o)
    per_head = sum(heads[0, :, t] @ w_o[:, t * d:(t + 1) * d].T for t in range(h_q))
    np.testing.assert_allclose(got, per_head, atol=1e-12)


@pytest.mark.parametrize("fn", [
    lambda a, w, r: R.out_proj_ref(a, w, None),                  # residual dropped
    lambda a, w, r: a @ w[:, ::-1].T + (0 if r is None else r),    # columns of W_O reversed
    lambda a, w, r: R.out_proj_ref(a, w, r) - (0 if r is None else 2 * r),   # residual subtracted
])
def test_out_proj_pins_catch_planted_mistakes(fn):
    assert not _out_pins_pass(fn)
