"""Pins of the fp64 oracle to facts fixed by the pages and by mathematics (no GPU).

Each test ties the oracle to something other than itself: a worked example the
pages print, a closed form, an invariant the pages state, a brute-force
restatement in pure Python, or a library routine on a special case.  The
last test plants mistakes in copies of the oracle and checks that the pins
catch every one of them.
"""
import cmath
import math

import numpy as np
import pytest
import torch

import gqa_inputs as gi
from oracle import gqa_ref as R
from tests.conftest import read_golden

THETA = 1.0e6


def rnd(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


# ---------------------------------------------------------------- head grouping
def test_head_group_worked_example():
    """Page 'Qwen2 architecture introduction' §4.1.2 (and nxmr.cn §2.2): heads 1-7 -> group 1, 8-14 -> 2."""
    rows = read_golden("head_groups_qwen2_7b.txt")
    h_q, h_kv = int(rows[0][0]), int(rows[0][1])
    g = h_q // h_kv
    assert g == 7
    for t1, u1 in rows[1:]:
        assert R.head_group(int(t1) - 1, g) + 1 == int(u1)


def test_table1_group_sizes_and_kv_ratio():
    """Table 1 shapes: d_model = h_q * d_k; MHA/GQA KV-cache ratio h_q/h_kv = 7 (7B), 8 (72B)."""
    for name, hidden, h_q, h_kv, d, ratio in read_golden("qwen2_table1_heads.txt"):
        hidden, h_q, h_kv, d = int(hidden), int(h_q), int(h_kv), int(d)
        if name != "0.5B":   # 0.5B: 14 * 64 = 896
            assert hidden == h_q * d
        else:
            assert hidden == 14 * 64
        if ratio != "-":
            seq = [32768]
            mha = R.decode_bytes(seq, h_q, h_q, d) - 2 * h_q * d * 2
            gqa = R.decode_bytes(seq, h_q, h_kv, d) - 2 * h_q * d * 2
            assert mha / gqa == pytest.approx(int(ratio))
            # page "Qwen2 / Qwen3 measured config differences" pitfall 2: 2 * h_kv * head_dim * seq_len
            assert gqa == 2 * h_kv * d * 32768 * 2


# ---------------------------------------------------------------- RoPE
def test_rope_is_complex_rotation():
    """Closed form: rotate-half RoPE == complex product (x_i + j x_{i+d/2}) * exp(j m theta^(-2i/d))."""
    d, P = 16, 9
    x = rnd((P, 3, d), 1)
    pos = np.array([0, 1, 2, 7, 100, 4095, 8191, 32767, 123456])
    got = R.rope(x, pos, THETA)
    h = d // 2
    for a, m in enumerate(pos):
        for hh in range(3):
            for i in range(h):
                w = cmath.exp(1j * m * THETA ** (-2.0 * i / d))
                z = complex(x[a, hh, i], x[a, hh, i + h]) * w
                assert got[a, hh, i] == pytest.approx(z.real, abs=1e-12)
                assert got[a, hh, i + h] == pytest.approx(z.imag, abs=1e-12)


def test_rope_identity_at_position_zero():
    x = rnd((1, 4, 128), 2)
    assert np.array_equal(R.rope(x, [0], THETA), x)


def test_rope_preserves_norm():
    """Page intelliparadigm.com §2.3: the rotation keeps each vector's length."""
    x = rnd((50, 5, 128), 3)
    pos = np.arange(50) * 661
    y = R.rope(x, pos, THETA)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)


def test_rope_scores_depend_only_on_offset():
    """Page aicoding.csdn.net §3.5.2: after RoPE, q_m . k_n depends on m - n only."""
    d = 128
    q = rnd((1, 1, d), 4)
    k = rnd((1, 1, d), 5)
    for m, n, s in [(5, 2, 1000), (0, 0, 31999), (30000, 17, 5), (1, 9, 777)]:
        a = np.dot(R.rope(q, [m], THETA).ravel(), R.rope(k, [n], THETA).ravel())
        b = np.dot(R.rope(q, [m + s], THETA).ravel(), R.rope(k, [n + s], THETA).ravel())
        assert a == pytest.approx(b, rel=1e-9, abs=1e-9)


def test_rope_pairings_are_the_same_rotation_up_to_permutation():
    """interleaved(x) == P^-1 rotate_half(P x) with P gathering even then odd dimensions."""
    d = 32
    x = rnd((7, 2, d), 6)
    pos = np.arange(7) * 13
    perm = np.concatenate([np.arange(0, d, 2), np.arange(1, d, 2)])
    inv = np.argsort(perm)
    a = R.rope_interleaved(x, pos, THETA)
    b = R.rope(x[..., perm], pos, THETA)[..., inv]
    np.testing.assert_allclose(a, b, atol=1e-13)


def test_inv_freq_geometric():
    """theta^(-2i/d): first term 1, constant ratio theta^(-2/d), last term theta^(-(d-2)/d)."""
    f = R.inv_freq(128, THETA)
    assert f[0] == 1.0
    np.testing.assert_allclose(f[1:] / f[:-1], THETA ** (-2.0 / 128), rtol=1e-13)
    assert f[-1] == pytest.approx(THETA ** (-126.0 / 128), rel=1e-13)


# ---------------------------------------------------------------- attention
def _small(B=2, L=37, h_q=6, h_kv=2, d=16, seed=11):
    q = rnd((B, L, h_q, d), seed)
    k = rnd((B, L, h_kv, d), seed + 1)
    v = rnd((B, L, h_kv, d), seed + 2)
    return q, k, v


def test_gqa_equals_mha_on_repeat_interleaved_kv():
    """Page 'Qwen2 / Qwen3 measured config differences' pitfall 2: expand K,V by repeat_interleave(g)."""
    q, k, v = _small()
    g = q.shape[2] // k.shape[2]
    ke = np.repeat(k, g, axis=2)
    ve = np.repeat(v, g, axis=2)
    np.testing.assert_allclose(R.prefill_ref(q, k, v, THETA), R.prefill_ref(q, ke, ve, THETA),
                               atol=1e-13)


def test_mqa_every_head_reads_the_single_group():
    """h_kv = 1 is MQA (aicoding.csdn.net §4.1.1): each head equals a one-head call on the same K,V."""
    q, k, v = _small(h_q=5, h_kv=1)
    full = R.prefill_ref(q, k, v, THETA)
    for t in range(5):
        one = R.prefill_ref(q[:, :, t:t + 1], k, v, THETA)
        np.testing.assert_allclose(full[:, :, t:t + 1], one, atol=1e-14)


def test_softmax_rows_sum_to_one():
    q, k, _ = _small(B=1, L=50, h_q=1, h_kv=1)
    pos = np.arange(50)
    a = R.causal_weights(R.rope(q, pos, THETA)[0, :, 0], pos, R.rope(k, pos, THETA)[0, :, 0])
    np.testing.assert_allclose(a.sum(axis=1), 1.0, rtol=1e-14)
    assert np.all(a[np.triu_indices(50, 1)] == 0.0)


def test_first_row_is_v0():
    """Row 0 sees only key 0, so out[b,0,t] = v[b,0,u] exactly."""
    q, k, v = _small()
    out = R.prefill_ref(q, k, v, THETA)
    g = q.shape[2] // k.shape[2]
    for t in range(q.shape[2]):
        assert np.array_equal(out[:, 0, t], v[:, 0, t // g])


def test_zero_query_gives_prefix_means():
    """q = 0 makes every score 0, so row i averages v rows 0..i of its group."""
    q, k, v = _small(h_q=8, h_kv=2)
    q[:] = 0.0
    out = R.prefill_ref(q, k, v, THETA)
    csum = np.cumsum(v, axis=1) / np.arange(1, v.shape[1] + 1)[None, :, None, None]
    for t in range(8):
        np.testing.assert_allclose(out[:, :, t], csum[:, :, t // 4], atol=1e-13)


def _bf_rope_row(vec, m, theta):
    d = len(vec)
    h = d // 2
    out = [0.0] * d
    for i in range(h):
        z = complex(vec[i], vec[i + h]) * cmath.exp(1j * m * theta ** (-2 * i / d))
        out[i], out[i + h] = z.real, z.imag
    return out


def _bf_attend(qrow, qpos, keys, vals, theta, d):
    qr = _bf_rope_row(qrow, qpos, theta)
    sc = []
    for j, kr in enumerate(keys):
        krr = _bf_rope_row(kr, j, theta)
        sc.append(sum(qr[c] * krr[c] for c in range(d)) / math.sqrt(d))
    mx = max(sc)
    w = [math.exp(s - mx) for s in sc]
    z = sum(w)
    return [sum(w[j] * vals[j][c] for j in range(len(vals))) / z for c in range(d)]


@pytest.mark.parametrize("B,L,h_q,h_kv,d", [(1, 5, 2, 1, 4), (2, 6, 4, 2, 8), (1, 4, 3, 3, 4)])
def test_prefill_matches_brute_force(B, L, h_q, h_kv, d):
    """Triple loop from the definition (page aicoding.csdn.net §4.1.2-4.1.3), 1-based grouping formula."""
    q, k, v = _small(B, L, h_q, h_kv, d, seed=B * 100 + L)
    theta = 10.0   # a small base makes every pair rotate visibly at these positions
    got = R.prefill_ref(q, k, v, theta)
    g = h_q // h_kv
    for b in range(B):
        for t1 in range(1, h_q + 1):
            u = (t1 - 1) // g + 1 - 1
            for i in range(L):
                keys = [list(k[b, j, u]) for j in range(i + 1)]
                vals = [list(v[b, j, u]) for j in range(i + 1)]
                ref = _bf_attend(list(q[b, i, t1 - 1]), i, keys, vals, theta, d)
                np.testing.assert_allclose(got[b, i, t1 - 1], ref, atol=1e-12)


def test_decode_matches_brute_force():
    h_q, h_kv, d = 4, 2, 8
    seqlens = [1, 3, 6]
    rng = np.random.default_rng(5)
    q = rng.standard_normal((3, h_q, d))
    kc = rng.standard_normal((10, h_kv, d))
    vc = rng.standard_normal((10, h_kv, d))
    got = R.decode_ref(q, kc, vc, seqlens, 10.0)
    off = 0
    for b, s in enumerate(seqlens):
        for t in range(h_q):
            u = t // (h_q // h_kv)
            ref = _bf_attend(list(q[b, t]), s, [list(kc[off + j, u]) for j in range(s)],
                             [list(vc[off + j, u]) for j in range(s)], 10.0, d)
            np.testing.assert_allclose(got[b, t], ref, atol=1e-12)
        off += s


def test_prefill_matches_torch_sdpa_fp64():
    """Library cross-check: torch SDPA (float64, causal) on K,V expanded per head, RoPE via complex numbers."""
    B, L, h_q, h_kv, d = 2, 40, 6, 3, 32
    q, k, v = _small(B, L, h_q, h_kv, d, seed=21)
    g = h_q // h_kv
    ang = np.arange(L)[:, None] * (THETA ** (-2.0 * np.arange(d // 2) / d))[None, :]
    w = np.exp(1j * ang)[None, :, None, :]

    def rot(x):
        z = (x[..., : d // 2] + 1j * x[..., d // 2:]) * w
        return np.concatenate([z.real, z.imag], axis=-1)

    qt = torch.from_numpy(rot(q)).permute(0, 2, 1, 3)
    kt = torch.from_numpy(np.repeat(rot(k), g, axis=2)).permute(0, 2, 1, 3)
    vt = torch.from_numpy(np.repeat(v, g, axis=2)).permute(0, 2, 1, 3)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True,
                                                           scale=1.0 / math.sqrt(d))
    np.testing.assert_allclose(R.prefill_ref(q, k, v, THETA), ref.permute(0, 2, 1, 3).numpy(),
                               atol=1e-12)


def test_prefill_rows_ref_matches_full():
    q, k, v = _small(B=2, L=70, h_q=4, h_kv=2, d=16)
    full = R.prefill_ref(q, k, v, THETA, row_block=16)
    rows = [0, 1, 15, 16, 33, 69]
    for b in range(2):
        for t in range(4):
            np.testing.assert_allclose(R.prefill_rows_ref(q, k, v, THETA, b, t, rows),
                                       full[b, rows, t], atol=1e-13)


def test_decode_self_reading_equals_last_prefill_row():
    """With the cache already holding token L-1 and q at L-1, decode == prefill row L-1."""
    q, k, v = _small(B=1, L=23, h_q=6, h_kv=2, d=16)
    pre = R.prefill_ref(q, k, v, THETA)
    dec = R.decode_ref(q[:, -1], k[0], v[0], [23], THETA, include_self=True)
    np.testing.assert_allclose(dec[0], pre[0, -1], atol=1e-13)


def test_decode_length_one_is_v0_and_zero_query_is_mean():
    rng = np.random.default_rng(9)
    q = rng.standard_normal((2, 4, 8))
    kc = rng.standard_normal((1 + 5, 2, 8))
    vc = rng.standard_normal((1 + 5, 2, 8))
    out = R.decode_ref(q, kc, vc, [1, 5], THETA)
    for t in range(4):
        assert np.array_equal(out[0, t], vc[0, t // 2])
    q[:] = 0
    out = R.decode_ref(q, kc, vc, [1, 5], THETA)
    for t in range(4):
        np.testing.assert_allclose(out[1, t], vc[1:6, t // 2].mean(axis=0), atol=1e-14)


def test_flop_and_byte_counts():
    assert R.prefill_flops(1, 128, 14, 64) == pytest.approx(2.959e7, rel=1e-3)
    assert R.prefill_flops(1, 4096, 28, 128) == pytest.approx(1.203e11, rel=1e-3)
    assert R.prefill_flops(4, 8192, 64, 128) == pytest.approx(4.399e12, rel=1e-3)
    assert R.prefill_flops(1, 32768, 28, 128) == pytest.approx(7.697e12, rel=1e-3)


def test_seeded_inputs_are_deterministic_bf16():
    w = gi.small("prefill", B=1, L=9, h_q=4, h_kv=2, d=8, seed=3)
    a = gi.prefill_inputs(w)
    b = gi.prefill_inputs(w)
    for x, y in zip(a, b):
        assert x.dtype == torch.bfloat16 and torch.equal(x, y)
    wd = gi.small("decode", B=3, max_len=50, h_q=4, h_kv=2, d=8, seed=3)
    s, q, kc, vc = gi.decode_inputs(wd)
    assert s.dtype == torch.int32 and int(s.min()) >= 1 and int(s.max()) <= 50
    assert kc.shape[0] == int(s.sum()) and vc.shape == kc.shape and q.shape == (3, 4, 8)


# ---------------------------------------------------------------- the pins catch planted mistakes
def _pins_pass(mod):
    """Run a subset of the pins against a (possibly mutated) oracle module; True if all pass."""
    try:
        q, k, v = _small(B=1, L=12, h_q=4, h_kv=2, d=8, seed=77)
        # brute force
        g = 2
        got = mod.prefill_ref(q, k, v, 10.0)
        for t in range(4):
            for i in range(12):
                u = t // g
                ref = _bf_attend(list(q[0, i, t]), i, [list(k[0, j, u]) for j in range(i + 1)],
                                 [list(v[0, j, u]) for j in range(i + 1)], 10.0, 8)
                if not np.allclose(got[0, i, t], ref, atol=1e-10):
                    return False
        # zero-query prefix means
        q0 = np.zeros_like(q)
        out = mod.prefill_ref(q0, k, v, THETA)
        csum = np.cumsum(v, axis=1) / np.arange(1, 13)[None, :, None, None]
        for t in range(4):
            if not np.allclose(out[:, :, t], csum[:, :, t // 2], atol=1e-12):
                return False
        # decode brute force
        dec = mod.decode_ref(q[0, -1:, :, :], k[0], v[0], [12], 10.0)
        ref = [_bf_attend(list(q[0, -1, t]), 12, [list(k[0, j, t // 2]) for j in range(12)],
                          [list(v[0, j, t // 2]) for j in range(12)], 10.0, 8) for t in range(4)]
        return bool(np.allclose(dec[0], np.array(ref), atol=1e-10))
    except Exception:
        return False


MUTATIONS = {
    "rope_sign": ("rope", lambda x, positions, theta: _mut_rope(x, positions, theta, sign=-1.0)),
    "rope_freq_uses_wrong_exponent": ("inv_freq", lambda d, theta: np.power(float(theta), -np.arange(d // 2) / d)),
    "group_modulo": ("head_group", lambda t, g: t % g),
    "mask_off_by_one": ("causal_weights", lambda qr, rp, kr: _mut_weights(qr, rp, kr, shift=1)),
    "no_scale": ("causal_weights", lambda qr, rp, kr: _mut_weights(qr, rp, kr, scale=1.0)),
}


def _mut_rope(x, positions, theta, sign):
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    h = d // 2
    ang = np.asarray(positions, dtype=np.float64)[:, None] * R.inv_freq(d, theta)[None, :]
    c = np.cos(ang)[:, None, :]
    s = sign * np.sin(ang)[:, None, :]
    return np.concatenate([x[..., :h] * c - x[..., h:] * s, x[..., h:] * c + x[..., :h] * s], -1)


def _mut_weights(qr, rp, kr, shift=0, scale=None):
    d = qr.shape[-1]
    s = (qr @ kr.T) * (scale if scale is not None else 1.0 / np.sqrt(d))
    j = np.arange(kr.shape[0])[None, :]
    s = np.where(j > np.asarray(rp)[:, None] - shift, -np.inf, s)
    return R.softmax_rows(s)


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name, monkeypatch):
    assert _pins_pass(R), "the unmutated oracle must pass the pins"
    attr, fn = MUTATIONS[name]
    monkeypatch.setattr(R, attr, fn)
    assert not _pins_pass(R), f"planted mistake {name} was not caught"
