"""Pins for the oracle's rotated-cache decode and rotated append (CPU only).

A cache that keeps its keys after RoPE (each row rotated at its own position when it was written) must
give the decode the same scores as a cache of raw keys rotated on load: the rotation of a key depends only
on its position, not on when it is applied (aicoding.csdn.net page, §4.1.3: RoPE acts on Q and K before
the dot product; closing paragraph: the cache holds the h_kv groups' keys).  The rotated rows here come
from an independent complex-number restatement of the rotation (pair i = dims i and i + d/2, angle m f_i,
f_i = theta^(-2i/d); intelliparadigm.com page, §2.3), and the decode is checked against a pure-Python brute
force on the raw cache, not against the oracle's own rope().
"""
import cmath
import math

import numpy as np
import pytest

from oracle import gqa_ref as R


def rotate_row(x, m, theta):
    """x [d] rotated at position m, as complex pairs z_i = x_i + j x_{i+d/2} times e^{j m f_i}."""
    d = len(x)
    h = d // 2
    out = [0.0] * d
    for i in range(h):
        z = complex(x[i], x[i + h]) * cmath.exp(1j * m * theta ** (-2.0 * i / d))
        out[i], out[i + h] = z.real, z.imag
    return out


def brute_decode(q, kcache, vcache, seqlens, theta, include_self=False):
    """Pure-Python decode on raw caches: rotate q at its position and every key at its row index."""
    B, h_q, d = q.shape
    h_kv = kcache.shape[1]
    g = h_q // h_kv
    out = np.zeros((B, h_q, d))
    off = 0
    for b in range(B):
        s = int(seqlens[b])
        p = s - 1 if include_self else s
        for t in range(h_q):
            u = t // g
            qr = rotate_row(list(q[b, t]), p, theta)
            sc = []
            for j in range(s):
                kr = rotate_row(list(kcache[off + j, u]), j, theta)
                sc.append(sum(a * c for a, c in zip(qr, kr)) / math.sqrt(d))
            mx = max(sc)
            w = [math.exp(x - mx) for x in sc]
            z = sum(w)
            for j in range(s):
                out[b, t] += (w[j] / z) * vcache[off + j, u]
        off += s
    return out


def rotated_cache(kcache, seqlens, theta):
    """The packed cache with every row rotated at its position within its sequence (complex restatement)."""
    out = np.array(kcache, dtype=np.float64, copy=True)
    off = 0
    for s in seqlens:
        for j in range(int(s)):
            for u in range(out.shape[1]):
                out[off + j, u] = rotate_row(list(kcache[off + j, u]), j, theta)
        off += int(s)
    return out


@pytest.mark.parametrize("include_self", [False, True])
@pytest.mark.parametrize("h_q,h_kv,d", [(4, 2, 8), (6, 1, 16), (3, 3, 4)])
def test_rotated_cache_decode_matches_brute_force_on_raw_cache(include_self, h_q, h_kv, d):
    rng = np.random.default_rng(h_q * 100 + d + include_self)
    seqlens = [5, 1, 9]
    N = sum(seqlens)
    q = rng.standard_normal((3, h_q, d))
    kc = rng.standard_normal((N, h_kv, d))
    vc = rng.standard_normal((N, h_kv, d))
    theta = 1.0e4
    expect = brute_decode(q, kc, vc, seqlens, theta, include_self)
    got = R.decode_ref(q, rotated_cache(kc, seqlens, theta), vc, seqlens, theta, include_self=include_self,
                       k_rotated=True)
    np.testing.assert_allclose(got, expect, rtol=0, atol=1e-12)


def test_rotated_paged_cache_matches_rotated_packed_cache():
    rng = np.random.default_rng(11)
    seqlens = [7, 3, 12]
    h_q, h_kv, d, page = 4, 2, 8, 4
    N = sum(seqlens)
    q = rng.standard_normal((3, h_q, d))
    kc = rotated_cache(rng.standard_normal((N, h_kv, d)), seqlens, 1.0e6)
    vc = rng.standard_normal((N, h_kv, d))
    # scatter the packed rows over pages in a scrambled order
    n_pages = sum((s + page - 1) // page for s in seqlens) + 2
    perm = rng.permutation(n_pages)
    kp = rng.standard_normal((n_pages, page, h_kv, d))
    vp = rng.standard_normal((n_pages, page, h_kv, d))
    bt = np.full((3, 4), -1, dtype=np.int64)
    nxt, off = 0, 0
    for b, s in enumerate(seqlens):
        for pi in range((s + page - 1) // page):
            bt[b, pi] = perm[nxt]
            nxt += 1
        for j in range(s):
            kp[bt[b, j // page], j % page] = kc[off + j]
            vp[bt[b, j // page], j % page] = vc[off + j]
        off += s
    packed = R.decode_ref(q, kc, vc, seqlens, 1.0e6, k_rotated=True)
    paged = R.decode_paged_ref(q, kp, vp, bt, seqlens, 1.0e6, k_rotated=True)
    np.testing.assert_array_equal(paged, packed)


def test_rotated_cache_under_yarn_equals_raw_cache_under_yarn():
    """With YaRN the cache keeps rope(k) as the oracle's rope defines it (scaled frequencies and the
    temperature on the row), so the two caches still give the same decode."""
    rng = np.random.default_rng(5)
    seqlens = [40, 17]
    N = sum(seqlens)
    q = rng.standard_normal((2, 4, 16))
    kc = rng.standard_normal((N, 2, 16))
    vc = rng.standard_normal((N, 2, 16))
    yarn = R.Yarn(base=1.0e6, factor=4.0, original_max=16)
    off = R.packed_offsets(seqlens)
    kr = np.concatenate([R.rope(kc[off[b]:off[b + 1]], np.arange(seqlens[b]), yarn) for b in range(2)])
    np.testing.assert_allclose(R.decode_ref(q, kr, vc, seqlens, yarn, k_rotated=True),
                               R.decode_ref(q, kc, vc, seqlens, yarn), rtol=0, atol=1e-12)


def test_rotated_append_stores_the_key_rotated_at_its_position():
    rng = np.random.default_rng(9)
    B, h_q, h_kv, d, dm, page = 3, 4, 2, 8, 12, 4
    x = rng.standard_normal((B, dm))
    w = rng.standard_normal(((h_q + 2 * h_kv) * d, dm))
    bias = rng.standard_normal((h_q + 2 * h_kv) * d)
    seqlens = np.array([0, 5, 9])
    bt = np.array([[0, 1, 2], [3, 4, 5], [6, 7, 8]])
    kp = np.zeros((9, page, h_kv, d))
    vp = np.zeros((9, page, h_kv, d))
    q0, k0, v0 = R.qkv_append_ref(x, w, bias, h_q, h_kv, d, seqlens, kp, vp, bt)
    q1, k1, v1 = R.qkv_append_ref(x, w, bias, h_q, h_kv, d, seqlens, kp, vp, bt, rotate_k=True, theta=1.0e4)
    np.testing.assert_array_equal(q1, q0)
    np.testing.assert_array_equal(v1, v0)
    for b in range(B):
        pos = int(seqlens[b])
        slot = (bt[b, pos // page], pos % page)
        for u in range(h_kv):
            np.testing.assert_allclose(k1[slot][u], rotate_row(list(k0[slot][u]), pos, 1.0e4), rtol=0, atol=1e-12)
    untouched = np.ones(k1.shape[:2], dtype=bool)
    for b in range(B):
        untouched[bt[b, int(seqlens[b]) // page], int(seqlens[b]) % page] = False
    np.testing.assert_array_equal(k1[untouched], k0[untouched])


def test_planted_mistake_rotating_a_rotated_cache_again_is_caught():
    """Treating a rotated cache as raw (rotating its keys a second time) must fail the brute force."""
    rng = np.random.default_rng(3)
    seqlens = [6, 4]
    N = sum(seqlens)
    q = rng.standard_normal((2, 4, 8))
    kc = rng.standard_normal((N, 2, 8))
    vc = rng.standard_normal((N, 2, 8))
    expect = brute_decode(q, kc, vc, seqlens, 1.0e4)
    wrong = R.decode_ref(q, rotated_cache(kc, seqlens, 1.0e4), vc, seqlens, 1.0e4)   # k_rotated left off
    assert np.abs(wrong - expect).max() > 1e-3
