"""Pins of the YaRN-scaled RoPE in the oracle (yudonglee.me page, §6.2: per-dimension interpolation
f_i / s * alpha_i with a ramp alpha_i from 1 to s; aicoding.csdn.net page, §5.3: a length-dependent
rescaling of the attention logits; §5.5: behaviour within the trained window unchanged).  The ramp bounds
and the temperature come from the published YaRN method, not the pages: these tests pin what the pages fix
(factor 1 is plain RoPE; slow pairs are interpolated by s, fast pairs kept; logits rescaled) and the
method's limits.  The constants themselves -- the ramp bounds of 1 and 32 turns and the temperature
0.1 ln s + 1 -- are parity unpinned by the pages: nothing on them fixes those numbers, and the tests that
mention them are consistency checks of the oracle's own choice."""
import numpy as np
import pytest

from oracle import gqa_ref as R

BASE, L0 = 1.0e6, 32768


def test_factor_one_is_plain_rope_exactly():
    rng = np.random.default_rng(1)
    q, k, v = rng.standard_normal((1, 9, 4, 16)), rng.standard_normal((1, 9, 2, 16)), rng.standard_normal((1, 9, 2, 16))
    y = R.Yarn(BASE, 1.0, L0)
    assert np.array_equal(R.inv_freq(16, y), R.inv_freq(16, BASE))
    assert R.rope_mscale(y) == 1.0
    assert np.array_equal(R.prefill_ref(q, k, v, y), R.prefill_ref(q, k, v, BASE))


@pytest.mark.parametrize("d,s,l0", [(128, 4.0, 32768), (64, 8.0, 4096), (128, 2.0, 8192)])
def test_ramp_keeps_fast_pairs_and_interpolates_slow_pairs(d, s, l0):
    f = R.inv_freq(d, BASE)
    fy = R.inv_freq(d, R.Yarn(BASE, s, l0))
    turns = l0 * f / (2 * np.pi)
    fast, slow = turns >= 32.0, turns <= 1.0
    assert fast.any() and slow.any()
    np.testing.assert_allclose(fy[fast], f[fast], rtol=1e-15)
    np.testing.assert_allclose(fy[slow], f[slow] / s, rtol=1e-15)
    alpha = fy / f * s                        # the pages' form: f' = f / s * alpha
    assert np.all(alpha >= 1.0 - 1e-12) and np.all(alpha <= s + 1e-12)
    mid = ~fast & ~slow
    assert np.all((alpha[mid] > 1.0) & (alpha[mid] < s))
    assert np.all(np.diff(alpha) <= 1e-12)    # frequencies fall with i, and so does alpha


def test_slow_pairs_at_position_p_turn_like_plain_rope_at_p_over_s():
    d, s = 64, 4.0
    y = R.Yarn(BASE, s, 4096)
    slow = 4096 * R.inv_freq(d, BASE) / (2 * np.pi) <= 1.0
    x = np.random.default_rng(2).standard_normal((3, 1, d))
    pos = np.array([5.0, 1000.0, 77777.0])
    a = R.rope(x, pos, y) / R.rope_mscale(y)
    b = R.rope(x, pos / s, BASE)
    h = d // 2
    idx = np.concatenate([np.where(slow)[0], np.where(slow)[0] + h])
    np.testing.assert_allclose(a[..., idx], b[..., idx], atol=1e-12)


def test_temperature_consistency_logits_scale_by_the_square_of_the_row_factor():
    """A consistency check, not a pin: the value m = rope_mscale(y) = 0.1 ln s + 1 is the published YaRN
    method's, which the pages do not give (parity unpinned by the pages), and it is restated here.  What
    this does check is how the oracle applies it: as a factor on every rotated Q and K row, so that the
    scores, and only the scores, scale by m^2.  With a huge original window every pair turns >= 32
    times, so no frequency changes and only the temperature remains: attention = softmax(m^2 * plain
    scores) V."""
    rng = np.random.default_rng(3)
    L, h_q, h_kv, d = 7, 2, 1, 16
    q, k, v = rng.standard_normal((1, L, h_q, d)), rng.standard_normal((1, L, h_kv, d)), rng.standard_normal((1, L, h_kv, d))
    y = R.Yarn(BASE, 4.0, 10 ** 12)
    assert np.allclose(R.inv_freq(d, y), R.inv_freq(d, BASE), rtol=0, atol=0)
    got = R.prefill_ref(q, k, v, y)
    m2 = (0.1 * np.log(4.0) + 1.0) ** 2
    pos = np.arange(L)
    qr, kr = R.rope(q[0], pos, BASE), R.rope(k[0], pos, BASE)
    for t in range(h_q):
        sc = m2 * (qr[:, t] @ kr[:, 0].T) / np.sqrt(d)
        sc = np.where(pos[None, :] > pos[:, None], -np.inf, sc)
        a = np.exp(sc - sc.max(1, keepdims=True))
        a /= a.sum(1, keepdims=True)
        np.testing.assert_allclose(got[0, :, t], a @ v[0, :, 0], atol=1e-12)


def _yarn_pins_pass(freq_fn, mscale_fn):
    try:
        for d, s, l0 in [(128, 4.0, 32768), (64, 8.0, 4096)]:
            f, fy = R.inv_freq(d, BASE), freq_fn(d, R.Yarn(BASE, s, l0))
            turns = l0 * f / (2 * np.pi)
            if not (np.allclose(fy[turns >= 32], f[turns >= 32], rtol=1e-14)
                    and np.allclose(fy[turns <= 1], f[turns <= 1] / s, rtol=1e-14)):
                return False
        return abs(mscale_fn(R.Yarn(BASE, 4.0, L0)) ** 2 - (0.1 * np.log(4.0) + 1.0) ** 2) < 1e-15
    except Exception:
        return False


def test_yarn_pins_catch_planted_mistakes():
    assert _yarn_pins_pass(R.inv_freq, R.rope_mscale)

    def ramp_reversed(d, y):
        f = R.inv_freq(d, y.base)
        g = 1.0 - np.clip((y.original_max * f / (2 * np.pi) - 1.0) / 31.0, 0, 1)
        return f / y.factor * (1 + g * (y.factor - 1))

    def factor_multiplied(d, y):
        return R.inv_freq(d, y) * y.factor ** 2

    assert not _yarn_pins_pass(ramp_reversed, R.rope_mscale)
    assert not _yarn_pins_pass(factor_multiplied, R.rope_mscale)
    assert not _yarn_pins_pass(R.inv_freq, lambda y: np.sqrt(R.rope_mscale(y)))   # temperature on one side only
