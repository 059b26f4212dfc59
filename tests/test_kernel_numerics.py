"""CPU checks of two numeric shortcuts inside the CUDA kernels, each restated here in fp32 NumPy.

The attention and decode parity tests cover these only end to end; here each is held to a bound of
its own, with the constants read from the kernel sources so the check follows the built code:

* exp2_poly / exp2_poly_x2 (the part of the softmax exponentials computed on the FMA pipe): a degree-3
  polynomial for 2^f on f in [-1/2, 1/2] after the range reduction 2^x = 2^n 2^f, n = round(x), with
  the 2^n applied by an integer add to the exponent field and x clamped below at -125.
* The decode kernel's RoPE angle recurrence: each lane starts from exact cos/sin of its row's angles
  and advances them 8 positions at a time by the angle-addition formulas in fp32, two steps per
  16-row block, re-anchored to exact values every REANCHOR blocks.  The drift after a full run of
  steps, at positions up to 32767 (the Qwen2 window of 32K positions, page "Qwen2 architecture
  introduction", aicoding.csdn.net, §5.1), must stay far below the bf16 rounding of the rotated keys.
"""
import os
import re

import numpy as np

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "grouped_query_attention_gqa_b200", "csrc")

f32 = np.float32


def _src(name):
    with open(os.path.join(CSRC, name), encoding="utf-8") as f:
        return f.read()


def _poly_coeffs():
    """(c3, c2, c1, c0) of exp2_poly, in the order the kernel's Horner steps use them."""
    body = re.search(r"float exp2_poly\(float x\) \{(.*?)\n\}", _src("sm100_ptx.cuh"), re.S).group(1)
    m1 = re.search(r"fmaf\(f, ([0-9.eE+-]+)f, ([0-9.eE+-]+)f\)", body)
    m2 = re.findall(r"fmaf\(p, f, ([0-9.eE+-]+)f\)", body)
    assert m1 and len(m2) == 2, "exp2_poly no longer has the expected Horner form"
    return f32(m1.group(1)), f32(m1.group(2)), f32(m2[0]), f32(m2[1])


def _fma32(a, b, c):
    # a*b is exact in float64 for float32 operands; one rounding of the sum to float32
    return (np.asarray(a, np.float64) * np.asarray(b, np.float64) + np.asarray(c, np.float64)).astype(f32)


def exp2_poly(x):
    """The kernel's exp2_poly, step for step in fp32."""
    c3, c2, c1, c0 = _poly_coeffs()
    x = np.maximum(np.asarray(x, f32), f32(-125.0))
    magic = f32(12582912.0)   # 1.5 * 2^23
    t = (x + magic).astype(f32)
    r = (t - magic).astype(f32)
    fr = (x - r).astype(f32)
    p = _fma32(fr, c3, c2)
    p = _fma32(p, fr, c1)
    p = _fma32(p, fr, c0)
    n = t.view(np.int32).astype(np.int64) - 0x4B400000
    return (p.view(np.int32).astype(np.int64) + (n << 23)).astype(np.int32).view(f32)


def test_exp2_poly_relative_error_on_the_reduced_interval():
    f = np.linspace(-0.5, 0.5, 200001, dtype=np.float64).astype(f32)
    got = exp2_poly(f).astype(np.float64)
    rel = np.abs(got / np.exp2(f.astype(np.float64)) - 1.0)
    assert rel.max() <= 7.5e-5, rel.max()
    # the fit is worth its name: equioscillating near its bound, not far inside it by luck
    assert rel.max() >= 6.5e-5


def test_exp2_poly_scales_by_powers_of_two():
    # Integers: the polynomial at 0 times 2^n; the exponent add must not be off by one anywhere.
    c0 = _poly_coeffs()[3]
    for n in range(-125, 128):
        got = exp2_poly(f32(n))
        assert got == np.ldexp(np.float64(c0), n).astype(f32), n
    # Half-integers and everything between, over the range the softmax uses (x <= 0) and beyond.
    rng = np.random.default_rng(5)
    x = np.concatenate([rng.uniform(-124.0, 100.0, 200000), np.arange(-124, 100) + 0.5,
                        np.arange(-124, 100) - 0.5]).astype(f32)
    rel = np.abs(exp2_poly(x).astype(np.float64) / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() <= 7.6e-5, rel.max()


def test_exp2_poly_clamp_at_minus_125():
    low = exp2_poly(f32(-125.0))
    for x in (-125.5, -126.0, -200.0, -1e30, -np.inf):
        got = exp2_poly(f32(x))
        assert got == low, x          # clamped, so never a denormal or a wrapped exponent
    assert 0.0 < low < 3e-38          # 2^-125 * p(0): tiny but NOT zero, which is why masked
    assert np.isfinite(low)           # scores never take this path in the kernel


# ------------------------------------------------------------------------ decode RoPE recurrence
def _decode_consts():
    s = _src("decode_sm100.cuh")
    rows = int(re.search(r"constexpr int ROWS = (\d+);", s).group(1))
    reanchor = int(re.search(r"constexpr int REANCHOR = (\d+);", s).group(1))
    return rows, reanchor


def _rot_step(C, S, Cr, Sr):
    """The kernel's rot_step in fp32: C' = C Cr - S Sr (two products, one subtraction),
    S' = fma(S, Cr, C Sr)."""
    c2 = ((C * Cr).astype(f32) - (S * Sr).astype(f32)).astype(f32)
    s2 = _fma32(S, Cr, (C * Sr).astype(f32))
    return c2, s2


def test_decode_rope_recurrence_drift_is_bounded():
    rows, reanchor = _decode_consts()
    assert rows == 16   # two 8-position steps per block, as restated here
    d, theta = 128, 1.0e6
    i = np.arange(d // 2, dtype=np.float64)
    freq = theta ** (-2.0 * i / d)                  # fp64 frequencies, as the kernel keeps them
    step8 = 8.0 * freq
    Cr, Sr = np.cos(step8).astype(f32), np.sin(step8).astype(f32)   # the per-step rotation, rounded
    worst = 0.0
    # Anchors at the start of the window, in the middle and as late as a run of REANCHOR blocks can
    # start below 32768, for every lane row offset t4 in 0..7.
    last = 32768 - rows * reanchor
    for anchor in (0, 1, 4093, 16384, last - 7, last):
        for t4 in range(8):
            pos0 = anchor + t4
            C = np.cos(pos0 * freq).astype(f32)     # exact anchor (the kernel's accurate sincos)
            S = np.sin(pos0 * freq).astype(f32)
            pos = pos0
            for _ in range(2 * reanchor):
                C, S = _rot_step(C, S, Cr, Sr)
                pos += 8
                err = max(np.abs(C - np.cos(pos * freq)).max(), np.abs(S - np.sin(pos * freq)).max())
                worst = max(worst, err)
            assert pos <= 32767 + 16
    # 2 * REANCHOR steps of a few fp32 roundings each (about 5e-6 measured); the rotated key is then
    # rounded to bf16 (relative 2^-9 = 2e-3), more than a hundred times coarser than the bound.
    assert worst <= 1.5e-5, worst


def test_decode_rope_recurrence_without_reanchoring_would_drift():
    # The bound above is not met by accident: running the same recurrence 64 times longer (no
    # re-anchoring over a whole 32K window) exceeds it.
    d, theta = 128, 1.0e6
    freq = theta ** (-2.0 * np.arange(d // 2) / d)
    Cr, Sr = np.cos(8.0 * freq).astype(f32), np.sin(8.0 * freq).astype(f32)
    C, S = np.ones(d // 2, f32), np.zeros(d // 2, f32)
    for _ in range(4096):
        C, S = _rot_step(C, S, Cr, Sr)
    pos = 8 * 4096
    err = max(np.abs(C - np.cos(pos * freq)).max(), np.abs(S - np.sin(pos * freq)).max())
    assert err > 1.5e-5, err
