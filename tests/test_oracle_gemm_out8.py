"""Pins for the FP8-bias and FP8-output parts of oracle/gemm.py.

The hand-worked fixture fixes the whole chain (bias dequantisation, product,
output cast with the ring's scale, amax, ring fold) on values whose float32
arithmetic is exact; the rest checks the acceptance interval against brute
force and planted mistakes.
"""

from fractions import Fraction

import numpy as np

from oracle import fp8_formats as F
from oracle import gemm as G
from oracle import recipe as R


def _codes(tokens):
    return np.array([int(t, 16) for t in tokens], dtype=np.uint8)


def _f(tokens):
    return np.array([float(t) for t in tokens])


def test_golden_hand_fp8_bias_and_fp8_output(golden):
    g = golden("gemm_out8_hand.txt")
    a = _codes(g["a_codes"]).reshape(2, 3)
    b = _codes(g["b_codes"]).reshape(2, 3)
    bias = G.bias_from_fp8(_codes(g["bias_codes"]), F.E4M3, float(g["bias_scale"][0]))
    assert np.array_equal(bias, _f(g["bias"]).astype(np.float32))
    ref, S = G.mm_fp8(a, b, F.E4M3, F.E4M3, float(g["sinv_a"][0]), float(g["sinv_b"][0]), bias)
    assert np.array_equal(ref.ravel(), _f(g["ref"]))
    assert np.array_equal(S.ravel(), _f(g["S"]))
    amax, tol = G.amax_range(ref, S)
    assert amax == float(g["amax"][0]) and 0 < tol < 1e-4
    for fmt, key in ((F.E4M3, "e4m3"), (F.E5M2, "e5m2")):
        s = float(g[f"{key}_scale"][0])
        # every value here is exact in float32, so the code is the definition's
        codes = R.scaled_codes(ref.astype(np.float32), s, fmt)
        assert np.array_equal(codes.ravel(), _codes(g[f"{key}_out"]))
        lo, hi = G.out8_code_range(ref, S, s, fmt)
        assert np.all(G.codes_within(codes, lo, hi, fmt))
        ring = R.Ring(scale=s)
        R.fold(ring, np.float32(amax), fmt)
        assert ring.history[0] == np.float32(19.0) and ring.idx == 1
        assert int(np.float32(ring.scale).view(np.uint32)) == int(g[f"{key}_next_scale_bits"][0], 16)
        assert ring.scale_inv == np.float32(float(g[f"{key}_scale_inv"][0]))


def test_bias_from_fp8_every_code_against_exact_products():
    """fp32(decode(c) * s) for every finite code of both formats and four
    scales: the float64 product of a <= 4-bit and a 24-bit significand is
    exact, so one rounding to float32 gives the correctly rounded value."""
    for fmt in (F.E4M3, F.E5M2):
        codes = np.arange(256, dtype=np.uint8)
        keep = np.isfinite(F.decode(codes, fmt))
        codes = codes[keep]
        for s in (1.0, 2.0 ** -3, 0.3, 3.7e-5):
            s32 = np.float32(s)
            exact = np.array([Fraction(float(v)) * Fraction(float(s32)) for v in F.decode(codes, fmt)])
            want = np.array([np.float32(float(e)) for e in exact], dtype=np.float32)  # float(Fraction) is exact here
            assert np.array_equal(G.bias_from_fp8(codes, fmt, s), want)


def test_out8_range_contains_every_float32_inside_the_bound():
    """Brute force: float32 values spread over [ref - b, ref + b] all encode
    inside (lo, hi), and lo / hi are the codes of the two ends (tight)."""
    rng = np.random.default_rng(5)
    ref = rng.normal(size=400) * np.exp2(rng.integers(-12, 10, 400))
    S = np.abs(ref) * rng.uniform(1, 4000, 400)
    for fmt in (F.E4M3, F.E5M2):
        for s in (1.0, 0.37, 2.0 ** 6):
            lo, hi = G.out8_code_range(ref, S, s, fmt)
            b = G.bound_f32(ref, S)
            for t in np.linspace(-1, 1, 41):
                y = (ref + t * b).astype(np.float32)
                inside = np.abs(y.astype(np.float64) - ref) <= b
                c = R.scaled_codes(y, s, fmt)
                assert np.all(G.codes_within(c, lo, hi, fmt)[inside])
            ends = [R.scaled_codes((ref - b).astype(np.float32), s, fmt), R.scaled_codes((ref + b).astype(np.float32), s, fmt)]
            assert np.array_equal(lo, ends[0]) and np.array_equal(hi, ends[1])


def test_out8_range_rejects_a_code_one_step_off():
    """Planted mistakes: away from rounding boundaries the range is one code,
    and its neighbours (one code up or down in magnitude) fall outside."""
    vals = np.array([1.0, 3.0, 40.0, -6.0, 0.125, 300.0])  # no ties in either format
    S = np.abs(vals)
    for fmt in (F.E4M3, F.E5M2):
        lo, hi = G.out8_code_range(vals, S, 1.0, fmt)
        exact = R.scaled_codes(vals.astype(np.float32), 1.0, fmt)
        assert np.array_equal(lo, exact) and np.array_equal(hi, exact)
        up = (exact & 0x80) | ((exact & 0x7F) + 1)
        down = (exact & 0x80) | ((exact & 0x7F) - 1)
        assert not np.any(G.codes_within(up.astype(np.uint8), lo, hi, fmt))
        assert not np.any(G.codes_within(down.astype(np.uint8), lo, hi, fmt))


def test_bound_f32_terms():
    """Closed form: 2^-20 * S + 2^-23 * |ref| + 2^-149."""
    assert G.bound_f32(8.0, 2.0 ** 20) == 1.0 + 2.0 ** -20 + 2.0 ** -149
    assert G.bound_f32(0.0, 0.0) == 2.0 ** -149
    assert G.amax_range(np.zeros((0, 3)), np.zeros((0, 3))) == (0.0, 0.0)
    assert G.amax_range(np.array([[1.0, -7.5], [2.0, 0.0]]), np.zeros((2, 2)))[0] == 7.5
