"""Pins for oracle/recipe.py: hand-worked fixtures, closed-form ring invariants, brute force.

The expected scales are computed here with exact rationals and a correctly
rounded float32 search, not with numpy's float32 division that the oracle uses.
"""

import struct
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import fp8_formats as F
from oracle import recipe as R


def _bits(x):
    return struct.unpack("<I", struct.pack("<f", float(x)))[0]


def _from_bits(b):
    return struct.unpack("<f", struct.pack("<I", b))[0]


def _f32_rn(fr):
    """Correctly rounded float32 of a positive Fraction (nearest, ties to even bits)."""
    b0 = _bits(np.float32(float(fr)))
    best = None
    for b in range(b0 - 2, b0 + 3):
        d = abs(Fraction(_from_bits(b)) - fr)
        if best is None or d < best[0] or (d == best[0] and b % 2 == 0):
            best = (d, b)
    return _from_bits(best[1])


def test_golden_e4m3_two_calls(golden):
    g = golden("quantize_e4m3_hand.txt")
    ring = R.Ring()
    x1 = torch.tensor([float(v) for v in g["call1_x"]], dtype=torch.bfloat16)[None, :]
    out, out_t, a = R.quantize(x1, F.E4M3, R.ROW, ring)
    assert out_t is None
    assert [int(c) for c in out[0]] == [int(c, 16) for c in g["call1_codes"]]
    assert _bits(a) == int(g["call1_amax"][0], 16)
    assert ring.idx == int(g["call1_idx"][0])
    assert _bits(ring.scale) == int(g["call1_scale"][0], 16)
    assert _bits(ring.scale_inv) == int(g["call1_scale_inv"][0], 16)
    x2 = torch.tensor([float(v) for v in g["call2_x"]], dtype=torch.bfloat16)[None, :]
    out, _, a = R.quantize(x2, F.E4M3, R.ROW, ring)
    assert [int(c) for c in out[0]] == [int(c, 16) for c in g["call2_codes"]]
    assert _bits(a) == int(g["call2_amax"][0], 16)
    assert ring.idx == int(g["call2_idx"][0])
    assert _bits(ring.scale) == int(g["call2_scale"][0], 16)
    assert _bits(ring.scale_inv) == int(g["call2_scale_inv"][0], 16)
    assert ring.history[0] == 480.0 and ring.history[1] == 0.9375


def test_golden_e5m2(golden):
    g = golden("quantize_e5m2_hand.txt")
    ring = R.Ring()
    x = np.array([float(v) for v in g["x"]], dtype=np.float32)[None, :]
    out, _, a = R.quantize(x, F.E5M2, R.ROW, ring)
    assert [int(c) for c in out[0]] == [int(c, 16) for c in g["codes"]]
    assert _bits(a) == int(g["amax"][0], 16)
    assert _bits(ring.scale) == int(g["scale"][0], 16)
    assert _bits(ring.scale_inv) == int(g["scale_inv"][0], 16)


@pytest.mark.parametrize("fmt", [F.E4M3, F.E5M2])
def test_ring_closed_form_over_40_steps(fmt):
    """After step t the ring holds the last min(t+1,16) amaxes at slots (t-j) mod 16,
    the published scale is FP8_MAX / max(window) and scale_inv inverts the scale used."""
    rng = np.random.default_rng(3)
    fmax = Fraction(int(F.fp8_max(fmt)))
    ring = R.Ring()
    amaxes = []
    prev_scale = 1.0
    for t in range(40):
        mag = float(np.float32(rng.uniform(0.1, 5.0) * 10.0 ** rng.integers(-3, 4)))
        if t in (5, 6):
            mag = 0.0  # zero steps must not reset the window maximum
        x = np.float32(rng.uniform(-1, 1, size=(3, 5))) * np.float32(mag) / 2
        x[1, 2] = -mag
        out, _, a = R.quantize(x, fmt, R.ROW, ring)
        amaxes.append(np.float32(mag))
        assert a == np.float32(mag)
        window = amaxes[max(0, t - 15): t + 1]
        for j in range(len(window)):
            assert ring.history[(t - j) % 16] == amaxes[t - j]
        assert ring.idx == (t + 1) % 16
        m = max(window)
        expect = _f32_rn(fmax / Fraction(float(m))) if m > 0 else prev_scale
        assert ring.scale == np.float32(expect)
        assert ring.scale_inv == np.float32(_f32_rn(1 / Fraction(float(prev_scale))))
        prev_scale = float(ring.scale)


def test_zero_history_keeps_scale():
    ring = R.Ring(scale=0.5)
    for _ in range(3):
        out, _, a = R.quantize(np.zeros((4, 4), np.float32), F.E4M3, R.ROW, ring)
        assert a == 0 and ring.scale == np.float32(0.5)
        assert np.all(out == 0)
    R.quantize(np.full((1, 1), 2.0, np.float32), F.E4M3, R.ROW, ring)
    assert ring.scale == np.float32(224.0)


def test_empty_input_folds_zero():
    ring = R.Ring()
    out, out_t, a = R.quantize(np.zeros((0, 7), np.float32), F.E4M3, R.DUAL, ring)
    assert out.shape == (0, 7) and out_t.shape == (7, 0)
    assert a == 0 and ring.idx == 1 and ring.scale == 1.0


def test_amax_is_over_raw_values_not_scaled():
    """The pages' amax fix: amax of the scaled values was ~448 and collapsed the scale."""
    ring = R.Ring(scale=1000.0)
    x = np.array([[0.5, -1.0, 0.75]], np.float32)
    out, _, a = R.quantize(x, F.E4M3, R.ROW, ring)
    assert a == 1.0
    assert ring.scale == np.float32(448.0)
    assert np.all(out[0] == [0x7E, 0xFE, 0x7E])  # 500, -1000, 750 all saturate


def test_layouts_transpose_and_dual():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((5, 3)).astype(np.float32)
    r0 = R.Ring(scale=3.0)
    r1 = r0.copy()
    r2 = r0.copy()
    out, _, _ = R.quantize(x, F.E4M3, R.ROW, r0)
    _, out_t, _ = R.quantize(x, F.E4M3, R.TRANSPOSED, r1)
    d, d_t, _ = R.quantize(x, F.E4M3, R.DUAL, r2)
    assert out.shape == (5, 3) and out_t.shape == (3, 5)
    for r in range(5):
        for c in range(3):
            assert out_t[c, r] == out[r, c]
    assert np.array_equal(d, out) and np.array_equal(d_t, out_t)
    assert r0.scale == r1.scale == r2.scale


def test_elementwise_codes_brute_force_with_fp32_product():
    """q = nearest FP8 to the float32-rounded product, for a scale that is not a power of 2."""
    rng = np.random.default_rng(11)
    x = (rng.standard_normal((4, 9)) * 30).astype(np.float32)
    scale = np.float32(0.7301)
    ring = R.Ring(scale=scale)
    out, _, _ = R.quantize(x, F.E5M2, R.ROW, ring)
    t = F.decode_table(F.E5M2)
    fin = [c for c in range(0x80) if np.isfinite(t[c])]
    for (i, j), v in np.ndenumerate(x):
        p = _f32_rn(abs(Fraction(float(v)) * Fraction(float(scale))))
        best = min(fin, key=lambda c: (abs(Fraction(t[c]) - Fraction(p)), c & 1))
        assert out[i, j] == (best | (0x80 if v < 0 else 0))


def test_no_scale_ratio_leak_across_steps():
    """Dequantising with scale_inv of the step recovers x to FP8 precision, whatever the scale."""
    ring = R.Ring()
    rng = np.random.default_rng(5)
    for step, mag in enumerate([1.0, 40.0, 0.02, 3.0]):
        x = (rng.uniform(-1, 1, (8, 8)) * mag).astype(np.float32)
        x[0, 0] = mag
        out, _, _ = R.quantize(x, F.E4M3, R.ROW, ring)
        deq = F.decode(out, F.E4M3) * float(ring.scale_inv)
        used = 1.0 / float(ring.scale_inv)
        in_range = np.abs(x * used) <= 448
        normal = np.abs(x * used) >= 2.0 ** -6
        sel = in_range & normal
        assert np.all(np.abs(deq[sel] - x[sel]) <= np.abs(x[sel]) * 2.0 ** -4 + 1e-30)


def test_nan_history_entry_is_ignored_by_the_window_max():
    """A NaN amax (only a caller-supplied amax can be one) is stored in its slot
    and skipped by the window maximum, like NaN elements in the amax itself:
    the scale is the one the same history without that entry gives, computed
    here with exact rationals."""
    for fmt, fmax in ((F.E4M3, 448), (F.E5M2, 57344)):
        ring = R.Ring()
        R.fold(ring, np.float32(3.0), fmt)
        s_before = ring.scale
        R.fold(ring, np.float32(np.nan), fmt)
        assert np.isnan(ring.history[1]) and ring.idx == 2
        assert _bits(ring.scale) == _bits(s_before) == _bits(_f32_rn(Fraction(fmax) / Fraction(3)))
        R.fold(ring, np.float32(0.75), fmt)  # a smaller finite amax: the max stays 3
        assert _bits(ring.scale) == _bits(_f32_rn(Fraction(fmax) / Fraction(3)))
        # Only NaN in the window: the maximum is 0 and the scale is kept.
        only = R.Ring(scale=0.625)
        R.fold(only, np.float32(np.nan), fmt)
        assert only.scale == np.float32(0.625) and only.scale_inv == np.float32(1.6)


@pytest.mark.parametrize("layout", [R.ROW, R.TRANSPOSED, R.DUAL])
@pytest.mark.parametrize("fmt", [F.E4M3, F.E5M2])
def test_quantize_local_then_fold_equals_quantize(layout, fmt):
    """The data-parallel split of a call: quantize_local leaves the ring alone,
    casts with the ring's scale and returns the raw amax and 1/scale; folding
    that amax gives the ring of one quantize call, and the codes are its codes.
    Checked over 5 delayed steps whose amax moves by orders of magnitude, so a
    cast with the post-fold scale or a stale scale_inv is caught."""
    ring_a, ring_b = R.Ring(), R.Ring()
    for step in range(5):
        g = torch.Generator().manual_seed(step)
        x = (torch.randn((37, 53), generator=g) * 10.0 ** (2 * (step % 3) - 2)).to(torch.bfloat16)
        before = (ring_b.history.copy(), ring_b.idx, ring_b.scale, ring_b.scale_inv)
        o1, t1, a1 = R.quantize(x, fmt, layout, ring_a)
        o2, t2, a2, sinv = R.quantize_local(x, fmt, layout, ring_b)
        assert np.array_equal(ring_b.history, before[0]) and ring_b.idx == before[1]
        assert ring_b.scale == before[2] and ring_b.scale_inv == before[3], "quantize_local must not touch the ring"
        assert _bits(a2) == _bits(np.max(np.abs(x.float().numpy())))
        assert _bits(sinv) == _bits(_f32_rn(1 / Fraction(float(ring_b.scale))))
        R.fold(ring_b, a2, fmt)
        for u, v in ((o1, o2), (t1, t2)):
            assert (u is None) == (v is None)
            if u is not None:
                assert np.array_equal(u, v)
        assert _bits(a1) == _bits(a2)
        assert np.array_equal(ring_a.history.view(np.uint32), ring_b.history.view(np.uint32))
        assert ring_a.idx == ring_b.idx
        assert _bits(ring_a.scale) == _bits(ring_b.scale) and _bits(ring_a.scale_inv) == _bits(ring_b.scale_inv)
        assert _bits(ring_b.scale_inv) == _bits(sinv)
    assert ring_b.scale != np.float32(1.0)
