"""Pins for oracle/gemm.py: a hand-summed case, exact integer arithmetic, rational brute force."""

from fractions import Fraction

import numpy as np
import torch

from oracle import fp8_formats as F
from oracle import gemm as G

from fp8_delayed_scaling_02_b200 import synthetic as S


def _codes(tokens):
    return np.array([int(t, 16) for t in tokens], dtype=np.uint8)


def test_golden_hand_gemm(golden):
    g = golden("gemm_nt_hand.txt")
    a = _codes(g["a_codes"]).reshape(2, 3)
    b = _codes(g["b_codes"]).reshape(2, 3)
    bias = np.array([float(v) for v in g["bias"]], np.float32)
    ref, Ssum = G.mm_fp8(a, b, F.E4M3, F.E4M3, float(g["sinv_a"][0]), float(g["sinv_b"][0]), bias)
    assert np.array_equal(ref.ravel(), np.array([float(v) for v in g["ref"]]))
    assert np.array_equal(Ssum.ravel(), np.array([float(v) for v in g["S"]]))


def test_e4m3_sum_exact_against_integer_matmul():
    """E4M3 values are multiples of 2^-9, so 2^9 * value is an integer; the int64
    product then gives the exact sum, which the float64 oracle must equal."""
    a = S.fp8_codes((37, 300), seed=1).numpy()
    b = S.fp8_codes((29, 300), seed=2).numpy()
    ai = (F.decode(a, F.E4M3) * 512).astype(np.int64)
    bi = (F.decode(b, F.E4M3) * 512).astype(np.int64)
    assert np.array_equal(ai, F.decode(a, F.E4M3) * 512)
    exact = ai @ bi.T  # int64, exact
    ref, _ = G.mm_fp8(a, b, F.E4M3, F.E4M3, 1.0, 1.0)
    assert np.array_equal(ref * (512 * 512), exact.astype(np.float64))


def test_mixed_formats_rational_brute_force():
    a = S.fp8_codes((3, 5), seed=3, fmt=F.E5M2).numpy()
    b = S.fp8_codes((4, 5), seed=4, fmt=F.E4M3).numpy()
    bias = np.array([0.5, -0.25, 3.0, 1e-3], np.float32)
    sa, sb = np.float32(0.37), np.float32(0.125)
    ref, Ssum = G.mm_fp8(a, b, F.E5M2, F.E4M3, sa, sb, bias)
    ta, tb = F.decode_table(F.E5M2), F.decode_table(F.E4M3)
    for i in range(3):
        for j in range(4):
            acc = sum(Fraction(ta[a[i, k]]) * Fraction(tb[b[j, k]]) for k in range(5))
            mag = sum(abs(Fraction(ta[a[i, k]]) * Fraction(tb[b[j, k]])) for k in range(5))
            sab = Fraction(float(sa)) * Fraction(float(sb))
            exact = acc * sab + Fraction(float(bias[j]))
            assert abs(Fraction(ref[i, j]) - exact) <= abs(exact) * Fraction(1, 2 ** 50)
            assert abs(Fraction(Ssum[i, j]) - mag * sab) <= mag * sab * Fraction(1, 2 ** 50)


def test_operand_orientation_non_square():
    """Y[i, j] = sum_k A[i, k] B[j, k]: a transposed operand would change the shape or values."""
    a = S.fp8_codes((2, 3), seed=5).numpy()
    b = S.fp8_codes((4, 3), seed=6).numpy()
    ref, _ = G.mm_fp8(a, b, F.E4M3, F.E4M3, 1.0, 1.0)
    assert ref.shape == (2, 4)
    ta = F.decode_table(F.E4M3)
    for i in range(2):
        for j in range(4):
            assert ref[i, j] == sum(ta[a[i, k]] * ta[b[j, k]] for k in range(3))


def test_batched_broadcast_equals_per_batch_loop():
    a = S.fp8_codes((3, 6, 32), seed=7).numpy()
    b = S.fp8_codes((1, 5, 32), seed=8).numpy()
    bias = S.uniform((5,), seed=9).numpy()
    ref, Ssum = G.mm_fp8(a, b, F.E4M3, F.E4M3, 0.5, 0.25, bias)
    assert ref.shape == (3, 6, 5)
    for z in range(3):
        r1, s1 = G.mm_fp8(a[z], b[0], F.E4M3, F.E4M3, 0.5, 0.25, bias)
        assert np.array_equal(ref[z], r1) and np.array_equal(Ssum[z], s1)


def test_rows_subset_matches_full():
    a = S.fp8_codes((20, 64), seed=10).numpy()
    b = S.fp8_codes((12, 64), seed=11).numpy()
    bias = S.uniform((12,), seed=12).numpy()
    full, fs = G.mm_fp8(a, b, F.E4M3, F.E4M3, 0.3, 0.7, bias)
    rows = np.array([0, 7, 19])
    sub, ss = G.mm_fp8_rows(a, b, F.E4M3, F.E4M3, 0.3, 0.7, bias, rows)
    assert np.array_equal(sub, full[rows]) and np.array_equal(ss, fs[rows])


def test_ulp_bf16_against_bit_successor():
    """ulp of bf16 at x equals next-representable minus x, found by incrementing bf16 bits."""
    xs = torch.tensor([1.0, 1.5, 2.0, 3.0, 255.0, 1e-3, 7e4, 2.0 ** -126, 1e-39], dtype=torch.bfloat16)
    nxt = (xs.view(torch.int16) + 1).view(torch.bfloat16)
    lib = (nxt.double() - xs.double()).numpy()
    ours = G.ulp_bf16(xs.double().numpy())
    assert np.array_equal(ours, lib)
    assert G.ulp_bf16(np.array([0.0]))[0] == 2.0 ** -133


def test_check_accepts_one_ulp_rejects_three():
    ref = np.array([100.0, -3.0])
    Ssum = np.zeros(2)
    assert G.check(ref + G.ulp_bf16(ref), ref, Ssum)[0]
    assert not G.check(ref + 3 * G.ulp_bf16(ref), ref, Ssum)[0]
    # The accumulation allowance widens the bound with sum |a.b|.
    assert G.check(ref + 2 * G.ulp_bf16(ref), ref, np.full(2, 2.0 ** 20 * 2.0))[0]
