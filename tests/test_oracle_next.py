"""Pins for the oracle's current-scaling quantize and bias-gradient sums."""

import numpy as np
import torch

from oracle import bias_grad as B
from oracle import fp8_formats as F
from oracle import recipe as R

from fp8_delayed_scaling_02_b200 import synthetic as S


def test_current_scaling_maps_amax_to_the_largest_code():
    """scale = FP8_MAX / amax, so the amax element lands on the largest finite code."""
    for fmt, top in ((F.E4M3, 0x7E), (F.E5M2, 0x7B)):
        for seed in range(5):
            x = S.quant_sweep_input(17, 33, "fp32", 10.0 ** (seed - 2), seed=seed)
            out, out_t, a, s, si = R.quantize_current(x, fmt, R.DUAL)
            idx = np.unravel_index(np.argmax(np.abs(x.numpy())), x.shape)
            assert (out[idx] & 0x7F) == top
            assert np.array_equal(out_t, out.T)
            assert a == np.float32(np.abs(x.numpy()).max())


def test_current_scaling_zero_and_hand_values():
    out, _, a, s, si = R.quantize_current(np.zeros((2, 3), np.float32), F.E4M3, R.ROW)
    assert a == 0 and s == 1.0 and si == 1.0 and np.all(out == 0)
    # amax 2 -> scale 224 exactly; 0.5*224 = 112 = 1.75*2^6 -> 0|1101|110 = 0x6E
    out, _, a, s, si = R.quantize_current(np.array([[2.0, -0.5]], np.float32), F.E4M3, R.ROW)
    assert s == 224.0 and si == np.float32(1 / 224.0)
    assert list(out[0]) == [0x7E, 0xEE]


def test_bias_grad_closed_forms():
    g = torch.ones((1000, 7), dtype=torch.bfloat16)
    assert np.array_equal(B.bias_grad(g), np.full(7, 1000.0))
    g = torch.arange(12, dtype=torch.float32).reshape(4, 3)
    assert np.array_equal(B.bias_grad(g), np.array([18.0, 22.0, 26.0]))  # 0+3+6+9, 1+4+7+10, ...


def test_bias_grad_brute_force_and_bound():
    g = S.normal_with_outliers((300, 5), seed=3, std=1e-3, dtype="bf16")
    gf = g.float().numpy().astype(np.float64)
    col = [sum(gf[r, c] for r in range(300)) for c in range(5)]
    assert np.allclose(B.bias_grad(g), col, rtol=0, atol=1e-15)
    # a float32 sequential sum stays inside the bound
    f32 = np.zeros(5, np.float32)
    for r in range(300):
        f32 = (f32 + g.float().numpy()[r]).astype(np.float32)
    assert np.all(np.abs(f32 - B.bias_grad(g)) <= B.bound(g))
