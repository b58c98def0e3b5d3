"""CPU check of the parity tests' fast path for 16-bit inputs: the oracle's
codes looked up by input bit pattern equal the oracle applied element by
element (every bf16 and fp16 pattern, scales that round in float32, both
formats, a random tensor), and the band rows hit every 128-row band."""

import numpy as np
import pytest
import torch

from fp8_delayed_scaling_02_b200 import synthetic as S
from gpu_helpers import OR, band_rows, oracle_codes


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("fmt", [0, 1])
def test_lookup_equals_elementwise_oracle(dtype, fmt):
    every = torch.arange(1 << 16, dtype=torch.int32).to(torch.int16).view(dtype).reshape(256, 256)
    rnd = S.quant_sweep_input(300, 77, "bf16" if dtype == torch.bfloat16 else "fp16", 10.0, seed=3)
    for x in (every, rnd):
        for s in (1.0, 0.3, 3.0 * 2.0 ** -7, 448.0 / 480.0):
            want = OR.scaled_codes(OR.to_float32(x), np.float32(s), fmt)
            assert np.array_equal(oracle_codes(x, s, fmt), want)


def test_float32_goes_through_the_oracle():
    x = S.quant_sweep_input(64, 33, "fp32", 1e3, seed=4)
    assert np.array_equal(oracle_codes(x, 0.37, 1), OR.scaled_codes(x.numpy(), np.float32(0.37), 1))


@pytest.mark.parametrize("M", [1, 127, 128, 129, 1000, 8192])
def test_band_rows_cover_every_band(M):
    r = band_rows(M, seed=M)
    assert r.min() == 0 and r.max() == M - 1
    assert set(range((M + 127) // 128)) == set((r // 128).tolist())
