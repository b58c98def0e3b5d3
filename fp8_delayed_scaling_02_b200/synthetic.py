"""Seeded synthetic inputs shared by the tests, the oracle checks and the bench.

This module only draws random numbers; it holds none of the quantize or GEMM
arithmetic.  Every generator uses a CPU ``torch.Generator`` so the same seed
gives the same tensor on any machine; callers move the result to the device.

Workloads (the shapes and distributions of the pages' benchmarks, made
synthetic because the pages' model weights and data are not available):

* linear_pr1      -- X bf16 [128,512], W bf16 [256,512], N(0,1) with 1% of
                     entries multiplied by 20, bias fp32 [256] ~ U(-1,1).
* linear_1p2b     -- the 1.2B-model linear shapes (hidden 1536, FFN 4096):
                     X [M,1536] N(0,1) with 0.5% x30 outliers, weights
                     [1536,1536] / [4096,1536] ~ N(0,0.02), gradient
                     G [M,N] ~ N(0,1e-3), bias fp32 ~ U(-1,1).
* quant_sweep     -- N(0,1) times {1, 1e-3, 1e3} in bf16/fp16/fp32.
* fp8_codes       -- uniform random FP8 codes over the finite codes.
"""

import torch

E4M3, E5M2 = 0, 1

_DTYPES = {"bf16": torch.bfloat16, "fp16": torch.float16, "fp32": torch.float32}


def _gen(seed):
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def _normal_outliers_from(g, shape, std, frac, mult, dtype):
    x = torch.randn(shape, generator=g, dtype=torch.float32) * std
    if frac > 0:
        mask = torch.rand(shape, generator=g) < frac
        x = torch.where(mask, x * mult, x)
    return x.to(_DTYPES[dtype] if isinstance(dtype, str) else dtype)


def normal_with_outliers(shape, seed, std=1.0, frac=0.0, mult=1.0, dtype="bf16"):
    """N(0, std^2) values; a Bernoulli(frac) mask (same generator) multiplies entries by ``mult``."""
    return _normal_outliers_from(_gen(seed), shape, std, frac, mult, dtype)


def uniform(shape, seed, lo=-1.0, hi=1.0):
    """float32 U(lo, hi)."""
    g = _gen(seed)
    return torch.rand(shape, generator=g, dtype=torch.float32) * (hi - lo) + lo


def finite_codes(fmt):
    """All 8-bit codes that are neither NaN nor infinite in the format (bit patterns only)."""
    if fmt == E4M3:
        bad = {0x7F, 0xFF}
    else:
        bad = {0x7C, 0x7D, 0x7E, 0x7F, 0xFC, 0xFD, 0xFE, 0xFF}
    return torch.tensor([c for c in range(256) if c not in bad], dtype=torch.uint8)


def fp8_codes(shape, seed, fmt=E4M3):
    """uint8 tensor of codes drawn uniformly from ``finite_codes(fmt)``."""
    g = _gen(seed)
    table = finite_codes(fmt)
    idx = torch.randint(0, table.numel(), shape, generator=g)
    return table[idx]


# --- named workloads -------------------------------------------------------

def linear_pr1_step(step):
    """One step of the small PR1 linear, steps 0, 1, 2 with fresh seeds 0, 1, 2.

    One generator seeded with the step draws X [128,512] and then W [256,512]
    (values, then the outlier mask, for each); the bias comes from seed 0.
    """
    g = _gen(step)
    x = _normal_outliers_from(g, (128, 512), 1.0, 0.01, 20.0, "bf16")
    w = _normal_outliers_from(g, (256, 512), 1.0, 0.01, 20.0, "bf16")
    bias = uniform((256,), seed=0)
    return x, w, bias


HIDDEN = 1536
FFN = 4096


def linear_1p2b_weights():
    """W1 [1536,1536], W2 [4096,1536] ~ N(0, 0.02) bf16 and their fp32 U(-1,1) biases."""
    w1 = normal_with_outliers((HIDDEN, HIDDEN), seed=11, std=0.02)
    w2 = normal_with_outliers((FFN, HIDDEN), seed=12, std=0.02)
    b1 = uniform((HIDDEN,), seed=13)
    b2 = uniform((FFN,), seed=14)
    return (w1, b1), (w2, b2)


def linear_1p2b_step(M, n_out, step):
    """Activations X [M,1536] (0.5% x30 outliers) and gradient G [M,n_out] ~ N(0,1e-3) for one step."""
    x = normal_with_outliers((M, HIDDEN), seed=100000 + 97 * step + M, frac=0.005, mult=30.0)
    gr = normal_with_outliers((M, n_out), seed=200000 + 89 * step + M + n_out, std=1e-3)
    return x, gr


def quant_sweep_input(rows, cols, dtype, value_scale, seed=0):
    """N(0,1) * value_scale in the named dtype."""
    x = normal_with_outliers((rows, cols), seed=seed, dtype="fp32") * value_scale
    return x.to(_DTYPES[dtype])
