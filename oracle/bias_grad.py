"""Bias gradient of the FP8 linear: column sums of the output gradient.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

The backward of Y = X.W^T + b gives db[n] = sum_m G[m, n] over all leading
(token) dimensions ("AstrAI commits, branch main, tests/extension": the
_LinearFp8 backward fix reduces grad_b over leading dims; the forward-to-
backward commit keeps G in bf16 for this sum).  The oracle sums the exact
float32 values of G in float64.  A float32 result summed in any order over
R rows is within (R - 1) * 2^-24 * sum_m |G[m, n]| of the exact sum (the
standard bound for recursive summation), plus half an ulp of its final
rounding to float32; ``bound`` returns that allowance.
"""

import numpy as np

from .recipe import to_float32


def bias_grad(g):
    """float64 column sums of a 2-D bf16/fp16/fp32 array or tensor."""
    gf = to_float32(g).astype(np.float64)
    assert gf.ndim == 2
    return gf.sum(axis=0)


def abs_col_sums(g):
    return np.abs(to_float32(g).astype(np.float64)).sum(axis=0)


def bound(g):
    """Allowed |db_fp32 - db_exact| per column."""
    rows = to_float32(g).shape[0]
    s = abs_col_sums(g)
    return max(rows - 1, 0) * 2.0 ** -24 * s + 2.0 ** -24 * s + 2.0 ** -149
