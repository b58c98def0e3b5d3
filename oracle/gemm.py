"""Scaled FP8 GEMM in float64 and its acceptance bound.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

What mm_fp8 computes ("AstrAI commits, branch main, tests/extension": the
bias-fusion commit and the 3D batched commit; the quantize split commit
fixes bf16 output):

    Y[b, m, n] = bf16( sinv_a * sinv_b * sum_k A[b, m, k] * B[b, n, k] + bias[n] )

A and B hold FP8 codes, K-major ("NT": both operands have K contiguous).
A batch stride of 0 broadcasts that operand over the batch.  The bias is
float32 [N], shared by every row and batch, optional.

The oracle returns the exact-as-possible float64 value ``ref`` (before the
bf16 rounding) and ``S = sinv_a * sinv_b * sum_k |A.B|``.  A result y
passes when ``|y - ref| <= ulp_bf16(ref) + 2^-20 * S``: one bf16 ulp for the
single output rounding plus an accumulation allowance proportional to the
sum of product magnitudes.

For E4M3 x E4M3 with K <= 8192 the float64 sum is exact: every decoded value
is a multiple of 2^-9 below 2^9, products are multiples of 2^-18 below 2^18,
and 8192 of them stay below 2^31, i.e. 49 significant bits.
"""

import numpy as np

from . import fp8_formats as F


def _batched(x, batch):
    """[batch, rows, K] view of a 2-D or 3-D array; a size-1 batch broadcasts."""
    x = np.asarray(x)
    if x.ndim == 2:
        x = x[None]
    if x.shape[0] == 1 and batch > 1:
        x = np.broadcast_to(x, (batch,) + x.shape[1:])
    assert x.shape[0] == batch
    return x


def mm_fp8(a_codes, b_codes, fmt_a, fmt_b, sinv_a, sinv_b, bias=None):
    """Return (ref, S), both float64 [batch, M, N] (or [M, N] for 2-D inputs)."""
    squeeze = np.asarray(a_codes).ndim == 2 and np.asarray(b_codes).ndim == 2
    batch = max(np.asarray(a_codes).shape[0] if np.asarray(a_codes).ndim == 3 else 1,
                np.asarray(b_codes).shape[0] if np.asarray(b_codes).ndim == 3 else 1)
    a = F.decode(_batched(a_codes, batch), fmt_a)
    b = F.decode(_batched(b_codes, batch), fmt_b)
    sab = float(np.float64(np.float32(sinv_a)) * np.float64(np.float32(sinv_b)))
    acc = np.matmul(a, np.swapaxes(b, 1, 2))
    mag = np.matmul(np.abs(a), np.swapaxes(np.abs(b), 1, 2))
    ref = acc * sab
    if bias is not None:
        ref = ref + np.asarray(bias, dtype=np.float32).astype(np.float64)[None, None, :]
    S = mag * abs(sab)
    if squeeze:
        return ref[0], S[0]
    return ref, S


def mm_fp8_rows(a_codes, b_codes, fmt_a, fmt_b, sinv_a, sinv_b, bias, rows):
    """(ref, S) for a subset of output rows of a 2-D product: [len(rows), N]."""
    a = F.decode(np.asarray(a_codes)[rows], fmt_a)
    b = F.decode(np.asarray(b_codes), fmt_b)
    sab = float(np.float64(np.float32(sinv_a)) * np.float64(np.float32(sinv_b)))
    ref = (a @ b.T) * sab
    if bias is not None:
        ref = ref + np.asarray(bias, dtype=np.float32).astype(np.float64)[None, :]
    S = (np.abs(a) @ np.abs(b).T) * abs(sab)
    return ref, S


def ulp_bf16(x):
    """Spacing of bf16 numbers at |x|: 2^(e - 7) for 2^e <= |x| < 2^(e+1), 2^-133 near 0."""
    x = np.abs(np.asarray(x, dtype=np.float64))
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(x > 0, x, 2.0 ** -140)))
    e = np.maximum(e, -126.0)
    return np.exp2(e - 7.0)


def bound(ref, S):
    """Allowed |y - ref|: one bf16 ulp of ref plus 2^-20 times the scaled |a.b| sum."""
    return ulp_bf16(ref) + np.ldexp(np.asarray(S, dtype=np.float64), -20)


def check(y, ref, S):
    """(ok, worst_ratio): ok iff every |y - ref| is within ``bound``; y is any float array."""
    y = np.asarray(y, dtype=np.float64)
    err = np.abs(y - ref)
    b = bound(ref, S)
    ratio = float(np.max(err / b)) if err.size else 0.0
    return bool(np.all(err <= b)), ratio
