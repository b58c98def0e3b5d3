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


# ---- FP8 bias storage and FP8 output (epilogue variants) -------------------
#
# "AstrAI commits, branch main, tests/extension" page: the bias_scale commit
# (FP8Params.bias becomes untyped with a bias_scale slot: without a scale the
# bias is used as stored, with one it is FP8 storage dequantised in the
# epilogue after the operand scaling and before any output quantisation) and
# the FP8-in/FP8-out GEMM commit (fp8_mm_prequant_fp8).  The pages fix no
# formula for either; the readings here are the plainest ones that match the
# rest of the recipe:
#   bias value  = fp32(decode(code) * bias_scale)        (one float32 multiply)
#   y           = sinv_a * sinv_b * sum_k a.b + bias     (the float32 epilogue value)
#   output code = encode(fp32(y * s)), s = out_ring.scale (the output tensor's
#                 delayed scale, one float32 multiply, saturating RNE)
#   out_ring    folds amax = max |y| over the output (NaN ignored) exactly as
#                 a quantize call folds the amax of its input.


def bias_from_fp8(codes, fmt, bias_scale):
    """float32 [N] bias of FP8 bias storage: fp32(decode(code) * bias_scale)."""
    vals = F.decode(np.asarray(codes, dtype=np.uint8), fmt).astype(np.float32)  # exact: FP8 values fit in float32
    return np.multiply(vals, np.float32(bias_scale), dtype=np.float32)


def bound_f32(ref, S):
    """Allowed |y - ref| for the float32 epilogue value y itself (no bf16 rounding):
    the accumulation allowance 2^-20 * S plus one float32 ulp of ref for the
    epilogue's fused multiply-add, plus the smallest float32 subnormal."""
    ref = np.abs(np.asarray(ref, dtype=np.float64))
    return np.ldexp(np.asarray(S, dtype=np.float64), -20) + np.ldexp(ref, -23) + 2.0 ** -149


def out8_code_range(ref, S, scale, fmt):
    """(lo, hi) uint8 codes: every float32 y within ``bound_f32`` of ``ref`` has
    encode(fp32(y * scale)) between the two (both encode steps are monotone in
    y, and a float32 y >= lo_end is >= fp32(lo_end)).  Where lo == hi the code
    is fixed exactly."""
    b = bound_f32(ref, S)
    lo_end = np.asarray(ref, dtype=np.float64) - b
    hi_end = np.asarray(ref, dtype=np.float64) + b
    with np.errstate(over="ignore"):
        lo32 = lo_end.astype(np.float32)
        hi32 = hi_end.astype(np.float32)
    s = np.float32(scale)
    with np.errstate(over="ignore"):
        lo = F.encode(np.multiply(lo32, s, dtype=np.float32), fmt)
        hi = F.encode(np.multiply(hi32, s, dtype=np.float32), fmt)
    return lo, hi


def codes_within(codes, lo, hi, fmt):
    """Boolean array: decode(lo) <= decode(codes) <= decode(hi), element-wise."""
    v = F.decode(np.asarray(codes, dtype=np.uint8), fmt)
    return (F.decode(lo, fmt) <= v) & (v <= F.decode(hi, fmt))


def amax_range(ref, S):
    """(amax_exact, tolerance) of max |y| over the output: the exact max |ref|
    and the largest per-element ``bound_f32`` (0, 0 for an empty output)."""
    ref = np.asarray(ref, dtype=np.float64)
    if ref.size == 0:
        return 0.0, 0.0
    return float(np.max(np.abs(ref))), float(np.max(bound_f32(ref, S)))
