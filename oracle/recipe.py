"""Per-tensor delayed scaling: amax, quantize in three layouts, ring fold.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

What one quantize call computes, in the pages' order:

1. ``s = ring.scale`` -- the scale this call uses was published by the
   previous call on the same ring (delayed scaling: "AstrAI commit 5244f1a8",
   "x/g scales delayed one step").
2. ``amax = max_i |x_i|`` over the raw input converted exactly to float32,
   not over the scaled values ("AstrAI commit 69f35c46, fix: quantize amax
   from raw values").  NaN elements are ignored (reading; unpinned).
3. ``q_i = encode(fp32(x_i * s))``: one float32 multiply with
   round-to-nearest-even, then the saturating RNE conversion of
   ``fp8_formats.encode``.  Rounding the product to float32 first is the
   precision the conversion instruction sees (reading).
4. Layouts ("tests/extension" page, quantize bindings commit: QuantLayout):
   ROW writes ``out[r, c]``, T writes ``out_t[c, r]`` (the [cols, rows]
   transpose), DUAL writes both from the same values.
5. Ring fold ("tests/extension" page, ring commit: the last block folds amax
   into the history window and publishes the next scale):
   ``hist[idx] = amax; idx = (idx + 1) mod 16; m = max(hist)``, where
   the maximum ignores NaN entries exactly as the amax of step 2 ignores
   NaN elements, and is 0 when every entry is NaN (reading: the pages state
   no NaN rule; a NaN can only reach the history through a caller-supplied
   amax, the data-parallel fold of a MAX-reduced amax);
   ``scale' = fp32(FP8_MAX / m)`` if m is positive and finite and the
   quotient is finite, else the scale is kept (a zero history keeps the
   previous scale).
6. ``scale_inv = fp32(1 / s)``: the inverse of the scale this call USED,
   so the GEMM dequantises with the quantize-time scale ("tests/extension"
   page, snapshot commit).
"""

import numpy as np

from . import fp8_formats as F

ROW, TRANSPOSED, DUAL = 0, 1, 2
HISTORY_LEN = 16


class Ring:
    """History ring state: 16 float32 amaxes, the next write slot, two scales."""

    def __init__(self, scale=1.0):
        self.history = np.zeros(HISTORY_LEN, dtype=np.float32)
        self.idx = 0
        self.scale = np.float32(scale)
        self.scale_inv = np.float32(1.0)

    def copy(self):
        r = Ring()
        r.history = self.history.copy()
        r.idx = self.idx
        r.scale = np.float32(self.scale)
        r.scale_inv = np.float32(self.scale_inv)
        return r


def to_float32(x):
    """Exact float32 value of a bf16 / fp16 / fp32 tensor or array."""
    try:
        import torch

        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu").to(torch.float32).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float32)


def amax(xf):
    """max |x| over the raw float32 values; NaN ignored; 0 for an empty input."""
    a = np.abs(np.asarray(xf, dtype=np.float32)).ravel()
    a = a[~np.isnan(a)]
    return np.float32(a.max()) if a.size else np.float32(0.0)


def scaled_codes(xf, scale, fmt):
    """encode(fp32(x * scale)) element-wise; shape of ``xf``."""
    prod = np.multiply(np.asarray(xf, dtype=np.float32), np.float32(scale), dtype=np.float32)
    return F.encode(prod, fmt)


def fold(ring, a, fmt):
    """Fold one amax into the ring and publish the next scale (in place).

    Returns the scale that was in effect before the fold (the one used).
    """
    s_used = np.float32(ring.scale)
    ring.history[ring.idx] = np.float32(a)
    ring.idx = (ring.idx + 1) % HISTORY_LEN
    h = ring.history[~np.isnan(ring.history)]
    m = np.float32(np.max(h)) if h.size else np.float32(0.0)
    fmax = np.float32(F.fp8_max(fmt))
    if m > 0 and np.isfinite(m):
        with np.errstate(over="ignore"):
            cand = np.float32(fmax / m)
        if np.isfinite(cand) and cand > 0:
            ring.scale = cand
    with np.errstate(divide="ignore"):
        ring.scale_inv = np.float32(np.float32(1.0) / s_used)
    return s_used


def quantize(x, fmt, layout, ring):
    """One quantize call: returns (out or None, out_t or None, amax); updates ``ring``.

    ``x`` is a 2-D [rows, cols] array/tensor in bf16, fp16 or fp32.
    """
    xf = to_float32(x)
    assert xf.ndim == 2
    s = np.float32(ring.scale)
    a = amax(xf)
    q = scaled_codes(xf, s, fmt)
    out = q if layout in (ROW, DUAL) else None
    out_t = np.ascontiguousarray(q.T) if layout in (TRANSPOSED, DUAL) else None
    fold(ring, a, fmt)
    return out, out_t, a


def current_scale(a, fmt):
    """Current (dynamic) scaling: fp32(FP8_MAX / amax) of this tensor's own amax.

    The pages' DynamicScaling path ("AstrAI commits, branch main,
    tests/extension", FP8Recipe commit: a dynamic flag, no rings, scales
    measured inline).  Reading: an amax of 0 (or a non-finite amax or
    quotient) gives scale 1.
    """
    a = np.float32(a)
    fmax = np.float32(F.fp8_max(fmt))
    if a > 0 and np.isfinite(a):
        with np.errstate(over="ignore"):
            c = np.float32(fmax / a)
        if np.isfinite(c) and c > 0:
            return c
    return np.float32(1.0)


def quantize_current(x, fmt, layout):
    """Current scaling: returns (out, out_t, amax, scale, scale_inv).

    amax over the raw values, scale from this amax, codes of fp32(x*scale),
    scale_inv = fp32(1/scale).  No history.
    """
    xf = to_float32(x)
    assert xf.ndim == 2
    a = amax(xf)
    s = current_scale(a, fmt)
    q = scaled_codes(xf, s, fmt)
    out = q if layout in (ROW, DUAL) else None
    out_t = np.ascontiguousarray(q.T) if layout in (TRANSPOSED, DUAL) else None
    return out, out_t, a, s, np.float32(np.float32(1.0) / s)


def quantize_local(x, fmt, layout, ring):
    """One shard's cast without the fold (data-parallel delayed scaling).

    Steps 1-4 above with the ring left untouched: the codes use ``ring.scale``
    and the shard's amax is returned for a cross-rank MAX.  The fold of that
    MAX with ``fold`` is the ring update of the whole tensor, because amax of
    a union is the max of the shards' amaxes (reading of the data-parallel
    scale-consistency item; the pages give no detail beyond the per-tensor
    ring of the "tests/extension" ring commit).

    Returns (out or None, out_t or None, amax, scale_inv) with
    scale_inv = fp32(1 / ring.scale).
    """
    xf = to_float32(x)
    assert xf.ndim == 2
    s = np.float32(ring.scale)
    a = amax(xf)
    q = scaled_codes(xf, s, fmt)
    out = q if layout in (ROW, DUAL) else None
    out_t = np.ascontiguousarray(q.T) if layout in (TRANSPOSED, DUAL) else None
    with np.errstate(divide="ignore"):
        sinv = np.float32(np.float32(1.0) / s)
    return out, out_t, a, sinv
