"""Shared helpers of the GPU parity tests: run the CUDA path, run the oracle, compare."""

import numpy as np
import pytest
import torch

from oracle import fp8_formats as OF
from oracle import gemm as OG
from oracle import recipe as OR

from fp8_delayed_scaling_02_b200 import ops


def require_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    ops.lib()  # raises if the library is missing: no silent fallback


def oracle_ring_from(ring_gpu):
    """Oracle Ring holding the same state as a GPU ring."""
    hist, idx, scale, scale_inv, _ = ring_gpu.state()
    r = OR.Ring()
    r.history = hist.numpy().astype(np.float32)
    r.idx = idx
    r.scale = np.float32(scale)
    r.scale_inv = np.float32(scale_inv)
    return r


def assert_ring_equal(ring_gpu, ring_ref):
    hist, idx, scale, scale_inv, scratch = ring_gpu.state()
    assert np.array_equal(hist.numpy().view(np.uint32), ring_ref.history.view(np.uint32)), (hist, ring_ref.history)
    assert idx == ring_ref.idx
    assert np.float32(scale).view(np.uint32) == np.float32(ring_ref.scale).view(np.uint32), (scale, ring_ref.scale)
    assert np.float32(scale_inv).view(np.uint32) == np.float32(ring_ref.scale_inv).view(np.uint32)
    assert all(int(v) == 0 for v in scratch), "scratch must self-reset"


def quantize_both(x_cpu, fmt, layout, ring_gpu, misalign=False):
    """Run one quantize on the GPU (through the C ABI) and on the oracle from the same
    ring state.  Returns (gpu_out, gpu_out_t, ref_out, ref_out_t, ref_ring).
    ``misalign``: False, True (one element past a 256-byte aligned base) or an
    element offset."""
    ref_ring = oracle_ring_from(ring_gpu)
    if misalign:
        k = int(misalign)
        flat = torch.empty(x_cpu.numel() + k, dtype=x_cpu.dtype, device="cuda")
        flat[k:].copy_(x_cpu.reshape(-1))
        x_dev = flat[k:].view(x_cpu.shape)
    else:
        x_dev = x_cpu.to("cuda")
    out, out_t = ops.quantize(x_dev, fmt, layout, ring_gpu)
    torch.cuda.synchronize()
    r_out, r_out_t, _ = OR.quantize(x_cpu, fmt, layout, ref_ring)
    return out, out_t, r_out, r_out_t, ref_ring


def oracle_codes(x_cpu, scale, fmt):
    """The oracle's codes encode(fp32(x * scale)) of a CPU tensor, element by element.

    A bf16 or fp16 tensor holds at most 65536 distinct values, so the oracle
    (``OR.scaled_codes``) is applied once to every 16-bit pattern and the
    result is looked up by each element's bit pattern: the same function,
    evaluated once per distinct input instead of once per element.  float32
    inputs go through ``OR.scaled_codes`` directly."""
    if x_cpu.dtype in (torch.bfloat16, torch.float16):
        pats = torch.arange(1 << 16, dtype=torch.int32).to(torch.int16).view(x_cpu.dtype)
        with np.errstate(over="ignore", invalid="ignore"):  # the table spans inf, NaN and huge patterns
            table = OR.scaled_codes(OR.to_float32(pats), np.float32(scale), fmt)
        bits = x_cpu.contiguous().view(torch.int16).numpy().view(np.uint16)
        return table[bits]
    return OR.scaled_codes(OR.to_float32(x_cpu), np.float32(scale), fmt)


def band_rows(M, seed, band=128):
    """Output rows that hit every 128-row band of an M-row result: each band's
    first and last row and one drawn at random inside it, so every M tile (and
    each half of a 256-row CTA-pair tile) is compared."""
    rng = np.random.default_rng(seed)
    rows = []
    for b0 in range(0, M, band):
        b1 = min(b0 + band, M) - 1
        rows += [b0, b1, int(rng.integers(b0, b1 + 1))]
    return np.unique(np.array(rows, dtype=np.int64))


def assert_bytes_equal(gpu, ref, what):
    g = gpu.cpu().numpy()
    assert g.shape == ref.shape, (what, g.shape, ref.shape)
    bad = np.nonzero(g != ref)
    assert bad[0].size == 0, f"{what}: {bad[0].size} mismatches, first at {tuple(b[0] for b in bad)}: " \
                             f"gpu {g[tuple(b[0] for b in bad)]:#x} ref {ref[tuple(b[0] for b in bad)]:#x}"


def mm_check(y_gpu, a_codes, b_codes, fmt_a, fmt_b, sinv_a, sinv_b, bias, rows=None):
    """Compare a GPU GEMM result (bf16) with the oracle bound; returns worst err/bound ratio."""
    y = y_gpu.float().cpu().numpy().astype(np.float64)
    if rows is None:
        ref, S = OG.mm_fp8(a_codes, b_codes, fmt_a, fmt_b, sinv_a, sinv_b, bias)
    else:
        ref, S = OG.mm_fp8_rows(a_codes, b_codes, fmt_a, fmt_b, sinv_a, sinv_b, bias, rows)
        y = y[rows]
    ok, ratio = OG.check(y, ref, S)
    assert ok, f"GEMM outside the bound: worst err/bound = {ratio:.3f}"
    return ratio


def f32(t):
    return float(t.cpu().item())


__all__ = ["require_gpu", "quantize_both", "assert_ring_equal", "assert_bytes_equal", "mm_check", "oracle_codes",
           "band_rows", "OF", "OG", "OR"]
