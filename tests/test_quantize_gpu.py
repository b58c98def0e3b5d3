"""GPU parity of fp8_quantize against the CPU oracle: bytes, amax, ring and scales bit-exact."""

import numpy as np
import pytest
import torch

from fp8_delayed_scaling_02_b200 import ops, synthetic as S
from gpu_helpers import OR, assert_bytes_equal, assert_ring_equal, oracle_codes, quantize_both, require_gpu

pytestmark = pytest.mark.gpu

DTYPES = ["bf16", "fp16", "fp32"]
FMTS = [ops.E4M3, ops.E5M2]
LAYOUTS = [ops.ROW, ops.TRANSPOSED, ops.DUAL]


@pytest.fixture(autouse=True)
def _gpu():
    require_gpu()


def _dev(x, misalign):
    if not misalign:
        return x.cuda()
    flat = torch.empty(x.numel() + 1, dtype=x.dtype, device="cuda")
    flat[1:].copy_(x.reshape(-1))
    return flat[1:].view(x.shape)


def _run_and_compare(x, fmt, layout, ring, misalign=False):
    # misalign: False, True (one element) or an element offset of the input base
    out, out_t, r_out, r_out_t, r_ring = quantize_both(x, fmt, layout, ring, misalign)
    if layout in (ops.ROW, ops.DUAL):
        assert_bytes_equal(out, r_out, "out")
    if layout in (ops.TRANSPOSED, ops.DUAL):
        assert_bytes_equal(out_t, r_out_t, "out_t")
    assert_ring_equal(ring, r_ring)


# Small shapes that span several 128x64 tiles and 16-element chunks and leave
# ragged tails in both dimensions, plus rows not a multiple of 4.
SMALL = [(1, 1), (3, 5), (7, 33), (130, 70), (301, 1537)]


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("layout", LAYOUTS)
@pytest.mark.parametrize("misalign", [False, True])
def test_small_shapes_two_calls(dtype, fmt, layout, misalign):
    for i, (r, c) in enumerate(SMALL):
        vs = [1.0, 1e-3, 1e3][i % 3]
        ring = ops.Ring()
        for step in range(2):  # second call uses the delayed scale published by the first
            x = S.quant_sweep_input(r, c, dtype, vs, seed=31 * i + step)
            _run_and_compare(x, fmt, layout, ring, misalign)


# Transposed / dual inputs whose rows are a multiple of 16 bytes but whose base
# is only element-aligned go through a 2-D map that starts at the base rounded
# down to 16 bytes (the shifted-base kernel); other element-aligned inputs go
# through the register tile kernel.  Every element offset of the base inside
# its 16-byte granule, ragged rows and columns, both kernels.
BASE_OFFSET_SHAPES = [(8, 8), (130, 64), (129, 72), (257, 1536), (9, 37), (255, 1001)]


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("layout", [ops.TRANSPOSED, ops.DUAL])
def test_every_base_offset(dtype, layout):
    per = 16 // (4 if dtype == "fp32" else 2)
    for i, (r, c) in enumerate(BASE_OFFSET_SHAPES):
        for off in range(per):
            ring = ops.Ring()
            for step in range(2):
                x = S.quant_sweep_input(r, c, dtype, [1.0, 1e-3][step], seed=97 * i + 7 * off + step)
                _run_and_compare(x, ops.E4M3 if (i + off) % 2 else ops.E5M2, layout, ring, off)


@pytest.mark.parametrize("dtype,shape", [("bf16", (257, 1536)), ("fp32", (130, 68)), ("bf16", (9, 37))])
def test_dual_row_output_at_every_byte_offset(dtype, shape):
    """DUAL's row-layout output written at every byte offset of an 8-byte word:
    interior tile rows take the widest aligned stores each offset allows
    (8, 4, 2 and 1 bytes)."""
    r, c = shape
    for off in range(8):
        ring = ops.Ring()
        ref = OR.Ring()
        x = S.quant_sweep_input(r, c, dtype, 1.0, seed=300 + off)
        flat = torch.empty(r * c + 8, dtype=torch.uint8, device="cuda")
        out = flat[off:off + r * c].view(r, c)
        out_t = torch.empty((c, r), dtype=torch.uint8, device="cuda")
        ops.quantize(x.cuda(), ops.E4M3, ops.DUAL, ring, out, out_t)
        torch.cuda.synchronize()
        r_out, r_out_t, _ = OR.quantize(x, ops.E4M3, ops.DUAL, ref)
        assert_bytes_equal(out, r_out, f"out (byte offset {off})")
        assert_bytes_equal(out_t, r_out_t, f"out_t (byte offset {off})")
        assert_ring_equal(ring, ref)


def test_pr1_linear_three_delayed_steps():
    """X [128,512] row and W [256,512] dual, E4M3, rings carried over 3 steps."""
    rx, rw = ops.Ring(), ops.Ring()
    for step in range(3):
        x, w, _ = S.linear_pr1_step(step)
        _run_and_compare(x, ops.E4M3, ops.ROW, rx)
        _run_and_compare(w, ops.E4M3, ops.DUAL, rw)
    assert ops.Ring().state()[2] == 1.0


def test_seventeen_steps_wrap_the_ring():
    ring = ops.Ring()
    for step in range(17):
        x = S.quant_sweep_input(64, 48, "bf16", 10.0 ** ((step % 5) - 2), seed=step)
        _run_and_compare(x, ops.E5M2, ops.ROW, ring)


def test_empty_and_zero_inputs_fold_the_ring():
    ring = ops.Ring(scale=0.5)
    for layout in LAYOUTS:
        x = torch.zeros((0, 9), dtype=torch.bfloat16)
        _run_and_compare(x, ops.E4M3, layout, ring)
    x = torch.zeros((5, 9), dtype=torch.float32)
    _run_and_compare(x, ops.E4M3, ops.DUAL, ring)
    assert ring.state()[2] == 0.5  # zero history keeps the scale


def test_saturation_and_specials():
    vals = torch.tensor([[0.0, -0.0, 1e-30, -1e-30, 480.0, -1e6, 65504.0, 3e38, float("inf"), -float("inf")]],
                        dtype=torch.float32)
    for fmt in FMTS:
        for layout in LAYOUTS:
            ring = ops.Ring()
            _run_and_compare(vals, fmt, layout, ring)


def _all_16bit_patterns(dtype, with_inf=True):
    """Every non-NaN bf16 or fp16 bit pattern (both zeros, subnormals, infinities
    unless left out), zero-padded to [rows, 256] so the aligned kernels run."""
    bits = torch.from_numpy(np.arange(1 << 16, dtype=np.uint16).view(np.int16).copy())
    x = bits.view(torch.bfloat16 if dtype == "bf16" else torch.float16)
    xf = x.float()
    x = x[~torch.isnan(xf) & (torch.isfinite(xf) | with_inf)]
    pad = (-x.numel()) % 256
    return torch.cat([x, torch.zeros(pad, dtype=x.dtype)]).view(-1, 256)


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("layout", LAYOUTS)
def test_every_16bit_input_pattern(dtype, fmt, layout):
    """All 16-bit inputs at scale 1 (subnormal, normal, saturating and infinite
    inputs), at two scales that are not powers of two (the scaled product rounds
    in float32 before the cast), then two delayed steps on the finite patterns:
    the second uses the scale the first folded from the largest finite value."""
    x = _all_16bit_patterns(dtype)
    for s in (1.0, 0.3, 3.0 * 2.0 ** -7):
        _run_and_compare(x, fmt, layout, ops.Ring(scale=s))
    ring = ops.Ring()
    finite = _all_16bit_patterns(dtype, with_inf=False)
    for _ in range(2):
        _run_and_compare(finite, fmt, layout, ring)
    assert ring.state()[2] != 1.0


# Full sizes of the quantize bandwidth sweep, in the launch configuration the
# bench times.  Every byte of out / out_t is compared with the oracle, and the
# ring bit for bit.  Each case runs the three layouts from the same ring state
# (one oracle evaluation serves all three) and then a second, delayed step.
FULL = [(128, 1536), (2048, 1536), (8192, 1536), (2048, 1537), (8192, 1537)]
VALUE_SCALES = [1.0, 1e-3, 1e3]


def _full_case(rows, cols, dtype, fmt, misalign, vs, seed):
    x = S.quant_sweep_input(rows, cols, dtype, vs, seed=seed)
    xd = _dev(x, misalign)
    rings = {lay: ops.Ring() for lay in LAYOUTS}
    ref = OR.Ring()
    xf = OR.to_float32(x)
    a = OR.amax(xf)
    for step in range(2):
        got = {lay: ops.quantize(xd, fmt, lay, rings[lay]) for lay in LAYOUTS}
        torch.cuda.synchronize()
        codes = oracle_codes(x, ref.scale, fmt)
        codes_t = np.ascontiguousarray(codes.T)
        OR.fold(ref, a, fmt)
        what = f"{rows}x{cols} {dtype} fmt{fmt} misalign={misalign} x{vs} step {step}"
        for lay, (out, out_t) in got.items():
            if out is not None:
                assert_bytes_equal(out, codes, f"out, layout {lay}, {what}")
            if out_t is not None:
                assert_bytes_equal(out_t, codes_t, f"out_t, layout {lay}, {what}")
            assert_ring_equal(rings[lay], ref)


@pytest.mark.parametrize("shape", FULL)
@pytest.mark.parametrize("dtype", DTYPES)
def test_full_size_whole_tensor(shape, dtype):
    """The whole dtype x format x base alignment x value-scale product."""
    rows, cols = shape
    for fmt in FMTS:
        for misalign in (False, True):
            for vs in VALUE_SCALES:
                _full_case(rows, cols, dtype, fmt, misalign, vs, seed=(rows ^ cols) + int(misalign) + 7 * fmt)


@pytest.mark.parametrize("dtype,fmt,misalign,vs", [("bf16", ops.E4M3, False, 1.0), ("fp16", ops.E5M2, True, 1e-3),
                                                   ("fp32", ops.E4M3, True, 1e3)])
def test_full_size_whole_tensor_67M(dtype, fmt, misalign, vs):
    """16384 x 4096 (67M elements: every TMA tile claim of a multi-wave launch)."""
    _full_case(16384, 4096, dtype, fmt, misalign, vs, seed=16384 + int(misalign))


def _fp32_rounding_boundaries():
    """Every sign, exponent and top-12 mantissa pattern of float32 with the low
    11 bits at 0, 1, 0x400 or 0x7FF (NaN removed): every tie between two FP8
    neighbours of either format, one float32 ulp either side of it, and every
    exact code, about 8.4M values."""
    hi = np.arange(1 << 21, dtype=np.uint32) << np.uint32(11)
    u = np.concatenate([hi | np.uint32(low) for low in (0, 1, 0x400, 0x7FF)])
    x = u.view(np.float32)
    x = x[~np.isnan(x)]
    pad = (-x.size) % 2048
    return torch.from_numpy(np.concatenate([x, np.zeros(pad, dtype=np.float32)]).reshape(-1, 2048))


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("scale", [1.0, 0.3])
def test_fp32_rounding_boundaries(fmt, scale):
    """The hardware cast on float32 inputs at every rounding boundary, through
    fp8_quantize (row layout), against the oracle's encoder byte for byte."""
    x = _fp32_rounding_boundaries()
    ring = ops.Ring(scale=scale)
    out, _ = ops.quantize(x.cuda(), fmt, ops.ROW, ring)
    torch.cuda.synchronize()
    assert_bytes_equal(out, OR.scaled_codes(x.numpy(), np.float32(scale), fmt), f"fp32 boundaries fmt{fmt} x{scale}")
    ref = OR.Ring(scale=scale)
    OR.fold(ref, OR.amax(x.numpy()), fmt)
    assert_ring_equal(ring, ref)


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("layout", LAYOUTS)
def test_nan_inputs_do_not_reach_amax(dtype, layout):
    """amax ignores NaN (reading of the pages' amax); the NaN elements' own codes
    are not compared (parity unpinned), every other byte and the ring are."""
    x = S.quant_sweep_input(256, 128, dtype, 1.0, seed=77).float()
    x[3, 5] = float("nan")
    x[200, 127] = float("nan")
    x = x.to({"bf16": torch.bfloat16, "fp16": torch.float16, "fp32": torch.float32}[dtype])
    ring = ops.Ring()
    out, out_t, r_out, r_out_t, r_ring = quantize_both(x, ops.E4M3, layout, ring)
    nan = torch.isnan(x.float()).numpy()
    if out is not None:
        g = out.cpu().numpy()
        assert np.array_equal(g[~nan], r_out[~nan])
    if out_t is not None:
        g = out_t.cpu().numpy()
        assert np.array_equal(g[~nan.T], r_out_t[~nan.T])
    assert_ring_equal(ring, r_ring)


# fp8_quantize_pair: two quantize calls (own rings) in one launch.  Each case
# runs 3 delayed steps and must equal the two separate fp8_quantize calls bit
# for bit (codes, rings).  Cases: paired TMA tiles (dual, transposed), paired
# ROW (aligned; element-offset bases), and the sequential fallbacks (different
# kernels, different formats, an empty side).
QPAIR = [
    (((8192, 1536), "bf16", 0, False), ((1536, 1536), "bf16", 0, False), ops.DUAL),
    (((2048, 1536), "fp32", 1, False), ((130, 64), "fp32", 1, False), ops.TRANSPOSED),
    (((8192, 1536), "bf16", 0, False), ((4096, 1536), "bf16", 0, False), ops.ROW),
    (((1000, 1537), "bf16", 0, True), ((7, 33), "bf16", 0, True), ops.ROW),
    (((2048, 1537), "bf16", 0, False), ((256, 512), "bf16", 0, False), ops.DUAL),
    (((256, 512), "bf16", 0, False), ((256, 512), "bf16", 1, False), ops.DUAL),
    (((0, 9), "bf16", 0, False), ((64, 64), "bf16", 0, False), ops.DUAL),
]


@pytest.mark.parametrize("s0,s1,layout", QPAIR)
def test_quantize_pair_equals_two_calls(s0, s1, layout):
    rings = [ops.Ring(), ops.Ring()]
    refs = [ops.Ring(), ops.Ring()]
    for step in range(3):
        qs, expect = [], []
        for i, ((rows, cols), dt, fmt, mis) in enumerate((s0, s1)):
            x = _dev(S.quant_sweep_input(rows, cols, dt, [1.0, 1e3, 1e-3][step], seed=600 + 10 * step + i), mis)
            qs.append(dict(x=x, fmt=fmt, layout=layout, ring=rings[i]))
            expect.append(ops.quantize(x, fmt, layout, refs[i]))
        got = ops.quantize_pair(qs[0], qs[1])
        torch.cuda.synchronize()
        for (o, t), (eo, et) in zip(got, expect):
            for a, b in ((o, eo), (t, et)):
                assert (a is None) == (b is None)
                if a is not None:
                    assert torch.equal(a, b)
        for r, e in zip(rings, refs):
            assert torch.equal(r.buf, e.buf)


QMULTI = [
    # A 1.2B-model linear's X, W and G (one launch: same dtype and layout, formats differ).
    [((8192, 1536), "bf16", 0), ((4096, 1536), "bf16", 0), ((8192, 4096), "bf16", 1)],
    # Eight tensors of very different sizes, one launch.
    [((2048, 1536), "fp32", 1), ((128, 64), "fp32", 0), ((130, 64), "fp32", 1), ((1, 4), "fp32", 0),
     ((64, 4), "fp32", 0), ((300, 68), "fp32", 1), ((1000, 128), "fp32", 0), ((129, 8), "fp32", 1)],
    # T / DUAL: not fusable (an odd width, an empty input), calls in order;
    # ROW: not fusable (an empty input).
    [((256, 512), "bf16", 0), ((300, 1537), "bf16", 1), ((0, 64), "bf16", 0)],
    [((777, 512), "fp16", 1)],
]


@pytest.mark.parametrize("layout", [ops.ROW, ops.TRANSPOSED, ops.DUAL])
@pytest.mark.parametrize("case", range(len(QMULTI)))
def test_quantize_multi_equals_the_single_calls(case, layout):
    specs = QMULTI[case]
    rings = [ops.Ring() for _ in specs]
    refs = [ops.Ring() for _ in specs]
    for step in range(3):
        qs, expect = [], []
        for i, ((rows, cols), dt, fmt) in enumerate(specs):
            x = S.quant_sweep_input(rows, cols, dt, [1.0, 1e3, 1e-3][step], seed=700 + 10 * step + i).cuda()
            qs.append(dict(x=x, fmt=fmt, layout=layout, ring=rings[i]))
            expect.append(ops.quantize(x, fmt, layout, refs[i]))
        got = ops.quantize_multi(qs)
        torch.cuda.synchronize()
        for (o, t), (eo, et) in zip(got, expect):
            for a, b in ((o, eo), (t, et)):
                assert (a is None) == (b is None)
                if a is not None:
                    assert torch.equal(a, b)
        for r, e in zip(rings, refs):
            assert torch.equal(r.buf, e.buf)


def test_quantize_multi_linear_matches_the_oracle():
    """X, W (E4M3) and G (E5M2) of the 1.2B-model FFN linear at M = 2048, dual
    layout, one launch per step over 3 delayed steps: every byte and ring
    against the oracle."""
    shapes = [((2048, 1536), ops.E4M3), ((4096, 1536), ops.E4M3), ((2048, 4096), ops.E5M2)]
    rings = [ops.Ring() for _ in shapes]
    refs = [OR.Ring() for _ in shapes]
    for step in range(3):
        xs = [S.quant_sweep_input(r, c, "bf16", [1.0, 30.0, 1e-3][step], seed=900 + 10 * step + i)
              for i, ((r, c), _) in enumerate(shapes)]
        got = ops.quantize_multi([dict(x=x.cuda(), fmt=f, layout=ops.DUAL, ring=rg)
                                  for x, ((_, f)), rg in zip(xs, shapes, rings)])
        torch.cuda.synchronize()
        for x, (_, f), (o, t), ref, rg in zip(xs, shapes, got, refs, rings):
            codes = oracle_codes(x, ref.scale, f)
            OR.fold(ref, OR.amax(OR.to_float32(x)), f)
            assert_bytes_equal(o, codes, "out")
            assert_bytes_equal(t, np.ascontiguousarray(codes.T), "out_t")
            assert_ring_equal(rg, ref)


def test_quantize_multi_with_one_ring_twice_runs_in_order():
    ring, other, ref, ref_other = ops.Ring(), ops.Ring(), ops.Ring(), ops.Ring()
    xs = [S.quant_sweep_input(512, 256, "bf16", v, seed=20 + i).cuda() for i, v in enumerate((1.0, 1e3, 1e-3))]
    got = ops.quantize_multi([dict(x=xs[0], fmt=ops.E4M3, layout=ops.DUAL, ring=ring),
                              dict(x=xs[1], fmt=ops.E4M3, layout=ops.DUAL, ring=other),
                              dict(x=xs[2], fmt=ops.E4M3, layout=ops.DUAL, ring=ring)])
    e0 = ops.quantize(xs[0], ops.E4M3, ops.DUAL, ref)
    e1 = ops.quantize(xs[1], ops.E4M3, ops.DUAL, ref_other)
    e2 = ops.quantize(xs[2], ops.E4M3, ops.DUAL, ref)
    torch.cuda.synchronize()
    for (o, t), (eo, et) in zip(got, (e0, e1, e2)):
        assert torch.equal(o, eo) and torch.equal(t, et)
    assert torch.equal(ring.buf, ref.buf) and torch.equal(other.buf, ref_other.buf)


def test_quantize_pair_with_one_ring_runs_in_order():
    """Naming the same ring twice is two calls in order (the second sees the
    scale the first published)."""
    ring, ref = ops.Ring(), ops.Ring()
    x0 = S.quant_sweep_input(512, 256, "bf16", 1.0, seed=1).cuda()
    x1 = S.quant_sweep_input(512, 256, "bf16", 1e3, seed=2).cuda()
    (o0, _), (o1, _) = ops.quantize_pair(dict(x=x0, fmt=ops.E4M3, layout=ops.ROW, ring=ring),
                                         dict(x=x1, fmt=ops.E4M3, layout=ops.ROW, ring=ring))
    e0, _ = ops.quantize(x0, ops.E4M3, ops.ROW, ref)
    e1, _ = ops.quantize(x1, ops.E4M3, ops.ROW, ref)
    torch.cuda.synchronize()
    assert torch.equal(o0, e0) and torch.equal(o1, e1) and torch.equal(ring.buf, ref.buf)
