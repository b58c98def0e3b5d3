"""GPU parity of fp8_mm_ex (FP8 bias storage, FP8 output with delayed output
scaling) against the CPU oracle.

FP8 output: every code lies in the oracle's interval (the codes of the exact
value +- the float32 epilogue bound), and equals the oracle's code wherever
that interval holds one code; the amax folded into the output ring is within
the bound of the exact max |y|; the ring then holds exactly the oracle fold
of that amax (history, index, both scales) and its scratch words are zero.
"""

import numpy as np
import pytest
import torch

from fp8_delayed_scaling_02_b200 import ops, synthetic as S
from gpu_helpers import OF, OG, OR, assert_ring_equal, mm_check, oracle_ring_from, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    require_gpu()


def _scalar(v):
    return torch.tensor([v], dtype=torch.float32, device="cuda")


def _inputs(M, N, K, seed, fmt_a=ops.E4M3, batch=None):
    shape_a = (M, K) if batch is None else (batch, M, K)
    a = S.fp8_codes(shape_a, seed=seed, fmt=fmt_a)
    b = S.fp8_codes((N, K), seed=seed + 1)
    return a, b


def _bias(N, kind, seed):
    """(bias tensor for the call, bias_scale or None, float32 bias for the oracle)."""
    if kind is None:
        return None, None, None
    if kind == "f32":
        bias = S.uniform((N,), seed=seed) * 4.0
        return bias.cuda(), None, bias.numpy()
    fmt = ops.E4M3 if kind == "e4m3" else ops.E5M2
    codes = S.fp8_codes((N,), seed=seed, fmt=fmt)
    bsc = 0.0625 if fmt == ops.E4M3 else 0.37
    return codes.cuda(), _scalar(bsc), OG.bias_from_fp8(codes.numpy(), fmt, bsc)


def _check_out8_step(out, ring, ref_ring_before, ref, S_, out_fmt):
    """Codes within the interval, amax within the bound, ring = oracle fold of the GPU amax."""
    s = np.float32(ref_ring_before.scale)
    lo, hi = OG.out8_code_range(ref, S_, s, out_fmt)
    g = out.cpu().numpy().reshape(ref.shape)
    ok = OG.codes_within(g, lo, hi, out_fmt)
    assert ok.all(), f"{int((~ok).sum())} codes outside the interval, first at {np.argwhere(~ok)[0]}"
    fixed = lo == hi
    assert np.array_equal(g[fixed], lo[fixed])
    hist, idx, scale, scale_inv, scratch = ring.state()
    a_gpu = hist.numpy()[ref_ring_before.idx]
    a_ref, tol = OG.amax_range(ref, S_)
    assert abs(float(a_gpu) - a_ref) <= tol, (float(a_gpu), a_ref, tol)
    expect = ref_ring_before.copy()
    OR.fold(expect, np.float32(a_gpu), out_fmt)
    assert_ring_equal(ring, expect)
    return float(np.mean(fixed))


# (M, N, K, batch, bias kind, A format, workspace): ragged M and N with byte
# stores, aligned 16-byte stores, an odd N, batched with B broadcast, and two
# shapes the chooser runs with a stream-K tail when given a workspace.
OUT8_CASES = [
    (130, 700, 512, None, None, ops.E4M3, False),
    (256, 512, 1024, None, "f32", ops.E4M3, False),
    (1000, 1537, 2048, None, "e4m3", ops.E5M2, False),
    (384, 256, 512, 3, "e5m2", ops.E4M3, False),
    (128, 256, 8192, None, "f32", ops.E4M3, True),
    (1000, 1537, 8192, None, None, ops.E5M2, True),
]


@pytest.mark.parametrize("out_fmt", [ops.E4M3, ops.E5M2])
@pytest.mark.parametrize("case", OUT8_CASES)
def test_fp8_output_three_delayed_steps(case, out_fmt):
    M, N, K, batch, bias_kind, fmt_a, use_ws = case
    a, b = _inputs(M, N, K, seed=M + N + K, fmt_a=fmt_a, batch=batch)
    bias, bsc, bias_ref = _bias(N, bias_kind, seed=N)
    bias_fmt = ops.E5M2 if bias_kind == "e5m2" else ops.E4M3
    sinv_a, sinv_b = 2.0 ** -7, 0.37
    ws = None
    if use_ws:
        need = ops.mm_workspace_bytes(M, N, K)
        assert need > 0, "expected a stream-K tail for this shape"
        ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    ref, S_ = OG.mm_fp8(a.numpy(), b.numpy(), fmt_a, ops.E4M3, sinv_a, sinv_b, bias_ref)
    ring = ops.Ring()
    ad, bd = a.cuda(), b.cuda()
    for step in range(3):  # scale 1, then the delayed scale folded from the previous output
        before = oracle_ring_from(ring)
        out = ops.mm_ex(ad, bd, _scalar(sinv_a), _scalar(sinv_b), bias=bias, bias_scale=bsc, bias_fmt=bias_fmt,
                        out_fmt=out_fmt, out_ring=ring, fmt_a=fmt_a, workspace=ws)
        torch.cuda.synchronize()
        frac = _check_out8_step(out, ring, before, ref, S_, out_fmt)
        assert frac > 0.9  # nearly every code is fixed by the oracle alone
    if ws is not None:
        assert int(ws[:1024].view(torch.int32).abs().sum()) == 0  # stream-K flags left clear


def test_fp8_output_full_size():
    """2048 x 4096 x 1536 (E4M3 operands, fp32 bias, E4M3 output), all elements."""
    M, N, K = 2048, 4096, 1536
    a, b = _inputs(M, N, K, seed=11)
    bias, _, bias_ref = _bias(N, "f32", seed=3)
    ref, S_ = OG.mm_fp8(a.numpy(), b.numpy(), ops.E4M3, ops.E4M3, 2.0 ** -7, 2.0 ** -6, bias_ref)
    ring = ops.Ring()
    for _ in range(2):
        before = oracle_ring_from(ring)
        out = ops.mm_ex(a.cuda(), b.cuda(), _scalar(2.0 ** -7), _scalar(2.0 ** -6), bias=bias,
                        out_fmt=ops.E4M3, out_ring=ring)
        torch.cuda.synchronize()
        _check_out8_step(out, ring, before, ref, S_, ops.E4M3)


@pytest.mark.parametrize("bias_kind", ["e4m3", "e5m2"])
def test_fp8_bias_with_bf16_output(bias_kind):
    for (M, N, K) in ((256, 512, 1024), (130, 700, 512), (1000, 1537, 2048)):
        a, b = _inputs(M, N, K, seed=7 * M)
        bias, bsc, bias_ref = _bias(N, bias_kind, seed=M)
        y = ops.mm_ex(a.cuda(), b.cuda(), _scalar(0.5), _scalar(0.25), bias=bias, bias_scale=bsc,
                      bias_fmt=ops.E5M2 if bias_kind == "e5m2" else ops.E4M3)
        torch.cuda.synchronize()
        mm_check(y, a.numpy(), b.numpy(), ops.E4M3, ops.E4M3, 0.5, 0.25, bias_ref)


def test_empty_and_k0_outputs_fold_the_ring():
    """M == 0: no codes, amax 0 folded; K == 0: y = bias, codes of bias * s."""
    ring = ops.Ring(scale=2.0)
    a = torch.zeros((0, 64), dtype=torch.uint8, device="cuda")
    b = torch.zeros((96, 64), dtype=torch.uint8, device="cuda")
    before = oracle_ring_from(ring)
    out = ops.mm_ex(a, b, _scalar(1.0), _scalar(1.0), out_fmt=ops.E4M3, out_ring=ring)
    torch.cuda.synchronize()
    assert out.shape == (0, 96)
    OR.fold(before, np.float32(0.0), OF.E4M3)
    assert_ring_equal(ring, before)
    for kind in ("f32", "e4m3"):
        bias, bsc, bias_ref = _bias(96, kind, seed=9)
        a = torch.zeros((5, 0), dtype=torch.uint8, device="cuda")
        b = torch.zeros((96, 0), dtype=torch.uint8, device="cuda")
        before = oracle_ring_from(ring)
        out = ops.mm_ex(a, b, _scalar(1.0), _scalar(1.0), bias=bias, bias_scale=bsc, out_fmt=ops.E5M2, out_ring=ring)
        torch.cuda.synchronize()
        want = OR.scaled_codes(np.broadcast_to(bias_ref, (5, 96)), before.scale, OF.E5M2)
        assert np.array_equal(out.cpu().numpy(), want)
        OR.fold(before, OR.amax(bias_ref), OF.E5M2)
        assert_ring_equal(ring, before)


def test_fp8_output_rejects_bad_arguments():
    a = torch.zeros((128, 64), dtype=torch.uint8, device="cuda")
    b = torch.zeros((128, 64), dtype=torch.uint8, device="cuda")
    one = _scalar(1.0)
    with pytest.raises(ValueError):
        ops.mm_ex(a, b, one, one, out_fmt=ops.E4M3)  # no ring
    with pytest.raises(ValueError):
        ops.mm_ex(a, b, one, one, bias=torch.zeros(128, device="cuda"), bias_scale=one)  # float32 bias with a scale


def test_data_parallel_shards_fold_the_global_amax():
    """Two row shards of one FP8 output (two data-parallel ranks emulated on
    one GPU): each shard's launch casts with the shared ring's scale, reports
    its own max |y| and leaves history, idx and scale alone; the MAX of the
    two, folded with fp8_ring_fold, gives the oracle's fold of that amax, and
    that amax is within the bound of the whole output's exact amax."""
    from fp8_delayed_scaling_02_b200 import dp

    M, N, K = 1000, 768, 1024
    a, b = _inputs(M, N, K, seed=21)
    bias, _, bias_ref = _bias(N, "f32", seed=4)
    ref, S_ = OG.mm_fp8(a.numpy(), b.numpy(), ops.E4M3, ops.E4M3, 2.0 ** -7, 0.5, bias_ref)
    ad, bd = a.cuda(), b.cuda()
    ring = ops.Ring()
    shards = (slice(0, 384), slice(384, M))
    for step in range(3):
        before = oracle_ring_from(ring)
        amax = torch.zeros(2, dtype=torch.float32, device="cuda")
        codes = []
        for i, rows in enumerate(shards):
            codes.append(ops.mm_ex(ad[rows], bd, _scalar(2.0 ** -7), _scalar(0.5), bias=bias, out_fmt=ops.E4M3,
                                   out_ring=ring, out_amax=amax[i:i + 1]))
        torch.cuda.synchronize()
        hist, idx, scale, scale_inv, scratch = ring.state()
        assert np.array_equal(hist.numpy(), before.history) and idx == before.idx  # no fold yet
        assert np.float32(scale) == before.scale
        assert np.float32(scale_inv) == np.float32(np.float32(1.0) / before.scale)
        assert all(int(v) == 0 for v in scratch)
        lo, hi = OG.out8_code_range(ref, S_, before.scale, OF.E4M3)
        g = torch.cat(codes).cpu().numpy()
        assert OG.codes_within(g, lo, hi, OF.E4M3).all()
        m = amax.max().reshape(1)  # what the MAX all-reduce of the ranks computes
        dp.all_reduce_amax(m)      # no process group here: a no-op
        ops.ring_fold(ring, ops.E4M3, m)
        torch.cuda.synchronize()
        a_ref, tol = OG.amax_range(ref, S_)
        assert abs(float(m.item()) - a_ref) <= tol
        expect = before.copy()
        OR.fold(expect, np.float32(m.item()), OF.E4M3)
        assert_ring_equal(ring, expect)
