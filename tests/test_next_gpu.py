"""GPU parity of the current-scaling quantize and the bias gradient against the oracle."""

import numpy as np
import pytest
import torch

from fp8_delayed_scaling_02_b200 import ops, synthetic as S
from gpu_helpers import assert_bytes_equal, assert_ring_equal, require_gpu
from oracle import bias_grad as OB
from oracle import recipe as OR

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    require_gpu()


def _bits(v):
    return np.float32(v).view(np.uint32)


def _check_current(x, fmt, layout, misalign=False):
    if misalign:
        flat = torch.empty(x.numel() + 1, dtype=x.dtype, device="cuda")
        flat[1:].copy_(x.reshape(-1))
        xd = flat[1:].view(x.shape)
    else:
        xd = x.cuda()
    cs = ops.CurrentScale()
    out, out_t = ops.quantize_current(xd, fmt, layout, cs)
    torch.cuda.synchronize()
    r_out, r_out_t, a, s, si = OR.quantize_current(x, fmt, layout)
    if out is not None:
        assert_bytes_equal(out, r_out, "out")
    if out_t is not None:
        assert_bytes_equal(out_t, r_out_t, "out_t")
    assert _bits(cs.scale.item()) == _bits(s)
    assert _bits(cs.scale_inv.item()) == _bits(si)
    assert _bits(cs.amax.item()) == _bits(a)
    assert all(int(v) == 0 for v in cs.scratch.cpu()), "scratch must self-reset"
    return cs


@pytest.mark.parametrize("dtype", ["bf16", "fp16", "fp32"])
@pytest.mark.parametrize("fmt", [ops.E4M3, ops.E5M2])
@pytest.mark.parametrize("layout", [ops.ROW, ops.TRANSPOSED, ops.DUAL])
def test_current_scaling_small_and_ragged(dtype, fmt, layout):
    for i, (r, c) in enumerate([(1, 1), (7, 33), (130, 70), (301, 1537), (256, 512)]):
        x = S.quant_sweep_input(r, c, dtype, [1.0, 1e-3, 1e3][i % 3], seed=50 + i)
        _check_current(x, fmt, layout, misalign=(i % 2 == 1))


@pytest.mark.parametrize("layout", [ops.ROW, ops.DUAL])
def test_current_scaling_full_size_and_repeat(layout):
    x = S.linear_1p2b_step(8192, 1536, 0)[0]
    cs1 = _check_current(x, ops.E4M3, layout)
    cs2 = _check_current(x, ops.E4M3, layout)  # fresh state, same answer
    assert cs1.scale.item() == cs2.scale.item()


def test_current_scaling_zero_input():
    cs = _check_current(torch.zeros((64, 48), dtype=torch.bfloat16), ops.E4M3, ops.DUAL)
    assert cs.scale.item() == 1.0


@pytest.mark.parametrize("dtype", ["bf16", "fp16", "fp32"])
@pytest.mark.parametrize("shape", [(1, 1), (7, 33), (1000, 1537), (8192, 1536), (8192, 4096)])
def test_bias_grad_within_bound_and_deterministic(dtype, shape):
    g = S.normal_with_outliers(shape, seed=shape[0] + shape[1], std=1e-3, dtype=dtype)
    gd = g.cuda()
    db1 = ops.bias_grad(gd)
    db2 = ops.bias_grad(gd)
    torch.cuda.synchronize()
    a, b = db1.cpu().numpy(), db2.cpu().numpy()
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32)), "bias gradient must be deterministic"
    ref = OB.bias_grad(g)
    assert np.all(np.abs(a.astype(np.float64) - ref) <= OB.bound(g))


def test_bias_grad_exact_on_integers_and_3d():
    g = torch.randint(-8, 9, (4, 300, 96), dtype=torch.int32).to(torch.bfloat16)
    db = ops.bias_grad(g.cuda())
    torch.cuda.synchronize()
    assert np.array_equal(db.cpu().numpy().astype(np.float64), OB.bias_grad(g.reshape(-1, 96)))


def test_linear_composite_matches_the_separate_calls_and_oracle():
    """fp8_linear_forward/backward over 3 delayed steps equal, bit for bit, the
    same sequence of individual calls, and the last step matches the oracle."""
    from oracle import gemm as OG

    M, N, K = 256, 384, 512
    lin = ops.Linear()
    rx, rw, rg = ops.Ring(), ops.Ring(), ops.Ring()
    for step in range(3):
        x = S.normal_with_outliers((M, K), seed=60 + step, frac=0.01, mult=20.0).cuda()
        w = S.normal_with_outliers((N, K), seed=70 + step, std=0.02).cuda()
        g = S.normal_with_outliers((M, N), seed=80 + step, std=1e-3).cuda()
        bias = S.uniform((N,), seed=90).cuda()
        y = lin.forward(x, w, bias)
        dx, dw, db = lin.backward(g)
        xq, _ = ops.quantize(x, ops.E4M3, ops.ROW, rx)
        wq, _ = ops.quantize(w, ops.E4M3, ops.ROW, rw)
        y2 = ops.mm(xq, wq, rx.scale_inv, rw.scale_inv, bias)
        gq, _ = ops.quantize(g, ops.E5M2, ops.ROW, rg)
        dx2 = ops.mm(gq, wq, rg.scale_inv, rw.scale_inv, fmt_a=ops.E5M2, b_mn_major=True)
        dw2 = ops.mm(gq, xq, rg.scale_inv, rx.scale_inv, fmt_a=ops.E5M2, a_mn_major=True, b_mn_major=True)
        db2 = ops.bias_grad(g)
        torch.cuda.synchronize()
        for a, b in ((y, y2), (dx, dx2), (dw, dw2), (db, db2)):
            assert torch.equal(a, b)
        for r1, r2 in ((lin.rx, rx), (lin.rw, rw), (lin.rg, rg)):
            assert torch.equal(r1.buf, r2.buf)
    ref, Ssum = OG.mm_fp8(xq.cpu().numpy(), wq.cpu().numpy(), 0, 0, rx.scale_inv.item(), rw.scale_inv.item(),
                          bias.cpu().numpy())
    assert OG.check(y.float().cpu().numpy(), ref, Ssum)[0]
    ref, Ssum = OG.mm_fp8(gq.cpu().numpy(), wq.cpu().numpy().T.copy(), 1, 0, rg.scale_inv.item(), rw.scale_inv.item())
    assert OG.check(dx.float().cpu().numpy(), ref, Ssum)[0]
    ref, Ssum = OG.mm_fp8(gq.cpu().numpy().T.copy(), xq.cpu().numpy().T.copy(), 1, 0, rg.scale_inv.item(),
                          rx.scale_inv.item())
    assert OG.check(dw.float().cpu().numpy(), ref, Ssum)[0]
    assert np.all(np.abs(db.cpu().numpy().astype(np.float64) - OB.bias_grad(g.cpu())) <= OB.bound(g.cpu()))


@pytest.mark.parametrize("dtype,fmt", [("bf16", ops.E4M3), ("fp32", ops.E5M2)])
@pytest.mark.parametrize("layout", [ops.ROW, ops.TRANSPOSED, ops.DUAL])
def test_quantize_local_then_fold_equals_quantize(dtype, fmt, layout):
    """fp8_quantize_local + fp8_ring_fold of its own amax = fp8_quantize, bit for bit, over 4 steps."""
    r1, r2 = ops.Ring(), ops.Ring()
    for step, (rows, cols) in enumerate([(256, 512), (130, 70), (8192, 1536), (7, 33)]):
        x = S.quant_sweep_input(rows, cols, dtype, [1.0, 1e-3, 1e3, 1.0][step], seed=400 + step).cuda()
        o1, t1 = ops.quantize(x, fmt, layout, r1)
        o2, t2, amax = ops.quantize_local(x, fmt, layout, r2)
        assert torch.equal(r2.scale_inv, r1.scale_inv), "scale_inv is published by the local cast"
        ops.ring_fold(r2, fmt, amax)
        torch.cuda.synchronize()
        for a, b in ((o1, o2), (t1, t2)):
            if a is not None:
                assert torch.equal(a, b)
        assert torch.equal(r1.buf, r2.buf)
        assert _bits(amax.item()) == _bits(OR.amax(OR.to_float32(x.cpu())))


def test_dp_two_shards_match_the_whole_tensor():
    """Two ranks emulated on one GPU: each casts its shard, the MAX of the two
    amaxes (taken on the device, as the collective would) is folded into both
    rings; codes and rings equal one quantize of the whole tensor and the oracle."""
    rows, cols = 2048, 1536
    r0, r1, rr = ops.Ring(), ops.Ring(), ops.Ring()
    ref = OR.Ring()
    for step in range(5):
        full = S.normal_with_outliers((rows, cols), seed=500 + step, frac=0.005, mult=10.0 * (1 + step % 3))
        x = full.cuda()
        o0, t0, a0 = ops.quantize_local(x[: rows // 2].contiguous(), ops.E4M3, ops.DUAL, r0)
        o1, t1, a1 = ops.quantize_local(x[rows // 2:].contiguous(), ops.E4M3, ops.DUAL, r1)
        g = torch.maximum(a0, a1)
        ops.ring_fold(r0, ops.E4M3, g)
        ops.ring_fold(r1, ops.E4M3, g)
        o, t = ops.quantize(x, ops.E4M3, ops.DUAL, rr)
        torch.cuda.synchronize()
        assert torch.equal(torch.cat([o0, o1]), o)
        assert torch.equal(torch.cat([t0, t1], dim=1), t)
        assert torch.equal(r0.buf, rr.buf) and torch.equal(r1.buf, rr.buf)
        r_out, r_out_t, _ = OR.quantize(full, OR.F.E4M3, OR.DUAL, ref)
        assert_bytes_equal(o, r_out, "out")
    assert_ring_equal(rr, ref)


def test_ring_fold_of_a_nan_amax_matches_the_oracle():
    """A caller-supplied NaN amax (a data-parallel fold) is stored in its slot
    and skipped by the window maximum on both sides; the scales stay those of
    the finite entries.  Then a finite fold, then a ring whose only entry is
    NaN (the scale is kept)."""
    for fmt in (ops.E4M3, ops.E5M2):
        ring, ref = ops.Ring(), OR.Ring()
        for a in (3.0, float("nan"), 0.75, float("nan"), 7.5):
            amax = torch.tensor([a], dtype=torch.float32, device="cuda")
            ops.ring_fold(ring, fmt, amax)
            OR.fold(ref, np.float32(a), fmt)
            torch.cuda.synchronize()
            assert_ring_equal(ring, ref)
        only, ref_only = ops.Ring(scale=0.625), OR.Ring(scale=0.625)
        ops.ring_fold(only, fmt, torch.tensor([float("nan")], dtype=torch.float32, device="cuda"))
        OR.fold(ref_only, np.float32("nan"), fmt)
        torch.cuda.synchronize()
        assert_ring_equal(only, ref_only)
