"""GPU parity of the current-scaling quantize and the bias gradient against the oracle."""

import numpy as np
import pytest
import torch

from fp8_delayed_scaling_02_b200 import ops, synthetic as S
from gpu_helpers import assert_bytes_equal, require_gpu
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
