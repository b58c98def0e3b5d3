"""The kernels' timeout path, made to run on purpose without faulting or hanging the GPU.

fp8_debug_wait shortens the budget of the waits on another role's progress
to 20 microseconds and names a wait site at which the next launches wait on
a barrier nothing completes: that wait runs out, records its site code in
the device error word, and the kernel stops early (the GEMM raises its abort
flag, lets its own copies and MMAs land with the full drain budget, frees
TMEM and returns; the quantize producer stops claiming, drains its copies
and the last CTA still folds and clears the ring's scratch; the row layout's
kernel streams with plain loads and has no waits).  Each test then
restores the defaults, checks fp8_device_error reports FP8_ERR_DEVICE_TIMEOUT
at that site, and runs the same call again, which must match the oracle.
"""

import numpy as np
import pytest
import torch

from fp8_delayed_scaling_02_b200 import ops, synthetic as S
from gpu_helpers import OG, OR, assert_bytes_equal, assert_ring_equal, mm_check, oracle_codes, require_gpu

pytestmark = pytest.mark.gpu

BUDGET_NS = 20_000


@pytest.fixture(autouse=True)
def _gpu():
    require_gpu()
    yield
    ops.debug_wait()  # defaults, whatever happened


def _stalled(site, fn):
    torch.cuda.synchronize()
    assert ops.device_error(clear=True)[0] == ops.FP8_OK
    ops.debug_wait(BUDGET_NS, site)
    try:
        fn()
        torch.cuda.synchronize()
    finally:
        ops.debug_wait()
    rc, where = ops.device_error(clear=True)
    assert rc == ops.FP8_ERR_DEVICE_TIMEOUT and where == site, (rc, where)


@pytest.mark.parametrize("shifted", [False, True])
@pytest.mark.parametrize("layout", [ops.TRANSPOSED, ops.DUAL])
def test_quantize_wait_runs_out_then_the_next_call_is_exact(layout, shifted):
    """The TMA tile kernels (transposed / dual of rows that are a multiple of
    16 bytes): 16-byte aligned base, and a base one element past 16 bytes."""
    x = S.quant_sweep_input(2048, 1536, "bf16", 1.0, seed=9)
    if shifted:
        flat = torch.empty(x.numel() + 1, dtype=x.dtype, device="cuda")
        flat[1:].copy_(x.reshape(-1))
        xd = flat[1:].view(x.shape)
    else:
        xd = x.cuda()
    failed = ops.Ring()
    _stalled(ops.SITE_QUANTIZE_TMA, lambda: ops.quantize(xd, ops.E4M3, layout, failed))
    assert all(int(v) == 0 for v in failed.state()[4]), "the stopped call still clears the scratch words"
    ring, ref = ops.Ring(), OR.Ring()
    out, out_t = ops.quantize(xd, ops.E4M3, layout, ring)
    torch.cuda.synchronize()
    codes = oracle_codes(x, ref.scale, OR.F.E4M3)
    OR.fold(ref, OR.amax(OR.to_float32(x)), OR.F.E4M3)
    if out is not None:
        assert_bytes_equal(out, codes, "out")
    if out_t is not None:
        assert_bytes_equal(out_t, np.ascontiguousarray(codes.T), "out_t")
    assert_ring_equal(ring, ref)


def test_gemm_wait_runs_out_then_the_next_call_is_within_the_bound():
    """One CTA (M = 128, N = 256: a single 128 x 256 tile), K = 4096."""
    a = S.fp8_codes((128, 4096), seed=1)
    b = S.fp8_codes((256, 4096), seed=2)
    ad, bd = a.cuda(), b.cuda()
    one = torch.ones(1, device="cuda")
    _stalled(ops.SITE_EPILOGUE_TMEM_FULL, lambda: ops.mm(ad, bd, one, one))
    y = ops.mm(ad, bd, one, one)
    torch.cuda.synchronize()
    mm_check(y, a.numpy(), b.numpy(), ops.E4M3, ops.E4M3, np.float32(1.0), np.float32(1.0), None)
