"""GPU parity of the 1.2B-model linear workload over 16 delayed-scaling steps (M = 512).

Per step and per linear shape (W1 [1536,1536], W2 [4096,1536]): X dual E4M3,
W dual E4M3, G dual E5M2, then fwd Y = Xq.Wq^T + b, dX = Gq.(W^T)q^T and
dW = (G^T)q.(X^T)q^T with each ring's scale_inv.  The three rings per linear
are checked against the oracle after every step (bit-exact: amax history,
idx, scale, scale_inv); the quantized bytes and the three GEMM outputs are
checked on sampled rows at the first and the last step.
"""

import numpy as np
import pytest
import torch

from fp8_delayed_scaling_02_b200 import ops, synthetic as S
from gpu_helpers import OG, OR, assert_ring_equal, require_gpu

pytestmark = pytest.mark.gpu

M = 512
STEPS = 16


@pytest.fixture(autouse=True)
def _gpu():
    require_gpu()


def _codes_rows(x, ring_scale, fmt, rows):
    """Oracle codes of rows `rows` of x quantized with the scale the call used."""
    return OR.scaled_codes(OR.to_float32(x)[rows], np.float32(ring_scale), fmt)


@pytest.mark.parametrize("which", [0, 1])
def test_linear_1p2b_sixteen_delayed_steps(which):
    (w1, b1), (w2, b2) = S.linear_1p2b_weights()
    w, bias = (w1, b1) if which == 0 else (w2, b2)
    n_out = w.shape[0]
    rx, rw, rg = ops.Ring(), ops.Ring(), ops.Ring()
    ox, ow, og = OR.Ring(), OR.Ring(), OR.Ring()
    wd, bd = w.cuda(), bias.cuda()
    rng = np.random.default_rng(which)
    for step in range(STEPS):
        x, g = S.linear_1p2b_step(M, n_out, step)
        sx, sw, sg = ox.scale, ow.scale, og.scale  # scales this step's quantizes use
        xq, xq_t = ops.quantize(x.cuda(), ops.E4M3, ops.DUAL, rx)
        wq, wq_t = ops.quantize(wd, ops.E4M3, ops.DUAL, rw)
        gq, gq_t = ops.quantize(g.cuda(), ops.E5M2, ops.DUAL, rg)
        y = ops.mm(xq, wq, rx.scale_inv, rw.scale_inv, bd)
        dx = ops.mm(gq, wq_t, rg.scale_inv, rw.scale_inv, None, fmt_a=ops.E5M2)
        dw = ops.mm(gq_t, xq_t, rg.scale_inv, rx.scale_inv, None, fmt_a=ops.E5M2)
        torch.cuda.synchronize()
        for ring_ref, t in ((ox, x), (ow, w), (og, g)):
            OR.fold(ring_ref, OR.amax(OR.to_float32(t)), 0 if ring_ref is not og else 1)
        assert_ring_equal(rx, ox)
        assert_ring_equal(rw, ow)
        assert_ring_equal(rg, og)
        if step not in (0, STEPS - 1):
            continue
        mr = np.unique(np.concatenate([rng.integers(0, M, 12), [0, M - 1]]))
        nr = np.unique(np.concatenate([rng.integers(0, n_out, 12), [0, n_out - 1]]))
        # quantized bytes (row and transposed layouts) on sampled rows
        x_rows = _codes_rows(x, sx, OR.F.E4M3, mr)
        assert np.array_equal(xq.cpu().numpy()[mr], x_rows)
        assert np.array_equal(xq_t.cpu().numpy()[:, mr].T, x_rows)
        g_rows = _codes_rows(g, sg, OR.F.E5M2, mr)
        assert np.array_equal(gq.cpu().numpy()[mr], g_rows)
        w_rows = _codes_rows(w, sw, OR.F.E4M3, nr)
        assert np.array_equal(wq.cpu().numpy()[nr], w_rows)
        # full codes needed as the other GEMM operand
        x_all = OR.scaled_codes(OR.to_float32(x), np.float32(sx), OR.F.E4M3)
        w_all = OR.scaled_codes(OR.to_float32(w), np.float32(sw), OR.F.E4M3)
        g_all = OR.scaled_codes(OR.to_float32(g), np.float32(sg), OR.F.E5M2)
        sinv_x, sinv_w, sinv_g = ox.scale_inv, ow.scale_inv, og.scale_inv
        ref, Ssum = OG.mm_fp8_rows(x_all, w_all, 0, 0, sinv_x, sinv_w, bias.numpy(), mr)
        ok, ratio = OG.check(y.float().cpu().numpy()[mr], ref, Ssum)
        assert ok, ("fwd", step, ratio)
        ref, Ssum = OG.mm_fp8_rows(g_all, np.ascontiguousarray(w_all.T), 1, 0, sinv_g, sinv_w, None, mr)
        ok, ratio = OG.check(dx.float().cpu().numpy()[mr], ref, Ssum)
        assert ok, ("dX", step, ratio)
        ref, Ssum = OG.mm_fp8_rows(np.ascontiguousarray(g_all.T), np.ascontiguousarray(x_all.T), 1, 0, sinv_g,
                                   sinv_x, None, nr)
        ok, ratio = OG.check(dw.float().cpu().numpy()[nr], ref, Ssum)
        assert ok, ("dW", step, ratio)
