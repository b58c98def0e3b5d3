"""GPU parity of the 1.2B-model linear workload over 16 delayed-scaling steps, M in {512, 2048, 8192}.

Per step and per linear shape (W1 [1536,1536], W2 [4096,1536]), in the launch
configurations the bench times: fwd Y = Xq.Wq^T + b (fp8_mm with the
stream-K workspace) and dX = Gq.Wq, dW = Gq^T.Xq in one fp8_mm_pair launch,
each GEMM with its rings' scale_inv, and X, W (E4M3) and G (E5M2) quantized
in one fp8_quantize_multi launch -- either in dual layout with NT backward
GEMMs on the transposed copies (the headline step), or in row layout only with
the backward GEMMs reading the row copies as MN-major operands (the layout-tag
step).  The three rings are checked
against the oracle after every step (bit-exact: amax history, idx, scale,
scale_inv).  At the first and the last step every byte of the six quantized
tensors is compared, and the three GEMM outputs on three rows of every
128-row band (every M tile and both halves of every CTA-pair tile; each row
spans every N tile).
"""

import numpy as np
import pytest
import torch

from fp8_delayed_scaling_02_b200 import ops, synthetic as S
from gpu_helpers import OG, OR, assert_bytes_equal, assert_ring_equal, band_rows, oracle_codes, require_gpu

pytestmark = pytest.mark.gpu

STEPS = 16
HIDDEN = 1536


@pytest.fixture(autouse=True)
def _gpu():
    require_gpu()


def _workspace(M, n_out):
    need = 0
    for (m, nn, k) in ((M, n_out, HIDDEN), (M, HIDDEN, n_out), (n_out, HIDDEN, M)):
        for amn, bmn in ((False, False), (False, True), (True, True)):
            need = max(need, ops.mm_workspace_bytes(m, nn, k, a_mn_major=amn, b_mn_major=bmn))
    return torch.zeros(max(need, 256), dtype=torch.uint8, device="cuda")


def _check_gemm(y, a_codes, b_codes, fmt_a, sinv_a, sinv_b, bias, rows, what):
    ref, Ssum = OG.mm_fp8_rows(a_codes, b_codes, fmt_a, 0, sinv_a, sinv_b, bias, rows)
    ok, ratio = OG.check(y.float().cpu().numpy()[rows], ref, Ssum)
    assert ok, (what, ratio)


@pytest.mark.parametrize("M", [512, 2048, 8192])
@pytest.mark.parametrize("which", [0, 1])
@pytest.mark.parametrize("layout_tag", [False, True])
def test_linear_1p2b_sixteen_delayed_steps(M, which, layout_tag):
    (w1, b1), (w2, b2) = S.linear_1p2b_weights()
    w, bias = (w1, b1) if which == 0 else (w2, b2)
    n_out = w.shape[0]
    rx, rw, rg = ops.Ring(), ops.Ring(), ops.Ring()
    ox, ow, og = OR.Ring(), OR.Ring(), OR.Ring()
    wd, bd = w.cuda(), bias.cuda()
    ws = _workspace(M, n_out)
    u8 = dict(dtype=torch.uint8, device="cuda")
    xq, xq_t = torch.empty((M, HIDDEN), **u8), torch.empty((HIDDEN, M), **u8)
    wq, wq_t = torch.empty((n_out, HIDDEN), **u8), torch.empty((HIDDEN, n_out), **u8)
    gq, gq_t = torch.empty((M, n_out), **u8), torch.empty((n_out, M), **u8)
    bf = dict(dtype=torch.bfloat16, device="cuda")
    y, dx, dw = torch.empty((M, n_out), **bf), torch.empty((M, HIDDEN), **bf), torch.empty((n_out, HIDDEN), **bf)
    w_amax = OR.amax(OR.to_float32(w))
    for step in range(STEPS):
        x, g = S.linear_1p2b_step(M, n_out, step)
        sx, sw, sg = ox.scale, ow.scale, og.scale  # scales this step's quantizes use
        lay = ops.ROW if layout_tag else ops.DUAL
        ops.quantize_multi([dict(x=x.cuda(), fmt=ops.E4M3, layout=lay, ring=rx, out=xq, out_t=xq_t),
                            dict(x=wd, fmt=ops.E4M3, layout=lay, ring=rw, out=wq, out_t=wq_t),
                            dict(x=g.cuda(), fmt=ops.E5M2, layout=lay, ring=rg, out=gq, out_t=gq_t)])
        ops.mm(xq, wq, rx.scale_inv, rw.scale_inv, bd, out=y, workspace=ws)
        if layout_tag:
            ops.mm_pair(dict(a=gq, b=wq, sinv_a=rg.scale_inv, sinv_b=rw.scale_inv, fmt_a=ops.E5M2, out=dx,
                             b_mn_major=True),
                        dict(a=gq, b=xq, sinv_a=rg.scale_inv, sinv_b=rx.scale_inv, fmt_a=ops.E5M2, out=dw,
                             a_mn_major=True, b_mn_major=True), workspace=ws)
        else:
            ops.mm_pair(dict(a=gq, b=wq_t, sinv_a=rg.scale_inv, sinv_b=rw.scale_inv, fmt_a=ops.E5M2, out=dx),
                        dict(a=gq_t, b=xq_t, sinv_a=rg.scale_inv, sinv_b=rx.scale_inv, fmt_a=ops.E5M2, out=dw),
                        workspace=ws)
        torch.cuda.synchronize()
        OR.fold(ox, OR.amax(OR.to_float32(x)), OR.F.E4M3)
        OR.fold(ow, w_amax, OR.F.E4M3)
        OR.fold(og, OR.amax(OR.to_float32(g)), OR.F.E5M2)
        assert_ring_equal(rx, ox)
        assert_ring_equal(rw, ow)
        assert_ring_equal(rg, og)
        if step not in (0, STEPS - 1):
            continue
        what = f"M={M} N={n_out} step {step} {'layout tag' if layout_tag else 'dual'}"
        x_all, w_all, g_all = oracle_codes(x, sx, OR.F.E4M3), oracle_codes(w, sw, OR.F.E4M3), \
            oracle_codes(g, sg, OR.F.E5M2)
        for got, ref, name in ((xq, x_all, "xq"), (wq, w_all, "wq"), (gq, g_all, "gq")):
            assert_bytes_equal(got, ref, f"{name} {what}")
        if not layout_tag:
            for got, ref, name in ((xq_t, x_all, "xq_t"), (wq_t, w_all, "wq_t"), (gq_t, g_all, "gq_t")):
                assert_bytes_equal(got, np.ascontiguousarray(ref.T), f"{name} {what}")
        sinv_x, sinv_w, sinv_g = ox.scale_inv, ow.scale_inv, og.scale_inv
        rows_m, rows_n = band_rows(M, seed=M + step), band_rows(n_out, seed=n_out + step)
        _check_gemm(y, x_all, w_all, 0, sinv_x, sinv_w, bias.numpy(), rows_m, f"fwd {what}")
        _check_gemm(dx, g_all, np.ascontiguousarray(w_all.T), 1, sinv_g, sinv_w, None, rows_m, f"dX {what}")
        _check_gemm(dw, np.ascontiguousarray(g_all.T), np.ascontiguousarray(x_all.T), 1, sinv_g, sinv_x, None,
                    rows_n, f"dW {what}")
