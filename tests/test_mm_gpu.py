"""GPU parity of fp8_mm against the float64 oracle: |y - ref| <= ulp_bf16(ref) + 2^-20 sum|ab| sinv_a sinv_b."""

import numpy as np
import pytest
import torch

from fp8_delayed_scaling_02_b200 import ops, synthetic as S
from gpu_helpers import OG, OR, band_rows, mm_check, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    require_gpu()


def _scalar(v):
    return torch.tensor([v], dtype=torch.float32, device="cuda")


def _run(M, N, K, fmt_a=ops.E4M3, fmt_b=ops.E4M3, sa=1.0, sb=1.0, with_bias=False, seed=0, rows=None):
    a = S.fp8_codes((M, K), seed=seed, fmt=fmt_a)
    b = S.fp8_codes((N, K), seed=seed + 1, fmt=fmt_b)
    bias = S.uniform((N,), seed=seed + 2) if with_bias else None
    y = ops.mm(a.cuda(), b.cuda(), _scalar(sa), _scalar(sb), bias.cuda() if bias is not None else None,
               fmt_a=fmt_a, fmt_b=fmt_b)
    torch.cuda.synchronize()
    assert y.shape == (M, N) and y.dtype == torch.bfloat16
    return mm_check(y, a.numpy(), b.numpy(), fmt_a, fmt_b, np.float32(sa), np.float32(sb),
                    bias.numpy() if bias is not None else None, rows)


# Ragged and tiny shapes: M/N tails inside a 128 x BN tile, K tails inside a
# 128-byte stage, several tiles in every dimension.
@pytest.mark.parametrize("M,N,K", [(1, 1, 16), (5, 7, 48), (128, 128, 128), (200, 300, 160), (130, 129, 4096),
                                   (257, 513, 272), (384, 1024, 640)])
@pytest.mark.parametrize("with_bias", [False, True])
def test_small_and_ragged(M, N, K, with_bias):
    _run(M, N, K, with_bias=with_bias, sa=0.37, sb=0.125, seed=M + N + K)


@pytest.mark.parametrize("fa,fb", [(ops.E5M2, ops.E4M3), (ops.E4M3, ops.E5M2), (ops.E5M2, ops.E5M2)])
def test_mixed_formats(fa, fb):
    _run(256, 384, 512, fmt_a=fa, fmt_b=fb, with_bias=True, sa=2.0 ** -10, sb=3.5)


# Square sweep; full comparison up to 2048^3, above it three rows of every
# 128-row band (each M tile and each half of a CTA-pair tile; every row spans
# all N tiles).
@pytest.mark.parametrize("n", [512, 1024, 1152, 2048, 3072, 4096, 8192])
def test_square_sweep(n):
    rows = None if n <= 2048 else band_rows(n, seed=n)
    _run(n, n, n, with_bias=(n % 3 == 0 or n == 1024), seed=n, rows=rows)


def test_square_8192_scaled_with_bias():
    _run(8192, 8192, 8192, sa=0.37, sb=0.125, with_bias=True, seed=5, rows=band_rows(8192, seed=5))


def test_skinny_and_odd():
    _run(64, 8192, 2048, seed=11)
    _run(1024, 1536, 2048, seed=12)
    _run(1000, 1537, 2048, with_bias=True, seed=13)


def _quantized_normal(shape, seed):
    """N(0,1) fp32 quantized E4M3 per tensor through fp8_quantize (second call uses 448/amax)."""
    x = S.normal_with_outliers(shape, seed=seed, dtype="fp32").cuda()
    ring = ops.Ring()
    flat = x.reshape(-1, shape[-1])
    ops.quantize(flat, ops.E4M3, ops.ROW, ring)
    q, _ = ops.quantize(flat, ops.E4M3, ops.ROW, ring)
    return q.view(shape), ring.scale_inv.clone()


def test_batched_and_broadcast():
    # 64 x (512^3), both operands batched.
    a, sa = _quantized_normal((64, 512, 512), 21)
    b, sb = _quantized_normal((64, 512, 512), 22)
    y = ops.mm(a, b, sa, sb)
    torch.cuda.synchronize()
    assert y.shape == (64, 512, 512)
    ref, Ssum = OG.mm_fp8(a.cpu().numpy(), b.cpu().numpy(), 0, 0, sa.item(), sb.item())
    ok, ratio = OG.check(y.float().cpu().numpy(), ref, Ssum)
    assert ok, ratio
    # 8 x (1024 x 2048 x 2048) with a size-1 B batch broadcast at stride 0, bias.
    a, sa = _quantized_normal((8, 1024, 2048), 23)
    b, sb = _quantized_normal((1, 2048, 2048), 24)
    bias = S.uniform((2048,), seed=25)
    y = ops.mm(a, b, sa, sb, bias.cuda())
    torch.cuda.synchronize()
    assert y.shape == (8, 1024, 2048)
    rows = band_rows(1024, seed=25)
    for z in range(8):
        ref, Ssum = OG.mm_fp8_rows(a[z].cpu().numpy(), b[0].cpu().numpy(), 0, 0, sa.item(), sb.item(),
                                   bias.numpy(), rows)
        ok, ratio = OG.check(y[z].float().cpu().numpy()[rows], ref, Ssum)
        assert ok, (z, ratio)


def test_k_zero_gives_bias_and_empty_is_noop():
    bias = S.uniform((37,), seed=3).cuda()
    a = torch.zeros((5, 0), dtype=torch.uint8, device="cuda")
    b = torch.zeros((37, 0), dtype=torch.uint8, device="cuda")
    y = ops.mm(a, b, _scalar(1.0), _scalar(1.0), bias)
    torch.cuda.synchronize()
    assert torch.equal(y.float().cpu(), bias.cpu().to(torch.bfloat16).float().expand(5, 37))
    e = ops.mm(torch.zeros((0, 32), dtype=torch.uint8, device="cuda"),
               torch.zeros((4, 32), dtype=torch.uint8, device="cuda"), _scalar(1.0), _scalar(1.0))
    assert e.shape == (0, 4)


def test_pr1_linear_end_to_end():
    """Quantize X (row) and W (dual) through their rings for 3 steps, then
    Y = Xq . Wq^T * sinv_x * sinv_w + bias with the scale_inv the quantize used."""
    rx, rw = ops.Ring(), ops.Ring()
    ox, ow = OR.Ring(), OR.Ring()
    for step in range(3):
        x, w, bias = S.linear_pr1_step(step)
        xq, _ = ops.quantize(x.cuda(), ops.E4M3, ops.ROW, rx)
        wq, wq_t = ops.quantize(w.cuda(), ops.E4M3, ops.DUAL, rw)
        y = ops.mm(xq, wq, rx.scale_inv, rw.scale_inv, bias.cuda())
        torch.cuda.synchronize()
        rxq, _, _ = OR.quantize(x, 0, OR.ROW, ox)
        rwq, _, _ = OR.quantize(w, 0, OR.DUAL, ow)
        assert np.array_equal(xq.cpu().numpy(), rxq) and np.array_equal(wq.cpu().numpy(), rwq)
        ref, Ssum = OG.mm_fp8(rxq, rwq, 0, 0, ox.scale_inv, ow.scale_inv, bias.numpy())
        ok, ratio = OG.check(y.float().cpu().numpy(), ref, Ssum)
        assert ok, (step, ratio)


def test_device_error_word_clear():
    rc, where = ops.device_error(clear=True)
    assert rc == ops.FP8_OK and where == 0


# MN-major operands (the layout tag): A stored [K, M] and/or B stored [K, N];
# the oracle multiplies the untransposed codes.  M/N multiples of 16 (row
# pitch of the stored operand); K tails inside a 128-deep stage; M <= 128 runs
# the single-CTA kernel, larger M the CTA pair.
@pytest.mark.parametrize("a_mn,b_mn", [(True, False), (False, True), (True, True)])
@pytest.mark.parametrize("M,N,K", [(64, 256, 256), (128, 128, 160), (208, 304, 400), (512, 1536, 640),
                                   (1536, 1536, 2048)])
def test_mn_major_layouts(M, N, K, a_mn, b_mn):
    a = S.fp8_codes((M, K), seed=M + K)
    b = S.fp8_codes((N, K), seed=N + K + 1)
    bias = S.uniform((N,), seed=7)
    ad = a.t().contiguous().cuda() if a_mn else a.cuda()
    bd = b.t().contiguous().cuda() if b_mn else b.cuda()
    y = ops.mm(ad, bd, _scalar(0.5), _scalar(0.25), bias.cuda(), a_mn_major=a_mn, b_mn_major=b_mn)
    torch.cuda.synchronize()
    assert y.shape == (M, N)
    mm_check(y, a.numpy(), b.numpy(), ops.E4M3, ops.E4M3, np.float32(0.5), np.float32(0.25), bias.numpy())


def test_mn_major_backward_shapes_mixed_formats():
    """The step's dX (B = W as quantized) and dW (A = G, B = X as quantized) with an E5M2 gradient."""
    Mtok, n_out, hid = 512, 4096, 1536
    g = S.fp8_codes((Mtok, n_out), seed=31, fmt=ops.E5M2)
    w = S.fp8_codes((n_out, hid), seed=32)
    x = S.fp8_codes((Mtok, hid), seed=33)
    dx = ops.mm(g.cuda(), w.cuda(), _scalar(0.01), _scalar(2.0), fmt_a=ops.E5M2, b_mn_major=True)
    dw = ops.mm(g.cuda(), x.cuda(), _scalar(0.01), _scalar(0.5), fmt_a=ops.E5M2, a_mn_major=True, b_mn_major=True)
    torch.cuda.synchronize()
    rows = band_rows(512, seed=1)
    mm_check(dx, g.numpy(), w.numpy().T.copy(), ops.E5M2, ops.E4M3, np.float32(0.01), np.float32(2.0), None, rows)
    rows = band_rows(4096, seed=2)
    mm_check(dw, g.numpy().T.copy(), x.numpy().T.copy(), ops.E5M2, ops.E4M3, np.float32(0.01), np.float32(0.5),
             None, rows)


def test_mn_major_batched_broadcast():
    a = S.fp8_codes((4, 256, 192), seed=41)            # [batch, K, M]
    b = S.fp8_codes((1, 256, 160), seed=42)            # [1, K, N] broadcast
    y = ops.mm(a.cuda(), b.cuda(), _scalar(1.0), _scalar(1.0), a_mn_major=True, b_mn_major=True)
    torch.cuda.synchronize()
    assert y.shape == (4, 192, 160)
    for z in range(4):
        ref, Ssum = OG.mm_fp8(a[z].numpy().T.copy(), b[0].numpy().T.copy(), 0, 0, 1.0, 1.0)
        ok, ratio = OG.check(y[z].float().cpu().numpy(), ref, Ssum)
        assert ok, (z, ratio)


# Stream-K through a caller workspace (fp8_mm_ws): the k-blocks of the last
# waves' tiles are dealt evenly to the CTAs, and pieces that start inside a
# tile hand float32 partials to the CTA holding the tile's first k-block.
# Shapes: dW GEMMs of the linears with long K (fewer tiles than CTA pairs), wide outputs
# with a wave of whole tiles before the stream-K tail (one ragged in M and
# N), a tiny output cut four ways per tile, and ragged ones on 128-wide pair
# tiles.  Checked against the oracle, deterministic across runs, flags left
# at zero, and an undersized workspace falls back to whole tiles.
@pytest.mark.parametrize("M,N,K,a_mn,b_mn", [(1536, 1536, 16384, False, False), (4096, 1536, 8192, True, True),
                                             (1536, 1536, 16384, True, True), (512, 19200, 4096, False, False),
                                             (500, 19199, 4096, False, False), (128, 256, 8192, False, False),
                                             (1000, 1537, 8192, False, False), (130, 700, 8192, False, False)])
def test_split_k_workspace(M, N, K, a_mn, b_mn):
    a = S.fp8_codes((M, K), seed=M + 3)
    b = S.fp8_codes((N, K), seed=N + 4)
    bias = S.uniform((N,), seed=5)
    need = ops.mm_workspace_bytes(M, N, K, a_mn_major=a_mn, b_mn_major=b_mn)
    assert need > 0, "this shape should use stream-K pieces"
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    ad = a.t().contiguous().cuda() if a_mn else a.cuda()
    bd = b.t().contiguous().cuda() if b_mn else b.cuda()
    args = (ad, bd, _scalar(0.37), _scalar(0.125), bias.cuda())
    y1 = ops.mm(*args, a_mn_major=a_mn, b_mn_major=b_mn, workspace=ws)
    y2 = ops.mm(*args, a_mn_major=a_mn, b_mn_major=b_mn, workspace=ws)
    small = torch.zeros(256, dtype=torch.uint8, device="cuda")
    y3 = ops.mm(*args, a_mn_major=a_mn, b_mn_major=b_mn, workspace=small)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2), "stream-K must be deterministic"
    assert int(ws[:1024].count_nonzero()) == 0, "piece flags (the first 1024 bytes) must return to zero"
    rows = band_rows(M, seed=M)
    for y in (y1, y3):
        mm_check(y, a.numpy(), b.numpy(), ops.E4M3, ops.E4M3, np.float32(0.37), np.float32(0.125), bias.numpy(),
                 rows)


# fp8_mm_pair: two independent GEMMs in one launch (the dX and dW of a
# linear), CTAs split between them.  Shapes: both linears' backward GEMMs
# (paired with CTA pairs), a single-CTA pairing (one problem with M <= 128),
# a ragged pair, and pairs the library runs one after the other (K = 0 on
# one side).  Each output is checked against the oracle on sampled rows.
PAIR_CASES = [
    ((8192, 1536, 1536, False, True), (1536, 1536, 8192, True, True)),
    ((8192, 1536, 4096, False, True), (4096, 1536, 8192, True, True)),
    ((128, 512, 4096, False, False), (2048, 2048, 1024, False, False)),
    ((1000, 1537, 512, False, False), (130, 700, 8192, False, False)),
    ((512, 256, 0, False, False), (256, 384, 1024, False, False)),
]


@pytest.mark.parametrize("c0,c1", PAIR_CASES)
def test_mm_pair_matches_the_oracle(c0, c1):
    probs, refs = [], []
    for i, (M, N, K, a_mn, b_mn) in enumerate((c0, c1)):
        a = S.fp8_codes((M, K), seed=M + K + i, fmt=ops.E5M2 if i == 1 else ops.E4M3)
        b = S.fp8_codes((N, K), seed=N + K + 7 * i)
        bias = S.uniform((N,), seed=11 + i) if i == 0 else None
        ad = a.t().contiguous().cuda() if a_mn else a.cuda()
        bd = b.t().contiguous().cuda() if b_mn else b.cuda()
        probs.append(dict(a=ad, b=bd, sinv_a=_scalar(0.5 + i), sinv_b=_scalar(0.25), bias=None if bias is None else
                          bias.cuda(), fmt_a=ops.E5M2 if i == 1 else ops.E4M3, a_mn_major=a_mn, b_mn_major=b_mn))
        refs.append((a, b, bias, M, i))
    y0, y1 = ops.mm_pair(probs[0], probs[1])
    torch.cuda.synchronize()
    for y, (a, b, bias, M, i) in zip((y0, y1), refs):
        rows = band_rows(M, seed=M + i)
        mm_check(y, a.numpy(), b.numpy(), ops.E5M2 if i == 1 else ops.E4M3, ops.E4M3, np.float32(0.5 + i),
                 np.float32(0.25), None if bias is None else bias.numpy(), rows)


def test_mm_pair_equals_separate_calls_when_the_shapes_match():
    """With one launch shape for both (256-wide CTA pairs, whole tiles) the
    paired results equal the single calls bit for bit."""
    # 48 long tiles (K = 8192) beside 256 short ones (K = 1024): paired, and
    # each alone also runs 256-wide CTA pairs over whole tiles.
    a0, b0 = S.fp8_codes((2048, 8192), seed=1).cuda(), S.fp8_codes((1536, 8192), seed=2).cuda()
    a1, b1 = S.fp8_codes((8192, 1024), seed=3).cuda(), S.fp8_codes((2048, 1024), seed=4).cuda()
    s = _scalar(1.0)
    y0, y1 = ops.mm_pair(dict(a=a0, b=b0, sinv_a=s, sinv_b=s), dict(a=a1, b=b1, sinv_a=s, sinv_b=s))
    z0 = ops.mm(a0, b0, s, s)
    z1 = ops.mm(a1, b1, s, s)
    torch.cuda.synchronize()
    assert torch.equal(y0, z0) and torch.equal(y1, z1)
