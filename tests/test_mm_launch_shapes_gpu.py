"""GPU parity of every launch shape the GEMM chooser can pick.

fp8_mm_launch_shape reports the tile width, cluster size, CTA count and
stream-K pieces of a call.  One problem per (tile width, cluster, stream-K)
class -- 64-, 128- and 256-wide tiles on single CTAs, 256-wide tiles on CTA
pairs, each with whole tiles only and with a stream-K tail -- is run with an
fp32 bias and checked against the oracle on three rows of every 128-row band
(every row of a small M); on a 148-SM B200 the test also asserts that the
problem lands in its class.  The cheaper problems also run with an E4M3
output and delayed output scaling, checked like the FP8-output tests: every
code in the oracle's interval, the folded amax within its bound, the ring
exactly the oracle's fold.
"""

import numpy as np
import pytest
import torch

from fp8_delayed_scaling_02_b200 import ops, synthetic as S
from gpu_helpers import OG, OR, assert_ring_equal, band_rows, oracle_ring_from, require_gpu

pytestmark = pytest.mark.gpu

# (bn, cluster, stream-K) -> (M, N, K): ragged M and N, odd N (unaligned rows:
# guarded stores), long K for the stream-K tails.
CASES = [
    ((64, 1, False), (130, 700, 512)),
    ((64, 1, True), (130, 256, 8192)),
    ((128, 1, False), (1000, 1536, 512)),
    ((128, 1, True), (130, 1537, 16384)),
    ((256, 1, False), (1536, 1537, 512)),
    ((256, 1, True), (384, 8192, 16384)),
    ((256, 2, False), (1536, 1537, 4096)),
    ((256, 2, True), (1536, 4096, 4096)),
]


@pytest.fixture(autouse=True)
def _gpu():
    require_gpu()


def _scalar(v):
    return torch.tensor([v], dtype=torch.float32, device="cuda")


def _b200():
    return torch.cuda.get_device_properties(0).multi_processor_count == 148


@pytest.mark.parametrize("cls,shape", CASES, ids=[f"bn{c[0]}x{c[1]}{'-sk' if c[2] else ''}" for c, _ in CASES])
def test_launch_shape_class_matches_the_oracle(cls, shape):
    bn, cluster, sk = cls
    M, N, K = shape
    ws_bytes = ops.mm_workspace_bytes(M, N, K) if sk else 0
    got = ops.mm_launch_shape(M, N, K, workspace_bytes=ws_bytes)
    if _b200():
        assert (got["bn"], got["cluster"], got["stream_k_pieces"] > 0) == cls, got
    ws = torch.zeros(max(ws_bytes, 256), dtype=torch.uint8, device="cuda") if sk else None
    a = S.fp8_codes((M, K), seed=M + K)
    b = S.fp8_codes((N, K), seed=N + K + 1)
    bias = S.uniform((N,), seed=N) * 2.0
    sinv_a, sinv_b = 2.0 ** -6, 0.375
    ad, bd = a.cuda(), b.cuda()
    y = ops.mm(ad, bd, _scalar(sinv_a), _scalar(sinv_b), bias.cuda(), workspace=ws)
    torch.cuda.synchronize()
    rows = np.arange(M) if M <= 512 else band_rows(M, seed=M)
    ref, Ssum = OG.mm_fp8_rows(a.numpy(), b.numpy(), 0, 0, sinv_a, sinv_b, bias.numpy(), rows)
    ok, ratio = OG.check(y.float().cpu().numpy()[rows], ref, Ssum)
    assert ok, (got, ratio)
    if ws is not None:
        assert int(ws[:1024].view(torch.int32).abs().sum()) == 0  # stream-K flags left clear
    if M * N * K > 4e9:
        return
    # E4M3 output with delayed output scaling, two steps (scale 1, then the folded one).
    ref, Ssum = OG.mm_fp8(a.numpy(), b.numpy(), 0, 0, sinv_a, sinv_b, bias.numpy())
    ring = ops.Ring()
    for _ in range(2):
        before = oracle_ring_from(ring)
        out = ops.mm_ex(ad, bd, _scalar(sinv_a), _scalar(sinv_b), bias=bias.cuda(), out_fmt=ops.E4M3,
                        out_ring=ring, workspace=ws)
        torch.cuda.synchronize()
        lo, hi = OG.out8_code_range(ref, Ssum, np.float32(before.scale), ops.E4M3)
        g = out.cpu().numpy().reshape(ref.shape)
        inside = OG.codes_within(g, lo, hi, ops.E4M3)
        assert inside.all(), f"{int((~inside).sum())} codes outside the interval, first at {np.argwhere(~inside)[0]}"
        fixed = lo == hi
        assert np.array_equal(g[fixed], lo[fixed])
        a_gpu = ring.state()[0].numpy()[before.idx]
        a_ref, tol = OG.amax_range(ref, Ssum)
        assert abs(float(a_gpu) - a_ref) <= tol, (float(a_gpu), a_ref, tol)
        expect = before.copy()
        OR.fold(expect, np.float32(a_gpu), ops.E4M3)
        assert_ring_equal(ring, expect)
