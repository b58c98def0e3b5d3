"""GPU check of fp8_quantize_static_scratch, the entry point for callers that
cannot allocate device memory (operator or plugin interfaces that receive only
input and output pointers, deployments that reserve all device memory up front).

It must produce exactly what fp8_quantize produces, with its four scratch words
taken from the library's static array instead of the ring.  Two calls in a row
check that the shared array is left clean for the next call.  The file is
named so that pytest collects it last.
"""

import ctypes

import numpy as np
import pytest
import torch

from fp8_delayed_scaling_02_b200 import build, ops, synthetic as S

pytestmark = pytest.mark.gpu


def _entry():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    build.build()
    L = ops.lib()
    f = L.fp8_quantize_static_scratch
    vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    f.argtypes = [vp, i32, i64, i64, i32, i32, ops.CRing, vp, vp, vp]
    f.restype = i32
    return f


def _ring_without_scratch(ring):
    c = ring.c()
    c.scratch = None
    return c


@pytest.mark.parametrize("dtype,fmt,layout,shape,misalign", [
    ("bf16", ops.E4M3, ops.DUAL, (301, 1537), False),
    ("fp32", ops.E5M2, ops.ROW, (2048, 1536), True),
    ("fp16", ops.E4M3, ops.TRANSPOSED, (130, 70), False),
])
def test_static_scratch_matches_fp8_quantize_on_two_calls(dtype, fmt, layout, shape, misalign):
    f = _entry()
    rows, cols = shape
    ring_ref, ring_new = ops.Ring(), ops.Ring()
    stream = torch.cuda.current_stream()
    for call in range(2):
        x = S.quant_sweep_input(rows, cols, dtype, [1.0, 1e3][call], seed=7 + call)
        if misalign:
            flat = torch.empty(x.numel() + 1, dtype=x.dtype, device="cuda")
            flat[1:].copy_(x.reshape(-1))
            xd = flat[1:].view(shape)
        else:
            xd = x.cuda()
        ref_out, ref_out_t = ops.quantize(xd, fmt, layout, ring_ref)
        out = torch.full((rows, cols), 0xAA, dtype=torch.uint8, device="cuda")
        out_t = torch.full((cols, rows), 0xAA, dtype=torch.uint8, device="cuda")
        rc = f(ctypes.c_void_p(xd.data_ptr()), ops.IN_DTYPE[xd.dtype], rows, cols, layout, fmt,
               _ring_without_scratch(ring_new), ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(out_t.data_ptr()),
               ctypes.c_void_p(stream.cuda_stream))
        assert rc == ops.FP8_OK, rc
        torch.cuda.synchronize()
        if ref_out is not None:
            assert torch.equal(out, ref_out), f"call {call}: row bytes differ"
        if ref_out_t is not None:
            assert torch.equal(out_t, ref_out_t), f"call {call}: transposed bytes differ"
        h_ref, i_ref, s_ref, si_ref, _ = ring_ref.state()
        h_new, i_new, s_new, si_new, _ = ring_new.state()
        assert np.array_equal(h_ref.numpy().view(np.uint32), h_new.numpy().view(np.uint32))
        assert i_ref == i_new
        assert np.float32(s_ref).view(np.uint32) == np.float32(s_new).view(np.uint32)
        assert np.float32(si_ref).view(np.uint32) == np.float32(si_new).view(np.uint32)
        assert all(int(v) == 0 for v in ring_new.scratch)  # the ring's own words stay unused


def test_static_scratch_rejects_bad_arguments():
    f = _entry()
    ring = ops.Ring()
    x = torch.zeros((4, 4), dtype=torch.bfloat16, device="cuda")
    o = torch.empty((4, 4), dtype=torch.uint8, device="cuda")
    args = lambda dt, lay: (ctypes.c_void_p(x.data_ptr()), dt, 4, 4, lay, 0, _ring_without_scratch(ring),  # noqa: E731
                            ctypes.c_void_p(o.data_ptr()), None, None)
    assert f(*args(5, 0)) == ops.FP8_ERR_INVALID_ARG
    assert f(*args(0, 1)) == ops.FP8_ERR_INVALID_ARG  # transposed layout without out_t
