"""CPU checks of the C ABI: the library loads, exports every declared symbol,
and rejects bad arguments on the host before touching CUDA."""

import ctypes
import os
import re

import pytest

from fp8_delayed_scaling_02_b200 import build, ops

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "fp8ds.h")


@pytest.fixture(scope="module")
def L():
    build.build()
    return ops.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fp8_[a-z_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    assert declared_functions() == sorted(
        ["fp8_quantize", "fp8_mm", "fp8_status_string", "fp8_device_error", "fp8_device_info",
         "fp8_quantize_static_scratch", "fp8_quantize_current", "fp8_bias_grad", "fp8_linear_forward",
         "fp8_linear_backward", "fp8_mm_ws", "fp8_mm_workspace_bytes", "fp8_quantize_local", "fp8_ring_fold",
         "fp8_mm_pair", "fp8_launch_count", "fp8_quantize_pair", "fp8_mm_ex", "fp8_debug_wait",
         "fp8_mm_launch_shape", "fp8_quantize_multi"])


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def test_status_strings(L):
    for code in (0, -1, -2, -3, -4, 7):
        s = L.fp8_status_string(code)
        assert isinstance(s, bytes) and len(s) > 0
    assert L.fp8_status_string(-4).startswith(b"FP8_ERR_DEVICE_TIMEOUT")


def _ring(addr=0x1000):
    return ops.CRing(addr, addr + 64, addr + 68, addr + 72, addr + 80)


def _q(L, dtype=0, rows=4, cols=4, layout=0, fmt=0, ring=None, out=0x2000, out_t=0x3000, inp=0x4000):
    return L.fp8_quantize(ctypes.c_void_p(inp), dtype, rows, cols, layout, fmt, ring or _ring(),
                          ctypes.c_void_p(out), ctypes.c_void_p(out_t), None)


def test_quantize_rejects_bad_arguments_without_cuda(L):
    assert _q(L, dtype=3) == ops.FP8_ERR_INVALID_ARG
    assert _q(L, fmt=2) == ops.FP8_ERR_INVALID_ARG
    assert _q(L, layout=3) == ops.FP8_ERR_INVALID_ARG
    assert _q(L, rows=-1) == ops.FP8_ERR_INVALID_ARG
    assert _q(L, ring=ops.CRing(0, 0, 0, 0, 0)) == ops.FP8_ERR_INVALID_ARG
    assert _q(L, inp=0) == ops.FP8_ERR_INVALID_ARG
    assert _q(L, layout=0, out=0) == ops.FP8_ERR_INVALID_ARG
    assert _q(L, layout=1, out_t=0) == ops.FP8_ERR_INVALID_ARG
    assert _q(L, layout=2, out_t=0) == ops.FP8_ERR_INVALID_ARG
    assert _q(L, dtype=2, inp=0x4002) == ops.FP8_ERR_UNSUPPORTED   # fp32 needs 4-byte alignment
    assert _q(L, dtype=0, inp=0x4001) == ops.FP8_ERR_UNSUPPORTED   # bf16 needs 2-byte alignment
    assert _q(L, ring=ops.CRing(0x1000, 0x1040, 0x1044, 0x1048, 0x104C)) == ops.FP8_ERR_UNSUPPORTED  # scratch % 8


def test_local_quantize_and_ring_fold_reject_bad_arguments_without_cuda(L):
    def ql(amax=0x5000, fmt=0, layout=0, ring=None, out=0x2000):
        return L.fp8_quantize_local(ctypes.c_void_p(0x4000), 0, 4, 4, layout, fmt, ring or _ring(),
                                    ctypes.c_void_p(amax), ctypes.c_void_p(out), ctypes.c_void_p(0x3000), None)
    assert ql(amax=0) == ops.FP8_ERR_INVALID_ARG
    assert ql(fmt=2) == ops.FP8_ERR_INVALID_ARG
    assert ql(layout=0, out=0) == ops.FP8_ERR_INVALID_ARG
    assert ql(ring=ops.CRing(0x1000, 0x1040, 0, 0x1048, 0x1050)) == ops.FP8_ERR_INVALID_ARG  # no scale
    assert L.fp8_ring_fold(_ring(), 0, None, None) == ops.FP8_ERR_INVALID_ARG
    assert L.fp8_ring_fold(_ring(), 2, ctypes.c_void_p(0x5000), None) == ops.FP8_ERR_INVALID_ARG
    assert L.fp8_ring_fold(ops.CRing(0, 0x1040, 0x1044, 0x1048, 0x1050), 0, ctypes.c_void_p(0x5000),
                           None) == ops.FP8_ERR_INVALID_ARG


def _mm(L, M=128, N=128, K=128, batch=1, strides=None, layout=0, A=0x10000, B=0x20000, out=0x30000,
        sa=0x40000, sb=0x40010):
    st = (ctypes.c_int64 * 3)(*strides) if strides is not None else None
    return L.fp8_mm(ctypes.c_void_p(A), ctypes.c_void_p(B), M, N, K, batch, st, layout, ctypes.c_void_p(sa),
                    ctypes.c_void_p(sb), None, ctypes.c_void_p(out), None)


def test_mm_rejects_bad_arguments_without_cuda(L):
    assert _mm(L, M=-1) == ops.FP8_ERR_INVALID_ARG
    assert _mm(L, batch=0) == ops.FP8_ERR_INVALID_ARG
    assert _mm(L, layout=1 << 2) == ops.FP8_ERR_INVALID_ARG
    assert _mm(L, layout=1 << 10) == ops.FP8_ERR_INVALID_ARG
    assert _mm(L, layout=ops.MM_A_MN_MAJOR, M=24) == ops.FP8_ERR_UNSUPPORTED  # [K, M] rows need M % 16 == 0
    assert _mm(L, layout=ops.MM_B_MN_MAJOR, N=40) == ops.FP8_ERR_UNSUPPORTED
    assert _mm(L, batch=2, strides=None) == ops.FP8_ERR_INVALID_ARG
    assert _mm(L, batch=2, strides=(-16, 0, 0)) == ops.FP8_ERR_INVALID_ARG
    assert _mm(L, out=0) == ops.FP8_ERR_INVALID_ARG
    assert _mm(L, sa=0) == ops.FP8_ERR_INVALID_ARG
    assert _mm(L, A=0) == ops.FP8_ERR_INVALID_ARG
    assert _mm(L, K=24) == ops.FP8_ERR_UNSUPPORTED
    assert _mm(L, out=0x30001) == ops.FP8_ERR_UNSUPPORTED
    assert _mm(L, A=0x10008) == ops.FP8_ERR_UNSUPPORTED
    assert _mm(L, batch=2, strides=(8, 0, 0)) == ops.FP8_ERR_UNSUPPORTED
    # Empty products are a no-op that needs no device.
    assert _mm(L, M=0) == ops.FP8_OK
    assert _mm(L, N=0, A=0, B=0) == ops.FP8_OK


def _mm_ex(L, out_kind=ops.MM_OUT_E4M3, layout=0, bias=None, bias_scale=None, out=0x30000, ring=None, M=128,
           amax=None):
    args = ops.CMmExArgs(0x10000, 0x20000, M, 128, 128, 1, None, layout, 0x40000, 0x40010, bias, bias_scale,
                         out_kind, out, ring if ring is not None else _ring(), amax)
    return L.fp8_mm_ex(ctypes.byref(args), None, 0, None)


def test_mm_ex_rejects_bad_arguments_without_cuda(L):
    assert L.fp8_mm_ex(None, None, 0, None) == ops.FP8_ERR_INVALID_ARG
    assert _mm_ex(L, out_kind=3) == ops.FP8_ERR_INVALID_ARG
    assert _mm_ex(L, out_kind=-1) == ops.FP8_ERR_INVALID_ARG
    assert _mm_ex(L, out=0) == ops.FP8_ERR_INVALID_ARG                      # FP8 output without codes
    assert _mm_ex(L, ring=ops.CRing(0x1000, 0x1040, 0, 0x1048, 0x1050)) == ops.FP8_ERR_INVALID_ARG  # no scale
    assert _mm_ex(L, ring=ops.CRing(0x1000, 0x1040, 0x1044, 0x1048, 0)) == ops.FP8_ERR_INVALID_ARG  # no scratch
    assert _mm_ex(L, ring=ops.CRing(0x1000, 0x1040, 0x1044, 0x1048, 0x1054)) == ops.FP8_ERR_UNSUPPORTED
    assert _mm_ex(L, layout=ops.MM_BIAS_E5M2) == ops.FP8_ERR_INVALID_ARG    # bias format bit without FP8 bias
    assert _mm_ex(L, out_kind=ops.MM_OUT_BF16, out=0) == ops.FP8_ERR_INVALID_ARG
    assert _mm_ex(L, out_kind=ops.MM_OUT_BF16, amax=0x50000) == ops.FP8_ERR_INVALID_ARG  # shard amax needs FP8 out


def test_mm_ex_binding_checks_arguments_on_the_host():
    """ops.mm_ex refuses inconsistent arguments before it touches the library."""
    import torch

    a = torch.zeros((128, 64), dtype=torch.uint8)
    b = torch.zeros((96, 64), dtype=torch.uint8)
    one = torch.ones(1)
    with pytest.raises(ValueError):
        ops.mm_ex(a, b, one, one, out_fmt=ops.E4M3)  # FP8 output without a ring
    with pytest.raises(ValueError):
        ops.mm_ex(a, b, one, one, bias=torch.zeros(96), bias_scale=one)  # float32 bias with a scale
    with pytest.raises(ValueError):
        ops.mm_ex(a, torch.zeros((96, 32), dtype=torch.uint8), one, one)  # K mismatch
    with pytest.raises(ValueError):
        ops.mm_ex(a.float(), b, one, one)  # operands are uint8 codes
    with pytest.raises(ValueError):
        ops.mm_ex(a, b, one, one, out=torch.zeros((128, 96), dtype=torch.uint8))  # bf16 output expected


def test_paired_entry_points_reject_bad_arguments_without_cuda(L):
    def mm_args(**kw):
        d = dict(A=0x10000, B=0x20000, M=128, N=128, K=128, batch=1, strides=None, layout=0, sinv_a=0x40000,
                 sinv_b=0x40010, bias=None, out_bf16=0x30000)
        d.update(kw)
        return ops.CMmArgs(*d.values())

    good = mm_args()
    assert L.fp8_mm_pair(None, ctypes.byref(good), None, 0, None) == ops.FP8_ERR_INVALID_ARG
    assert L.fp8_mm_pair(ctypes.byref(good), ctypes.byref(mm_args(M=-1)), None, 0, None) == ops.FP8_ERR_INVALID_ARG
    assert L.fp8_mm_pair(ctypes.byref(mm_args(K=24)), ctypes.byref(good), None, 0, None) == ops.FP8_ERR_UNSUPPORTED
    assert L.fp8_mm_pair(ctypes.byref(good), ctypes.byref(mm_args(layout=1 << 10)), None, 0,
                         None) == ops.FP8_ERR_INVALID_ARG  # the FP8-bias bit belongs to fp8_mm_ex

    def q_args(**kw):
        d = dict(inp=0x10000, dtype=0, rows=64, cols=64, layout=0, fmt=0, ring=_ring(), out=0x20000, out_t=0x30000)
        d.update(kw)
        return ops.CQuantArgs(*d.values())

    gq = q_args()
    assert L.fp8_quantize_pair(None, ctypes.byref(gq), None) == ops.FP8_ERR_INVALID_ARG
    assert L.fp8_quantize_pair(ctypes.byref(gq), ctypes.byref(q_args(dtype=3)), None) == ops.FP8_ERR_INVALID_ARG
    assert L.fp8_quantize_pair(ctypes.byref(q_args(fmt=2)), ctypes.byref(gq), None) == ops.FP8_ERR_INVALID_ARG
    assert L.fp8_quantize_pair(ctypes.byref(gq), ctypes.byref(q_args(ring=ops.CRing(0, 0, 0, 0, 0))),
                               None) == ops.FP8_ERR_INVALID_ARG

    def arr(*qs):
        return (ops.CQuantArgs * len(qs))(*qs)

    assert L.fp8_quantize_multi(None, 1, None) == ops.FP8_ERR_INVALID_ARG
    assert L.fp8_quantize_multi(arr(gq), 0, None) == ops.FP8_ERR_INVALID_ARG
    assert L.fp8_quantize_multi(arr(*([gq] * 9)), 9, None) == ops.FP8_ERR_INVALID_ARG
    # Every call is checked before anything launches: a bad third call
    # returns its own status (here, with no GPU, a launch would give FP8_ERR_CUDA).
    assert L.fp8_quantize_multi(arr(gq, gq, q_args(layout=3)), 3, None) == ops.FP8_ERR_INVALID_ARG
    assert L.fp8_quantize_multi(arr(gq, q_args(inp=0x10001), gq), 3, None) == ops.FP8_ERR_UNSUPPORTED
    assert L.fp8_quantize_multi(arr(gq, q_args(layout=2, out_t=0)), 2, None) == ops.FP8_ERR_INVALID_ARG


def test_linear_composites_check_every_call_before_launching(L):
    """A linear call that one of its GEMMs (or the bias gradient) would reject
    returns that status before any kernel is enqueued, so its rings stay as
    they were.  With no GPU here, a quantize enqueued first would have failed
    with FP8_ERR_CUDA instead."""
    vp = ctypes.c_void_p
    ring = _ring()

    def fwd(M=128, N=128, K=128, xq=0x50000, wq=0x60000, y=0x70000, x=0x10000, w=0x20000):
        return L.fp8_linear_forward(vp(x), 0, vp(w), 0, M, N, K, None, ring, _ring(0x1100), vp(xq), vp(wq), vp(y),
                                    None)

    assert fwd(K=24) == ops.FP8_ERR_UNSUPPORTED          # K % 16
    assert fwd(y=0) == ops.FP8_ERR_INVALID_ARG           # no output
    assert fwd(xq=0x50008) == ops.FP8_ERR_UNSUPPORTED     # FP8 operand not 16-byte aligned
    assert fwd(y=0x70001) == ops.FP8_ERR_UNSUPPORTED      # bf16 output not 2-byte aligned

    def bwd(M=128, N=128, K=128, dx=0x80000, dw=0x90000, db=0xA0000, g=0x10000, gq=0x30000, g_dtype=0):
        return L.fp8_linear_backward(vp(g), g_dtype, M, N, K, ring, vp(0x50000), vp(0x60000), vp(0x40000),
                                     vp(0x40010), vp(gq), vp(dx) if dx else None, vp(dw) if dw else None,
                                     vp(db) if db else None, None)

    assert bwd(M=24) == ops.FP8_ERR_UNSUPPORTED           # dW reduces over M: M % 16
    assert bwd(N=40) == ops.FP8_ERR_UNSUPPORTED           # dX reduces over N: N % 16
    assert bwd(N=40, dx=0) == ops.FP8_ERR_UNSUPPORTED     # dW's MN-major A needs N % 16 too
    assert bwd(K=24, dw=0) == ops.FP8_ERR_UNSUPPORTED     # dX's MN-major B needs K % 16
    assert bwd(gq=0x30008) == ops.FP8_ERR_UNSUPPORTED     # Gq is a GEMM operand: 16-byte aligned
    assert bwd(g=0x10001) == ops.FP8_ERR_UNSUPPORTED      # bias gradient input alignment
    assert bwd(g_dtype=2, g=0x10002, dx=0, dw=0) == ops.FP8_ERR_UNSUPPORTED  # fp32 G, 4-byte alignment


def test_static_scratch_entry_point_checks_before_cuda(L):
    """Argument errors that need no device come back before any CUDA call."""
    f = L.fp8_quantize_static_scratch
    vp = ctypes.c_void_p
    f.argtypes = [vp, ctypes.c_int, ctypes.c_int64, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ops.CRing, vp, vp,
                  vp]
    f.restype = ctypes.c_int
    assert f(vp(0x4000), 0, 4, 4, 0, 0, ops.CRing(0, 0, 0, 0, 0), vp(0x2000), None, None) == ops.FP8_ERR_INVALID_ARG


def test_debug_wait_checks_its_arguments(L):
    assert L.fp8_debug_wait(0, 0) == ops.FP8_ERR_INVALID_ARG
    assert L.fp8_debug_wait(2_000_000_001, 0) == ops.FP8_ERR_INVALID_ARG
    assert L.fp8_debug_wait(1000, 5) == ops.FP8_ERR_INVALID_ARG   # only sites 4 and 6 can stall
    assert L.fp8_debug_wait(1000, 4) == ops.FP8_OK
    assert L.fp8_debug_wait(2_000_000_000, 0) == ops.FP8_OK      # back to the defaults


def test_launch_shape_query_checks_its_arguments(L):
    """Argument errors come before any device query, so they show on a CPU host too."""
    shape = (ctypes.c_int32 * 4)()
    assert L.fp8_mm_launch_shape(128, 128, 128, 1, 0, 0, None) == ops.FP8_ERR_INVALID_ARG
    for M, N, K, batch in ((0, 128, 128, 1), (128, -1, 128, 1), (128, 128, 0, 1), (128, 128, 128, 0)):
        assert L.fp8_mm_launch_shape(M, N, K, batch, 0, 0, shape) == ops.FP8_ERR_INVALID_ARG
