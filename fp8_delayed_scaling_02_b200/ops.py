"""Thin ctypes binding of the fp8ds C ABI (``include/fp8ds.h``).

Argument marshalling only: every step of quantize_fp8 and mm_fp8 runs in the
CUDA kernels of ``libfp8ds.so``.  There is no CPU fallback -- if the library
is missing or no CUDA device is present the calls raise.  torch provides the
device memory and the current stream.
"""

import ctypes
import os

import torch

from . import build as _build

E4M3, E5M2 = 0, 1
ROW, TRANSPOSED, DUAL = 0, 1, 2
IN_DTYPE = {torch.bfloat16: 0, torch.float16: 1, torch.float32: 2}
MM_NT = 0
MM_A_MN_MAJOR = 1 << 0
MM_B_MN_MAJOR = 1 << 1
MM_A_E5M2 = 1 << 8
MM_B_E5M2 = 1 << 9
MM_BIAS_E5M2 = 1 << 10
MM_OUT_BF16, MM_OUT_E4M3, MM_OUT_E5M2 = 0, 1, 2
HISTORY_LEN = 16

FP8_OK = 0
FP8_ERR_INVALID_ARG = -1
FP8_ERR_UNSUPPORTED = -2
FP8_ERR_CUDA = -3
FP8_ERR_DEVICE_TIMEOUT = -4


class CRing(ctypes.Structure):
    """Mirror of ``fp8_ring``: five device pointers."""

    _fields_ = [
        ("history", ctypes.c_void_p),
        ("idx", ctypes.c_void_p),
        ("scale", ctypes.c_void_p),
        ("scale_inv", ctypes.c_void_p),
        ("scratch", ctypes.c_void_p),
    ]


_LIB = None


def lib_path():
    return _build.LIB


def lib():
    """The loaded library; raises if it has not been built."""
    global _LIB
    if _LIB is None:
        path = lib_path()
        if not os.path.exists(path):
            raise RuntimeError(
                f"{path} is missing: build it with `python -m fp8_delayed_scaling_02_b200.build` "
                "(there is no CPU fallback)")
        L = ctypes.CDLL(path)
        vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        L.fp8_quantize.argtypes = [vp, i32, i64, i64, i32, i32, CRing, vp, vp, vp]
        L.fp8_quantize.restype = i32
        L.fp8_mm.argtypes = [vp, vp, i64, i64, i64, i64, vp, i32, vp, vp, vp, vp, vp]
        L.fp8_mm.restype = i32
        L.fp8_status_string.argtypes = [i32]
        L.fp8_status_string.restype = ctypes.c_char_p
        L.fp8_device_error.argtypes = [i32, ctypes.POINTER(ctypes.c_uint32)]
        L.fp8_device_error.restype = i32
        L.fp8_device_info.argtypes = [ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_char_p)]
        L.fp8_device_info.restype = i32
        L.fp8_quantize_current.argtypes = [vp, i32, i64, i64, i32, i32, vp, vp, vp, vp, vp, vp, vp]
        L.fp8_quantize_current.restype = i32
        L.fp8_bias_grad.argtypes = [vp, i32, i64, i64, vp, vp]
        L.fp8_bias_grad.restype = i32
        L.fp8_mm_ws.argtypes = [vp, vp, i64, i64, i64, i64, vp, i32, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
        L.fp8_mm_ws.restype = i32
        L.fp8_mm_workspace_bytes.argtypes = [i64, i64, i64, i64, i32]
        L.fp8_mm_workspace_bytes.restype = ctypes.c_size_t
        L.fp8_mm_launch_shape.argtypes = [i64, i64, i64, i64, i32, ctypes.c_size_t, ctypes.POINTER(ctypes.c_int32)]
        L.fp8_mm_launch_shape.restype = i32
        L.fp8_linear_forward.argtypes = [vp, i32, vp, i32, i64, i64, i64, vp, CRing, CRing, vp, vp, vp, vp]
        L.fp8_linear_forward.restype = i32
        L.fp8_linear_backward.argtypes = [vp, i32, i64, i64, i64, CRing, vp, vp, vp, vp, vp, vp, vp, vp, vp]
        L.fp8_linear_backward.restype = i32
        L.fp8_debug_wait.argtypes = [ctypes.c_uint64, ctypes.c_uint32]
        L.fp8_debug_wait.restype = i32
        L.fp8_quantize_local.argtypes = [vp, i32, i64, i64, i32, i32, CRing, vp, vp, vp, vp]
        L.fp8_quantize_local.restype = i32
        L.fp8_ring_fold.argtypes = [CRing, i32, vp, vp]
        L.fp8_ring_fold.restype = i32
        L.fp8_mm_pair.argtypes = [vp, vp, vp, ctypes.c_size_t, vp]
        L.fp8_mm_pair.restype = i32
        L.fp8_quantize_pair.argtypes = [vp, vp, vp]
        L.fp8_quantize_pair.restype = i32
        L.fp8_quantize_multi.argtypes = [vp, i32, vp]
        L.fp8_quantize_multi.restype = i32
        L.fp8_mm_ex.argtypes = [vp, vp, ctypes.c_size_t, vp]
        L.fp8_mm_ex.restype = i32
        L.fp8_launch_count.argtypes = []
        L.fp8_launch_count.restype = ctypes.c_uint64
        _LIB = L
    return _LIB


class Fp8Error(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__(f"{what}: {lib().fp8_status_string(status).decode()} ({status})")


def _check(rc, what):
    if rc != FP8_OK:
        raise Fp8Error(rc, what)


_raw_stream = torch._C._cuda_getCurrentRawStream


def _stream(stream, device_index):
    """Raw cudaStream_t (as an int) of ``stream`` or of the device's current stream."""
    if stream is None:
        return _raw_stream(device_index)
    return stream.cuda_stream


def _ptr(t):
    return t.data_ptr() if t is not None else None


class Ring:
    """One tensor's delayed-scaling state in a single device buffer.

    Layout (32-bit words): history[0:16] | idx[16] | scale[17] | scale_inv[18] | pad[19] |
    scratch[20:24] (amax bits, block ticket, tile counter, spare; 8-byte aligned).
    """

    WORDS = 24

    def __init__(self, device="cuda", scale=1.0):
        self.buf = torch.zeros(self.WORDS, dtype=torch.int32, device=device)
        f = self.buf.view(torch.float32)
        f[17] = float(scale)
        f[18] = 1.0

    @property
    def history(self):
        return self.buf[0:HISTORY_LEN].view(torch.float32)

    @property
    def idx(self):
        return self.buf[16:17]

    @property
    def scale(self):
        return self.buf[17:18].view(torch.float32)

    @property
    def scale_inv(self):
        return self.buf[18:19].view(torch.float32)

    @property
    def scratch(self):
        return self.buf[20:24]

    def c(self):
        c = getattr(self, "_c", None)
        if c is None:
            base = self.buf.data_ptr()
            c = self._c = CRing(base, base + 16 * 4, base + 17 * 4, base + 18 * 4, base + 20 * 4)
        return c

    def state(self):
        """Host copy: (history float32[16], idx, scale, scale_inv, scratch[4])."""
        h = self.buf.cpu()
        f = h.view(torch.float32)
        return f[:16].clone(), int(h[16]), float(f[17]), float(f[18]), h[20:24].clone()


def quantize(x, fmt, layout, ring, out=None, out_t=None, stream=None):
    """fp8_quantize on a 2-D CUDA tensor ``x`` (bf16/fp16/fp32, contiguous).

    Returns (out, out_t) as uint8 tensors (None where the layout has none).
    """
    if x.dim() != 2 or not x.is_contiguous():
        raise ValueError("x must be a contiguous 2-D tensor")
    rows, cols = x.shape
    if layout in (ROW, DUAL) and out is None:
        out = torch.empty((rows, cols), dtype=torch.uint8, device=x.device)
    if layout in (TRANSPOSED, DUAL) and out_t is None:
        out_t = torch.empty((cols, rows), dtype=torch.uint8, device=x.device)
    rc = (_LIB or lib()).fp8_quantize(x.data_ptr(), IN_DTYPE[x.dtype], rows, cols, layout, fmt, ring.c(),
                                      _ptr(out if layout in (ROW, DUAL) else None),
                                      _ptr(out_t if layout in (TRANSPOSED, DUAL) else None),
                                      _stream(stream, x.get_device()))
    _check(rc, "fp8_quantize")
    return (out if layout in (ROW, DUAL) else None), (out_t if layout in (TRANSPOSED, DUAL) else None)


class CQuantArgs(ctypes.Structure):
    """Mirror of ``fp8_quantize_args``."""

    _fields_ = [("in_", ctypes.c_void_p), ("dtype", ctypes.c_int), ("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("layout", ctypes.c_int), ("fmt", ctypes.c_int), ("ring", CRing), ("out", ctypes.c_void_p),
                ("out_t", ctypes.c_void_p)]


def _quant_args(qs):
    """CQuantArgs and (out, out_t) for a sequence of ``quantize`` argument dicts."""
    args, res = [], []
    for q in qs:
        x, layout = q["x"], q["layout"]
        if x.dim() != 2 or not x.is_contiguous():
            raise ValueError("x must be a contiguous 2-D tensor")
        rows, cols = x.shape
        out, out_t = q.get("out"), q.get("out_t")
        if layout in (ROW, DUAL) and out is None:
            out = torch.empty((rows, cols), dtype=torch.uint8, device=x.device)
        if layout in (TRANSPOSED, DUAL) and out_t is None:
            out_t = torch.empty((cols, rows), dtype=torch.uint8, device=x.device)
        out = out if layout in (ROW, DUAL) else None
        out_t = out_t if layout in (TRANSPOSED, DUAL) else None
        args.append(CQuantArgs(x.data_ptr(), IN_DTYPE[x.dtype], rows, cols, layout, q["fmt"], q["ring"].c(),
                               _ptr(out), _ptr(out_t)))
        res.append((out, out_t))
    return args, res


def quantize_pair(q0, q1, stream=None):
    """fp8_quantize_pair: two quantize calls (own rings) in one launch, e.g. a linear's X and W.

    q0, q1: dicts of ``quantize`` arguments (x, fmt, layout, ring and
    optionally out, out_t).  Returns ((out0, out_t0), (out1, out_t1)).
    """
    args, res = _quant_args((q0, q1))
    rc = (_LIB or lib()).fp8_quantize_pair(ctypes.byref(args[0]), ctypes.byref(args[1]),
                                           _stream(stream, q0["x"].get_device()))
    _check(rc, "fp8_quantize_pair")
    return res[0], res[1]


def quantize_multi(qs, stream=None):
    """fp8_quantize_multi: up to 8 quantize calls (own rings) in one launch, e.g. a linear's X, W and G.

    qs: a sequence of dicts of ``quantize`` arguments (x, fmt, layout, ring and
    optionally out, out_t).  Returns a list of (out, out_t).
    """
    qs = list(qs)
    if not qs:
        raise ValueError("quantize_multi needs at least one call")
    args, res = _quant_args(qs)
    arr = (CQuantArgs * len(args))(*args)
    rc = (_LIB or lib()).fp8_quantize_multi(arr, len(args), _stream(stream, qs[0]["x"].get_device()))
    _check(rc, "fp8_quantize_multi")
    return res


def quantize_local(x, fmt, layout, ring, amax=None, out=None, out_t=None, stream=None):
    """fp8_quantize_local: the cast of ``quantize`` without the ring fold.

    Writes ring.scale_inv (1 / the scale used) and this shard's amax into
    ``amax`` (a one-element float32 CUDA tensor, allocated when None).
    Returns (out, out_t, amax); fold later with ``ring_fold`` after the
    ranks have MAX-reduced ``amax``.
    """
    if x.dim() != 2 or not x.is_contiguous():
        raise ValueError("x must be a contiguous 2-D tensor")
    rows, cols = x.shape
    if layout in (ROW, DUAL) and out is None:
        out = torch.empty((rows, cols), dtype=torch.uint8, device=x.device)
    if layout in (TRANSPOSED, DUAL) and out_t is None:
        out_t = torch.empty((cols, rows), dtype=torch.uint8, device=x.device)
    if amax is None:
        amax = torch.zeros(1, dtype=torch.float32, device=x.device)
    rc = (_LIB or lib()).fp8_quantize_local(x.data_ptr(), IN_DTYPE[x.dtype], rows, cols, layout, fmt, ring.c(),
                                            amax.data_ptr(), _ptr(out if layout in (ROW, DUAL) else None),
                                            _ptr(out_t if layout in (TRANSPOSED, DUAL) else None),
                                            _stream(stream, x.get_device()))
    _check(rc, "fp8_quantize_local")
    return (out if layout in (ROW, DUAL) else None), (out_t if layout in (TRANSPOSED, DUAL) else None), amax


def ring_fold(ring, fmt, amax, stream=None):
    """fp8_ring_fold: fold the amax in the one-element float32 CUDA tensor ``amax`` into ``ring``."""
    rc = (_LIB or lib()).fp8_ring_fold(ring.c(), fmt, amax.data_ptr(), _stream(stream, amax.get_device()))
    _check(rc, "fp8_ring_fold")


def launch_count():
    """Kernels launched through the library by this process so far (fp8_launch_count)."""
    return int((_LIB or lib()).fp8_launch_count())


def mm_workspace_bytes(M, N, K, batch=1, a_mn_major=False, b_mn_major=False):
    """Bytes of workspace fp8_mm_ws would use (0 when whole tiles are as fast)."""
    layout = (MM_A_MN_MAJOR if a_mn_major else 0) | (MM_B_MN_MAJOR if b_mn_major else 0)
    return int((_LIB or lib()).fp8_mm_workspace_bytes(M, N, K, batch, layout))


def mm_launch_shape(M, N, K, batch=1, a_mn_major=False, b_mn_major=False, workspace_bytes=0):
    """The launch shape fp8_mm / fp8_mm_ws picks: dict(bn, cluster, ctas, stream_k_pieces)."""
    layout = (MM_A_MN_MAJOR if a_mn_major else 0) | (MM_B_MN_MAJOR if b_mn_major else 0)
    shape = (ctypes.c_int32 * 4)()
    rc = (_LIB or lib()).fp8_mm_launch_shape(M, N, K, batch, layout, workspace_bytes, shape)
    _check(rc, "fp8_mm_launch_shape")
    return dict(bn=shape[0], cluster=shape[1], ctas=shape[2], stream_k_pieces=shape[3])


def _shape2d(a, b, a_mn_major, b_mn_major, out):
    """(M, N, K, out) of a 2-D fp8_mm call; checks strides and allocates out."""
    if (a_mn_major or b_mn_major) and not (a.is_contiguous() and b.is_contiguous()):
        raise ValueError("operands must be contiguous")
    K, M = a.shape if a_mn_major else (a.shape[1], a.shape[0])
    Kb, N = b.shape if b_mn_major else (b.shape[1], b.shape[0])
    if Kb != K:
        raise ValueError("K mismatch")
    if not (a_mn_major or b_mn_major) and K > 0 and (
            (M > 1 and a.stride(0) != K) or a.stride(1) != 1 or (N > 1 and b.stride(0) != K) or b.stride(1) != 1):
        raise ValueError("operands must be K-contiguous")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=a.device)
    elif not out.is_contiguous() or out.shape != (M, N):
        raise ValueError("out must be a contiguous [M, N] bf16 tensor")
    return M, N, K, out


def _layout(fmt_a, fmt_b, a_mn_major, b_mn_major):
    return (MM_NT | (MM_A_E5M2 if fmt_a == E5M2 else 0) | (MM_B_E5M2 if fmt_b == E5M2 else 0)
            | (MM_A_MN_MAJOR if a_mn_major else 0) | (MM_B_MN_MAJOR if b_mn_major else 0))


class CMmArgs(ctypes.Structure):
    """Mirror of ``fp8_mm_args``."""

    _fields_ = [("A", ctypes.c_void_p), ("B", ctypes.c_void_p), ("M", ctypes.c_int64), ("N", ctypes.c_int64),
                ("K", ctypes.c_int64), ("batch", ctypes.c_int64), ("strides", ctypes.c_void_p),
                ("layout", ctypes.c_int), ("sinv_a", ctypes.c_void_p), ("sinv_b", ctypes.c_void_p),
                ("bias", ctypes.c_void_p), ("out_bf16", ctypes.c_void_p)]


def mm_pair(p0, p1, workspace=None, stream=None):
    """fp8_mm_pair: two independent 2-D GEMMs in one launch (e.g. dX and dW).

    p0, p1: dicts of ``mm`` keyword arguments (a, b, sinv_a, sinv_b and
    optionally bias, fmt_a, fmt_b, out, a_mn_major, b_mn_major).  Returns
    (out0, out1).
    """
    args, outs = [], []
    for q in (p0, p1):
        a, b = q["a"], q["b"]
        if a.dtype != torch.uint8 or b.dtype != torch.uint8 or a.dim() != 2 or b.dim() != 2:
            raise ValueError("a and b are 2-D uint8 FP8 codes")
        amn, bmn = q.get("a_mn_major", False), q.get("b_mn_major", False)
        M, N, K, out = _shape2d(a, b, amn, bmn, q.get("out"))
        outs.append(out)
        args.append(CMmArgs(a.data_ptr(), b.data_ptr(), M, N, K, 1, None,
                            _layout(q.get("fmt_a", E4M3), q.get("fmt_b", E4M3), amn, bmn),
                            q["sinv_a"].data_ptr(), q["sinv_b"].data_ptr(), _ptr(q.get("bias")), out.data_ptr()))
    ws, wsb = (workspace.data_ptr(), workspace.numel() * workspace.element_size()) if workspace is not None else (None, 0)
    rc = (_LIB or lib()).fp8_mm_pair(ctypes.byref(args[0]), ctypes.byref(args[1]), ws, wsb,
                                     _stream(stream, p0["a"].get_device()))
    _check(rc, "fp8_mm_pair")
    return outs[0], outs[1]


def mm(a, b, sinv_a, sinv_b, bias=None, fmt_a=E4M3, fmt_b=E4M3, out=None, stream=None,
       a_mn_major=False, b_mn_major=False, workspace=None):
    """fp8_mm: Y = bf16(A . B^T * sinv_a * sinv_b + bias).

    a: uint8 [M, K] or [Ba, M, K] (K contiguous), or with a_mn_major=True the
    stored [K, M] / [Ba, K, M] (M contiguous); b likewise [N, K] or, with
    b_mn_major=True, [K, N].  A size-1 (or 2-D) operand broadcasts over the
    batch at stride 0.  sinv_a / sinv_b: one-element float32 CUDA tensors.
    bias: float32 [N] or None.  workspace: optional zero-initialised uint8 CUDA
    tensor (256-byte aligned) that lets the library spread the last waves' k-blocks
    over all CTAs (stream-K, fp8_mm_ws).
    """
    if a.dtype != torch.uint8 or b.dtype != torch.uint8:
        raise ValueError("a and b hold FP8 codes as uint8")
    layout = (MM_NT | (MM_A_E5M2 if fmt_a == E5M2 else 0) | (MM_B_E5M2 if fmt_b == E5M2 else 0)
              | (MM_A_MN_MAJOR if a_mn_major else 0) | (MM_B_MN_MAJOR if b_mn_major else 0))
    L = _LIB or lib()
    if a.dim() == 2 and b.dim() == 2:
        M, N, K, out = _shape2d(a, b, a_mn_major, b_mn_major, out)
        if workspace is None:
            rc = L.fp8_mm(a.data_ptr(), b.data_ptr(), M, N, K, 1, None, layout, sinv_a.data_ptr(),
                          sinv_b.data_ptr(), _ptr(bias), out.data_ptr(), _stream(stream, a.get_device()))
        else:
            rc = L.fp8_mm_ws(a.data_ptr(), b.data_ptr(), M, N, K, 1, None, layout, sinv_a.data_ptr(),
                             sinv_b.data_ptr(), _ptr(bias), out.data_ptr(), workspace.data_ptr(),
                             workspace.numel() * workspace.element_size(), _stream(stream, a.get_device()))
        _check(rc, "fp8_mm")
        return out
    a3 = a if a.dim() == 3 else a.unsqueeze(0)
    b3 = b if b.dim() == 3 else b.unsqueeze(0)
    batch = max(a3.shape[0], b3.shape[0])
    K, M = (a3.shape[1], a3.shape[2]) if a_mn_major else (a3.shape[2], a3.shape[1])
    Kb, N = (b3.shape[1], b3.shape[2]) if b_mn_major else (b3.shape[2], b3.shape[1])
    if Kb != K:
        raise ValueError("K mismatch")
    for t in (a3, b3):
        if t.shape[0] not in (1, batch) or (t.numel() > 0 and (t.stride(2) != 1 or t.stride(1) != t.shape[2])):
            raise ValueError("operands must be contiguous in their last two dims with matching batch")
    sa = 0 if a3.shape[0] == 1 else a3.stride(0)
    sb = 0 if b3.shape[0] == 1 else b3.stride(0)
    if out is None:
        out = torch.empty((batch, M, N), dtype=torch.bfloat16, device=a.device)
    out3 = out if out.dim() == 3 else out.unsqueeze(0)
    strides = (ctypes.c_int64 * 3)(sa, sb, out3.stride(0) if batch > 1 else M * N)
    if workspace is None:
        rc = L.fp8_mm(a3.data_ptr(), b3.data_ptr(), M, N, K, batch, strides, layout, sinv_a.data_ptr(),
                      sinv_b.data_ptr(), _ptr(bias), out3.data_ptr(), _stream(stream, a.get_device()))
    else:
        rc = L.fp8_mm_ws(a3.data_ptr(), b3.data_ptr(), M, N, K, batch, strides, layout, sinv_a.data_ptr(),
                         sinv_b.data_ptr(), _ptr(bias), out3.data_ptr(), workspace.data_ptr(),
                         workspace.numel() * workspace.element_size(), _stream(stream, a.get_device()))
    _check(rc, "fp8_mm")
    return out


class CMmExArgs(ctypes.Structure):
    """Mirror of ``fp8_mm_ex_args``."""

    _fields_ = [("A", ctypes.c_void_p), ("B", ctypes.c_void_p), ("M", ctypes.c_int64), ("N", ctypes.c_int64),
                ("K", ctypes.c_int64), ("batch", ctypes.c_int64), ("strides", ctypes.c_void_p),
                ("layout", ctypes.c_int), ("sinv_a", ctypes.c_void_p), ("sinv_b", ctypes.c_void_p),
                ("bias", ctypes.c_void_p), ("bias_scale", ctypes.c_void_p), ("out_kind", ctypes.c_int),
                ("out", ctypes.c_void_p), ("out_ring", CRing), ("out_amax", ctypes.c_void_p)]


def mm_ex(a, b, sinv_a, sinv_b, bias=None, bias_scale=None, bias_fmt=E4M3, out_fmt=None, out_ring=None,
          fmt_a=E4M3, fmt_b=E4M3, out=None, a_mn_major=False, b_mn_major=False, workspace=None, stream=None,
          out_amax=None):
    """fp8_mm_ex: ``mm`` with an FP8 bias and / or an FP8 output.

    bias: float32 [N], or (with bias_scale, a one-element float32 CUDA tensor)
    uint8 FP8 codes [N] in format bias_fmt, dequantised as code * bias_scale.
    out_fmt: None for bf16 output, or E4M3 / E5M2 for FP8 codes of
    y * out_ring.scale, with max |y| folded into ``out_ring`` (a Ring) in the
    same launch -- or, with out_amax (a one-element float32 CUDA tensor), max |y|
    written there and the fold left to ``ring_fold`` (a data-parallel shard).
    Operands and batching as ``mm``.  Returns out.
    """
    if a.dtype != torch.uint8 or b.dtype != torch.uint8:
        raise ValueError("a and b hold FP8 codes as uint8")
    if out_fmt is not None and out_ring is None:
        raise ValueError("an FP8 output needs out_ring")
    if bias_scale is not None and bias is not None and bias.dtype != torch.uint8:
        raise ValueError("with bias_scale the bias holds FP8 codes (uint8)")
    a3 = a if a.dim() == 3 else a.unsqueeze(0)
    b3 = b if b.dim() == 3 else b.unsqueeze(0)
    batch = max(a3.shape[0], b3.shape[0])
    K, M = (a3.shape[1], a3.shape[2]) if a_mn_major else (a3.shape[2], a3.shape[1])
    Kb, N = (b3.shape[1], b3.shape[2]) if b_mn_major else (b3.shape[2], b3.shape[1])
    if Kb != K:
        raise ValueError("K mismatch")
    for t in (a3, b3):
        if t.shape[0] not in (1, batch) or (t.numel() > 0 and (t.stride(2) != 1 or (t.shape[1] > 1 and t.stride(1) != t.shape[2]))):
            raise ValueError("operands must be contiguous in their last two dims with matching batch")
    sa = 0 if a3.shape[0] == 1 else a3.stride(0)
    sb = 0 if b3.shape[0] == 1 else b3.stride(0)
    dtype = torch.bfloat16 if out_fmt is None else torch.uint8
    two_d = a.dim() == 2 and b.dim() == 2
    if out is None:
        out = torch.empty((M, N) if two_d else (batch, M, N), dtype=dtype, device=a.device)
    out3 = out if out.dim() == 3 else out.unsqueeze(0)
    if out.dtype != dtype or not out.is_contiguous() or tuple(out3.shape) != (batch, M, N):
        raise ValueError(f"out must be a contiguous [batch, M, N] {dtype} tensor")
    strides = (ctypes.c_int64 * 3)(sa, sb, out3.stride(0) if batch > 1 else M * N)
    layout = _layout(fmt_a, fmt_b, a_mn_major, b_mn_major)
    if bias_scale is not None and bias_fmt == E5M2:
        layout |= MM_BIAS_E5M2
    kind = MM_OUT_BF16 if out_fmt is None else (MM_OUT_E5M2 if out_fmt == E5M2 else MM_OUT_E4M3)
    ring = out_ring.c() if out_ring is not None else CRing()
    args = CMmExArgs(a3.data_ptr(), b3.data_ptr(), M, N, K, batch, ctypes.cast(strides, ctypes.c_void_p), layout,
                     sinv_a.data_ptr(), sinv_b.data_ptr(), _ptr(bias), _ptr(bias_scale), kind,
                     out3.data_ptr(), ring, _ptr(out_amax))
    ws, wsb = (workspace.data_ptr(), workspace.numel() * workspace.element_size()) if workspace is not None else (None, 0)
    rc = (_LIB or lib()).fp8_mm_ex(ctypes.byref(args), ws, wsb, _stream(stream, a.get_device()))
    _check(rc, "fp8_mm_ex")
    return out


class CurrentScale:
    """Device state of current (dynamic) scaling: scale, scale_inv, amax and 4 scratch words."""

    def __init__(self, device="cuda"):
        self.buf = torch.zeros(8, dtype=torch.int32, device=device)

    @property
    def scale(self):
        return self.buf[0:1].view(torch.float32)

    @property
    def scale_inv(self):
        return self.buf[1:2].view(torch.float32)

    @property
    def amax(self):
        return self.buf[2:3].view(torch.float32)

    @property
    def scratch(self):
        return self.buf[4:8]


def quantize_current(x, fmt, layout, cs, out=None, out_t=None, stream=None):
    """fp8_quantize_current: scale from this tensor's amax (no history).

    ``cs`` is a CurrentScale; after the call it holds scale, scale_inv and amax.
    Returns (out, out_t) like ``quantize``.
    """
    if x.dim() != 2 or not x.is_contiguous():
        raise ValueError("x must be a contiguous 2-D tensor")
    rows, cols = x.shape
    if layout in (ROW, DUAL) and out is None:
        out = torch.empty((rows, cols), dtype=torch.uint8, device=x.device)
    if layout in (TRANSPOSED, DUAL) and out_t is None:
        out_t = torch.empty((cols, rows), dtype=torch.uint8, device=x.device)
    rc = (_LIB or lib()).fp8_quantize_current(
        x.data_ptr(), IN_DTYPE[x.dtype], rows, cols, layout, fmt, cs.scale.data_ptr(), cs.scale_inv.data_ptr(),
        cs.amax.data_ptr(), cs.scratch.data_ptr(), _ptr(out if layout in (ROW, DUAL) else None),
        _ptr(out_t if layout in (TRANSPOSED, DUAL) else None), _stream(stream, x.get_device()))
    _check(rc, "fp8_quantize_current")
    return (out if layout in (ROW, DUAL) else None), (out_t if layout in (TRANSPOSED, DUAL) else None)


def bias_grad(g, out=None, stream=None):
    """fp8_bias_grad: float32 column sums of a 2-D (or flattened) gradient."""
    g2 = g.reshape(-1, g.shape[-1])
    if not g2.is_contiguous():
        raise ValueError("g must be contiguous")
    rows, cols = g2.shape
    if out is None:
        out = torch.empty(cols, dtype=torch.float32, device=g.device)
    rc = (_LIB or lib()).fp8_bias_grad(g2.data_ptr(), IN_DTYPE[g2.dtype], rows, cols, out.data_ptr(),
                                       _stream(stream, g.get_device()))
    _check(rc, "fp8_bias_grad")
    return out


class Linear:
    """One FP8 delayed-scaling linear through fp8_linear_forward / fp8_linear_backward.

    Holds the three rings (x, w, g) and the quantized operands the backward
    reuses; weights and bias are passed per call (they change every step).
    """

    def __init__(self, device="cuda"):
        self.rx, self.rw, self.rg = Ring(device), Ring(device), Ring(device)
        self.xq = self.wq = self.gq = None

    def forward(self, x, w, bias=None, y=None, stream=None):
        M, K = x.shape
        N = w.shape[0]
        dev = x.device
        if self.xq is None or self.xq.shape != (M, K):
            self.xq = torch.empty((M, K), dtype=torch.uint8, device=dev)
        if self.wq is None or self.wq.shape != (N, K):
            self.wq = torch.empty((N, K), dtype=torch.uint8, device=dev)
        if y is None:
            y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        rc = (_LIB or lib()).fp8_linear_forward(
            x.data_ptr(), IN_DTYPE[x.dtype], w.data_ptr(), IN_DTYPE[w.dtype], M, N, K, _ptr(bias), self.rx.c(),
            self.rw.c(), self.xq.data_ptr(), self.wq.data_ptr(), y.data_ptr(), _stream(stream, x.get_device()))
        _check(rc, "fp8_linear_forward")
        return y

    def backward(self, g, need_dx=True, need_dw=True, need_db=True, stream=None):
        M, N = g.shape
        K = self.xq.shape[1]
        dev = g.device
        if self.gq is None or self.gq.shape != (M, N):
            self.gq = torch.empty((M, N), dtype=torch.uint8, device=dev)
        dx = torch.empty((M, K), dtype=torch.bfloat16, device=dev) if need_dx else None
        dw = torch.empty((N, K), dtype=torch.bfloat16, device=dev) if need_dw else None
        db = torch.empty(N, dtype=torch.float32, device=dev) if need_db else None
        rc = (_LIB or lib()).fp8_linear_backward(
            g.data_ptr(), IN_DTYPE[g.dtype], M, N, K, self.rg.c(), self.xq.data_ptr(), self.wq.data_ptr(),
            self.rx.scale_inv.data_ptr(), self.rw.scale_inv.data_ptr(), self.gq.data_ptr(), _ptr(dx), _ptr(dw),
            _ptr(db), _stream(stream, g.get_device()))
        _check(rc, "fp8_linear_backward")
        return dx, dw, db


WAIT_BUDGET_DEFAULT_NS = 2_000_000_000
SITE_EPILOGUE_TMEM_FULL = 4   # fp8_mm: the epilogue's wait for an accumulator
SITE_QUANTIZE_TMA = 6         # fp8_quantize: the producer / consumer waits


def debug_wait(budget_ns=WAIT_BUDGET_DEFAULT_NS, stall_site=0):
    """fp8_debug_wait (testing only): the budget of the kernels' bounded waits and
    a wait site at which later launches wait on a barrier nothing completes."""
    _check((_LIB or lib()).fp8_debug_wait(int(budget_ns), int(stall_site)), "fp8_debug_wait")


def device_error(clear=True):
    """(status, site) of the library's device error word; synchronises the device."""
    where = ctypes.c_uint32(0)
    rc = lib().fp8_device_error(1 if clear else 0, ctypes.byref(where))
    return rc, where.value
