"""Thin Python binding of the quantized-matmul C ABI (``include/qgemm.h``).

Argument marshalling only: every step of every operation runs in the CUDA
kernels of ``libqgemm.so``.  Tensors are torch CUDA tensors (PyTorch provides
device memory and streams); sizes and element strides are read from them.
There is no CPU fallback: if the library is missing, importing this package
raises ImportError, and a failing call raises QGError with the library's
status code.

The function names are those of the C ABI:
  quantize_rows_a8, pack_w4_g32, qgemm_a8w4_f32,
  qgemm_pack_b_s8, qgemm_s8s8_requant, qgemm_s8s8_requant_packed,
  qconv2d_s8_im2col, qg_requant_params, qg_device_status,
  quantize_rows_a8_sym, qconv2d_f32_dyn_a8w4
plus the *_bytes / *_workspace_bytes size queries.
"""
from __future__ import annotations

import ctypes
import math
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqgemm.so")

QG_OK = 0
STATUS = {
    0: "QG_OK", -1: "QG_ERR_INVALID_ARG", -2: "QG_ERR_MISALIGNED", -3: "QG_ERR_OVERFLOW_BOUND",
    -4: "QG_ERR_UNSUPPORTED", -5: "QG_ERR_CUDA", -6: "QG_ERR_TIMEOUT", -7: "QG_ERR_WORKSPACE",
    -8: "QG_ERR_NO_DEVICE",
}


class QGError(RuntimeError):
    def __init__(self, status, where=""):
        self.status = int(status)
        msg = lib.qg_status_string(self.status).decode()
        super().__init__(f"{where}: {msg} ({self.status})" if where else msg)


if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is not built; run `python gemv_zero_point_b200/build.py` "
        "(nvcc with sm_100a) first")

lib = ctypes.CDLL(LIB_PATH)

_i32, _i64, _sz, _vp, _f32, _f64 = (ctypes.c_int, ctypes.c_int64, ctypes.c_size_t,
                                    ctypes.c_void_p, ctypes.c_float, ctypes.c_double)


class RequantParams(ctypes.Structure):
    """Mirror of qg_requant_t."""
    _fields_ = [
        ("a_zero_point", ctypes.c_int32), ("b_zero_point", ctypes.c_int32),
        ("bias", _vp), ("bias_abs_max", ctypes.c_int32), ("per_channel", ctypes.c_int32),
        ("multiplier0", ctypes.c_int32), ("shift0", ctypes.c_int32),
        ("multiplier", _vp), ("shift", _vp),
        ("out_zero_point", ctypes.c_int32), ("clamp_min", ctypes.c_int32),
        ("clamp_max", ctypes.c_int32),
    ]


def _sig(name, res, args):
    f = getattr(lib, name)
    f.restype = res
    f.argtypes = args
    return f


_sig("qg_status_string", ctypes.c_char_p, [_i32])
_sig("qg_version", _i32, [])
_sig("qg_device_status", _i32, [_i32])
_sig("qg_test_arm_stall", _i32, [_i32])
_sig("qg_requant_params", _i32, [_f64, ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int32)])
_sig("qgemm_s8s8_workspace_bytes", _sz, [_i32, _i32, _i32])
_sig("qgemm_s8s8_requant", _i32, [_i32, _i32, _i32, _vp, _i64, _vp, _i64, _vp, _i64,
                                  ctypes.POINTER(RequantParams), _vp, _i64, _vp, _sz, _vp])
_sig("qgemm_pack_b_s8_bytes", _sz, [_i32, _i32])
_sig("qgemm_pack_b_s8", _i32, [_i32, _i32, _vp, _i64, _vp, _sz, _vp])
_sig("qgemm_s8s8_packed_workspace_bytes", _sz, [_i32, _i32])
_sig("qgemm_s8s8_requant_packed", _i32, [_i32, _i32, _i32, _vp, _i64, _vp, _vp, _i64,
                                         ctypes.POINTER(RequantParams), _vp, _i64, _vp, _sz, _vp])
_sig("qconv2d_s8_workspace_bytes", _sz, [_i32] * 11)
_sig("qconv2d_s8_im2col", _i32, [_i32] * 11 + [_vp, _vp, _vp, ctypes.POINTER(RequantParams),
                                               _vp, _vp, _sz, _vp])
_sig("qconv2d_s8_pack_w_bytes", _sz, [_i32] * 4)
_sig("qconv2d_s8_pack_w", _i32, [_i32] * 4 + [_vp, _vp, _sz, _vp])
_sig("qconv2d_s8_im2col_packed", _i32, [_i32] * 11 + [_vp, _vp, _vp, ctypes.POINTER(RequantParams),
                                                      _vp, _vp])
_sig("quantize_rows_a8", _i32, [_i32, _i32, _vp, _i64, _vp, _i64, _vp, _vp, _vp])
_sig("pack_w4_g32_bytes", _sz, [_i32, _i32])
_sig("pack_w4_g32", _i32, [_i32, _i32, _vp, _i64, _vp, _vp, _sz, _vp])
_sig("qgemm_a8w4_workspace_bytes", _sz, [_i32, _i32, _i32])
_sig("qgemm_a8w4_f32", _i32, [_i32, _i32, _i32, _vp, _i64, _vp, _vp, _f32, _f32, _vp, _i64,
                              _vp, _vp, _vp, _vp, _sz, _vp])
_sig("qgemm_a8w4_f32_actblock", _i32, [_i32, _i32, _i32, _vp, _i64, _vp, _vp, _f32, _f32, _vp,
                                       _i64, _vp, _vp, _vp, _vp, _sz, _vp])
_sig("pack_w4_g32_asym_bytes", _sz, [_i32, _i32])
_sig("pack_w4_g32_asym", _i32, [_i32, _i32, _vp, _i64, _vp, _vp, _vp, _sz, _vp])
_sig("qgemm_a8w4_f32_asym", _i32, [_i32, _i32, _i32, _vp, _i64, _vp, _vp, _f32, _f32, _vp,
                                   _i64, _vp, _vp, _vp, _vp, _sz, _vp])
_sig("quantize_rows_a8_sym", _i32, [_i32, _i32, _vp, _i64, _vp, _i64, _vp, _vp])
_sig("qconv2d_f32_dyn_a8w4_workspace_bytes", _sz, [_i32] * 11)
_sig("qconv2d_f32_dyn_a8w4", _i32, [_i32] * 11 + [_vp, _vp, _vp, _f32, _f32, _i32, _vp, _vp, _vp,
                                                  _vp, _vp, _sz, _vp])
_sig("pack_w4_g32_bf16_bytes", _sz, [_i32, _i32])
_sig("pack_w4_g32_bf16", _i32, [_i32, _i32, _vp, _i64, _vp, _vp, _sz, _vp])
_sig("qgemm_a8w4_f32_bf16s", _i32, [_i32, _i32, _i32, _vp, _i64, _vp, _vp, _f32, _f32, _vp,
                                    _i64, _vp, _vp, _vp, _vp, _sz, _vp])


def _check(rc, where):
    if rc != QG_OK:
        raise QGError(rc, where)


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ld(t):
    """Row stride (elements) of a 2-D row-major tensor view."""
    assert t.dim() == 2 and t.stride(1) == 1, "expected a row-major 2-D view"
    return t.stride(0)


def _empty_bytes(n, device):
    import torch
    # 256-byte alignment comes with the caching allocator
    return torch.empty(max(int(n), 1), dtype=torch.uint8, device=device)


# ---------------------------------------------------------------------------
# Status and requant parameters
# ---------------------------------------------------------------------------
def qg_device_status(reset=True):
    return lib.qg_device_status(1 if reset else 0)


def qg_test_arm_stall(which):
    """Test hook: arm one stalled pipeline for the next launch of a kernel
    family (1 = INT8 GEMM one-CTA kernel, 2 = A8W4 tensor-core kernel, 0 =
    disarm); see include/qgemm.h."""
    _check(lib.qg_test_arm_stall(int(which)), "qg_test_arm_stall")


def qg_requant_params(ratio):
    m0, sh = ctypes.c_int32(), ctypes.c_int32()
    _check(lib.qg_requant_params(float(ratio), ctypes.byref(m0), ctypes.byref(sh)), "qg_requant_params")
    return m0.value, sh.value


def make_requant(*, a_zero_point, b_zero_point=0, bias=None, bias_abs_max=None,
                 multiplier=None, shift=None, out_zero_point=0, clamp_min=-128,
                 clamp_max=127):
    """Build a qg_requant_t.  ``multiplier``/``shift`` are ints (per tensor)
    or int32 CUDA tensors [N] (per channel).  The returned object keeps the
    tensors it points to alive."""
    import torch
    rq = RequantParams()
    rq.a_zero_point, rq.b_zero_point = int(a_zero_point), int(b_zero_point)
    rq.bias = None if bias is None else bias.data_ptr()
    if bias is not None and bias_abs_max is None:
        bias_abs_max = int(bias.abs().max().item()) if bias.numel() else 0
    rq.bias_abs_max = int(bias_abs_max or 0)
    if isinstance(multiplier, torch.Tensor):
        rq.per_channel = 1
        rq.multiplier, rq.shift = multiplier.data_ptr(), shift.data_ptr()
    else:
        rq.per_channel = 0
        rq.multiplier0, rq.shift0 = int(multiplier), int(shift)
    rq.out_zero_point, rq.clamp_min, rq.clamp_max = int(out_zero_point), int(clamp_min), int(clamp_max)
    rq._keep = (bias, multiplier, shift)
    return rq


# ---------------------------------------------------------------------------
# A8W4
# ---------------------------------------------------------------------------
def quantize_rows_a8(x, q, scale, zero_point, stream=None):
    M, K = x.shape
    _check(lib.quantize_rows_a8(M, K, _p(x), _ld(x), _p(q), _ld(q), _p(scale), _p(zero_point),
                                _stream(stream)), "quantize_rows_a8")


def pack_w4_g32_bytes(N, K):
    return lib.pack_w4_g32_bytes(N, K)


def pack_w4_g32(w, group_scales, packed=None, stream=None, bf16_scales=False):
    """Pack int4 weights [N][K] and f32 group scales; with bf16_scales the
    scales are stored rounded to bf16 (use with qgemm_a8w4_f32_bf16s)."""
    N, K = w.shape
    bytes_fn = lib.pack_w4_g32_bf16_bytes if bf16_scales else lib.pack_w4_g32_bytes
    pack_fn = lib.pack_w4_g32_bf16 if bf16_scales else lib.pack_w4_g32
    nbytes = bytes_fn(N, K)
    if packed is None:
        packed = _empty_bytes(nbytes, w.device)
    _check(pack_fn(N, K, _p(w), _ld(w), _p(group_scales), _p(packed), packed.numel(),
                   _stream(stream)), pack_fn.__name__)
    return packed


def pack_w4_g32_bf16(w, group_scales, packed=None, stream=None):
    return pack_w4_g32(w, group_scales, packed, stream, bf16_scales=True)


def qgemm_a8w4_workspace_bytes(M, N, K):
    return lib.qgemm_a8w4_workspace_bytes(M, N, K)


def qgemm_a8w4_f32(x, packed_w, N, bias, clamp_min, clamp_max, y, q_out=None, scale_out=None,
                   zp_out=None, workspace=None, stream=None, bf16_scales=False):
    """A8W4 linear; bf16_scales selects weights packed by pack_w4_g32_bf16."""
    M, K = x.shape
    wsb = lib.qgemm_a8w4_workspace_bytes(M, N, K)
    if wsb and workspace is None:
        workspace = _empty_bytes(wsb, x.device)
    fn = lib.qgemm_a8w4_f32_bf16s if bf16_scales else lib.qgemm_a8w4_f32
    _check(fn(M, N, K, _p(x), _ld(x), _p(packed_w), _p(bias),
              float(clamp_min), float(clamp_max), _p(y), _ld(y), _p(q_out),
              _p(scale_out), _p(zp_out), _p(workspace),
              0 if workspace is None else workspace.numel(), _stream(stream)), fn.__name__)


def _a8w4_workspace(M, N, K, workspace, device):
    wsb = lib.qgemm_a8w4_workspace_bytes(M, N, K)
    if wsb and workspace is None:
        workspace = _empty_bytes(wsb, device)
    return workspace


def qgemm_a8w4_f32_actblock(x, packed_w, N, bias, clamp_min, clamp_max, y, q_out=None,
                            scale_out=None, zp_out=None, workspace=None, stream=None):
    """A8W4 linear with the activations quantized per 32-wide K block;
    scale_out / zp_out, when given, receive [M][K/32] values."""
    M, K = x.shape
    workspace = _a8w4_workspace(M, N, K, workspace, x.device)
    _check(lib.qgemm_a8w4_f32_actblock(M, N, K, _p(x), _ld(x), _p(packed_w), _p(bias),
                                       float(clamp_min), float(clamp_max), _p(y), _ld(y),
                                       _p(q_out), _p(scale_out), _p(zp_out), _p(workspace),
                                       0 if workspace is None else workspace.numel(),
                                       _stream(stream)),
           "qgemm_a8w4_f32_actblock")


def pack_w4_g32_asym(w, group_scales, group_zeros, packed=None, stream=None):
    """Pack int4 weights with f32 group scales and f32 group zeros."""
    N, K = w.shape
    if packed is None:
        packed = _empty_bytes(lib.pack_w4_g32_asym_bytes(N, K), w.device)
    _check(lib.pack_w4_g32_asym(N, K, _p(w), _ld(w), _p(group_scales), _p(group_zeros),
                                _p(packed), packed.numel(), _stream(stream)), "pack_w4_g32_asym")
    return packed


def qgemm_a8w4_f32_asym(x, packed_w, N, bias, clamp_min, clamp_max, y, q_out=None,
                        scale_out=None, zp_out=None, workspace=None, stream=None):
    """A8W4 linear with asymmetric int4 weights (pack_w4_g32_asym)."""
    M, K = x.shape
    workspace = _a8w4_workspace(M, N, K, workspace, x.device)
    _check(lib.qgemm_a8w4_f32_asym(M, N, K, _p(x), _ld(x), _p(packed_w), _p(bias),
                                   float(clamp_min), float(clamp_max), _p(y), _ld(y),
                                   _p(q_out), _p(scale_out), _p(zp_out), _p(workspace),
                                   0 if workspace is None else workspace.numel(),
                                   _stream(stream)),
           "qgemm_a8w4_f32_asym")


def qgemm_a8w4_f32_bf16s(x, packed_w, N, bias, clamp_min, clamp_max, y, **kw):
    return qgemm_a8w4_f32(x, packed_w, N, bias, clamp_min, clamp_max, y, bf16_scales=True, **kw)


# ---------------------------------------------------------------------------
# INT8 GEMM / conv
# ---------------------------------------------------------------------------
def qgemm_pack_b_s8_bytes(K, N):
    return lib.qgemm_pack_b_s8_bytes(K, N)


def qgemm_pack_b_s8(B, N=None, packed=None, stream=None):
    K = B.shape[0]
    N = B.shape[1] if N is None else N
    nbytes = lib.qgemm_pack_b_s8_bytes(K, N)
    if packed is None:
        packed = _empty_bytes(nbytes, B.device)
    _check(lib.qgemm_pack_b_s8(K, N, _p(B), _ld(B), _p(packed), packed.numel(), _stream(stream)),
           "qgemm_pack_b_s8")
    return packed


def qgemm_s8s8_workspace_bytes(M, N, K):
    return lib.qgemm_s8s8_workspace_bytes(M, N, K)


def qgemm_s8s8_packed_workspace_bytes(M, K):
    return lib.qgemm_s8s8_packed_workspace_bytes(M, K)


def qgemm_s8s8_requant(A, B, C, rq, K=None, N=None, acc_out=None, workspace=None, stream=None):
    M = A.shape[0]
    K = A.shape[1] if K is None else K
    N = C.shape[1] if N is None else N
    wsb = lib.qgemm_s8s8_workspace_bytes(M, N, K)
    if workspace is None:
        workspace = _empty_bytes(wsb, A.device)
    _check(lib.qgemm_s8s8_requant(M, N, K, _p(A), _ld(A), _p(B), _ld(B), _p(C), _ld(C),
                                  ctypes.byref(rq), _p(acc_out),
                                  0 if acc_out is None else _ld(acc_out), _p(workspace),
                                  workspace.numel(), _stream(stream)), "qgemm_s8s8_requant")


def qgemm_s8s8_requant_packed(A, packed_b, N, C, rq, K=None, acc_out=None, workspace=None,
                              stream=None):
    M = A.shape[0]
    K = A.shape[1] if K is None else K
    wsb = lib.qgemm_s8s8_packed_workspace_bytes(M, K)
    if workspace is None:
        workspace = _empty_bytes(wsb, A.device)
    _check(lib.qgemm_s8s8_requant_packed(M, N, K, _p(A), _ld(A), _p(packed_b), _p(C), _ld(C),
                                         ctypes.byref(rq), _p(acc_out),
                                         0 if acc_out is None else _ld(acc_out), _p(workspace),
                                         workspace.numel(), _stream(stream)),
           "qgemm_s8s8_requant_packed")


def conv_out_hw(H, W, KH, KW, stride, pad):
    return (H + 2 * pad[0] - KH) // stride[0] + 1, (W + 2 * pad[1] - KW) // stride[1] + 1


def qconv2d_s8_workspace_bytes(x_shape, w_shape, stride, pad):
    Nb, H, W, Cin = x_shape
    Cout, KH, KW, _ = w_shape
    return lib.qconv2d_s8_workspace_bytes(Nb, H, W, Cin, Cout, KH, KW, stride[0], stride[1],
                                          pad[0], pad[1])


def qconv2d_s8_im2col(x, w, y, rq, stride, pad, acc_out=None, workspace=None, stream=None):
    Nb, H, W, Cin = x.shape
    Cout, KH, KW, Cin2 = w.shape
    assert Cin == Cin2 and x.is_contiguous() and w.is_contiguous() and y.is_contiguous()
    wsb = qconv2d_s8_workspace_bytes(x.shape, w.shape, stride, pad)
    if workspace is None:
        workspace = _empty_bytes(wsb, x.device)
    _check(lib.qconv2d_s8_im2col(Nb, H, W, Cin, Cout, KH, KW, stride[0], stride[1], pad[0],
                                 pad[1], _p(x), _p(w), _p(y), ctypes.byref(rq), _p(acc_out),
                                 _p(workspace), workspace.numel(), _stream(stream)),
           "qconv2d_s8_im2col")


def qconv2d_s8_pack_w(w, packed=None, stream=None):
    """Pack conv weights [Cout][KH][KW][Cin] once (weights-stationary)."""
    Cout, KH, KW, Cin = w.shape
    assert w.is_contiguous()
    if packed is None:
        packed = _empty_bytes(lib.qconv2d_s8_pack_w_bytes(Cout, KH, KW, Cin), w.device)
    _check(lib.qconv2d_s8_pack_w(Cout, KH, KW, Cin, _p(w), _p(packed), packed.numel(),
                                 _stream(stream)), "qconv2d_s8_pack_w")
    return packed


def qconv2d_s8_im2col_packed(x, packed_w, w_shape, y, rq, stride, pad, acc_out=None,
                             stream=None):
    """INT8 conv from weights packed by qconv2d_s8_pack_w (one launch)."""
    Nb, H, W, Cin = x.shape
    Cout, KH, KW, Cin2 = w_shape
    assert Cin == Cin2 and x.is_contiguous() and y.is_contiguous()
    _check(lib.qconv2d_s8_im2col_packed(Nb, H, W, Cin, Cout, KH, KW, stride[0], stride[1], pad[0],
                                        pad[1], _p(x), _p(packed_w), _p(y), ctypes.byref(rq),
                                        _p(acc_out), _stream(stream)),
           "qconv2d_s8_im2col_packed")


def quantize_rows_a8_sym(x, q, scale, stream=None):
    """Symmetric per-row int8 quantization (zero-point 0)."""
    M, K = x.shape
    _check(lib.quantize_rows_a8_sym(M, K, _p(x), _ld(x), _p(q), _ld(q), _p(scale),
                                    _stream(stream)), "quantize_rows_a8_sym")


def qconv2d_f32_dyn_a8w4_workspace_bytes(x_shape, Cout, KH, KW, stride, pad):
    Nb, H, W, Cin = x_shape
    return lib.qconv2d_f32_dyn_a8w4_workspace_bytes(Nb, H, W, Cin, Cout, KH, KW, stride[0],
                                                    stride[1], pad[0], pad[1])


def qconv2d_f32_dyn_a8w4(x, packed_w, Cout, KH, KW, stride, pad, bias, clamp_min, clamp_max, y,
                         symmetric=False, q_out=None, scale_out=None, zp_out=None,
                         workspace=None, stream=None):
    """Float NHWC input x [Nb][H][W][Cin], unrolled and quantized per output
    pixel, times int4 weights packed by pack_w4_g32 from [Cout][KH*KW*Cin];
    y f32 NHWC [Nb][OH][OW][Cout]."""
    Nb, H, W, Cin = x.shape
    assert x.is_contiguous() and y.is_contiguous()
    if workspace is None:
        workspace = _empty_bytes(qconv2d_f32_dyn_a8w4_workspace_bytes(x.shape, Cout, KH, KW,
                                                                      stride, pad), x.device)
    _check(lib.qconv2d_f32_dyn_a8w4(Nb, H, W, Cin, Cout, KH, KW, stride[0], stride[1], pad[0],
                                    pad[1], _p(x), _p(packed_w), _p(bias), float(clamp_min),
                                    float(clamp_max), 1 if symmetric else 0, _p(y), _p(q_out),
                                    _p(scale_out), _p(zp_out), _p(workspace), workspace.numel(),
                                    _stream(stream)), "qconv2d_f32_dyn_a8w4")


def exported_symbols():
    """Function names declared in include/qgemm.h (for export checks)."""
    import re
    hdr = os.path.join(os.path.dirname(_HERE), "include", "qgemm.h")
    txt = open(hdr).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b([a-z][a-z0-9_]*)\s*\(", txt)) - {"sizeof"})
