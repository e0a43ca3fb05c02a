"""Host-only checks of the C ABI: the library loads without a GPU, exports
every function the header declares, and rejects invalid arguments with the
documented status before touching the device.  No compute call is made."""
import ctypes
import math

import numpy as np
import pytest

import oracle

qg = pytest.importorskip("gemv_zero_point_b200")
lib = qg.lib
NULL = None


def test_exports_every_declared_symbol():
    names = qg.exported_symbols()
    for expected in ["quantize_rows_a8", "pack_w4_g32", "qgemm_a8w4_f32", "qgemm_s8s8_requant",
                     "pack_w4_g32_bf16", "qgemm_a8w4_f32_bf16s", "qgemm_a8w4_f32_actblock",
                     "pack_w4_g32_asym", "qgemm_a8w4_f32_asym",
                     "quantize_rows_a8_sym", "qconv2d_f32_dyn_a8w4",
                     "qconv2d_f32_dyn_a8w4_workspace_bytes",
                     "qconv2d_s8_im2col", "qgemm_pack_b_s8", "qgemm_s8s8_requant_packed",
                     "qg_requant_params", "qg_status_string", "qg_device_status"]:
        assert expected in names
    for n in names:
        assert hasattr(lib, n), f"libqgemm.so does not export {n}"


def test_status_strings_and_version():
    assert lib.qg_version() == 2
    for code, name in qg.STATUS.items():
        assert lib.qg_status_string(code).decode().startswith(name)
    assert lib.qg_status_string(12345).decode() == "QG_ERR_UNKNOWN"


def test_requant_params_match_oracle_bit_exact():
    rng = np.random.default_rng(0)
    ratios = list(np.exp(rng.uniform(np.log(1e-9), np.log(0.9999), 2000)))
    ratios += [0.5, 0.25, 0.75, 2.0 ** -10, 2.0 ** -31, 0.999999999, 1e-4, 1e-2,
               0.5 - 2.0 ** -34, 0.25 - 2.0 ** -35, 0.5 - 2.0 ** -31]
    for r in ratios:
        try:
            ref = oracle.requant_params(r)
        except ValueError:
            with pytest.raises(qg.QGError):
                qg.qg_requant_params(r)
            continue
        assert qg.qg_requant_params(r) == ref, r
    for bad in (0.0, 1.0, 2.0, -1.0, float("nan"), float("inf"), 1e-12):
        m0, sh = ctypes.c_int32(), ctypes.c_int32()
        assert lib.qg_requant_params(bad, ctypes.byref(m0), ctypes.byref(sh)) == -4
    assert lib.qg_requant_params(0.5, None, None) == -1


def test_workspace_queries():
    assert qg.pack_w4_g32_bytes(14336, 4096) == 14336 * 2048 + 14336 * 128 * 4
    assert qg.pack_w4_g32_bytes(10, 33) == 0          # K % 32 != 0
    assert lib.pack_w4_g32_bf16_bytes(14336, 4096) == 14336 * 2048 + 14336 * 128 * 2
    assert lib.pack_w4_g32_bf16_bytes(10, 33) == 0
    assert qg.qgemm_a8w4_workspace_bytes(1, 14336, 4096) == 0  # fused GEMV needs none
    assert qg.qgemm_a8w4_workspace_bytes(128, 4096, 4096) >= 128 * 4096 + 2 * 128 * 4
    assert qg.qgemm_pack_b_s8_bytes(129, 70) >= 256 * 256 + 256 * 4
    assert qg.qgemm_s8s8_workspace_bytes(130, 70, 129) >= qg.qgemm_pack_b_s8_bytes(129, 70)
    assert qg.qgemm_pack_b_s8_bytes(0, 5) == 0


def _rq(**kw):
    d = dict(a_zero_point=0, b_zero_point=0, multiplier=2 ** 30, shift=0)
    d.update(kw)
    return qg.make_requant(**d)


FAKE = ctypes.c_void_p(0x10000)  # never dereferenced: these calls fail validation first


def _gemm(M, N, K, rq, lda=None, ldb=None, ldc=None, A=FAKE, ws=FAKE, wsb=1 << 30):
    return lib.qgemm_s8s8_requant(M, N, K, A, lda or K, FAKE, ldb or N, FAKE, ldc or N,
                                  ctypes.byref(rq), NULL, 0, ws, wsb, NULL)


def test_gemm_rejects_overflow_bound():
    # 33026*65025 > INT32_MAX: rejected whatever else is valid
    assert _gemm(4, 4, 33026, _rq()) == -3
    rq = _rq()
    rq.bias = 0x20000
    rq.bias_abs_max = 2 ** 31 - 1 - 33025 * 65025 + 1
    assert _gemm(4, 4, 33025, rq) == -3


def test_gemm_rejects_invalid_args():
    assert _gemm(4, 0, 8, _rq()) == -1
    assert _gemm(4, 4, 0, _rq()) == -1
    assert _gemm(4, 4, 8, _rq(), lda=7) == -1          # lda < K
    assert _gemm(4, 4, 8, _rq(), ldc=3) == -1          # ldc < N
    assert _gemm(4, 4, 8, _rq(), ldb=3) == -1          # ldb < N
    assert _gemm(4, 4, 8, _rq(a_zero_point=200)) == -1
    assert _gemm(4, 4, 8, _rq(clamp_min=5, clamp_max=4)) == -1
    assert _gemm(4, 4, 8, _rq(shift=32)) == -1
    assert _gemm(4, 4, 8, _rq(), ws=None, wsb=0) == -7  # workspace required
    assert lib.qgemm_s8s8_requant(4, 4, 8, FAKE, 8, FAKE, 4, FAKE, 4, None, NULL, 0, FAKE,
                                  1 << 30, NULL) == -1
    assert _gemm(0, 4, 8, _rq()) == 0                  # empty M is a no-op


def test_pack_and_a8w4_validation():
    assert lib.pack_w4_g32(4, 48, FAKE, 48, FAKE, FAKE, 1 << 20, NULL) == -4      # K % 32
    assert lib.pack_w4_g32(4, 64, FAKE, 63, FAKE, FAKE, 1 << 20, NULL) == -1      # ldw < K
    assert lib.pack_w4_g32(4, 64, FAKE, 64, FAKE, ctypes.c_void_p(0x10008), 1 << 20, NULL) == -2
    assert lib.pack_w4_g32(4, 64, FAKE, 64, FAKE, FAKE, 10, NULL) == -7           # too small
    f = lib.qgemm_a8w4_f32
    assert f(1, 8, 48, FAKE, 48, FAKE, NULL, -1.0, 1.0, FAKE, 8, NULL, NULL, NULL, NULL, 0, NULL) == -4
    assert f(1, 8, 64, FAKE, 64, FAKE, NULL, 1.0, -1.0, FAKE, 8, NULL, NULL, NULL, NULL, 0, NULL) == -1
    assert f(1, 8, 64, FAKE, 64, FAKE, NULL, float("nan"), 1.0, FAKE, 8, NULL, NULL, NULL, NULL, 0, NULL) == -1
    assert f(1, 8, 64, FAKE, 63, FAKE, NULL, -1.0, 1.0, FAKE, 8, NULL, NULL, NULL, NULL, 0, NULL) == -1
    assert f(0, 8, 64, FAKE, 64, FAKE, NULL, -1.0, 1.0, FAKE, 8, NULL, NULL, NULL, NULL, 0, NULL) == 0
    assert lib.quantize_rows_a8(2, 8, FAKE, 7, FAKE, 8, FAKE, FAKE, NULL) == -1


def test_conv_validation():
    rq = _rq(a_zero_point=-5)
    c = lib.qconv2d_s8_im2col
    args = [1, 8, 8, 4, 4, 3, 3, 1, 1, 1, 1]
    assert c(*args[:9], 3, 1, FAKE, FAKE, FAKE, ctypes.byref(rq), NULL, FAKE, 1 << 30, NULL) == -4
    bad = list(args); bad[7] = 0
    assert c(*bad, FAKE, FAKE, FAKE, ctypes.byref(rq), NULL, FAKE, 1 << 30, NULL) == -1
    rqb = _rq(a_zero_point=-5, b_zero_point=3)
    assert c(*args, FAKE, FAKE, FAKE, ctypes.byref(rqb), NULL, FAKE, 1 << 30, NULL) == -4
    big = [1, 8, 8, 4000, 4, 3, 3, 1, 1, 1, 1]         # K = 36000 breaks the bound
    assert c(*big, FAKE, FAKE, FAKE, ctypes.byref(rq), NULL, FAKE, 1 << 30, NULL) == -3


def test_bf16_scale_entry_points_validate_like_f32_ones():
    p = lib.pack_w4_g32_bf16
    assert p(4, 48, FAKE, 48, FAKE, FAKE, 1 << 20, NULL) == -4      # K % 32
    assert p(4, 64, FAKE, 63, FAKE, FAKE, 1 << 20, NULL) == -1      # ldw < K
    assert p(4, 64, FAKE, 64, FAKE, ctypes.c_void_p(0x10008), 1 << 20, NULL) == -2
    assert p(4, 64, FAKE, 64, FAKE, FAKE, 4 * 32 + 4 * 2 * 2 - 1, NULL) == -7   # one byte short
    f = lib.qgemm_a8w4_f32_bf16s
    assert f(1, 8, 48, FAKE, 48, FAKE, NULL, -1.0, 1.0, FAKE, 8, NULL, NULL, NULL, NULL, 0, NULL) == -4
    assert f(1, 8, 64, FAKE, 64, FAKE, NULL, 1.0, -1.0, FAKE, 8, NULL, NULL, NULL, NULL, 0, NULL) == -1
    assert f(0, 8, 64, FAKE, 64, FAKE, NULL, -1.0, 1.0, FAKE, 8, NULL, NULL, NULL, NULL, 0, NULL) == 0


def test_actblock_gemv_validation():
    f = lib.qgemm_a8w4_f32_actblock
    args = (FAKE, NULL, -1.0, 1.0, FAKE, 8, NULL, NULL, NULL)
    assert f(2, 8, 96, FAKE, 96, *args, FAKE, 1 << 20, NULL) == -4      # M > 1, K % 64 != 0
    assert f(2, 8, 16384, FAKE, 16384, *args, FAKE, 1 << 30, NULL) == -4  # M > 1, K > 8192
    assert f(2, 8, 128, FAKE, 128, *args, NULL, 0, NULL) == -7         # M > 1 needs a workspace
    need = lib.qgemm_a8w4_workspace_bytes(2, 8, 128)
    assert need > 0
    assert f(2, 8, 128, FAKE, 128, *args, FAKE, need - 1, NULL) == -7  # too small
    assert f(2, 8, 128, FAKE, 128, *args, ctypes.c_void_p(0x10010), need, NULL) == -2
    assert f(1, 8, 96, FAKE, 96, *args, NULL, 0, NULL) == -4           # M == 1, K % 128
    assert f(1, 8, 48, FAKE, 48, *args, NULL, 0, NULL) == -4           # K % 32
    assert f(1, 8, 128, FAKE, 128, FAKE, NULL, 1.0, -1.0, FAKE, 8, NULL, NULL, NULL, NULL, 0, NULL) == -1
    assert f(1, 8, 128, FAKE, 127, *args, NULL, 0, NULL) == -1         # ldx < K
    assert f(0, 8, 128, FAKE, 128, *args, NULL, 0, NULL) == 0          # empty


def test_asym_entry_points_validation():
    assert lib.pack_w4_g32_asym_bytes(14336, 4096) == 14336 * 2048 + 2 * 14336 * 128 * 4
    assert lib.pack_w4_g32_asym_bytes(10, 33) == 0
    p = lib.pack_w4_g32_asym
    assert p(4, 64, FAKE, 64, FAKE, NULL, FAKE, 1 << 20, NULL) == -1      # zeros missing
    assert p(4, 48, FAKE, 48, FAKE, FAKE, FAKE, 1 << 20, NULL) == -4      # K % 32
    assert p(4, 64, FAKE, 64, FAKE, ctypes.c_void_p(0x10002), FAKE, 1 << 20, NULL) == -2
    assert p(4, 64, FAKE, 64, FAKE, FAKE, FAKE, 4 * 32 + 2 * 4 * 2 * 4 - 1, NULL) == -7
    f = lib.qgemm_a8w4_f32_asym
    args = (FAKE, NULL, -1.0, 1.0, FAKE, 8, NULL, NULL, NULL)
    assert f(2, 8, 96, FAKE, 96, *args, FAKE, 1 << 20, NULL) == -4      # M > 1, K % 64 != 0
    assert f(2, 8, 128, FAKE, 128, *args, NULL, 0, NULL) == -7         # M > 1 needs a workspace
    assert f(1, 8, 96, FAKE, 96, *args, NULL, 0, NULL) == -4           # M == 1, K % 128
    assert f(1, 8, 128, FAKE, 128, FAKE, NULL, 1.0, -1.0, FAKE, 8, NULL, NULL, NULL, NULL, 0, NULL) == -1
    assert f(0, 8, 128, FAKE, 128, *args, NULL, 0, NULL) == 0


def test_symmetric_quantization_validation():
    f = lib.quantize_rows_a8_sym
    assert f(0, 16, NULL, 16, NULL, 16, NULL, NULL) == 0                  # empty
    assert f(-1, 16, FAKE, 16, FAKE, 16, FAKE, NULL) == -1
    assert f(2, 16, FAKE, 15, FAKE, 16, FAKE, NULL) == -1                 # ldx < K
    assert f(2, 16, FAKE, 16, FAKE, 15, FAKE, NULL) == -1                 # ldq < K
    assert f(2, 16, NULL, 16, FAKE, 16, FAKE, NULL) == -1
    assert f(2, 16, ctypes.c_void_p(0x10002), 16, FAKE, 16, FAKE, NULL) == -2


def test_dynamic_conv_workspace_and_validation():
    ws = lib.qconv2d_f32_dyn_a8w4_workspace_bytes
    # 56x56x64 3x3 pad 1: 3136 unrolled rows of K = 576 codes, scales, zero-points
    assert ws(1, 56, 56, 64, 64, 3, 3, 1, 1, 1, 1) >= 3136 * 576 + 2 * 3136 * 4
    assert ws(1, 56, 56, 60, 64, 3, 3, 1, 1, 1, 1) == 0                   # K % 32
    assert ws(1, 4, 4, 32, 8, 5, 5, 1, 1, 0, 0) == 0                      # kernel larger than image
    assert ws(1, 8, 8, 1024, 8, 5, 5, 1, 1, 2, 2) > 0                     # K = 25600: the limit
    assert ws(1, 8, 8, 25632, 8, 1, 1, 1, 1, 0, 0) == 0                   # K = 25632: over it
    f = lib.qconv2d_f32_dyn_a8w4
    geo = [1, 8, 8, 32, 16, 3, 3, 1, 1, 1, 1]
    big = 1 << 30

    def call(g=geo, x=FAKE, w=FAKE, lo=-1.0, hi=1.0, sym=0, y=FAKE, ws_=FAKE, wsb=big, s=NULL):
        return f(*g, x, w, NULL, lo, hi, sym, y, NULL, s, NULL, ws_, wsb, NULL)

    assert call(g=[1, 8, 8, 30, 16, 3, 3, 1, 1, 1, 1]) == -4             # K = 270, not % 32
    assert call(g=[1, 8, 8, 32, 16, 3, 3, 0, 1, 1, 1]) == -1             # stride 0
    assert call(g=[1, 8, 8, 32, 16, 3, 3, 1, 1, -1, 1]) == -1            # negative pad
    assert call(g=[1, 2, 8, 32, 16, 5, 3, 1, 1, 1, 1]) == -1             # KH > H + 2*pad
    assert call(g=[1, 8, 8, 3200, 16, 3, 3, 1, 1, 1, 1]) == -4           # K = 28800 > 25600
    assert call(g=[200, 56, 56, 32, 16, 1, 1, 1, 1, 0, 0]) == -4         # 627200 unrolled rows
    assert call(sym=2) == -1
    assert call(lo=1.0, hi=-1.0) == -1
    assert call(lo=float("nan")) == -1
    assert call(x=NULL) == -1 and call(w=NULL) == -1 and call(y=NULL) == -1
    assert call(w=ctypes.c_void_p(0x10008)) == -2                        # packed 16-byte aligned
    assert call(x=ctypes.c_void_p(0x10002)) == -2
    assert call(s=ctypes.c_void_p(0x10002)) == -2
    assert call(ws_=NULL) == -7
    need = ws(*geo)
    assert call(wsb=need - 1) == -7
    assert call(ws_=ctypes.c_void_p(0x10080)) == -2                     # workspace 256-byte aligned
