"""GPU parity of symmetric row quantization and of the float-input dynamic
convolution (unrolled rows quantized per output pixel, int4 weights) against
the CPU oracle, through the C ABI.

Quantized rows (codes, scales, zero-points) must match bit-exactly; f32
outputs within |y - y_ref| <= 1e-4 * max(|y_ref|, 1), as the A8W4 linear
(tests/a8w4_tol.py)."""
import numpy as np
import pytest

import oracle
import workloads
from a8w4_tol import assert_a8w4_close

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


@pytest.fixture(autouse=True)
def _clean_status(lib, cuda):
    lib.qg_device_status(True)
    yield
    assert lib.qg_device_status(True) == 0


# ---------------------------------------------------------------------------
# symmetric row quantization
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("M,K,pad", [(1, 4096, 0), (128, 4096, 0), (3, 33, 5), (5, 1, 0),
                                     (2, 1000, 3), (7, 12345, 1), (9, 64, 0)])
def test_quantize_rows_sym_bit_exact(lib, M, K, pad):
    rng = np.random.default_rng(M * 1000 + K + 7)
    x = (rng.standard_normal((M, K + pad)) * rng.uniform(0.1, 10, (M, 1))).astype(np.float32)
    if M >= 3:
        x[1] = 0.0                       # all-zero row
        x[2] = -3.25                     # constant negative row
    q_ref, s_ref, _ = oracle.quantize_rows_a8_sym(x[:, :K])
    xd = _dev(x)
    q = torch.full((M, K + 2), 99, dtype=torch.int8, device="cuda")
    s = torch.empty(M, dtype=torch.float32, device="cuda")
    lib.quantize_rows_a8_sym(xd[:, :K], q[:, :K], s)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(q[:, :K].cpu().numpy(), q_ref)
    assert (q[:, K:].cpu().numpy() == 99).all()          # ldq padding untouched
    np.testing.assert_array_equal(s.cpu().numpy().view(np.int32), s_ref.view(np.int32))


# ---------------------------------------------------------------------------
# float-input dynamic convolution
# ---------------------------------------------------------------------------
def _run_dynconv(lib, w, symmetric):
    Nb, H, W, Cin, Cout = w["Nb"], w["H"], w["W"], w["Cin"], w["Cout"]
    KH, KW, K = w["KH"], w["KW"], w["K"]
    OH, OW = lib.conv_out_hw(H, W, KH, KW, w["stride"], w["pad"])
    P = Nb * OH * OW
    packed = lib.pack_w4_g32(_dev(w["qw"].reshape(Cout, K)), _dev(w["sw"]))
    y = torch.full((Nb, OH, OW, Cout), float("nan"), dtype=torch.float32, device="cuda")
    q = torch.empty((P, K), dtype=torch.int8, device="cuda")
    s = torch.empty(P, dtype=torch.float32, device="cuda")
    z = torch.empty(P, dtype=torch.int32, device="cuda")
    lib.qconv2d_f32_dyn_a8w4(_dev(w["x"]), packed, Cout, KH, KW, w["stride"], w["pad"],
                             _dev(w["bias"]), w["clamp_min"], w["clamp_max"], y,
                             symmetric=symmetric, q_out=q, scale_out=s, zp_out=z)
    torch.cuda.synchronize()
    y_ref, q_ref, s_ref, z_ref = oracle.qconv2d_f32_dyn_a8w4(
        w["x"], w["qw"], w["sw"], w["stride"], w["pad"], w["bias"], w["clamp_min"],
        w["clamp_max"], symmetric=symmetric)
    np.testing.assert_array_equal(q.cpu().numpy(), q_ref)
    np.testing.assert_array_equal(s.cpu().numpy().view(np.int32), s_ref.view(np.int32))
    np.testing.assert_array_equal(z.cpu().numpy(), z_ref)
    assert_a8w4_close(y.cpu().numpy(), y_ref,
                      f"dynconv {'sym' if symmetric else 'asym'} {Nb}x{H}x{W}x{Cin}->{Cout} "
                      f"{KH}x{KW}")
    return y_ref


@pytest.mark.parametrize("symmetric", [False, True])
def test_dynconv_56x56x64_3x3(lib, symmetric):
    _run_dynconv(lib, workloads.a8w4_conv_f32_56x56x64_3x3(), symmetric)


@pytest.mark.parametrize("symmetric", [False, True])
@pytest.mark.parametrize("Nb,H,W,Cin,Cout,KH,KW,stride,pad", [
    (2, 9, 7, 32, 13, 3, 3, (1, 1), (1, 1)),      # P = 126, odd Cout
    (1, 14, 14, 64, 40, 3, 3, (2, 2), (1, 1)),    # strided
    (3, 5, 6, 96, 7, 1, 1, (1, 1), (0, 0)),       # pointwise
    (1, 11, 10, 32, 16, 5, 5, (2, 1), (2, 0)),    # mixed stride and pad
    (1, 4, 4, 128, 33, 4, 4, (1, 1), (0, 0)),     # kernel the size of the image: P = 1
    (1, 7, 7, 32, 9, 3, 3, (3, 3), (2, 2)),       # pixels with mostly pad taps
    (1, 6, 6, 2048, 8, 3, 3, (1, 1), (1, 1)),     # K = 18432
    (1, 9, 9, 4, 10, 4, 4, (1, 1), (1, 1)),       # Cin % 8 != 0 on tensor cores (K = 64)
    (2, 8, 7, 12, 6, 4, 4, (1, 1), (2, 1)),       # Cin % 8 != 0, K = 192, uneven pads
])
def test_dynconv_shapes(lib, symmetric, Nb, H, W, Cin, Cout, KH, KW, stride, pad):
    w = workloads.a8w4_conv_f32(Nb, H, W, Cin, Cout, KH, KW, stride, pad,
                                seed=Nb * 100 + H * 10 + KH + Cout)
    _run_dynconv(lib, w, symmetric)


@pytest.mark.parametrize("symmetric", [False, True])
def test_dynconv_zero_image_gives_the_clamped_bias(lib, symmetric):
    w = workloads.a8w4_conv_f32(1, 6, 5, 32, 12, 3, 3, (1, 1), (1, 1), seed=77,
                                clamp=(-0.05, 0.05))
    w["x"] = np.zeros_like(w["x"])
    y_ref = _run_dynconv(lib, w, symmetric)
    expect = np.clip(w["bias"], np.float32(-0.05), np.float32(0.05))
    assert (y_ref == expect[None, None, None, :]).all()
