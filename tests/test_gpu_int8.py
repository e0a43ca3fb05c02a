"""GPU parity of the INT8 GEMM and INT8 convolution against the CPU oracle,
through the C ABI.  Integer outputs (int8 C and the int32 accumulators) must
match bit-exactly."""
import numpy as np
import pytest

import oracle
import workloads

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


@pytest.fixture(autouse=True)
def _clean_status(lib, cuda):
    lib.qg_device_status(True)
    yield
    assert lib.qg_device_status(True) == 0


def _params(lib, w):
    """(library requant struct args, oracle m0/shift) from the workload's ratios."""
    ratios = np.atleast_1d(w["ratio"])
    lib_p = [lib.qg_requant_params(float(r)) for r in ratios]
    ora_p = [oracle.requant_params(float(r)) for r in ratios]
    assert lib_p == ora_p
    m0 = np.array([p[0] for p in ora_p], np.int64)
    sh = np.array([p[1] for p in ora_p], np.int64)
    if w.get("per_channel", False) or ratios.size > 1:
        mult = _dev(m0.astype(np.int32))
        shift = _dev(sh.astype(np.int32))
    else:
        mult, shift, m0, sh = int(m0[0]), int(sh[0]), int(m0[0]), int(sh[0])
    return mult, shift, m0, sh


def run_gemm(lib, w, packed=False, with_acc=True, rows=None, ldc_pad=0):
    M, N, K = w["M"], w["N"], w["K"]
    A = _dev(w["A"])[:, :K]
    B = _dev(w["B"])[:, :N]
    mult, shift, m0, sh = _params(lib, w)
    bias = None if w["bias"] is None else _dev(w["bias"])
    rq = lib.make_requant(a_zero_point=w["za"], b_zero_point=w["zb"], bias=bias,
                          multiplier=mult, shift=shift, out_zero_point=w["out_zp"],
                          clamp_min=w["clamp_min"], clamp_max=w["clamp_max"])
    C = torch.full((M, N + ldc_pad), 55, dtype=torch.int8, device="cuda")
    acc = torch.full((M, N), 7, dtype=torch.int32, device="cuda") if with_acc else None
    if packed:
        pb = lib.qgemm_pack_b_s8(B)
        lib.qgemm_s8s8_requant_packed(A, pb, N, C[:, :N], rq, K=K, acc_out=acc)
    else:
        lib.qgemm_s8s8_requant(A, B, C[:, :N], rq, K=K, N=N, acc_out=acc)
    torch.cuda.synchronize()
    Cn = C.cpu().numpy()
    if ldc_pad:
        assert (Cn[:, N:] == 55).all()
    return Cn[:, :N], (acc.cpu().numpy() if with_acc else None), m0, sh


def check_gemm(lib, w, rows=None, **kw):
    C, acc, m0, sh = run_gemm(lib, w, **kw)
    K, N = w["K"], w["N"]
    Ar = w["A"][:, :K] if rows is None else w["A"][rows, :K]
    C_ref, acc_ref = oracle.qgemm_s8s8_requant(Ar, w["B"][:, :N], w["za"], w["zb"], w["bias"],
                                               m0, sh, w["out_zp"], w["clamp_min"],
                                               w["clamp_max"])
    Cg = C if rows is None else C[rows]
    np.testing.assert_array_equal(Cg, C_ref)
    if acc is not None:
        np.testing.assert_array_equal(acc if rows is None else acc[rows], acc_ref)
    return C, C_ref


def test_gemm_130x70x129_bit_exact(lib):
    w = workloads.int8_gemm_130x70x129()
    C, C_ref = check_gemm(lib, w)
    # the outputs are not trivially saturated
    assert 0.05 < np.mean(np.abs(C_ref.astype(int)) < 127)


def test_gemm_130x70x129_packed_bit_exact(lib):
    check_gemm(lib, workloads.int8_gemm_130x70x129(), packed=True, ldc_pad=3)


# Kernel choice: M <= 128 -> one CTA per 128 x 256 tile; M <= 256 -> the same
# while its tiles fit in one wave (129x257: 4 tiles; 256x16: 2), else CTA
# pairs (200x19000: 2 x 75 = 150 one-CTA tiles, more than the 148 SMs).
SHAPES = [(1, 1, 1), (2, 16, 31), (127, 70, 129), (128, 256, 128), (129, 257, 256),
          (256, 16, 200), (200, 19000, 64), (300, 600, 300), (64, 40, 1000), (257, 513, 130)]


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("per_channel,zb", [(False, None), (True, 0)])
def test_gemm_shapes(lib, M, N, K, per_channel, zb):
    seed = M * 10007 + N * 101 + K + (1 if per_channel else 0)
    w = workloads.int8_gemm(M, N, K, seed, per_channel=per_channel, zb=zb,
                            lda=K + (seed % 5), ldb=N + (seed % 3))
    check_gemm(lib, w)


# M > 256 runs on CTA pairs (as does M > 128 when one-CTA tiles would take
# more than one wave).  Rows the tensor-copy engine cannot address
# (pitch or base not a multiple of 16 bytes) are first copied to a 16-byte
# pitch.  Cases: pitches 8, 4 and 1 (mod 16), a base offset into the
# allocation, b_zero_point != 0 (row sums), ragged M / N / K, and more tiles
# than resident CTA pairs (the stage ring wraps across tiles).
PAIR_UNALIGNED = [
    # M,   N,    K,   lda, a_off, zb
    (300, 300, 264, 264, 0, 0),       # pitch = 8 (mod 16)
    (257, 520, 1000, 1004, 0, 0),     # pitch = 4 (mod 8)
    (384, 256, 1000, 1000, 8, 0),     # base 8 bytes into the allocation
    (300, 300, 264, 264, 4, 5),       # base 4 bytes in, b zero-point (row sums)
    (260, 130, 131, 131, 0, 0),       # odd pitch
    (4096, 2560, 136, 136, 0, 0),     # 160 pair tiles
]


@pytest.mark.parametrize("M,N,K,lda,a_off,zb", PAIR_UNALIGNED)
def test_gemm_pair_unaligned_rows(lib, M, N, K, lda, a_off, zb):
    w = workloads.int8_gemm(M, N, K, 7000 + M + lda, zb=zb, per_channel=True, lda=lda,
                            ratio_range=(1e-5, 1e-3))
    flat = torch.full((M * lda + a_off + 16,), 99, dtype=torch.int8, device="cuda")
    flat[a_off:a_off + M * lda].copy_(_dev(w["A"]).reshape(-1))
    A = torch.as_strided(flat, (M, K), (lda, 1), a_off)
    B = _dev(w["B"])[:, :N]
    mult, shift, m0, sh = _params(lib, w)
    rq = lib.make_requant(a_zero_point=w["za"], b_zero_point=w["zb"], bias=_dev(w["bias"]),
                          multiplier=mult, shift=shift, out_zero_point=w["out_zp"],
                          clamp_min=w["clamp_min"], clamp_max=w["clamp_max"])
    C = torch.full((M, N), 55, dtype=torch.int8, device="cuda")
    acc = torch.full((M, N), 7, dtype=torch.int32, device="cuda")
    lib.qgemm_s8s8_requant_packed(A, lib.qgemm_pack_b_s8(B), N, C, rq, K=K, acc_out=acc)
    torch.cuda.synchronize()
    C_ref, acc_ref = oracle.qgemm_s8s8_requant(w["A"][:, :K], w["B"][:, :N], w["za"], w["zb"],
                                               w["bias"], m0, sh, w["out_zp"], w["clamp_min"],
                                               w["clamp_max"])
    np.testing.assert_array_equal(acc.cpu().numpy(), acc_ref)
    np.testing.assert_array_equal(C.cpu().numpy(), C_ref)


def test_gemm_relu_clamp_and_no_bias(lib):
    w = workloads.int8_gemm(200, 96, 200, seed=77, with_bias=False, out_zp=-10,
                            clamp=(-10, 127))
    check_gemm(lib, w)


def test_gemm_extreme_bound(lib):
    # all terms at the worst magnitude 255*255 with K at the page's example size
    K = 129
    w = workloads.int8_gemm(130, 70, K, seed=1, za=-128, zb=127, with_bias=False)
    w["A"][:] = 127
    w["B"][:] = -128
    w["ratio"] = np.array([1e-7])
    C, acc, m0, sh = run_gemm(lib, w)
    assert (acc == -K * 65025).all()


@pytest.mark.parametrize("M", [64, 200, 300])
def test_gemm_k_at_the_overflow_bound(lib, M):
    # K = 33025 is the largest K with K*65025 <= 2^31 - 1 (no bias): every term
    # at the worst magnitude gives an accumulator of -2,147,450,625, inside
    # int32 by 33,022.  M = 64 and 200 run the one-CTA kernel (one and two row
    # tiles), M = 300 the CTA pairs.
    K = 33025
    w = workloads.int8_gemm(M, 64, K, seed=3, za=-128, zb=127, with_bias=False)
    w["A"][:] = 127
    w["B"][:] = -128
    w["ratio"] = np.array([1e-9])
    C, acc, m0, sh = run_gemm(lib, w)
    assert (acc == -K * 65025).all()
    assert (C == w["out_zp"] + np.int64(oracle.rq_round(np.int64(-K * 65025), m0, sh))).all()


def test_gemm_deterministic(lib):
    w = workloads.int8_gemm(300, 300, 500, seed=9)
    C1, a1, *_ = run_gemm(lib, w)
    C2, a2, *_ = run_gemm(lib, w)
    np.testing.assert_array_equal(C1, C2)
    np.testing.assert_array_equal(a1, a2)


def test_gemm_8192x8192x8200_sampled_rows(lib):
    # direct int64 definition on rows at tile edges (the full check below
    # goes through the exact float64 route)
    w = workloads.int8_gemm_8192x8192x8200()
    rows = np.array([0, 1, 127, 128, 129, 2047, 4096, 5000, 8063, 8064, 8190, 8191])
    C, C_ref = check_gemm(lib, w, packed=True, rows=rows)
    # every column of the sampled rows is checked; outputs are not all saturated
    assert np.mean(np.abs(C_ref.astype(int)) < 127) > 0.05


@pytest.mark.parametrize("packed", [True, False])
def test_gemm_8192x8192x8200_every_output(lib, packed):
    """All 67,108,864 outputs (int8 C and the int32 accumulators) of the
    8192x8192x8200 GEMM against the oracle's exact float64 accumulation
    (pinned to the int64 definition on the CPU) and its requantization.
    packed=True is the weights-stationary call the benchmark times."""
    w = workloads.int8_gemm_8192x8192x8200()
    C, acc, m0, sh = run_gemm(lib, w, packed=packed)
    K, N = w["K"], w["N"]
    B = w["B"][:, :N]
    for r0 in range(0, w["M"], 2048):
        rows = slice(r0, r0 + 2048)
        acc_ref = oracle.int8_gemm_acc_f64(w["A"][rows, :K], B, w["za"], w["zb"], w["bias"])
        bad = np.argwhere(acc[rows] != acc_ref)
        assert bad.size == 0, f"first accumulator mismatch at row {r0 + bad[0][0]}, col {bad[0][1]}"
        C_ref = oracle.requantize(acc_ref, m0, sh, w["out_zp"], w["clamp_min"], w["clamp_max"])
        bad = np.argwhere(C[rows] != C_ref)
        assert bad.size == 0, f"first output mismatch at row {r0 + bad[0][0]}, col {bad[0][1]}"


# ---------------------------------------------------------------------------
# convolution
# ---------------------------------------------------------------------------
def run_conv(lib, w, with_acc=True, packed=False, x_offset=0):
    mult, shift, m0, sh = _params(lib, dict(ratio=w["ratio"], per_channel=True))
    bias = None if w["bias"] is None else _dev(w["bias"])
    rq = lib.make_requant(a_zero_point=w["za"], bias=bias, multiplier=mult, shift=shift,
                          out_zero_point=w["out_zp"], clamp_min=w["clamp_min"],
                          clamp_max=w["clamp_max"])
    OH, OW = lib.conv_out_hw(w["H"], w["W"], w["KH"], w["KW"], w["stride"], w["pad"])
    y = torch.empty((w["Nb"], OH, OW, w["Cout"]), dtype=torch.int8, device="cuda")
    acc = torch.empty((w["Nb"], OH, OW, w["Cout"]), dtype=torch.int32, device="cuda") if with_acc else None
    x = _dev(w["x"])
    if x_offset:  # the same image at an address that is not 16-byte aligned
        buf = torch.empty(x.numel() + x_offset, dtype=torch.int8, device="cuda")
        x = buf[x_offset:].view(x.shape)
        x.copy_(_dev(w["x"]))
    if packed:
        pw = lib.qconv2d_s8_pack_w(_dev(w["w"]))
        lib.qconv2d_s8_im2col_packed(x, pw, w["w"].shape, y, rq, w["stride"], w["pad"],
                                     acc_out=acc)
    else:
        lib.qconv2d_s8_im2col(x, _dev(w["w"]), y, rq, w["stride"], w["pad"], acc_out=acc)
    torch.cuda.synchronize()
    y_ref, acc_ref = oracle.qconv2d_s8(w["x"], w["w"], w["stride"], w["pad"], w["za"], w["bias"],
                                       m0, sh, w["out_zp"], w["clamp_min"], w["clamp_max"])
    np.testing.assert_array_equal(y.cpu().numpy(), y_ref)
    if with_acc:
        np.testing.assert_array_equal(acc.cpu().numpy(), acc_ref)
    return y_ref


def test_conv_56x56x64_bit_exact(lib):
    y_ref = run_conv(lib, workloads.int8_conv_56x56x64_3x3())
    assert (y_ref == -10).mean() > 0.05      # the ReLU floor at the out zero-point binds


@pytest.mark.parametrize("x_offset", [0, 3])
def test_conv_56x56x64_packed_weights_bit_exact(lib, x_offset):
    # weights packed once; x_offset = 3 takes the byte-gather path
    run_conv(lib, workloads.int8_conv_56x56x64_3x3(), packed=True, x_offset=x_offset)


def test_conv_more_tiles_than_sms(lib):
    # 12 x 40 x 40 output pixels = 150 row tiles of 128 on a 148-SM grid: some
    # CTAs run two tiles, so the stage ring and the two TMEM accumulators wrap
    # across tiles
    w = workloads.int8_conv(12, 40, 40, 16, 8, 3, 3, (1, 1), (1, 1), seed=4411)
    run_conv(lib, w, packed=True)


def test_gemm_one_cta_more_tiles_than_sms(lib):
    # M <= 128: the one-CTA kernel; 149 column tiles of 256 on 148 CTAs
    w = workloads.int8_gemm(64, 38000, 64, seed=4412, per_channel=True)
    check_gemm(lib, w)


@pytest.mark.parametrize("Nb,H,W,Cin,Cout,KH,KW,s,p", [
    (2, 17, 19, 32, 96, 3, 3, 1, 1), (1, 40, 33, 16, 300, 5, 5, 2, 2), (3, 9, 9, 48, 40, 1, 3, 1, 0),
    (1, 12, 12, 3, 8, 7, 7, 2, 3), (1, 300, 3, 64, 64, 3, 3, 1, 1)])
def test_conv_packed_shapes(lib, Nb, H, W, Cin, Cout, KH, KW, s, p):
    w = workloads.int8_conv(Nb, H, W, Cin, Cout, KH, KW, (s, s), (p, p), seed=H * 3 + Cin + Cout,
                            relu=(Cout % 2 == 0))
    run_conv(lib, w, packed=True)


@pytest.mark.parametrize("Nb,H,W,Cin,Cout,KH,KW,s,p", [
    (1, 9, 7, 8, 5, 3, 3, 1, 1), (2, 15, 16, 3, 33, 3, 3, 2, 1), (1, 8, 8, 64, 300, 1, 1, 1, 0),
    (3, 11, 13, 20, 64, 5, 3, 2, 2), (1, 30, 30, 130, 17, 3, 3, 1, 0)])
def test_conv_shapes(lib, Nb, H, W, Cin, Cout, KH, KW, s, p):
    w = workloads.int8_conv(Nb, H, W, Cin, Cout, KH, KW, (s, s), (p, p), seed=H * W + Cin + Cout,
                            relu=(Cout % 2 == 1))
    run_conv(lib, w)
