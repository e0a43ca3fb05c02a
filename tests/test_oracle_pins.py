"""Pins for the CPU oracle, run without a GPU.

Each test ties an oracle function to something other than itself: numbers
printed on the pages (fixtures under tests/golden/, each with its source),
closed forms, invariants, or brute force on tiny inputs written as plain
Python loops.  A dropped term, a wrong sign, a transposed operand or a wrong
group index in the oracle fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------------------
# P1: the 130x70x129 worked example (quantized GEMM case study, section 3)
# ---------------------------------------------------------------------------
def test_p1_tiling_counts_match_page():
    g = _golden("qg_tiling_130x70x129.json")
    w = workloads.int8_gemm_130x70x129()
    assert (w["M"], w["N"], w["K"]) == (g["M"], g["N"], g["K"])
    A, B = w["A"][:, :w["K"]], w["B"][:, :w["N"]]
    acc_t, st = oracle.tiled_int8_gemm(A, B, w["za"], w["zb"], w["bias"],
                                       g["Tm"], g["Tn"], g["Tk"])
    assert st["tiles_mnk"] == (g["tiles_m"], g["tiles_n"], g["tiles_k"])
    assert st["tiles"] == g["tiles"]
    assert st["useful_macs"] == g["useful_macs"]
    assert st["slots"] == g["slots"]
    assert round(100 * st["shape_efficiency"], 2) == g["shape_efficiency_percent_approx"]
    # level 3 of the verification ladder: the tiled model equals the full GEMM
    acc = oracle.int8_gemm_acc(A, B, w["za"], w["zb"], w["bias"])
    np.testing.assert_array_equal(acc_t, acc)


def test_p1_buffer_budget_matches_page():
    g = _golden("qg_tiling_130x70x129.json")
    b = oracle.tile_budget_bytes(g["Tm"], g["Tn"], g["Tk"], g["reserve_bytes"])
    assert b["S_input"] == g["S_input_bytes"]
    assert b["S_acc"] == g["S_acc_bytes"]
    assert b["S_total"] == g["S_total_bytes"]


# ---------------------------------------------------------------------------
# P2: INT32 overflow bound (section 4)
# ---------------------------------------------------------------------------
def test_p2_overflow_constants():
    g = _golden("qg_overflow_bound.json")
    assert oracle.worst_zp_corrected_magnitude() == g["worst_magnitude"]
    assert oracle.overflow_bound(1, 0) == g["product_bound"]
    assert oracle.fits_int32(g["K_safe_example"], 5000)
    assert oracle.overflow_bound(129, 0) == 129 * 65025 == 8388225


def test_p2_extreme_case_reaches_bound_exactly():
    K = 129
    A = np.full((2, K), 127, np.int8)
    B = np.full((K, 3), -128, np.int8)
    acc = oracle.int8_gemm_acc(A, B, za=-128, zb=127)
    assert (acc == -K * 65025).all()
    A2 = np.full((1, K), -128, np.int8)
    acc2 = oracle.int8_gemm_acc(A2, B, za=127, zb=127)
    assert (acc2 == K * 65025).all()


def test_p2_bound_edge_and_rejection():
    # 33025*65025 = 2147450625 <= 2^31-1 < 33026*65025 = 2147515650
    assert oracle.fits_int32(33025, 0)
    assert not oracle.fits_int32(33026, 0)
    assert not oracle.fits_int32(33025, 2 ** 31 - 1 - 2147450625 + 1)
    A = np.zeros((1, 33026), np.int8)
    B = np.zeros((33026, 1), np.int8)
    with pytest.raises(OverflowError):
        oracle.qgemm_s8s8_requant(A, B, 0, 0, None, 2 ** 30, 0, 0, -128, 127)


# ---------------------------------------------------------------------------
# P3: padding stands for real zero (section 2)
# ---------------------------------------------------------------------------
def test_p3_zero_point_padding_invariance():
    w = workloads.int8_gemm_130x70x129()
    A, B = w["A"][:, :129], w["B"][:, :70]
    za, zb = 11, -7        # non-zero on both sides so raw-zero padding is visible
    acc = oracle.int8_gemm_acc(A, B, za, zb, w["bias"])
    Ap = np.full((130, 256), za, np.int8); Ap[:, :129] = A
    Bp = np.full((256, 70), zb, np.int8); Bp[:129] = B
    np.testing.assert_array_equal(oracle.int8_gemm_acc(Ap, Bp, za, zb, w["bias"]), acc)
    A0 = np.zeros((130, 256), np.int8); A0[:, :129] = A
    B0 = np.zeros((256, 70), np.int8); B0[:129] = B
    assert (oracle.int8_gemm_acc(A0, B0, za, zb, w["bias"]) != acc).any()


def _im2col_zp(x, KH, KW, stride, pad, za):
    Nb, H, W, C = x.shape
    OH = oracle.conv_out_size(H, KH, stride[0], pad[0])
    OW = oracle.conv_out_size(W, KW, stride[1], pad[1])
    xp = np.full((Nb, H + 2 * pad[0], W + 2 * pad[1], C), za, np.int8)
    xp[:, pad[0]:pad[0] + H, pad[1]:pad[1] + W] = x
    cols = np.empty((Nb, OH, OW, KH, KW, C), np.int8)
    for kh in range(KH):
        for kw in range(KW):
            cols[:, :, :, kh, kw] = xp[:, kh:kh + stride[0] * OH:stride[0],
                                       kw:kw + stride[1] * OW:stride[1]]
    return cols.reshape(Nb * OH * OW, KH * KW * C)


def test_p3_conv_equals_zp_padded_im2col_gemm():
    w = workloads.int8_conv(1, 9, 7, 8, 5, 3, 3, (1, 1), (1, 1), seed=7)
    acc = oracle.qconv2d_s8_acc(w["x"], w["w"], w["stride"], w["pad"], w["za"], w["bias"])
    cols = _im2col_zp(w["x"], 3, 3, w["stride"], w["pad"], w["za"])
    Bm = w["w"].reshape(w["Cout"], -1).T
    acc2 = oracle.int8_gemm_acc(cols, Bm, w["za"], 0, w["bias"])
    np.testing.assert_array_equal(acc.reshape(-1, w["Cout"]), acc2)
    # raw-zero padding would be wrong
    cols0 = _im2col_zp(w["x"], 3, 3, w["stride"], w["pad"], 0)
    assert (oracle.int8_gemm_acc(cols0, Bm, w["za"], 0, w["bias"]) != acc2).any()


def test_conv_brute_force_loops():
    rng = np.random.default_rng(3)
    Nb, H, W, Cin, Cout, KH, KW = 2, 4, 5, 3, 2, 3, 2
    sh, sw_, ph, pw = 2, 1, 1, 0
    x = rng.integers(-128, 128, (Nb, H, W, Cin)).astype(np.int8)
    wt = rng.integers(-127, 128, (Cout, KH, KW, Cin)).astype(np.int8)
    za = -5
    bias = rng.integers(-50, 50, Cout).astype(np.int32)
    OH, OW = (H + 2 * ph - KH) // sh + 1, (W + 2 * pw - KW) // sw_ + 1
    ref = np.zeros((Nb, OH, OW, Cout), np.int64)
    for n in range(Nb):
        for oh in range(OH):
            for ow in range(OW):
                for co in range(Cout):
                    s = int(bias[co])
                    for kh in range(KH):
                        for kw in range(KW):
                            for ci in range(Cin):
                                ih, iw = oh * sh + kh - ph, ow * sw_ + kw - pw
                                v = int(x[n, ih, iw, ci]) if (0 <= ih < H and 0 <= iw < W) else za
                                s += (v - za) * int(wt[co, kh, kw, ci])
                    ref[n, oh, ow, co] = s
    got = oracle.qconv2d_s8_acc(x, wt, (sh, sw_), (ph, pw), za, bias)
    np.testing.assert_array_equal(got, ref)


# ---------------------------------------------------------------------------
# P4: accumulate across K, requantize once (section 4)
# ---------------------------------------------------------------------------
def test_p4_k_block_accumulation():
    w = workloads.int8_gemm_130x70x129()
    A, B = w["A"][:, :129], w["B"][:, :70]
    acc = oracle.int8_gemm_acc(A, B, w["za"], w["zb"])
    parts = [oracle.int8_gemm_acc(A[:, k:k + 32], B[k:k + 32], w["za"], w["zb"])
             for k in range(0, 129, 32)]
    np.testing.assert_array_equal(sum(parts), acc)
    m0, sh = oracle.requant_params(float(w["ratio"][0]))
    once = oracle.rq_round(acc, m0, sh)
    # requantizing every block partial changes the result somewhere
    m0b, shb = oracle.requant_params(0.37)
    y1 = oracle.requantize(acc, m0b, shb, 0, -128, 127).astype(np.int64)
    y2 = sum(oracle.requantize(p, m0b, shb, 0, -128, 127).astype(np.int64) for p in parts)
    assert (np.clip(y2, -128, 127) != y1).any()
    assert once.shape == acc.shape


# ---------------------------------------------------------------------------
# P5: brute force (pure Python loops) and float dequant reference
# ---------------------------------------------------------------------------
def test_p5_gemm_brute_force_loops():
    rng = np.random.default_rng(11)
    M, N, K = 3, 4, 5
    A = rng.integers(-128, 128, (M, K)).astype(np.int8)
    B = rng.integers(-128, 128, (K, N)).astype(np.int8)
    za, zb = -17, 9
    bias = rng.integers(-5000, 5001, N).astype(np.int32)
    ref = [[int(bias[n]) + sum((int(A[m, k]) - za) * (int(B[k, n]) - zb) for k in range(K))
            for n in range(N)] for m in range(M)]
    np.testing.assert_array_equal(oracle.int8_gemm_acc(A, B, za, zb, bias), np.array(ref))


def test_p5_float64_accumulation_is_exact_against_int64_loops():
    # The float64 route equals the int64 definition on random blocks with
    # several row blocks, zero-points and a bias, and on the all-worst-case
    # operands at K = 8200, where every product is -65025 and the sum reaches
    # -533,205,000: far past float32's exact range (2^24), inside float64's.
    rng = np.random.default_rng(21)
    for M, N, K, za, zb in [(37, 29, 8200, 7, 0), (300, 64, 1000, -20, 13), (5, 3, 1, 0, 0)]:
        A = rng.integers(-128, 128, (M, K)).astype(np.int8)
        B = rng.integers(-128, 128, (K, N)).astype(np.int8)
        bias = rng.integers(-5000, 5001, N).astype(np.int32)
        ref = oracle.int8_gemm_acc(A, B, za, zb, bias)
        np.testing.assert_array_equal(oracle.int8_gemm_acc_f64(A, B, za, zb, bias, row_block=16),
                                      ref)
    K = 8200
    A = np.full((3, K), 127, np.int8)
    B = np.full((K, 4), -128, np.int8)
    acc = oracle.int8_gemm_acc_f64(A, B, za=-128, zb=127)
    assert (acc == -K * 65025).all()
    # that sum is not a float32 value: an accumulation in float32 would fail here
    assert int(np.float32(K * 65025)) != K * 65025
    # a few brute-force entries with plain Python integers
    A = rng.integers(-128, 128, (4, 50)).astype(np.int8)
    B = rng.integers(-128, 128, (50, 6)).astype(np.int8)
    f = oracle.int8_gemm_acc_f64(A, B, 3, -5)
    for m in range(4):
        for n in range(6):
            assert f[m, n] == sum((int(A[m, k]) - 3) * (int(B[k, n]) + 5) for k in range(50))


def test_p5_float64_accumulation_refuses_k_past_the_exact_range():
    K = 2 ** 53 // 65025 + 1
    A = np.broadcast_to(np.int8(0), (1, K))        # views: nothing of size K is allocated
    B = np.broadcast_to(np.int8(0), (K, 1))
    with pytest.raises(ValueError):
        oracle.int8_gemm_acc_f64(A, B, 0, 0)


def test_p5_float_dequant_reference():
    w = workloads.int8_gemm(37, 23, 129, seed=5)
    A, B = w["A"], w["B"]
    rng = np.random.default_rng(1)
    sA = 0.02
    sB = rng.uniform(1e-3, 1e-1, w["N"])
    acc = oracle.int8_gemm_acc(A, B, w["za"], w["zb"])
    real = (sA * (A.astype(np.float64) - w["za"])) @ (sB[None, :] * (B.astype(np.float64) - w["zb"]))
    np.testing.assert_allclose(sA * sB[None, :] * acc, real, rtol=1e-12, atol=1e-9)


def test_p5_requant_within_one_lsb_of_real_ratio():
    rng = np.random.default_rng(2)
    acc = rng.integers(-2 ** 24, 2 ** 24, 20000)
    worst, mism = 0, 0
    for ratio in np.exp(rng.uniform(np.log(1e-6), np.log(0.99), 50)):
        m0, sh = oracle.requant_params(ratio)
        y = oracle.rq_round(acc, m0, sh)
        ref = np.rint(acc * ratio).astype(np.int64)
        d = np.abs(y - ref)
        worst = max(worst, int(d.max()))
        mism += int((d != 0).sum())
    assert worst <= 1
    assert mism < 0.01 * 50 * 20000


def test_requant_params_closed_forms():
    assert oracle.requant_params(0.5) == (2 ** 30, 0)
    assert oracle.requant_params(0.25) == (2 ** 30, 1)
    assert oracle.requant_params(2.0 ** -10) == (2 ** 30, 9)
    assert oracle.requant_params(0.75) == (3 * 2 ** 29, 0)
    rng = np.random.default_rng(4)
    for r in np.exp(rng.uniform(np.log(1e-9), np.log(0.999), 200)):
        m0, sh = oracle.requant_params(r)
        assert 2 ** 30 <= m0 < 2 ** 31
        assert abs(m0 * 2.0 ** -(31 + sh) - r) <= 2.0 ** -(32 + sh)
    for bad in (0.0, 1.0, 1.5, -0.1, 1e-12):
        with pytest.raises(ValueError):
            oracle.requant_params(bad)


def test_requant_params_carry_into_the_next_power_of_two():
    # f = 1 - 2^-33 rounds to 2^31 at 31 bits, which does not fit int32: the
    # multiplier becomes 2^30 one binade up, i.e. exactly 0.5 (resp. 0.25)
    assert oracle.requant_params(0.5 - 2.0 ** -34) == (2 ** 30, 0)
    assert oracle.requant_params(0.25 - 2.0 ** -35) == (2 ** 30, 1)
    # one step further from the power of two stays below it
    assert oracle.requant_params(0.5 - 2.0 ** -31) == (2 ** 31 - 2, 1)


def test_requant_round_half_even_cases():
    m0, sh = oracle.requant_params(0.5)            # divides by exactly 2
    acc = np.array([3, 5, 7, -3, -5, -7, 1, -1, 4])
    y = oracle.requantize(acc, m0, sh, 0, -128, 127)
    np.testing.assert_array_equal(y, [2, 2, 4, -2, -2, -4, 0, 0, 2])
    y = oracle.requantize(np.array([1000, -1000]), m0, sh, 3, -128, 127)
    np.testing.assert_array_equal(y, [127, -128])   # saturating clamp
    y = oracle.requantize(np.array([-40, 40]), m0, sh, -10, -10, 127)
    np.testing.assert_array_equal(y, [-10, 10])     # ReLU floor at the out zero-point


# ---------------------------------------------------------------------------
# P6: dynamic activation quantization specials
# ---------------------------------------------------------------------------
def test_p6_quantization_specials():
    for case in _golden("qg_dynamic_quant_specials.json")["cases"]:
        q, s, z = oracle.quantize_rows_a8(np.array([case["x"]], np.float32))
        assert s[0] == np.float32(case["scale"])
        assert z[0] == case["zp"]
        np.testing.assert_array_equal(q[0], case["q"])


def test_p6_constant_row_and_error_bound():
    q, s, z = oracle.quantize_rows_a8(np.full((1, 10), 1.0, np.float32))
    assert z[0] == -128 and (q == 127).all()
    x = np.random.default_rng(9).standard_normal((16, 333)).astype(np.float32) * 3
    q, s, z = oracle.quantize_rows_a8(x)
    assert (s > 0).all()
    # real 0.0 is exactly representable: it maps to the zero-point
    xz = np.concatenate([x[:, :5], np.zeros((16, 1), np.float32)], 1)
    q0, _, z0 = oracle.quantize_rows_a8(xz)
    np.testing.assert_array_equal(q0[:, -1], z0)
    err = np.abs(oracle.dequantize_rows(q, s, z) - x.astype(np.float64))
    assert (err <= 0.5 * s[:, None] * (1 + 1e-5)).all()
    # each row reaches an end of the code range at its extreme value
    assert ((q.min(1) == -128) | (q.max(1) == 127)).all()


def test_p6_grid_exact_round_trip():
    rng = np.random.default_rng(12)
    zp = -40
    s = np.float32(0.125)                 # power of two: exact arithmetic
    codes = rng.integers(-128, 128, (1, 300))
    codes[0, 0], codes[0, 1] = -128, 127  # pin the range so min/max give s, zp
    x = ((codes - zp) * s).astype(np.float32)
    q, sc, z = oracle.quantize_rows_a8(x)
    assert sc[0] == s and z[0] == zp
    np.testing.assert_array_equal(q[0], codes[0])


# ---------------------------------------------------------------------------
# P7: A8W4 special case and brute force
# ---------------------------------------------------------------------------
def test_p7_a8w4_integer_special_case():
    rng = np.random.default_rng(21)
    N, K = 40, 128
    x = rng.integers(-100, 156, (1, K)).astype(np.float32)
    x[0, 0], x[0, 1] = -100, 155          # scale (155+100)/255 = 1 exactly
    qw = rng.integers(-8, 8, (N, K)).astype(np.int8)
    sw = np.ones((N, K // 32), np.float32)
    bias = rng.integers(-9, 10, N).astype(np.float32)
    y, q, s, z = oracle.qgemm_a8w4_f32(x, qw, sw, bias, -np.inf, np.inf)
    assert s[0] == 1.0 and z[0] == -28
    exact = qw.astype(np.int64) @ x[0].astype(np.int64) + bias.astype(np.int64)
    np.testing.assert_array_equal(y[0], exact.astype(np.float32))


def test_p7_a8w4_brute_force_loops():
    rng = np.random.default_rng(22)
    M, N, K = 2, 3, 64
    x = rng.standard_normal((M, K)).astype(np.float32)
    qw = rng.integers(-8, 8, (N, K)).astype(np.int8)
    sw = rng.uniform(0.01, 0.1, (N, K // 32)).astype(np.float32)
    bias = rng.normal(0, 0.1, N).astype(np.float32)
    y, q, s, z = oracle.qgemm_a8w4_f32(x, qw, sw, bias, -0.5, 0.5)
    for m in range(M):
        for n in range(N):
            t = float(bias[n])
            for k in range(K):
                t += float(s[m]) * (int(q[m, k]) - int(z[m])) * float(sw[n, k // 32]) * int(qw[n, k])
            assert abs(float(y[m, n]) - min(max(t, -0.5), 0.5)) <= 1e-6 * max(1.0, abs(t))


def test_p7_a8w4_float_reference():
    w = workloads.a8w4(3, 50, 256, seed=8, clamp=(-np.inf, np.inf))
    y, q, s, z = oracle.qgemm_a8w4_f32(w["x"], w["qw"], w["sw"], w["bias"], -np.inf, np.inf)
    xa = oracle.dequantize_rows(q, s, z)
    wd = np.repeat(w["sw"].astype(np.float64), 32, axis=1) * w["qw"]
    ref = xa @ wd.T + w["bias"].astype(np.float64)
    np.testing.assert_allclose(y, ref, rtol=1e-6, atol=1e-6)
    # and the quantized activations approximate x to within half a step
    assert (np.abs(xa - w["x"]) <= 0.5 * s[:, None] * (1 + 1e-5)).all()


# ---------------------------------------------------------------------------
# P8: W4 packed layout (this library's own format, reading R6)
# ---------------------------------------------------------------------------
def test_p8_w4_pack_round_trip_and_bytes():
    w = workloads.a8w4(1, 7, 96, seed=9)
    packed = oracle.pack_w4_g32(w["qw"], w["sw"])
    assert packed.size == oracle.pack_w4_g32_bytes(7, 96)
    qw2, sw2 = oracle.unpack_w4_g32(packed, 7, 96)
    np.testing.assert_array_equal(qw2, w["qw"])
    np.testing.assert_array_equal(sw2, w["sw"])
    # hand-derived pattern: q[k] = (k % 16) - 8 -> nibble value k % 16
    qw = ((np.arange(32) % 16) - 8).astype(np.int8)[None, :]
    p = oracle.pack_w4_g32(qw, np.ones((1, 1), np.float32))
    # word j covers k = 8j..8j+7: low nibble of byte b = k0+b, high = k0+4+b
    expect = []
    for j in range(4):
        for b in range(4):
            lo, hi = (8 * j + b) % 16, (8 * j + 4 + b) % 16
            expect.append(lo | (hi << 4))
    np.testing.assert_array_equal(p[:16], expect)
    assert p[16:20].view(np.float32)[0] == 1.0


# ---------------------------------------------------------------------------
# P9: bf16 group scales (reading R12: f32 -> bf16 round to nearest, ties to
# even; the method uses the bf16 value)
# ---------------------------------------------------------------------------
def test_p9_bf16_rounding_hand_derived_cases():
    # bf16 keeps 7 fraction bits: around 1.0 the spacing is 2^-7
    cases = [
        (1.0, 0x3F80),
        (1 + 2 ** -8, 0x3F80),              # exactly half way: tie -> even (0x3F80)
        (1 + 3 * 2 ** -8, 0x3F82),          # half way between 0x3F81 and 0x3F82 -> even
        (1 + 2 ** -8 + 2 ** -23, 0x3F81),   # just above half way -> up
        (1 + 2 ** -8 - 2 ** -23, 0x3F80),   # just below half way -> down
        (-(1 + 2 ** -8), 0xBF80),           # the sign does not change the rounding
        (2.0 ** -126, 0x0080),              # smallest normal, exact
        (0.1, 0x3DCD),                      # 0x3DCCCCCD: low half 0xCCCD > 0x8000 -> up
        (65280.0, 0x477F),                  # 255 * 256 exact
    ]
    x = np.array([c[0] for c in cases], np.float32)
    got = oracle.f32_to_bf16_bits(x)
    assert [int(v) for v in got] == [c[1] for c in cases]
    # round trip of exact bf16 values is the identity
    np.testing.assert_array_equal(oracle.bf16_bits_to_f32(got)[[0, 6, 8]],
                                  np.array([1.0, 2.0 ** -126, 65280.0], np.float32))


def test_p9_bf16_rounding_matches_library_conversion():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(12)
    x = rng.standard_normal(20000).astype(np.float32) * np.float32(10.0) ** rng.integers(-6, 6, 20000)
    # exact ties: an f32 whose low 16 bits are 0x8000, both parities of bit 16
    ties = (rng.integers(0x3000, 0x4F00, 4000).astype(np.uint32) << 16) | 0x8000
    x = np.concatenate([x, ties.view(np.float32)])
    lib = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(oracle.f32_to_bf16_bits(x), lib)


def test_p9_bf16_pack_layout_and_scales():
    w = workloads.a8w4(1, 5, 64, seed=4)
    p = oracle.pack_w4_g32_bf16(w["qw"], w["sw"])
    assert p.size == oracle.pack_w4_g32_bf16_bytes(5, 64) == 5 * 32 + 5 * 2 * 2
    # the nibble region is the f32 packing's, byte for byte
    np.testing.assert_array_equal(p[:160], oracle.pack_w4_g32(w["qw"], w["sw"])[:160])
    bits = p[160:].view("<u2").reshape(5, 2)
    np.testing.assert_array_equal(bits, oracle.f32_to_bf16_bits(w["sw"]))
    # the rounded scale is within half a bf16 step (2^-8 relative) of the f32 scale
    rel = np.abs(oracle.bf16_scales(w["sw"]) - w["sw"]) / w["sw"]
    assert rel.max() <= 2.0 ** -8


def test_p9_bf16_linear_equals_f32_linear_on_representable_scales():
    # with scales that are exact in bf16 (powers of two) the two methods agree
    w = workloads.a8w4(3, 40, 128, seed=5)
    sw = (2.0 ** np.round(np.log2(w["sw"]))).astype(np.float32)
    np.testing.assert_array_equal(oracle.bf16_scales(sw), sw)
    y16 = oracle.qgemm_a8w4_f32_bf16s(w["x"], w["qw"], sw, w["bias"], -6.0, 6.0)[0]
    y32 = oracle.qgemm_a8w4_f32(w["x"], w["qw"], sw, w["bias"], -6.0, 6.0)[0]
    np.testing.assert_array_equal(y16, y32)
    # and with general scales they differ only through the rounded scales
    y16g = oracle.qgemm_a8w4_f32_bf16s(w["x"], w["qw"], w["sw"], w["bias"], -6.0, 6.0)[0]
    y32r = oracle.qgemm_a8w4_f32(w["x"], w["qw"], oracle.bf16_scales(w["sw"]), w["bias"], -6.0, 6.0)[0]
    np.testing.assert_array_equal(y16g, y32r)


# ---------------------------------------------------------------------------
# P10: per-block activation quantization (reading R13: 32-wide K blocks, the
# per-row rule applied to each block)
# ---------------------------------------------------------------------------
def test_p10_one_block_per_row_is_the_per_row_rule():
    x = np.random.default_rng(3).standard_normal((4, 256)).astype(np.float32)
    qb, sb, zb = oracle.quantize_blocks_a8(x, 256)
    qr, sr, zr = oracle.quantize_rows_a8(x)
    np.testing.assert_array_equal(qb, qr)
    np.testing.assert_array_equal(sb[:, 0], sr)
    np.testing.assert_array_equal(zb[:, 0], zr)


def test_p10_block_specials_and_reconstruction():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((2, 128)).astype(np.float32) * np.repeat(
        np.float32(10.0) ** rng.integers(-3, 3, (2, 4)), 32, axis=1)
    x[0, 32:64] = 0.0                           # an all-zero block
    x[1, 64:96] = 2.5                           # a constant positive block
    q, s, z = oracle.quantize_blocks_a8(x, 32)
    assert s[0, 1] == 1.0 and z[0, 1] == -128 and (q[0, 32:64] == -128).all()
    # constant 2.5: range [0, 2.5], scale 2.5/255, zp -128, codes 127
    assert s[1, 2] == np.float32(np.float32(2.5) / np.float32(255.0)) and z[1, 2] == -128
    assert (q[1, 64:96] == 127).all()
    # every value is reconstructed within half a step of its own block's scale
    rec = (s.repeat(32, axis=1).astype(np.float64)
           * (q.astype(np.float64) - z.repeat(32, axis=1)))
    assert (np.abs(rec - x) <= 0.5 * s.repeat(32, axis=1) * (1 + 1e-5) + 1e-30).all()


def test_p10_blockwise_linear_equals_rowwise_when_blocks_share_the_range():
    # every block holds the row's min and max: block scales = row scale
    w = workloads.a8w4(2, 24, 128, seed=6)
    x = np.asarray(w["x"][:, :128], np.float32).copy()
    for m in range(2):
        lo, hi = x[m].min(), x[m].max()
        for g in range(4):
            x[m, 32 * g], x[m, 32 * g + 1] = lo, hi
    yb, qb, sb, zb = oracle.qgemm_a8w4_f32_actblock(x, w["qw"], w["sw"], w["bias"], -6.0, 6.0)
    yr, qr, sr, zr = oracle.qgemm_a8w4_f32(x, w["qw"], w["sw"], w["bias"], -6.0, 6.0)
    np.testing.assert_array_equal(sb, np.repeat(sr[:, None], 4, axis=1))
    np.testing.assert_array_equal(qb, qr)
    np.testing.assert_array_equal(yb, yr)


def test_p10_blockwise_brute_force_loops():
    w = workloads.a8w4(1, 3, 64, seed=8)
    x = np.asarray(w["x"][:, :64], np.float32)
    y, q, s, z = oracle.qgemm_a8w4_f32_actblock(x, w["qw"], w["sw"], w["bias"], -1e30, 1e30)
    for n in range(3):
        tot = 0.0
        for g in range(2):
            I = sum((int(q[0, k]) - int(z[0, g])) * int(w["qw"][n, k]) for k in range(32 * g, 32 * g + 32))
            tot += float(w["sw"][n, g]) * float(s[0, g]) * I
        tot += float(w["bias"][n])
        assert y[0, n] == np.float32(tot)


# ---------------------------------------------------------------------------
# P11: asymmetric int4 weights (reading R14: w_real = sw*w + zw per group)
# ---------------------------------------------------------------------------
def _asym_case(M, N, K, seed):
    w = workloads.a8w4(M, N, K, seed=seed)
    zw = (w["sw"] * np.random.default_rng(seed).uniform(-8, 8, w["sw"].shape)).astype(np.float32)
    return w, zw


def test_p11_zero_zeros_reduce_to_the_symmetric_method():
    w, _ = _asym_case(3, 20, 128, 21)
    zw = np.zeros_like(w["sw"])
    ya = oracle.qgemm_a8w4_f32_asym(w["x"], w["qw"], w["sw"], zw, w["bias"], -6.0, 6.0)[0]
    ys = oracle.qgemm_a8w4_f32(w["x"], w["qw"], w["sw"], w["bias"], -6.0, 6.0)[0]
    np.testing.assert_array_equal(ya, ys)


def test_p11_equals_dense_float_product_of_dequantized_operands():
    # a different computation: dequantize both operands, one float64 matmul
    w, zw = _asym_case(4, 30, 256, 22)
    K = 256
    y = oracle.qgemm_a8w4_f32_asym(w["x"][:, :K], w["qw"], w["sw"], zw, w["bias"], -1e30, 1e30)[0]
    qA, sA, za = oracle.quantize_rows_a8(w["x"][:, :K])
    xa = oracle.dequantize_rows(qA, sA, za)                                   # [M][K]
    wr = (np.repeat(w["sw"].astype(np.float64), 32, axis=1) * w["qw"].astype(np.float64)
          + np.repeat(zw.astype(np.float64), 32, axis=1))                     # [N][K]
    ref = xa @ wr.T + w["bias"].astype(np.float64)
    np.testing.assert_allclose(y.astype(np.float64), ref, rtol=1e-6, atol=1e-6)


def test_p11_pack_layout():
    w, zw = _asym_case(1, 6, 64, 23)
    p = oracle.pack_w4_g32_asym(w["qw"], w["sw"], zw)
    assert p.size == oracle.pack_w4_g32_asym_bytes(6, 64) == 6 * 32 + 2 * 6 * 2 * 4
    np.testing.assert_array_equal(p[:6 * 32 + 6 * 2 * 4], oracle.pack_w4_g32(w["qw"], w["sw"]))
    np.testing.assert_array_equal(p[6 * 32 + 6 * 2 * 4:].view(np.float32).reshape(6, 2), zw)


# ---------------------------------------------------------------------------
# P12: symmetric dynamic activation quantization (reading R15: amax/127,
# codes in [-127, 127], zero-point 0)
# ---------------------------------------------------------------------------
def test_p12_symmetric_hand_derived_rows():
    # amax 2: quant scale 63.5, so -1 -> -63.5 (tie, to even -64), 0.5 -> 31.75 -> 32
    # amax 4: quant scale 31.75, so 1 -> 31.75 -> 32, 3 -> 95.25 -> 95
    x = np.array([[2.0, -1.0, 0.5, 0.0], [-4.0, 1.0, 3.0, 0.0], [0.0, 0.0, 0.0, 0.0]],
                 np.float32)
    q, s, z = oracle.quantize_rows_a8_sym(x)
    assert q.tolist() == [[127, -64, 32, 0], [-127, 32, 95, 0], [0, 0, 0, 0]]
    assert s[0] == np.float32(2.0) / np.float32(127.0)
    assert s[1] == np.float32(4.0) / np.float32(127.0)
    assert s[2] == 1.0
    assert z.tolist() == [0, 0, 0]


def test_p12_symmetric_invariants():
    rng = np.random.default_rng(12)
    x = (rng.standard_normal((16, 96)) * rng.uniform(0.01, 50, (16, 1))).astype(np.float32)
    q, s, z = oracle.quantize_rows_a8_sym(x)
    assert (z == 0).all() and q.min() >= -127 and q.max() <= 127
    # the largest magnitude takes the end code, with its sign
    am = np.abs(x).argmax(axis=1)
    assert (q[np.arange(16), am] == np.sign(x[np.arange(16), am]) * 127).all()
    # odd symmetry: negating the row negates the codes and keeps the scale
    qn, sn, _ = oracle.quantize_rows_a8_sym(-x)
    assert (qn == -q).all() and (sn == s).all()
    # a power-of-two scaling of the row scales the scale and keeps the codes
    q2, s2, _ = oracle.quantize_rows_a8_sym(x * np.float32(8.0))
    assert (q2 == q).all() and (s2 == s * np.float32(8.0)).all()
    # reconstruction within half a step (plus the float32 rounding of the scales)
    err = np.abs(x.astype(np.float64) - s.astype(np.float64)[:, None] * q)
    assert (err <= s.astype(np.float64)[:, None] * 0.5001).all()


def test_p12_symmetric_brute_force_nearest_code():
    rng = np.random.default_rng(121)
    x = rng.uniform(-3, 3, (4, 40)).astype(np.float32)
    q, _, _ = oracle.quantize_rows_a8_sym(x)
    for m in range(4):
        amax = max(abs(float(v)) for v in x[m])
        for k in range(40):
            t = float(x[m, k]) * 127.0 / amax
            if abs(abs(t - math.floor(t)) - 0.5) < 1e-4:
                continue  # too close to a tie for a float64 search to decide
            best = min(range(-127, 128), key=lambda c: abs(c - t))
            assert q[m, k] == best


# ---------------------------------------------------------------------------
# P13: convolution with a float input quantized per unrolled row (reading R16)
# ---------------------------------------------------------------------------
def _direct_dyn_conv(x, qw, sw, stride, pad, bias, lo, hi, symmetric):
    """Brute force by output pixel: read the taps inside the image with
    explicit bounds tests, quantize that pixel's values (a pad tap is the
    value 0, which never widens the range), and sum the dequantized products
    in float64 with the weight group taken from the (kh, kw, ci) position."""
    Nb, H, W, Cin = x.shape
    Cout, KH, KW, _ = qw.shape
    sh, sw_ = stride
    ph, pw = pad
    OH = (H + 2 * ph - KH) // sh + 1
    OW = (W + 2 * pw - KW) // sw_ + 1
    quant = oracle.quantize_rows_a8_sym if symmetric else oracle.quantize_rows_a8
    y = np.zeros((Nb, OH, OW, Cout), np.float32)
    for n in range(Nb):
        for oh in range(OH):
            for ow in range(OW):
                taps = []
                for kh in range(KH):
                    for kw in range(KW):
                        ih, iw = oh * sh + kh - ph, ow * sw_ + kw - pw
                        if 0 <= ih < H and 0 <= iw < W:
                            for ci in range(Cin):
                                taps.append((kh, kw, ci, float(x[n, ih, iw, ci])))
                vals = np.array([[t[3] for t in taps] + [0.0]], np.float32)
                q, s, z = quant(vals)
                for co in range(Cout):
                    acc = 0.0
                    for j, (kh, kw, ci, _) in enumerate(taps):
                        g = ((kh * KW + kw) * Cin + ci) // 32
                        acc += (float(s[0]) * (int(q[0, j]) - int(z[0]))
                                * float(sw[co, g]) * int(qw[co, kh, kw, ci]))
                    if bias is not None:
                        acc += float(bias[co])
                    y[n, oh, ow, co] = min(max(np.float32(acc), np.float32(lo)), np.float32(hi))
    return y


def _conv_case(Nb, H, W, Cin, Cout, KH, KW, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((Nb, H, W, Cin)).astype(np.float32)
    qw = rng.integers(-8, 8, size=(Cout, KH, KW, Cin)).astype(np.int8)
    sw = rng.uniform(0.01, 0.1, (Cout, KH * KW * Cin // 32)).astype(np.float32)
    bias = rng.standard_normal(Cout).astype(np.float32)
    return x, qw, sw, bias


@pytest.mark.parametrize("symmetric", [False, True])
@pytest.mark.parametrize("H,W,Cin,KH,KW,stride,pad", [
    (5, 6, 32, 3, 3, (1, 1), (1, 1)),
    (7, 5, 32, 3, 2, (2, 1), (1, 0)),
    (4, 4, 64, 1, 1, (2, 2), (0, 0)),
])
def test_p13_dynamic_conv_equals_direct_brute_force(symmetric, H, W, Cin, KH, KW, stride, pad):
    x, qw, sw, bias = _conv_case(2, H, W, Cin, 3, KH, KW, seed=H * 10 + KH)
    y, _, _, _ = oracle.qconv2d_f32_dyn_a8w4(x, qw, sw, stride, pad, bias, -50.0, 50.0,
                                             symmetric=symmetric)
    y_bf = _direct_dyn_conv(x, qw, sw, stride, pad, bias, -50.0, 50.0, symmetric)
    np.testing.assert_allclose(y, y_bf, rtol=1e-6, atol=1e-6)


def test_p13_pointwise_conv_is_the_linear():
    # a 1x1 conv with unit stride and no pad is the A8W4 linear on [Nb*H*W, Cin]
    x, qw, sw, bias = _conv_case(2, 3, 4, 64, 5, 1, 1, seed=131)
    y, qA, sA, za = oracle.qconv2d_f32_dyn_a8w4(x, qw, sw, (1, 1), (0, 0), bias, -6.0, 6.0)
    y2, qA2, sA2, za2 = oracle.qgemm_a8w4_f32(x.reshape(24, 64), qw.reshape(5, 64), sw, bias,
                                              -6.0, 6.0)
    assert (y.reshape(24, 5) == y2).all()
    assert (qA == qA2).all() and (sA == sA2).all() and (za == za2).all()


def test_p13_whole_image_kernel_is_the_linear_on_the_flattened_image():
    # a kernel the size of the image gives one output pixel: the linear on
    # the image flattened in (h, w, c) order, which fixes the K order
    x, qw, sw, bias = _conv_case(3, 2, 3, 32, 4, 2, 3, seed=132)
    y, _, _, _ = oracle.qconv2d_f32_dyn_a8w4(x, qw, sw, (1, 1), (0, 0), bias, -60.0, 60.0)
    y2, _, _, _ = oracle.qgemm_a8w4_f32(x.reshape(3, 2 * 3 * 32), qw.reshape(4, 2 * 3 * 32), sw,
                                        bias, -60.0, 60.0)
    assert y.shape == (3, 1, 1, 4) and (y.reshape(3, 4) == y2).all()


def test_p13_padding_does_not_move_the_quantization_of_a_row():
    # zero taps never widen the range (0 is always inside it), so an unrolled
    # row with pad taps has the parameters of its in-image values alone
    x, _, _, _ = _conv_case(1, 3, 3, 32, 1, 3, 3, seed=133)
    cols = oracle.im2col_f32(x, 3, 3, (1, 1), (1, 1))
    corner = cols[0]                                   # output pixel (0, 0): 5 pad taps
    inside = corner.reshape(3, 3, 32)[1:, 1:].reshape(1, -1)
    for quant in (oracle.quantize_rows_a8, oracle.quantize_rows_a8_sym):
        _, s1, z1 = quant(corner[None, :])
        _, s2, z2 = quant(inside)
        assert s1[0] == s2[0] and z1[0] == z2[0]
    assert (corner.reshape(3, 3, 32)[0] == 0).all() and (corner.reshape(3, 3, 32)[:, 0] == 0).all()


def test_p13_codes_entry_matches_the_linear():
    x, qw, sw, bias = _conv_case(1, 4, 8, 32, 6, 1, 1, seed=134)
    x2 = x.reshape(32, 32)
    qA, sA, za = oracle.quantize_rows_a8(x2)
    y = oracle.a8w4_from_codes(qA, sA, za, qw.reshape(6, 32), sw, bias, -6.0, 6.0)
    y2, _, _, _ = oracle.qgemm_a8w4_f32(x2, qw.reshape(6, 32), sw, bias, -6.0, 6.0)
    assert (y == y2).all()
