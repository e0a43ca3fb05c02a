"""GPU parity of the A8W4 path against the CPU oracle, through the C ABI.

Quantized activations (q, scale, zero-point) and packed weights must match
bit-exactly.  f32 outputs must satisfy |y - y_ref| <= 1e-4 * max(|y_ref|, 1)
against the float64 oracle: relative 1e-4 where |y| >= 1, absolute 1e-4
below, because the float32 rounding of a sum of group terms is set by the
size of the terms, not of y (tests/a8w4_tol.py; the observed errors are
printed at the end of the run)."""
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
# dynamic quantization
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("M,K,pad", [(1, 4096, 0), (128, 4096, 0), (3, 33, 5), (5, 1, 0),
                                     (2, 1000, 3), (7, 12345, 1)])
def test_quantize_rows_bit_exact(lib, M, K, pad):
    rng = np.random.default_rng(M * 1000 + K)
    x = (rng.standard_normal((M, K + pad)) * rng.uniform(0.1, 10, (M, 1))).astype(np.float32)
    if M >= 3:
        x[1] = 0.0                       # all-zero row
        x[2] = 3.25                      # constant positive row
    q_ref, s_ref, z_ref = oracle.quantize_rows_a8(x[:, :K])
    xd = _dev(x)
    q = torch.full((M, K + 2), 99, dtype=torch.int8, device="cuda")
    s = torch.empty(M, dtype=torch.float32, device="cuda")
    z = torch.empty(M, dtype=torch.int32, device="cuda")
    lib.quantize_rows_a8(xd[:, :K], q[:, :K], s, z)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(q[:, :K].cpu().numpy(), q_ref)
    assert (q[:, K:].cpu().numpy() == 99).all()          # ldq padding untouched
    np.testing.assert_array_equal(s.cpu().numpy().view(np.int32), s_ref.view(np.int32))
    np.testing.assert_array_equal(z.cpu().numpy(), z_ref)


def test_quantize_rows_golden_specials(lib):
    import json, os
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                    "qg_dynamic_quant_specials.json")))
    for case in g["cases"]:
        x = np.array([case["x"]], np.float32)
        xd = _dev(x)
        q = torch.empty(x.shape, dtype=torch.int8, device="cuda")
        s = torch.empty(1, dtype=torch.float32, device="cuda")
        z = torch.empty(1, dtype=torch.int32, device="cuda")
        lib.quantize_rows_a8(xd, q, s, z)
        torch.cuda.synchronize()
        assert s.item() == case["scale"] and z.item() == case["zp"]
        assert q.cpu().numpy()[0].tolist() == case["q"]


# ---------------------------------------------------------------------------
# W4 pack
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("N,K,ldw", [(7, 96, 100), (300, 1024, 1024), (14336, 4096, 4096)])
def test_pack_w4_bit_exact(lib, N, K, ldw):
    w = workloads.a8w4(1, N, K, seed=N + K)
    qw = np.zeros((N, ldw), np.int8)
    qw[:, :K] = w["qw"]
    packed = lib.pack_w4_g32(_dev(qw)[:, :K], _dev(w["sw"]))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(packed.cpu().numpy(), oracle.pack_w4_g32(w["qw"], w["sw"]))


def test_pack_w4_out_of_range_recorded(lib):
    qw = np.zeros((2, 32), np.int8)
    qw[1, 5] = 9                                       # not an int4 value
    lib.pack_w4_g32(_dev(qw), _dev(np.ones((2, 1), np.float32)))
    assert lib.qg_device_status(True) == -1


# ---------------------------------------------------------------------------
# A8W4 linear
# ---------------------------------------------------------------------------
def _run_a8w4(lib, w, ldy_pad=0, with_outputs=True, bf16=False):
    M, N, K = w["M"], w["N"], w["K"]
    packed = lib.pack_w4_g32(_dev(w["qw"]), _dev(w["sw"]), bf16_scales=bf16)
    x = _dev(w["x"])[:, :K]
    y = torch.full((M, N + ldy_pad), 7.0, dtype=torch.float32, device="cuda")
    q = torch.empty((M, K), dtype=torch.int8, device="cuda") if with_outputs else None
    s = torch.empty(M, dtype=torch.float32, device="cuda") if with_outputs else None
    z = torch.empty(M, dtype=torch.int32, device="cuda") if with_outputs else None
    bias = None if w["bias"] is None else _dev(w["bias"])
    lib.qgemm_a8w4_f32(x, packed, N, bias, w["clamp_min"], w["clamp_max"], y[:, :N], q, s, z,
                       bf16_scales=bf16)
    torch.cuda.synchronize()
    y_np = y.cpu().numpy()
    if ldy_pad:
        assert (y_np[:, N:] == 7.0).all()
    out = (y_np[:, :N],)
    if with_outputs:
        out += (q.cpu().numpy(), s.cpu().numpy(), z.cpu().numpy())
    return out


def _check_a8w4(lib, w, bf16=False, **kw):
    y, q, s, z = _run_a8w4(lib, w, bf16=bf16, **kw)
    ref = oracle.qgemm_a8w4_f32_bf16s if bf16 else oracle.qgemm_a8w4_f32
    y_ref, q_ref, s_ref, z_ref = ref(w["x"][:, :w["K"]], w["qw"], w["sw"], w["bias"],
                                     w["clamp_min"], w["clamp_max"])
    np.testing.assert_array_equal(q, q_ref)
    np.testing.assert_array_equal(s.view(np.int32), s_ref.view(np.int32))
    np.testing.assert_array_equal(z, z_ref)
    M, N, K = w["M"], w["N"], w["K"]
    kind = "gemv" if M == 1 else ("tc" if K % 64 == 0 and K <= 8192 else "simt")
    assert_a8w4_close(y, y_ref, f"a8w4{'_bf16s' if bf16 else ''} {kind} {M}x{N}x{K}")
    return y, y_ref


def test_gemv_full_size_1x14336x4096(lib):
    w = workloads.a8w4_gemv_1x14336x4096()
    y, y_ref = _check_a8w4(lib, w)
    # the clamp binds on a large share of outputs at this scale; both sides agree where it does
    assert ((np.abs(y_ref) == 6.0) == (np.abs(y) == 6.0)).mean() > 0.999


@pytest.mark.parametrize("N,K,bias,clamp", [
    (1, 32, True, (-np.inf, np.inf)), (7, 96, False, (-np.inf, np.inf)),
    (300, 1024, True, (-2.0, 2.0)), (1000, 2080, True, (-np.inf, np.inf)),
    (33, 8192, True, (-np.inf, np.inf)), (17, 12288, False, (-np.inf, np.inf)),
    (5000, 4096, True, (-6.0, 6.0))])
def test_gemv_shapes(lib, N, K, bias, clamp):
    w = workloads.a8w4(1, N, K, seed=N * 7 + K, clamp=clamp, with_bias=bias, ldx=K + 3)
    _check_a8w4(lib, w, ldy_pad=2)


# (64, 256, 320) and (40, 128, 448) take 5 and 7 split-K ranks, whose last
# rank owns fewer rows of the tile (24 of 26, 14 of 19) in the reduction.
@pytest.mark.parametrize("M,N,K", [(2, 64, 64), (9, 300, 1024), (17, 1000, 4096), (128, 256, 4096),
                                   (129, 520, 384), (200, 132, 128), (3, 4096, 8192),
                                   (256, 8, 2048), (5, 96, 96), (64, 256, 320), (40, 128, 448)])
def test_a8w4_gemm_shapes(lib, M, N, K):
    w = workloads.a8w4(M, N, K, seed=M * 31 + N + K, clamp=(-np.inf, np.inf), ldx=K + 1)
    _check_a8w4(lib, w, ldy_pad=1)


# Degenerate activation rows through every A8W4 path (the GEMV for M = 1,
# the quantization tiles + tensor-core kernel for M > 1 with K % 64 == 0,
# the CUDA-core kernel otherwise): an all-zero row (scale 1, zero-point
# -128), constant positive and negative rows (the range includes 0), a
# single spike among zeros, values near the f32 subnormal range, and a row
# whose extremes are the clamp bounds of the codes.
def _degenerate_rows(M, K, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K), dtype=np.float32)
    specials = [np.zeros(K, np.float32), np.full(K, 3.25, np.float32),
                np.full(K, -0.75, np.float32), np.zeros(K, np.float32),
                rng.standard_normal(K).astype(np.float32) * np.float32(1e-30),
                np.linspace(-1e4, 1e4, K).astype(np.float32)]
    specials[3][K // 3] = 1e3
    for i, row in enumerate(specials[:M]):
        x[i] = row
    return x


@pytest.mark.parametrize("M,N,K", [(1, 300, 1024), (6, 200, 1024), (6, 200, 96), (130, 64, 512)])
def test_a8w4_degenerate_rows(lib, M, N, K):
    w = workloads.a8w4(M, N, K, seed=900 + M + K, clamp=(-np.inf, np.inf))
    w["x"] = _degenerate_rows(M, K, 901 + M)
    _check_a8w4(lib, w)


def test_a8w4_gemm_full_size_128x4096x4096(lib):
    _check_a8w4(lib, workloads.a8w4_gemm_128x4096x4096())


def test_gemv_without_optional_outputs_matches(lib):
    w = workloads.a8w4(1, 640, 4096, seed=3)
    (y,) = _run_a8w4(lib, w, with_outputs=False)
    y2, *_ = _run_a8w4(lib, w)
    np.testing.assert_array_equal(y, y2)


def test_gemv_chain_on_one_stream(lib):
    """Back-to-back M = 1 calls on one stream, each reading the previous call's
    y as its x.  A call may start while the previous one finishes (it fetches
    its weights early); it must still quantize the finished y."""
    K = 4096
    ws = [workloads.a8w4(1, K, K, seed=40 + i) for i in range(3)]
    packed = [lib.pack_w4_g32(_dev(w["qw"]), _dev(w["sw"])) for w in ws]
    ys = [torch.empty((1, K), dtype=torch.float32, device="cuda") for _ in ws]
    cur = _dev(ws[0]["x"])[:, :K]
    for w, p, y in zip(ws, packed, ys):
        lib.qgemm_a8w4_f32(cur, p, K, _dev(w["bias"]), w["clamp_min"], w["clamp_max"], y)
        cur = y
    torch.cuda.synchronize()
    xin = ws[0]["x"][:, :K]
    for w, y in zip(ws, ys):
        y_ref = oracle.qgemm_a8w4_f32(xin, w["qw"], w["sw"], w["bias"], w["clamp_min"],
                                      w["clamp_max"])[0]
        y_np = y.cpu().numpy()
        assert_a8w4_close(y_np, y_ref, "a8w4 gemv chain")
        xin = y_np


# ---------------------------------------------------------------------------
# A8W4 with bf16 group scales (pack_w4_g32_bf16 / qgemm_a8w4_f32_bf16s)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("N,K", [(7, 96), (300, 1024), (14336, 4096)])
def test_pack_w4_bf16_bit_exact(lib, N, K):
    w = workloads.a8w4(1, N, K, seed=N + K + 1)
    packed = lib.pack_w4_g32_bf16(_dev(w["qw"]), _dev(w["sw"]))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(packed.cpu().numpy(), oracle.pack_w4_g32_bf16(w["qw"], w["sw"]))


def test_gemv_bf16_scales_full_size_1x14336x4096(lib):
    _check_a8w4(lib, workloads.a8w4_gemv_1x14336x4096(), bf16=True)


@pytest.mark.parametrize("M,N,K", [
    (1, 300, 1024),      # streaming GEMV, one group per lane
    (1, 300, 1536),      # streaming GEMV, 2 groups per lane (48 of 64 slots live), split rows
    (1, 5000, 2048),     # streaming GEMV, 2 groups per lane, whole and split rows
    (1, 777, 3072),      # streaming GEMV, 4 groups per lane (96 of 128 slots live)
    (1, 1111, 8192),     # streaming GEMV, 8 groups per lane
    (1, 1000, 2080),     # plain GEMV (K % 128 != 0)
    (1, 17, 12288),      # plain GEMV (K > 8192)
    (9, 300, 1024),      # tensor cores
    (129, 520, 384),     # tensor cores, ragged M
    (5, 96, 96),         # CUDA cores (K % 128 != 0)
])
def test_a8w4_bf16_scales_shapes(lib, M, N, K):
    w = workloads.a8w4(M, N, K, seed=M * 13 + N + K, clamp=(-np.inf, np.inf), ldx=K + 1)
    _check_a8w4(lib, w, bf16=True, ldy_pad=1)


def test_a8w4_bf16_scales_full_size_128x4096x4096(lib):
    _check_a8w4(lib, workloads.a8w4_gemm_128x4096x4096(), bf16=True)


# ---------------------------------------------------------------------------
# A8W4 GEMV with the activations quantized per 32-wide K block
# ---------------------------------------------------------------------------
def _check_actblock(lib, w):
    M, N, K = w["M"], w["N"], w["K"]
    packed = lib.pack_w4_g32(_dev(w["qw"]), _dev(w["sw"]))
    x = _dev(w["x"])[:, :K]
    y = torch.full((M, N + 1), 7.0, dtype=torch.float32, device="cuda")
    q = torch.empty((M, K), dtype=torch.int8, device="cuda")
    s = torch.empty((M, K // 32), dtype=torch.float32, device="cuda")
    z = torch.empty((M, K // 32), dtype=torch.int32, device="cuda")
    bias = None if w["bias"] is None else _dev(w["bias"])
    lib.qgemm_a8w4_f32_actblock(x, packed, N, bias, w["clamp_min"], w["clamp_max"], y[:, :N],
                                q, s, z)
    torch.cuda.synchronize()
    y_ref, q_ref, s_ref, z_ref = oracle.qgemm_a8w4_f32_actblock(
        w["x"][:, :K], w["qw"], w["sw"], w["bias"], w["clamp_min"], w["clamp_max"])
    np.testing.assert_array_equal(q.cpu().numpy(), q_ref)
    np.testing.assert_array_equal(s.cpu().numpy().view(np.int32), s_ref.view(np.int32))
    np.testing.assert_array_equal(z.cpu().numpy(), z_ref)
    y_np = y.cpu().numpy()
    assert (y_np[:, N:] == 7.0).all()
    assert_a8w4_close(y_np[:, :N], y_ref, f"actblock {'gemv' if M == 1 else 'tc'} {M}x{N}x{K}")


def test_gemv_actblock_full_size_1x14336x4096(lib):
    _check_actblock(lib, workloads.a8w4_gemv_1x14336x4096())


@pytest.mark.parametrize("N,K", [(1, 128), (300, 1024), (1000, 2048), (33, 8192), (5000, 4096)])
def test_gemv_actblock_shapes(lib, N, K):
    w = workloads.a8w4(1, N, K, seed=N * 3 + K, clamp=(-np.inf, np.inf), ldx=K + 3)
    # blocks of very different magnitudes and a zero block
    scale = np.float32(10.0) ** np.random.default_rng(N).integers(-3, 3, K // 32)
    w["x"][:, :K] *= np.repeat(scale, 32)[None, :]
    w["x"][:, 32:64] = 0.0
    _check_actblock(lib, w)


def test_a8w4_actblock_full_size_128x4096x4096(lib):
    _check_actblock(lib, workloads.a8w4_gemm_128x4096x4096())


@pytest.mark.parametrize("M,N,K", [(2, 64, 64), (9, 300, 1024), (17, 1000, 4096),
                                   (129, 520, 384), (200, 132, 128), (3, 4096, 8192),
                                   (40, 128, 448)])
def test_a8w4_actblock_gemm_shapes(lib, M, N, K):
    w = workloads.a8w4(M, N, K, seed=M * 17 + N + K, clamp=(-np.inf, np.inf), ldx=K + 1)
    # blocks of magnitudes 10^-2 .. 10^0 (a 1000x spread); with a 10^5 spread
    # the float32 group sum of y near 0 cancels terms of size 10^3 and its
    # absolute error reaches ~1e-4 on any float32 path
    scale = np.float32(10.0) ** np.random.default_rng(M + N).integers(-2, 1, (M, K // 32))
    w["x"][:, :K] *= np.repeat(scale, 32, axis=1)
    w["x"][0, 32:64] = 0.0                                 # a zero block
    _check_actblock(lib, w)


def test_gemv_actblock_rejects_what_it_does_not_cover(lib):
    y = torch.empty((2, 64), dtype=torch.float32, device="cuda")
    w = workloads.a8w4(2, 64, 96, seed=1)
    packed = lib.pack_w4_g32(_dev(w["qw"]), _dev(w["sw"]))
    with pytest.raises(lib.QGError):                       # M > 1 with K % 64 != 0
        lib.qgemm_a8w4_f32_actblock(_dev(w["x"])[:, :96], packed, 64, None, -1.0, 1.0, y)
    w = workloads.a8w4(1, 64, 96, seed=2)
    packed = lib.pack_w4_g32(_dev(w["qw"]), _dev(w["sw"]))
    with pytest.raises(lib.QGError):                       # M == 1 with K % 128 != 0
        lib.qgemm_a8w4_f32_actblock(_dev(w["x"])[:, :96], packed, 64, None, -1.0, 1.0, y[:1])


# ---------------------------------------------------------------------------
# A8W4 GEMV with asymmetric int4 weights (f32 zero per group)
# ---------------------------------------------------------------------------
def _asym_zeros(w, seed):
    rng = np.random.default_rng(seed)
    return (w["sw"] * rng.uniform(-8, 8, w["sw"].shape)).astype(np.float32)


def _check_asym(lib, w, zw):
    M, N, K = w["M"], w["N"], w["K"]
    packed = lib.pack_w4_g32_asym(_dev(w["qw"]), _dev(w["sw"]), _dev(zw))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(packed.cpu().numpy(),
                                  oracle.pack_w4_g32_asym(w["qw"], w["sw"], zw))
    x = _dev(w["x"])[:, :K]
    y = torch.full((M, N + 1), 7.0, dtype=torch.float32, device="cuda")
    q = torch.empty((M, K), dtype=torch.int8, device="cuda")
    s = torch.empty(M, dtype=torch.float32, device="cuda")
    z = torch.empty(M, dtype=torch.int32, device="cuda")
    bias = None if w["bias"] is None else _dev(w["bias"])
    lib.qgemm_a8w4_f32_asym(x, packed, N, bias, w["clamp_min"], w["clamp_max"], y[:, :N], q, s, z)
    torch.cuda.synchronize()
    y_ref, q_ref, s_ref, z_ref = oracle.qgemm_a8w4_f32_asym(
        w["x"][:, :K], w["qw"], w["sw"], zw, w["bias"], w["clamp_min"], w["clamp_max"])
    np.testing.assert_array_equal(q.cpu().numpy(), q_ref)
    np.testing.assert_array_equal(s.cpu().numpy().view(np.int32), s_ref.view(np.int32))
    np.testing.assert_array_equal(z.cpu().numpy(), z_ref)
    y_np = y.cpu().numpy()
    assert (y_np[:, N:] == 7.0).all()
    assert_a8w4_close(y_np[:, :N], y_ref, f"asym {'gemv' if M == 1 else 'tc'} {M}x{N}x{K}")


def test_gemv_asym_full_size_1x14336x4096(lib):
    w = workloads.a8w4_gemv_1x14336x4096()
    _check_asym(lib, w, _asym_zeros(w, 31))


@pytest.mark.parametrize("N,K", [(1, 128), (300, 1024), (1000, 2048), (33, 8192), (5000, 4096)])
def test_gemv_asym_shapes(lib, N, K):
    w = workloads.a8w4(1, N, K, seed=N * 5 + K, clamp=(-np.inf, np.inf), ldx=K + 3)
    _check_asym(lib, w, _asym_zeros(w, N + K))


def test_a8w4_asym_full_size_128x4096x4096(lib):
    w = workloads.a8w4_gemm_128x4096x4096()
    _check_asym(lib, w, _asym_zeros(w, 33))


@pytest.mark.parametrize("M,N,K", [(2, 64, 64), (9, 300, 1024), (17, 1000, 4096),
                                   (129, 520, 384), (200, 132, 128), (3, 4096, 8192),
                                   (40, 128, 448)])
def test_a8w4_asym_gemm_shapes(lib, M, N, K):
    w = workloads.a8w4(M, N, K, seed=M * 19 + N + K, clamp=(-np.inf, np.inf), ldx=K + 1)
    _check_asym(lib, w, _asym_zeros(w, M + N + K))


def test_gemv_asym_with_zero_zeros_matches_symmetric_entry(lib):
    w = workloads.a8w4(1, 640, 4096, seed=32)
    N, K = 640, 4096
    zw = np.zeros_like(w["sw"])
    pa = lib.pack_w4_g32_asym(_dev(w["qw"]), _dev(w["sw"]), _dev(zw))
    ps = lib.pack_w4_g32(_dev(w["qw"]), _dev(w["sw"]))
    x = _dev(w["x"])[:, :K]
    ya = torch.empty((1, N), dtype=torch.float32, device="cuda")
    ys = torch.empty((1, N), dtype=torch.float32, device="cuda")
    lib.qgemm_a8w4_f32_asym(x, pa, N, _dev(w["bias"]), -6.0, 6.0, ya)
    lib.qgemm_a8w4_f32(x, ps, N, _dev(w["bias"]), -6.0, 6.0, ys)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(ya.cpu().numpy(), ys.cpu().numpy())
