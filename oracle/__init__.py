"""CPU oracle for quantized integer matrix multiplication.

TEST INFRASTRUCTURE ONLY.  This package is the plain, slow, obviously
correct reference that the CUDA library is checked against.  Only the test
suite, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may
import it; the library itself never calls it, and it shares no code with the
CUDA path (``gemv_zero_point_b200``).

Every result is computed from its definition, in int64 for integer work and
in float64 where the definition has real arithmetic.  Where a step decides
an integer from floating point (dynamic activation quantization) it is done
in float32, the precision the GPU kernel uses, with one IEEE rounding per
operation and no fused multiply-add.

Sources (web pages), cited by title and section:
  [QG]   xidianedu, "量化 GEMM：数值契约、SRAM、DMA 与结果验证" (quantized GEMM:
         numeric contract, SRAM, DMA and result verification), sections
         1 (固定量化语义, fixed quantization semantics), 2 (Padding 必须代表实数零,
         padding must mean real zero), 3 (切块与容量预算, tiling and capacity
         budget), 4 (跨 K 保留累加器, keep the accumulator across K),
         6 (四级验证, four-level verification).
  [MNN]  MNN source/backend/cpu/compute/ConvInt8TiledExecutor.cpp:
         initializeConvInt8QuantInfo, _computeReorderQuantInfo,
         BatchAsyDynamicQuant, BatchSymDynamicQuant, the low-memory
         float im2col path, tileSplitFunction (QuanPostTreatParameters).
  [KAI]  pytorch/ao PR #997 "Kleidi 4b blockwise gemv prototype".

Where the pages are silent the oracle takes the plainest reading and names
it R1..R16 at the function that uses it, stating the reading in that
function's docstring or the comment above it: R1 requant rounding (one
round-half-even on the exact 64-bit product), R2 bias in accumulator scale
added once after all of K, R5 min/max dynamic quantization in float32 with
one rounding per operation, R6 the packed int4 layout, R8 clamp after bias,
R12 bf16 scales rounded to nearest even, R13 one activation block per 32-wide
weight group, R14 an f32 zero per weight group, R15 absolute-maximum
symmetric quantization, R16 the unrolled float input of the dynamic conv.

Parity pins: every function below is pinned by tests in
``tests/test_oracle_pins.py`` against the pages' printed numbers, closed
forms or brute force, except ``pack_w4_g32`` whose byte layout is this
library's own format (R6): it is pinned by a round trip and a hand-derived
byte pattern, not by the pages.
"""
from __future__ import annotations

import math

import numpy as np

INT8_MIN, INT8_MAX = -128, 127
INT32_MIN, INT32_MAX = -(2 ** 31), 2 ** 31 - 1
GROUP = 32  # A8W4: one weight scale per 32 consecutive K ([KAI], qsi4c32)


# ---------------------------------------------------------------------------
# Overflow bound  ([QG] section 4)
# ---------------------------------------------------------------------------
def worst_zp_corrected_magnitude() -> int:
    """Largest |q - zero_point| for int8 q and int8 zero-point: 127-(-128)."""
    return INT8_MAX - INT8_MIN


def overflow_bound(K: int, max_abs_bias: int) -> int:
    """Conservative INT32 bound of [QG] section 4: K * 255^2 + |bias|."""
    p = worst_zp_corrected_magnitude() ** 2
    return int(K) * p + int(max_abs_bias)


def fits_int32(K: int, max_abs_bias: int) -> bool:
    return overflow_bound(K, max_abs_bias) <= INT32_MAX


# ---------------------------------------------------------------------------
# Fixed-point requantization  (R1; [QG] section 1 names an integer
# multiplier/shift approximation of the scale ratio and ONNX QuantizeLinear
# rounding, which is round-half-to-even)
# ---------------------------------------------------------------------------
def requant_params(ratio: float):
    """ratio = sA*sB/sO as (M0, shift) with ratio ~= M0 * 2^-(31+shift).

    frexp(ratio) = f * 2^e with f in [0.5, 1); M0 = round(f * 2^31) with
    ties away from zero (f*2^31 is exact in double); if M0 reaches 2^31 it is
    halved and e raised by one; shift = -e.  Supported: 0 < ratio < 1 and
    0 <= shift <= 31, else ValueError.
    """
    ratio = float(ratio)
    if not (ratio > 0.0 and ratio < 1.0 and math.isfinite(ratio)):
        raise ValueError("requant ratio must lie in (0, 1)")
    f, e = math.frexp(ratio)
    m0 = math.floor(f * 2.0 ** 31 + 0.5)
    if m0 == 2 ** 31:
        m0 //= 2
        e += 1
    shift = -e
    if not (0 <= shift <= 31):
        raise ValueError("requant shift out of [0, 31]")
    return int(m0), int(shift)


def round_half_even_shift(p, s):
    """round_half_even(p / 2^s) for int64 p and s >= 1 (elementwise)."""
    p = np.asarray(p, dtype=np.int64)
    s = np.asarray(s, dtype=np.int64)
    q = p >> s                      # floor division by 2^s
    r = p - (q << s)                # remainder in [0, 2^s)
    half = np.int64(1) << (s - 1)
    up = (r > half) | ((r == half) & ((q & 1) == 1))
    return q + up.astype(np.int64)


def rq_round(acc, m0, shift):
    """rne(acc * M0 / 2^(31+shift)) as int64  (R1).

    The product acc*M0 is exact in int64 (|acc| < 2^31, M0 < 2^31), so the
    result is rounded once.  ``m0``/``shift`` broadcast along the last axis
    (per output column) or are scalars.
    """
    acc = np.asarray(acc, dtype=np.int64)
    m0 = np.asarray(m0, dtype=np.int64)
    shift = np.asarray(shift, dtype=np.int64)
    return round_half_even_shift(acc * m0, 31 + shift)


def requantize(acc, m0, shift, out_zp, clamp_min, clamp_max):
    """y = clamp(out_zp + rq_round(acc, M0, shift), lo, hi) as int8, with
    int8 clamp bounds ([MNN] QuanPostTreatParameters maxValue/minValue)."""
    assert INT8_MIN <= int(clamp_min) <= int(clamp_max) <= INT8_MAX
    q = rq_round(acc, m0, shift)
    y = np.clip(q + int(out_zp), int(clamp_min), int(clamp_max))
    return y.astype(np.int8)


# ---------------------------------------------------------------------------
# O1: affine INT8 GEMM  ([QG] sections 1, 2, 4; [MNN] QuanPostTreatParameters)
# ---------------------------------------------------------------------------
def int8_gemm_acc(A, B, za, zb, bias=None):
    """acc[m,n] = sum_k (A[m,k]-za)(B[k,n]-zb) + bias[n], exact (int64).

    Direct form of the affine contract real = scale*(q - zero_point): the
    zero-points are subtracted before the product, then the int32 bias in
    accumulator scale is added once after all of K (R2).
    """
    A = np.asarray(A, dtype=np.int64) - int(za)
    B = np.asarray(B, dtype=np.int64) - int(zb)
    acc = A @ B
    if bias is not None:
        acc = acc + np.asarray(bias, dtype=np.int64)[None, :]
    return acc


F64_EXACT_LIMIT = 2 ** 53  # every integer of magnitude <= 2^53 is a float64


def int8_gemm_acc_f64(A, B, za, zb, bias=None, row_block=1024):
    """The accumulator of int8_gemm_acc computed with a float64 matrix
    product, for sizes where the int64 product is too slow to check every
    output.

    Each factor (A[m,k]-za)(B[k,n]-zb) is an integer of magnitude at most
    255*255 = 65025 ([QG] section 4), so every partial sum of any summation
    order has magnitude at most K*65025.  While K*65025 <= 2^53 each partial
    sum is an integer that float64 represents, every addition is exact, and
    the product equals the int64 definition whatever blocking the BLAS
    routine uses.  Larger K is refused.  Returns int64 [M, N], bias added in
    int64 after the product (R2).
    """
    A = np.asarray(A)
    B = np.asarray(B)
    K = A.shape[1]
    if K * worst_zp_corrected_magnitude() ** 2 > F64_EXACT_LIMIT:
        raise ValueError("K too large for an exact float64 accumulation")
    Bf = B.astype(np.float64) - float(zb)
    blocks = [np.zeros((0, B.shape[1]), np.int64)]
    for r0 in range(0, A.shape[0], row_block):
        Af = A[r0:r0 + row_block].astype(np.float64) - float(za)
        blocks.append((Af @ Bf).astype(np.int64))
    out = np.concatenate(blocks)
    if bias is not None:
        out += np.asarray(bias, dtype=np.int64)[None, :]
    return out


def qgemm_s8s8_requant(A, B, za, zb, bias, m0, shift, out_zp, clamp_min,
                       clamp_max, max_abs_bias=None):
    """C = requantize(int8_gemm_acc(...)) -> (C int8 [M,N], acc int32 [M,N]).

    Raises OverflowError when the bound of [QG] section 4 does not hold for
    this K and bias (the library must reject such calls), and AssertionError
    if an accumulator ever leaves that bound.
    """
    K = np.asarray(A).shape[1]
    if max_abs_bias is None:
        max_abs_bias = 0 if bias is None else int(np.abs(np.asarray(bias, np.int64)).max(initial=0))
    if not fits_int32(K, max_abs_bias):
        raise OverflowError("K*65025 + |bias| exceeds INT32_MAX")
    acc = int8_gemm_acc(A, B, za, zb, bias)
    assert np.abs(acc).max(initial=0) <= overflow_bound(K, max_abs_bias)
    C = requantize(acc, m0, shift, out_zp, clamp_min, clamp_max)
    return C, acc.astype(np.int32)


# ---------------------------------------------------------------------------
# Tiled model  ([QG] section 3 tile count / MAC slots, section 2 zero-point
# padding, section 4 accumulator kept across K blocks; level 3 of the
# four-level verification in section 6)
# ---------------------------------------------------------------------------
def tiled_int8_gemm(A, B, za, zb, bias=None, Tm=64, Tn=64, Tk=128):
    """Full-size tiles over zero-point-padded operands.

    A is padded to (ceil(M/Tm)*Tm, ceil(K/Tk)*Tk) with za and B to
    (ceil(K/Tk)*Tk, ceil(N/Tn)*Tn) with zb, so padded products are
    (za-za)(zb-zb) = 0.  Each output tile's INT32 accumulator is zeroed at its
    first K block, accumulated over the rest, and the bias is added only after
    the last one.  Returns (acc int64 [M,N], stats) where stats counts tiles,
    useful MACs, physical MAC slots and their ratio.
    """
    A = np.asarray(A, dtype=np.int64)
    B = np.asarray(B, dtype=np.int64)
    M, K = A.shape
    N = B.shape[1]
    mt, nt, kt = -(-M // Tm), -(-N // Tn), -(-K // Tk)
    Ap = np.full((mt * Tm, kt * Tk), int(za), dtype=np.int64)
    Ap[:M, :K] = A
    Bp = np.full((kt * Tk, nt * Tn), int(zb), dtype=np.int64)
    Bp[:K, :N] = B
    out = np.zeros((mt * Tm, nt * Tn), dtype=np.int64)
    tiles = 0
    for i in range(mt):
        for j in range(nt):
            accum = np.zeros((Tm, Tn), dtype=np.int64)   # zeroed at first K block
            for b in range(kt):
                a_t = Ap[i * Tm:(i + 1) * Tm, b * Tk:(b + 1) * Tk] - int(za)
                b_t = Bp[b * Tk:(b + 1) * Tk, j * Tn:(j + 1) * Tn] - int(zb)
                accum += a_t @ b_t
                tiles += 1
            out[i * Tm:(i + 1) * Tm, j * Tn:(j + 1) * Tn] = accum
    acc = out[:M, :N]
    if bias is not None:
        acc = acc + np.asarray(bias, dtype=np.int64)[None, :]
    slots = tiles * Tm * Tn * Tk
    useful = M * N * K
    stats = dict(tiles=tiles, tiles_mnk=(mt, nt, kt), useful_macs=useful,
                 slots=slots, shape_efficiency=useful / slots)
    return acc, stats


def tile_budget_bytes(Tm=64, Tn=64, Tk=128, reserve=16384):
    """[QG] section 3 buffer budget: double-buffered int8 A/B tiles, one int32
    accumulator tile, plus a reserve for output, scales and descriptors."""
    s_input = 2 * (Tm * Tk + Tk * Tn)
    s_acc = 4 * Tm * Tn
    return dict(S_input=s_input, S_acc=s_acc, S_total=s_input + s_acc + reserve)


# ---------------------------------------------------------------------------
# O2: INT8 convolution  ([MNN] tileSplitFunction im2col with the input
# zero-point as pad value; [QG] section 2)
# ---------------------------------------------------------------------------
def conv_out_size(H, KH, stride, pad):
    return (H + 2 * pad - KH) // stride + 1


def qconv2d_s8_acc(x, w, stride, pad, za, bias=None):
    """Direct NHWC convolution: acc[n,oh,ow,co] = sum over taps inside the
    image of (x[n,ih,iw,ci]-za)*w[co,kh,kw,ci] + bias[co].

    A tap outside the image reads the pad value, which is the input
    zero-point za, so it contributes (za-za)*w = 0; it is skipped by an
    explicit bounds test.
    """
    x = np.asarray(x, dtype=np.int64)
    w = np.asarray(w, dtype=np.int64)
    Nb, H, W, Cin = x.shape
    Cout, KH, KW, Cin2 = w.shape
    assert Cin == Cin2
    sh, sw = stride
    ph, pw = pad
    OH, OW = conv_out_size(H, KH, sh, ph), conv_out_size(W, KW, sw, pw)
    xc = x - int(za)
    acc = np.zeros((Nb, OH, OW, Cout), dtype=np.int64)
    for kh in range(KH):
        ih = np.arange(OH) * sh + kh - ph
        oh_ok = np.nonzero((ih >= 0) & (ih < H))[0]
        for kw in range(KW):
            iw = np.arange(OW) * sw + kw - pw
            ow_ok = np.nonzero((iw >= 0) & (iw < W))[0]
            if oh_ok.size == 0 or ow_ok.size == 0:
                continue
            patch = xc[:, ih[oh_ok]][:, :, iw[ow_ok]]          # (Nb, h, w, Cin)
            contrib = np.einsum("nhwc,oc->nhwo", patch, w[:, kh, kw, :])
            acc[np.ix_(np.arange(Nb), oh_ok, ow_ok, np.arange(Cout))] += contrib
    if bias is not None:
        acc = acc + np.asarray(bias, dtype=np.int64)
    return acc


def qconv2d_s8(x, w, stride, pad, za, bias, m0, shift, out_zp, clamp_min,
               clamp_max):
    """Convolution followed by the same requant epilogue as O1 (per output
    channel M0/shift; fused ReLU is clamp_min = out_zp, [MNN]
    QuanPostTreatParameters minValue).  -> (y int8 NHWC, acc int32)."""
    K = w.shape[1] * w.shape[2] * w.shape[3]
    mab = 0 if bias is None else int(np.abs(np.asarray(bias, np.int64)).max(initial=0))
    if not fits_int32(K, mab):
        raise OverflowError("K*65025 + |bias| exceeds INT32_MAX")
    acc = qconv2d_s8_acc(x, w, stride, pad, za, bias)
    y = requantize(acc, m0, shift, out_zp, clamp_min, clamp_max)
    return y, acc.astype(np.int32)


# ---------------------------------------------------------------------------
# O3: dynamic per-row asymmetric int8 activation quantization  (R5; [MNN]
# BatchAsyDynamicQuant: min/max -> scale/zero, quantize with clamp to
# [-128,127]; [KAI] qai8dx = int8 dynamic per-row asymmetric)
# ---------------------------------------------------------------------------
def quantize_rows_a8(x):
    """Per row m of x[M][K] (float32):
        rmin = min(0, min_k x), rmax = max(0, max_k x)
        scale = (rmax - rmin) / 255            (scale = 1 if that is 0)
        inv = 1 / scale
        zp = clamp(rne(-128 - rmin*inv), -128, 127)
        q[k] = clamp(rne(x[k]*inv) + zp, -128, 127)
    every operation in float32 with one rounding each.
    Returns q int8 [M][K], scale float32 [M], zp int32 [M].
    """
    x = np.asarray(x, dtype=np.float32)
    M, K = x.shape
    f32 = np.float32
    q = np.empty((M, K), dtype=np.int8)
    scale = np.empty(M, dtype=np.float32)
    zp = np.empty(M, dtype=np.int32)
    for m in range(M):
        row = x[m]
        rmin = min(f32(0.0), row.min()) if K else f32(0.0)
        rmax = max(f32(0.0), row.max()) if K else f32(0.0)
        s = f32(f32(rmax) - f32(rmin)) / f32(255.0)
        s = f32(s)
        if s == f32(0.0):
            s = f32(1.0)
        inv = f32(f32(1.0) / s)
        t = f32(f32(rmin) * inv)
        z = int(np.clip(np.rint(f32(f32(-128.0) - t)), INT8_MIN, INT8_MAX))
        r = np.rint((row * inv).astype(np.float32)).astype(np.int64)
        q[m] = np.clip(r + z, INT8_MIN, INT8_MAX).astype(np.int8)
        scale[m] = s
        zp[m] = z
    return q, scale, zp


def quantize_blocks_a8(x, block):
    """Per-block dynamic quantization ([MNN] ConvInt8TiledExecutor: with the
    dynamic-quant option 2 the input is quantized in as many K blocks as the
    weights have quant blocks, each with its own scale and zero-point).
    READING R13: block = the weight group size; every block of `block`
    consecutive k of a row is quantized by the per-row rule above (R5).
    Returns q int8 [M][K], scale float32 [M][K/block], zp int32 [M][K/block].
    """
    x = np.asarray(x, dtype=np.float32)
    M, K = x.shape
    assert K % block == 0
    q, s, z = quantize_rows_a8(x.reshape(M * (K // block), block))
    return q.reshape(M, K), s.reshape(M, K // block), z.reshape(M, K // block)


def dequantize_rows(q, scale, zp):
    """real = scale * (q - zero_point)  ([QG] section 1), in float64."""
    return (np.asarray(scale, np.float64)[:, None]
            * (np.asarray(q, np.int64) - np.asarray(zp, np.int64)[:, None]))


# ---------------------------------------------------------------------------
# A8W4 packed weight format  (R6: this library's own layout; [MNN] stores
# int4 weights as two nibbles per byte with an offset of 8, and
# _computeReorderQuantInfo keeps per-block scales beside them)
# ---------------------------------------------------------------------------
def pack_w4_g32_bytes(N, K):
    return N * (K // 2) + N * (K // GROUP) * 4


def pack_w4_g32(qw, sw):
    """qw int8 [N][K] in [-8,7], sw float32 [N][K/32] -> packed uint8 buffer.

    Region 1, N rows of K/2 bytes: for each row n and each run of 8
    consecutive k starting at k0 = 8*j, bytes 4j..4j+3 hold
        byte[4j+b] = (qw[n,k0+b]+8) | ((qw[n,k0+4+b]+8) << 4),  b = 0..3
    so one little-endian 32-bit word carries k0..k0+3 in its low nibbles and
    k0+4..k0+7 in its high nibbles, and 16 bytes carry one 32-wide group.
    Region 2, right after: the float32 scales sw[N][K/32], row-major.
    """
    qw = np.asarray(qw, dtype=np.int64)
    N, K = qw.shape
    assert K % GROUP == 0
    assert qw.min(initial=0) >= -8 and qw.max(initial=0) <= 7
    u = (qw + 8).reshape(N, K // 8, 2, 4)           # [n][j][half][b]
    nib = (u[:, :, 0, :] | (u[:, :, 1, :] << 4)).astype(np.uint8)
    w_bytes = nib.reshape(N, K // 2)
    s_bytes = np.ascontiguousarray(np.asarray(sw, dtype=np.float32)).view(np.uint8).reshape(-1)
    return np.concatenate([w_bytes.reshape(-1), s_bytes])


def unpack_w4_g32(packed, N, K):
    """Inverse of pack_w4_g32 -> (qw int8 [N][K], sw float32 [N][K/32])."""
    packed = np.asarray(packed, dtype=np.uint8)
    nb = N * (K // 2)
    b = packed[:nb].reshape(N, K // 8, 4).astype(np.int64)
    lo = (b & 0xF) - 8
    hi = (b >> 4) - 8
    qw = np.concatenate([lo, hi], axis=2).reshape(N, K).astype(np.int8)
    sw = packed[nb:nb + N * (K // GROUP) * 4].view(np.float32).reshape(N, K // GROUP)
    return qw, sw.copy()


# ---------------------------------------------------------------------------
# O5: bf16 group scales ([KAI] review of the packing call: the Kleidi packing
# is passed a bf16 type for the group scales, kept as bf16 to save space).
# READING R12: f32 -> bf16 rounds to nearest, ties to even; the method then
# uses that bf16 value as the group scale.
# ---------------------------------------------------------------------------
def f32_to_bf16_bits(a):
    """bfloat16 bit patterns (uint16) of finite float32 values, rounded to
    nearest with ties to even.  bf16 keeps the top 16 bits of the f32 pattern.
    Patterns order like magnitudes within one sign, so adding 0x7FFF plus the
    lowest kept bit and dropping the low 16 bits rounds the magnitude to
    nearest, a tie (low half exactly 0x8000) going to the even pattern."""
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    assert np.isfinite(a).all()
    u = a.view(np.uint32).astype(np.uint64)
    kept_lsb = (u >> 16) & 1
    return ((u + 0x7FFF + kept_lsb) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b):
    """bf16 bit patterns -> the float32 values they denote (exact)."""
    b = np.ascontiguousarray(np.asarray(b, dtype=np.uint16))
    return (b.astype(np.uint32) << 16).view(np.float32)


def pack_w4_g32_bf16_bytes(N, K):
    return N * (K // 2) + N * (K // GROUP) * 2


def pack_w4_g32_bf16(qw, sw):
    """As pack_w4_g32, with region 2 the bf16 patterns of sw[N][K/32] (R12),
    little-endian, row-major."""
    qw = np.asarray(qw)
    N, K = qw.shape
    nib = pack_w4_g32(qw, sw)[:N * (K // 2)]
    bits = f32_to_bf16_bits(np.asarray(sw, np.float32).reshape(N, K // GROUP))
    return np.concatenate([nib, bits.reshape(-1).astype("<u2").view(np.uint8)])


def bf16_scales(sw):
    """The group scales the bf16-scale method uses: sw rounded to bf16 (R12)."""
    sw = np.asarray(sw, np.float32)
    return bf16_bits_to_f32(f32_to_bf16_bits(sw)).reshape(sw.shape)


# ---------------------------------------------------------------------------
# O4: A8W4 blockwise GEMV/GEMM  ([KAI] matmul_clamp_f32_qai8dxp_qsi4c32p:
# f32 out = clamp(dequant(int8 dyn act) x dequant(int4 g32 weights) + bias);
# weight zero-points are absent (nullptr or all zero); bias before clamp R8)
# ---------------------------------------------------------------------------
def qgemm_a8w4_f32(x, qw, sw, bias, clamp_min, clamp_max):
    """y[m,n] = clamp(f32( sum_g sw[n,g]*sA[m]*I[m,n,g] + bias[n] ), lo, hi)
    with I[m,n,g] = sum_{k in group g} (qA[m,k]-za[m]) * qw[n,k]  (exact int)
    and the combination over groups in float64.
    Returns (y float32 [M,N], qA int8, sA float32 [M], za int32 [M]).
    """
    qA, sA, za = quantize_rows_a8(x)
    qw = np.asarray(qw, dtype=np.int64)
    N, K = qw.shape
    G = K // GROUP
    M = qA.shape[0]
    swd = np.asarray(sw, dtype=np.float64)
    wg = qw.reshape(N, G, GROUP)
    y = np.empty((M, N), dtype=np.float32)
    lo, hi = np.float32(clamp_min), np.float32(clamp_max)
    for m in range(M):
        a = (qA[m].astype(np.int64) - int(za[m])).reshape(G, GROUP)
        I = np.einsum("gj,ngj->ng", a, wg)                       # exact
        comb = (swd * np.float64(sA[m]) * I.astype(np.float64)).sum(axis=1)
        if bias is not None:
            comb = comb + np.asarray(bias, np.float64)
        y[m] = np.minimum(np.maximum(comb.astype(np.float32), lo), hi)
    return y, qA, sA, za


def qgemm_a8w4_f32_bf16s(x, qw, sw, bias, clamp_min, clamp_max):
    """O4 with every group scale replaced by its bf16 value (O5, R12)."""
    return qgemm_a8w4_f32(x, qw, bf16_scales(sw), bias, clamp_min, clamp_max)


def qgemm_a8w4_f32_actblock(x, qw, sw, bias, clamp_min, clamp_max):
    """O4 with the activations quantized per 32-wide K block (O6, R13):
        y[m,n] = clamp(f32( sum_g sw[n,g]*sA[m,g]*I[m,n,g] + bias[n] ), lo, hi)
        I[m,n,g] = sum_{k in group g} (qA[m,k]-za[m,g]) * qw[n,k]   (exact int)
    with the combination over groups in float64.
    Returns (y float32 [M,N], qA int8 [M,K], sA float32 [M,G], za int32 [M,G]).
    """
    qw = np.asarray(qw, dtype=np.int64)
    N, K = qw.shape
    G = K // GROUP
    qA, sA, za = quantize_blocks_a8(x, GROUP)
    M = qA.shape[0]
    swd = np.asarray(sw, dtype=np.float64)
    wg = qw.reshape(N, G, GROUP)
    y = np.empty((M, N), dtype=np.float32)
    lo, hi = np.float32(clamp_min), np.float32(clamp_max)
    for m in range(M):
        a = qA[m].astype(np.int64).reshape(G, GROUP) - za[m].astype(np.int64)[:, None]
        I = np.einsum("gj,ngj->ng", a, wg)                       # exact
        comb = (swd * sA[m].astype(np.float64)[None, :] * I.astype(np.float64)).sum(axis=1)
        if bias is not None:
            comb = comb + np.asarray(bias, np.float64)
        y[m] = np.minimum(np.maximum(comb.astype(np.float32), lo), hi)
    return y, qA, sA, za


# ---------------------------------------------------------------------------
# O7: asymmetric int4 weights ([MNN] ConvInt8TiledExecutor, asymmetric quant
# info: each (output channel, block) carries a zero and an alpha, and the
# weight is alpha * code + zero).  READING R14: w_real[n,k] = sw[n,g]*w[n,k]
# + zw[n,g] with the int4 code w in [-8,7] as in the symmetric packing and a
# float32 zero zw per (row, 32-wide group).
# ---------------------------------------------------------------------------
def pack_w4_g32_asym_bytes(N, K):
    return N * (K // 2) + 2 * N * (K // GROUP) * 4


def pack_w4_g32_asym(qw, sw, zw):
    """pack_w4_g32's nibbles and f32 scales, then the f32 zeros zw[N][K/32]."""
    packed = pack_w4_g32(qw, sw)
    z_bytes = np.ascontiguousarray(np.asarray(zw, dtype=np.float32)).view(np.uint8).reshape(-1)
    return np.concatenate([packed, z_bytes])


def qgemm_a8w4_f32_asym(x, qw, sw, zw, bias, clamp_min, clamp_max):
    """y[m,n] = clamp(f32( sum_g sA[m]*(sw[n,g]*I[m,n,g] + zw[n,g]*S[m,g]) + bias[n] ))
    with I as in O4 and S[m,g] = sum_{k in g} (qA[m,k]-za[m]) (exact int):
    the dequantized activations times (sw*w + zw), grouped.  The combination
    is in float64.  Returns (y float32 [M,N], qA, sA, za) as O4."""
    qA, sA, za = quantize_rows_a8(x)
    qw = np.asarray(qw, dtype=np.int64)
    N, K = qw.shape
    G = K // GROUP
    M = qA.shape[0]
    swd = np.asarray(sw, dtype=np.float64)
    zwd = np.asarray(zw, dtype=np.float64)
    wg = qw.reshape(N, G, GROUP)
    y = np.empty((M, N), dtype=np.float32)
    lo, hi = np.float32(clamp_min), np.float32(clamp_max)
    for m in range(M):
        a = (qA[m].astype(np.int64) - int(za[m])).reshape(G, GROUP)
        I = np.einsum("gj,ngj->ng", a, wg)                       # exact
        S = a.sum(axis=1)                                        # exact
        sa = np.float64(sA[m])
        comb = (swd * sa * I.astype(np.float64) + zwd * sa * S.astype(np.float64)[None, :]).sum(axis=1)
        if bias is not None:
            comb = comb + np.asarray(bias, np.float64)
        y[m] = np.minimum(np.maximum(comb.astype(np.float32), lo), hi)
    return y, qA, sA, za



# ---------------------------------------------------------------------------
# O8: dynamic per-row symmetric int8 activation quantization ([MNN]
# ConvInt8TiledExecutor, BatchSymDynamicQuant: the absolute maximum of each
# row gives a quantizing scale and a dequantizing scale, the codes are taken
# with that scale and the zero-point is 0).
# READING R15: amax = max_k |x[k]|; dequant scale = amax/127 and quant scale
# = 127/amax, each one float32 division (both 1 when amax is 0);
# q = clamp(rne(x * quant scale), -127, 127); zero-point 0.
# ---------------------------------------------------------------------------
def quantize_rows_a8_sym(x):
    """Per row m of x[M][K] (float32):
        amax = max_k |x[m,k]|   (0 for an empty or all-zero row)
        dscale = amax / 127, qscale = 127 / amax   (both 1 if amax == 0)
        q[k] = clamp(rne(x[k] * qscale), -127, 127)
    every operation in float32 with one rounding each.
    Returns q int8 [M][K], dscale float32 [M], zp int32 [M] (all zero).
    """
    x = np.asarray(x, dtype=np.float32)
    M, K = x.shape
    f32 = np.float32
    q = np.empty((M, K), dtype=np.int8)
    scale = np.empty(M, dtype=np.float32)
    for m in range(M):
        row = x[m]
        amax = f32(np.abs(row).max()) if K else f32(0.0)
        if amax == f32(0.0):
            ds, qs = f32(1.0), f32(1.0)
        else:
            ds = f32(amax / f32(127.0))
            qs = f32(f32(127.0) / amax)
        r = np.rint((row * qs).astype(np.float32)).astype(np.int64)
        q[m] = np.clip(r, -127, 127).astype(np.int8)
        scale[m] = ds
    return q, scale, np.zeros(M, dtype=np.int32)


# ---------------------------------------------------------------------------
# O9: convolution with a float input quantized on the fly ([MNN]
# ConvInt8TiledExecutor, low-memory path: the float input of a tile of output
# pixels is unrolled by im2col, each unrolled row is quantized dynamically,
# asymmetric (BatchAsyDynamicQuant) or symmetric (BatchSymDynamicQuant), and
# the int8 rows meet the int4 block-quantized weights; [QG] section 2: a pad
# tap stands for the real value zero).
# READING R16: x float32 NHWC [Nb][H][W][Cin]; int4 codes w[Cout][KH][KW][Cin]
# flattened to K = KH*KW*Cin in (kh, kw, ci) order, one scale per 32
# consecutive k of that order; the unrolled row of output pixel (n, oh, ow)
# holds x[n, oh*sh+kh-ph, ow*sw+kw-pw, ci], 0.0 for a tap outside the image;
# each unrolled row is quantized on its own (R5, or R15 when symmetric) and
# y[n,oh,ow,:] is O4 on that row, output NHWC float32.
# ---------------------------------------------------------------------------
def im2col_f32(x, KH, KW, stride, pad):
    """Unrolled float input: cols[(n*OH+oh)*OW+ow, (kh*KW+kw)*Cin+ci]."""
    x = np.asarray(x, dtype=np.float32)
    Nb, H, W, Cin = x.shape
    sh, sw = stride
    ph, pw = pad
    OH, OW = conv_out_size(H, KH, sh, ph), conv_out_size(W, KW, sw, pw)
    cols = np.zeros((Nb, OH, OW, KH, KW, Cin), dtype=np.float32)
    for kh in range(KH):
        for kw in range(KW):
            for oh in range(OH):
                ih = oh * sh + kh - ph
                if ih < 0 or ih >= H:
                    continue
                for ow in range(OW):
                    iw = ow * sw + kw - pw
                    if iw < 0 or iw >= W:
                        continue
                    cols[:, oh, ow, kh, kw, :] = x[:, ih, iw, :]
    return cols.reshape(Nb * OH * OW, KH * KW * Cin)


def a8w4_from_codes(qA, sA, za, qw, sw, bias, clamp_min, clamp_max):
    """O4's combination for activations already quantized:
        y[m,n] = clamp(f32( sum_g sw[n,g]*sA[m]*I[m,n,g] + bias[n] ), lo, hi)
        I[m,n,g] = sum_{k in group g} (qA[m,k]-za[m]) * qw[n,k]   (exact int)
    with the combination over groups in float64."""
    qw = np.asarray(qw, dtype=np.int64)
    N, K = qw.shape
    G = K // GROUP
    M = qA.shape[0]
    swd = np.asarray(sw, dtype=np.float64)
    wg = qw.reshape(N, G, GROUP)
    y = np.empty((M, N), dtype=np.float32)
    lo, hi = np.float32(clamp_min), np.float32(clamp_max)
    for m in range(M):
        a = (qA[m].astype(np.int64) - int(za[m])).reshape(G, GROUP)
        I = np.einsum("gj,ngj->ng", a, wg)                       # exact
        comb = (swd * np.float64(sA[m]) * I.astype(np.float64)).sum(axis=1)
        if bias is not None:
            comb = comb + np.asarray(bias, np.float64)
        y[m] = np.minimum(np.maximum(comb.astype(np.float32), lo), hi)
    return y


def qconv2d_f32_dyn_a8w4(x, qw, sw, stride, pad, bias, clamp_min, clamp_max,
                         symmetric=False):
    """Float-input convolution with dynamic int8 activations and int4 g32
    weights (O9, R16).  qw int4 codes [Cout][KH][KW][Cin], sw [Cout][K/32].
    Returns (y float32 [Nb][OH][OW][Cout], qA int8 [P][K], sA float32 [P],
    za int32 [P]) with P = Nb*OH*OW unrolled rows."""
    qw = np.asarray(qw)
    Cout, KH, KW, Cin = qw.shape
    Nb, H, W, _ = np.asarray(x).shape
    OH, OW = conv_out_size(H, KH, stride[0], pad[0]), conv_out_size(W, KW, stride[1], pad[1])
    cols = im2col_f32(x, KH, KW, stride, pad)
    qA, sA, za = quantize_rows_a8_sym(cols) if symmetric else quantize_rows_a8(cols)
    y = a8w4_from_codes(qA, sA, za, qw.reshape(Cout, KH * KW * Cin), sw, bias,
                        clamp_min, clamp_max)
    return y.reshape(Nb, OH, OW, Cout), qA, sA, za
