"""Seeded synthetic inputs for the quantized-matmul workloads.

This module only draws random numbers with the shapes and distributions of
the five workloads; it holds none of the method's arithmetic (no
quantization, no requantization, no packing, no matmul).  Both the CPU oracle
tests and the GPU tests / benchmark take their inputs from here, so the two
sides see identical data.

Generator: ``numpy.random.default_rng(seed)`` (PCG64).  Seeds 1001..1006 are
the standard workloads listed in ``WORKLOADS``.

Workload shapes follow the quantized GEMM case study (xidianedu, "量化 GEMM：
数值契约、SRAM、DMA 与结果验证", "明确范围": M=130, N=70, K=129) and the A8W4
blockwise GEMV of pytorch/ao PR #997 (int8 dynamic activations x int4
weights with one scale per 32-wide K group, f32 output with clamp).
"""
from __future__ import annotations

import numpy as np

INT8_MIN, INT8_MAX = -128, 127


def _rng(seed: int) -> np.random.Generator:
    return np.random.default_rng(int(seed))


def _int8(rng, shape, lo=INT8_MIN, hi=INT8_MAX):
    return rng.integers(lo, hi + 1, size=shape, dtype=np.int8)


def _log_uniform(rng, shape, lo, hi, dtype=np.float32):
    u = rng.random(size=shape)
    return np.exp(np.log(lo) + u * (np.log(hi) - np.log(lo))).astype(dtype)


# --------------------------------------------------------------------------
# INT8 GEMM workloads (row-major A[M][lda], B[K][ldb])
# --------------------------------------------------------------------------
def int8_gemm(M, N, K, seed, *, za=None, zb=None, za_range=(-20, 20),
              zb_range=(-20, 20), b_symmetric=False, per_channel=False,
              ratio_range=(1e-4, 1e-2), ratio_scale=None, out_zp=3,
              clamp=(INT8_MIN, INT8_MAX), bias_range=(-5000, 5000),
              lda=None, ldb=None, with_bias=True):
    """Random affine INT8 GEMM problem.

    Returns a dict with A (M x lda int8, logical M x K), B (K x ldb int8,
    logical K x N), zero-points, int32 bias[N] (or None), the float64
    requant ratio(s) (one per tensor or one per column), out zero-point and
    clamp bounds.  Padding columns of A/B beyond the logical shape hold
    random bytes: a correct implementation never reads them.
    """
    rng = _rng(seed)
    lda = K if lda is None else lda
    ldb = N if ldb is None else ldb
    A = _int8(rng, (M, lda))
    if b_symmetric:
        B = _int8(rng, (K, ldb), -127, 127)
    else:
        B = _int8(rng, (K, ldb))
    za = int(rng.integers(za_range[0], za_range[1] + 1)) if za is None else int(za)
    zb = int(rng.integers(zb_range[0], zb_range[1] + 1)) if zb is None else int(zb)
    bias = (rng.integers(bias_range[0], bias_range[1] + 1, size=N).astype(np.int32)
            if with_bias else None)
    if per_channel:
        if ratio_scale is not None:
            sB = _log_uniform(rng, N, 1e-3, 1e-1, np.float64)
            ratio = (ratio_scale * sB).astype(np.float64)
        else:
            ratio = np.exp(np.log(ratio_range[0]) + rng.random(N)
                           * (np.log(ratio_range[1]) - np.log(ratio_range[0])))
    else:
        ratio = np.array([rng.uniform(ratio_range[0], ratio_range[1])])
    return dict(M=M, N=N, K=K, A=A, lda=lda, B=B, ldb=ldb, za=za, zb=zb,
                bias=bias, ratio=ratio, per_channel=per_channel,
                out_zp=int(out_zp), clamp_min=int(clamp[0]), clamp_max=int(clamp[1]))


def int8_gemm_130x70x129(seed=1001):
    """Affine INT8 GEMM M=130, N=70, K=129 (tails in all three dims)."""
    return int8_gemm(130, 70, 129, seed)


def int8_gemm_8192x8192x8200(seed=1005):
    """INT8 GEMM M=N=8192, K=8200 (K tail 8 past 64 blocks of 128), za=7,
    symmetric B with per-column scales log-uniform [1e-3, 1e-1],
    sA/sO = 0.01 so per-column ratios lie in [1e-5, 1e-3]."""
    return int8_gemm(8192, 8192, 8200, seed, za=7, zb=0, b_symmetric=True,
                     per_channel=True, ratio_scale=0.01, out_zp=0)


# --------------------------------------------------------------------------
# INT8 convolution workload (NHWC input, OHWI weights)
# --------------------------------------------------------------------------
def int8_conv(Nb, H, W, Cin, Cout, KH, KW, stride, pad, seed, *, za=-5,
              out_zp=-10, s_in_over_s_out=0.1, relu=True, with_bias=True):
    rng = _rng(seed)
    x = _int8(rng, (Nb, H, W, Cin))
    w = _int8(rng, (Cout, KH, KW, Cin), -127, 127)
    sW = _log_uniform(rng, Cout, 1e-3, 1e-1, np.float64)
    bias = (rng.integers(-5000, 5001, size=Cout).astype(np.int32)
            if with_bias else None)
    ratio = (s_in_over_s_out * sW).astype(np.float64)
    lo = int(out_zp) if relu else INT8_MIN
    return dict(Nb=Nb, H=H, W=W, Cin=Cin, Cout=Cout, KH=KH, KW=KW,
                stride=tuple(stride), pad=tuple(pad), x=x, w=w, za=int(za),
                bias=bias, ratio=ratio, out_zp=int(out_zp), clamp_min=lo,
                clamp_max=INT8_MAX)


def int8_conv_56x56x64_3x3(seed=1002):
    """1x56x56x64 -> 64, 3x3, stride 1, pad 1, input zp -5 (also the pad
    value), per-Cout weight scales, fused ReLU (clamp floor = out zp)."""
    return int8_conv(1, 56, 56, 64, 64, 3, 3, (1, 1), (1, 1), seed)


# --------------------------------------------------------------------------
# A8W4 workloads
# --------------------------------------------------------------------------
def a8w4(M, N, K, seed, *, clamp=(-6.0, 6.0), with_bias=True, ldx=None):
    """f32 activations N(0,1) [M][ldx]; int4 weights uniform in [-8,7] stored
    one per int8 as qw[N][K]; f32 group scales sw[N][K/32] log-uniform
    [1e-3, 1e-1]; f32 bias N(0, 0.1); output clamp."""
    assert K % 32 == 0
    rng = _rng(seed)
    ldx = K if ldx is None else ldx
    x = rng.standard_normal((M, ldx), dtype=np.float32)
    qw = _int8(rng, (N, K), -8, 7)
    sw = _log_uniform(rng, (N, K // 32), 1e-3, 1e-1)
    bias = (rng.normal(0.0, 0.1, size=N).astype(np.float32) if with_bias else None)
    return dict(M=M, N=N, K=K, x=x, ldx=ldx, qw=qw, sw=sw, bias=bias,
                clamp_min=float(clamp[0]), clamp_max=float(clamp[1]))


def a8w4_gemv_1x14336x4096(seed=1003):
    """A8W4 GEMV M=1, N=14336, K=4096."""
    return a8w4(1, 14336, 4096, seed)


def a8w4_gemm_128x4096x4096(seed=1004):
    """A8W4 GEMM M=128, N=4096, K=4096."""
    return a8w4(128, 4096, 4096, seed)


def a8w4_conv_f32(Nb, H, W, Cin, Cout, KH, KW, stride, pad, seed, *, clamp=(-6.0, 6.0)):
    """f32 NHWC input N(0,1) [Nb][H][W][Cin]; int4 weight codes uniform in
    [-8,7] stored one per int8 as qw[Cout][KH][KW][Cin]; f32 group scales
    sw[Cout][KH*KW*Cin/32] log-uniform [1e-3, 1e-1]; f32 bias N(0, 0.1);
    output clamp."""
    K = KH * KW * Cin
    assert K % 32 == 0
    rng = _rng(seed)
    x = rng.standard_normal((Nb, H, W, Cin), dtype=np.float32)
    qw = _int8(rng, (Cout, KH, KW, Cin), -8, 7)
    sw = _log_uniform(rng, (Cout, K // 32), 1e-3, 1e-1)
    bias = rng.normal(0.0, 0.1, size=Cout).astype(np.float32)
    return dict(Nb=Nb, H=H, W=W, Cin=Cin, Cout=Cout, KH=KH, KW=KW, stride=tuple(stride),
                pad=tuple(pad), K=K, x=x, qw=qw, sw=sw, bias=bias,
                clamp_min=float(clamp[0]), clamp_max=float(clamp[1]))


def a8w4_conv_f32_56x56x64_3x3(seed=1006):
    """Float-input dynamic conv: Nb=1, 56x56, Cin=Cout=64, 3x3, stride 1,
    pad 1 (the INT8 conv's shape, K = 576)."""
    return a8w4_conv_f32(1, 56, 56, 64, 64, 3, 3, (1, 1), (1, 1), seed)


WORKLOADS = {
    "int8_gemm_130x70x129": int8_gemm_130x70x129,
    "int8_conv_56x56x64_3x3": int8_conv_56x56x64_3x3,
    "a8w4_gemv_1x14336x4096": a8w4_gemv_1x14336x4096,
    "a8w4_gemm_128x4096x4096": a8w4_gemm_128x4096x4096,
    "int8_gemm_8192x8192x8200": int8_gemm_8192x8192x8200,
    "a8w4_conv_f32_56x56x64_3x3": a8w4_conv_f32_56x56x64_3x3,
}
