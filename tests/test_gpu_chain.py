"""Calls chained through their buffers on one stream, against the CPU oracle.

The library launches its kernels as programmatic dependents of the work
before them on the stream: a call's CTAs may start while the previous call
is still running and wait for it on the device before they read activations
or workspace or write any output.  These tests chain calls the way a network
does, with nothing between the launches:

  - read after write: each call's input is the previous call's output;
  - write after read: with two buffers in ping-pong, each call overwrites
    the buffer the call just before it read.

If a call read its input before the previous call had finished writing it,
or wrote its output while the previous call was still reading that buffer,
the chain would drift from the oracle's.  Integer chains are compared bit
for bit at every link (the oracle runs the same chain); float chains keep
their last three buffers and check the last two links against the oracle
applied to the library's own inputs, within the A8W4 tolerance.
"""
import numpy as np
import pytest

import oracle
import workloads
from a8w4_tol import assert_a8w4_close

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")

LINKS = 8


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


@pytest.fixture(autouse=True)
def _clean_status(lib, cuda):
    lib.qg_device_status(True)
    yield
    assert lib.qg_device_status(True) == 0


def _requant(lib, ratios, za, zb, bias, out_zp, lo, hi):
    params = [oracle.requant_params(float(r)) for r in ratios]
    m0 = np.array([p[0] for p in params], np.int64)
    sh = np.array([p[1] for p in params], np.int64)
    rq = lib.make_requant(a_zero_point=za, b_zero_point=zb, bias=bias,
                          multiplier=_dev(m0.astype(np.int32)), shift=_dev(sh.astype(np.int32)),
                          out_zero_point=out_zp, clamp_min=lo, clamp_max=hi)
    return rq, m0, sh


def _not_degenerate(v):
    v = np.asarray(v, np.int64)
    assert v.std() > 4 and np.mean((v == 127) | (v == -128)) < 0.5, "chain saturated"


def test_int8_conv_chain_ping_pong(lib):
    # 64 -> 64 channels so an output feeds the next call; one launch per call
    w = workloads.int8_conv(1, 24, 20, 64, 64, 3, 3, (1, 1), (1, 1), seed=3101, relu=False,
                            s_in_over_s_out=0.02)
    bias = _dev(w["bias"])
    rq, m0, sh = _requant(lib, w["ratio"], w["za"], 0, bias, w["out_zp"], -128, 127)
    pw = lib.qconv2d_s8_pack_w(_dev(w["w"]))
    bufs = [_dev(w["x"]), torch.empty_like(_dev(w["x"]))]
    for i in range(LINKS):
        lib.qconv2d_s8_im2col_packed(bufs[i % 2], pw, w["w"].shape, bufs[(i + 1) % 2], rq,
                                     w["stride"], w["pad"])
    torch.cuda.synchronize()
    x = w["x"]
    for i in range(LINKS):
        x, _ = oracle.qconv2d_s8(x, w["w"], w["stride"], w["pad"], w["za"], w["bias"], m0, sh,
                                 w["out_zp"], -128, 127)
    _not_degenerate(x)
    np.testing.assert_array_equal(bufs[LINKS % 2].cpu().numpy(), x)


@pytest.mark.parametrize("M,K", [(100, 96), (100, 100), (200, 100), (300, 100)])
def test_int8_gemm_chain_ping_pong(lib, M, K):
    # N = K: C feeds the next call as A.  (100, 96): one-CTA kernel, A read
    # in place; (100, 100) and (200, 100): row pitch 100 bytes, so each call
    # stages A first, then the one-CTA kernel (one wave of tiles); (300, 100):
    # the CTA-pair kernel after the staging pass.
    w = workloads.int8_gemm(M, K, K, seed=3200 + M + K, per_channel=True, ratio_scale=0.05,
                            out_zp=2)
    bias = _dev(w["bias"])
    rq, m0, sh = _requant(lib, w["ratio"], w["za"], w["zb"], bias, w["out_zp"], -128, 127)
    pb = lib.qgemm_pack_b_s8(_dev(w["B"]))
    bufs = [_dev(w["A"]), torch.empty((M, K), dtype=torch.int8, device="cuda")]
    for i in range(LINKS):
        lib.qgemm_s8s8_requant_packed(bufs[i % 2], pb, K, bufs[(i + 1) % 2], rq, K=K)
    torch.cuda.synchronize()
    a = w["A"]
    for i in range(LINKS):
        a, _ = oracle.qgemm_s8s8_requant(a, w["B"], w["za"], w["zb"], w["bias"], m0, sh,
                                         w["out_zp"], -128, 127)
    _not_degenerate(a)
    np.testing.assert_array_equal(bufs[LINKS % 2].cpu().numpy(), a)


@pytest.mark.parametrize("M,K,gain", [(1, 4096, 0.04), (64, 1024, 0.12)])
def test_a8w4_chain_ring(lib, M, K, gain):
    # N = K: y feeds the next call as x.  M = 1: the fused GEMV; M = 64: the
    # quantization grid and the tensor-core kernel.  A ring of three buffers
    # keeps the last two links' inputs for the check.  The group scales are
    # scaled down so that a link neither saturates the clamp nor decays to
    # the bias (found by running the oracle's chain): the standard deviation
    # of x stays between 0.13 and 0.7 over the eight links.
    w = workloads.a8w4(M, K, K, seed=3300 + M, clamp=(-6.0, 6.0))
    w["sw"] = (w["sw"] * gain).astype(np.float32)
    packed = lib.pack_w4_g32(_dev(w["qw"]), _dev(w["sw"]))
    bias = _dev(w["bias"])
    bufs = [_dev(w["x"])] + [torch.empty((M, K), dtype=torch.float32, device="cuda")
                             for _ in range(2)]
    for i in range(LINKS):
        lib.qgemm_a8w4_f32(bufs[i % 3], packed, K, bias, -6.0, 6.0, bufs[(i + 1) % 3])
    torch.cuda.synchronize()
    host = [b.cpu().numpy() for b in bufs]
    last = LINKS % 3
    for k in (1, 2):
        y_gpu = host[(last - k + 1) % 3]
        x_in = host[(last - k) % 3]
        assert np.std(x_in) > 0.12 and np.mean(np.abs(x_in) >= 6.0) < 0.1, "chain degenerate"
        y_ref = oracle.qgemm_a8w4_f32(x_in, w["qw"], w["sw"], w["bias"], -6.0, 6.0)[0]
        assert_a8w4_close(y_gpu, y_ref, f"a8w4 chain {M}x{K}x{K} link -{k}")


def test_inputs_written_by_a_preceding_torch_kernel(lib):
    # Each call's input is written by a torch copy kernel launched right
    # before it on the same stream (a grid that does not signal dependents
    # early): the A8W4 quantization grid, the INT8 staging pass and the
    # implicit-GEMM conv must still read the new values.
    w = workloads.a8w4(64, 384, 1024, seed=3401, clamp=(-6.0, 6.0))
    packed = lib.pack_w4_g32(_dev(w["qw"]), _dev(w["sw"]))
    bias = _dev(w["bias"])
    srcs = [_dev((w["x"] * s).astype(np.float32)) for s in (0.5, 1.0, 2.0)]
    x = torch.empty_like(srcs[0])
    ys = [torch.empty((64, 384), dtype=torch.float32, device="cuda") for _ in srcs]
    for src, y in zip(srcs, ys):
        x.copy_(src)
        lib.qgemm_a8w4_f32(x, packed, 384, bias, -6.0, 6.0, y)
    torch.cuda.synchronize()
    for s, y in zip((0.5, 1.0, 2.0), ys):
        x_in = (w["x"] * s).astype(np.float32)
        y_ref = oracle.qgemm_a8w4_f32(x_in, w["qw"], w["sw"], w["bias"], -6.0, 6.0)[0]
        assert_a8w4_close(y.cpu().numpy(), y_ref, f"a8w4 after torch copy, scale {s}")

    g = workloads.int8_gemm(300, 96, 100, seed=3402, per_channel=True, ratio_scale=0.05, out_zp=2)
    rq, m0, sh = _requant(lib, g["ratio"], g["za"], g["zb"], _dev(g["bias"]), g["out_zp"], -128, 127)
    pb = lib.qgemm_pack_b_s8(_dev(g["B"]))
    rng = np.random.default_rng(3403)
    a_list = [rng.integers(-128, 128, size=g["A"].shape, dtype=np.int8) for _ in range(3)]
    a = torch.empty((300, 100), dtype=torch.int8, device="cuda")
    cs = [torch.empty((300, 96), dtype=torch.int8, device="cuda") for _ in a_list]
    for a_host, c in zip(a_list, cs):
        a.copy_(_dev(a_host))
        lib.qgemm_s8s8_requant_packed(a, pb, 96, c, rq, K=100)
    torch.cuda.synchronize()
    for a_host, c in zip(a_list, cs):
        ref, _ = oracle.qgemm_s8s8_requant(a_host, g["B"], g["za"], g["zb"], g["bias"], m0, sh,
                                          g["out_zp"], -128, 127)
        np.testing.assert_array_equal(c.cpu().numpy(), ref)

    v = workloads.int8_conv(1, 12, 10, 16, 8, 3, 3, (1, 1), (1, 1), seed=3404, relu=False)
    rq, m0, sh = _requant(lib, v["ratio"], v["za"], 0, _dev(v["bias"]), v["out_zp"], -128, 127)
    pw = lib.qconv2d_s8_pack_w(_dev(v["w"]))
    x_list = [rng.integers(-128, 128, size=v["x"].shape, dtype=np.int8) for _ in range(3)]
    xc = torch.empty(v["x"].shape, dtype=torch.int8, device="cuda")
    outs = []
    for x_host in x_list:
        xc.copy_(_dev(x_host))
        o = torch.empty((1, 12, 10, 8), dtype=torch.int8, device="cuda")
        lib.qconv2d_s8_im2col_packed(xc, pw, v["w"].shape, o, rq, v["stride"], v["pad"])
        outs.append(o)
    torch.cuda.synchronize()
    for x_host, o in zip(x_list, outs):
        ref, _ = oracle.qconv2d_s8(x_host, v["w"], v["stride"], v["pad"], v["za"], v["bias"], m0, sh,
                                   v["out_zp"], -128, 127)
        np.testing.assert_array_equal(o.cpu().numpy(), ref)
