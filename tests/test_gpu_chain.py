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


@pytest.mark.parametrize("M,K", [(100, 96), (100, 100), (200, 100)])
def test_int8_gemm_chain_ping_pong(lib, M, K):
    # N = K: C feeds the next call as A.  (100, 96): one-CTA kernel, A read
    # in place; (100, 100): row pitch 100 bytes, so each call stages A first;
    # (200, 100): the CTA-pair kernel after the staging pass.
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
