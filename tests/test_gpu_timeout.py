"""The bounded-wait path of the tensor-core kernels, exercised on the GPU
without a fault.

qg_test_arm_stall makes the next launch of a kernel family skip one pipeline
stage: nothing is issued for that stage, so its consumer waits on a barrier
that no copy will ever complete.  With the short poll limit the hook also
sets, that wait runs out: the kernel must record QG_ERR_TIMEOUT in the device
status word, wait for its own copies and MMAs still in flight, free its
tensor memory and return.  The context must stay usable: the next call on
the same inputs is checked bit for bit (or within the A8W4 tolerance)
against the CPU oracle.  No test here traps, faults or hangs a GPU."""
import numpy as np
import pytest

import oracle
import workloads
from a8w4_tol import assert_a8w4_close

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")

QG_ERR_TIMEOUT = -6


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _gemm_call(lib, w, C, acc):
    m0, sh = lib.qg_requant_params(float(w["ratio"][0]))
    rq = lib.make_requant(a_zero_point=w["za"], b_zero_point=w["zb"], bias=_dev(w["bias"]),
                          multiplier=m0, shift=sh, out_zero_point=w["out_zp"],
                          clamp_min=w["clamp_min"], clamp_max=w["clamp_max"])
    lib.qgemm_s8s8_requant(_dev(w["A"])[:, :w["K"]], _dev(w["B"])[:, :w["N"]], C, rq,
                           K=w["K"], N=w["N"], acc_out=acc)
    return m0, sh


@pytest.mark.parametrize("M,N,K", [(64, 200, 1000), (128, 600, 4096)])
def test_int8_gemm_stalled_pipeline_times_out_then_recovers(lib, cuda, M, N, K):
    assert lib.qg_device_status(True) in (0, QG_ERR_TIMEOUT)
    w = workloads.int8_gemm(M, N, K, seed=M + N + K)
    C = torch.zeros((M, N), dtype=torch.int8, device="cuda")
    acc = torch.zeros((M, N), dtype=torch.int32, device="cuda")
    lib.qg_test_arm_stall(1)
    _gemm_call(lib, w, C, acc)
    assert lib.qg_device_status(True) == QG_ERR_TIMEOUT
    # the context is intact and the next call (not stalled) is exact
    m0, sh = _gemm_call(lib, w, C, acc)
    torch.cuda.synchronize()
    C_ref, acc_ref = oracle.qgemm_s8s8_requant(w["A"][:, :K], w["B"][:, :N], w["za"], w["zb"],
                                               w["bias"], m0, sh, w["out_zp"], w["clamp_min"],
                                               w["clamp_max"])
    np.testing.assert_array_equal(acc.cpu().numpy(), acc_ref)
    np.testing.assert_array_equal(C.cpu().numpy(), C_ref)
    assert lib.qg_device_status(True) == 0


def test_stall_hook_is_one_shot_and_disarmable(lib, cuda):
    lib.qg_device_status(True)
    w = workloads.int8_gemm(64, 64, 512, seed=3)
    C = torch.zeros((64, 64), dtype=torch.int8, device="cuda")
    acc = torch.zeros((64, 64), dtype=torch.int32, device="cuda")
    lib.qg_test_arm_stall(1)
    lib.qg_test_arm_stall(0)                  # disarmed before any launch
    _gemm_call(lib, w, C, acc)
    assert lib.qg_device_status(True) == 0
    with pytest.raises(lib.QGError):
        lib.qg_test_arm_stall(7)


@pytest.mark.parametrize("M,N,K", [(128, 512, 4096), (20, 300, 1024)])
def test_a8w4_tc_stalled_pipeline_times_out_then_recovers(lib, cuda, M, N, K):
    lib.qg_device_status(True)
    w = workloads.a8w4(M, N, K, seed=M + N, clamp=(-np.inf, np.inf))
    packed = lib.pack_w4_g32(_dev(w["qw"]), _dev(w["sw"]))
    x = _dev(w["x"])
    bias = _dev(w["bias"])
    y = torch.zeros((M, N), dtype=torch.float32, device="cuda")
    lib.qg_test_arm_stall(2)
    lib.qgemm_a8w4_f32(x, packed, N, bias, -np.inf, np.inf, y)
    assert lib.qg_device_status(True) == QG_ERR_TIMEOUT
    lib.qgemm_a8w4_f32(x, packed, N, bias, -np.inf, np.inf, y)
    torch.cuda.synchronize()
    y_ref = oracle.qgemm_a8w4_f32(w["x"], w["qw"], w["sw"], w["bias"], -np.inf, np.inf)[0]
    assert_a8w4_close(y.cpu().numpy(), y_ref, f"a8w4 tc after a stall {M}x{N}x{K}")
    assert lib.qg_device_status(True) == 0
