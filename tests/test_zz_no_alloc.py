"""The allocation-free A8W4 entry point, called through the C ABI.

qgemm_a8w4_f32_noalloc serves callers that cannot give the library a
workspace: a plugin whose host framework owns the device allocator and
offers none, or a serving loop that must not call cudaMalloc after start-up
(it can synchronise the device).  Its scratch is a fixed device array inside
the library.  Two calls in a row, with different inputs and row counts, must
each match the CPU oracle and the workspace-taking entry point
qgemm_a8w4_f32 within the A8W4 tolerance (tests/a8w4_tol.py); the M = 1 call
(fused GEMV, scratch in shared memory) is covered too.  This file is
collected last on purpose.
"""
import ctypes

import numpy as np
import pytest

import oracle
import workloads
from a8w4_tol import assert_a8w4_close

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")

QG_ERR_WORKSPACE = -7
QG_ERR_UNSUPPORTED = -4


def _fn(lib):
    f = lib.lib.qgemm_a8w4_f32_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_int64,
                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_float, ctypes.c_float,
                  ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p]
    return f


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def test_noalloc_matches_oracle_and_workspace_entry_point_twice(lib, cuda):
    f = _fn(lib)
    lib.qg_device_status(True)
    N, K = 384, 1024
    w = workloads.a8w4(32, N, K, seed=4242, clamp=(-np.inf, np.inf))
    packed = lib.pack_w4_g32(_dev(w["qw"]), _dev(w["sw"]))
    bias = _dev(w["bias"])
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # second call: fewer rows and different activations, so stale scratch
    # from the first call would show up in its result; the third is M = 1
    x2 = np.random.default_rng(7).standard_normal((8, K)).astype(np.float32) * 3.0
    x3 = np.random.default_rng(8).standard_normal((1, K)).astype(np.float32)
    for x in (w["x"], x2, x3):
        M = x.shape[0]
        xd = _dev(x)
        y = torch.full((M, N), 123.0, dtype=torch.float32, device="cuda")
        rc = f(M, N, K, _p(xd), K, _p(packed), _p(bias), float("-inf"), float("inf"), _p(y), N,
               stream)
        assert rc == 0, lib.lib.qg_status_string(rc)
        y_lib = torch.empty((M, N), dtype=torch.float32, device="cuda")
        lib.qgemm_a8w4_f32(xd, packed, N, bias, float("-inf"), float("inf"), y_lib)
        torch.cuda.synchronize()
        y_np = y.cpu().numpy()
        y_ref = oracle.qgemm_a8w4_f32(x, w["qw"], w["sw"], w["bias"], -np.inf, np.inf)[0]
        assert_a8w4_close(y_np, y_ref, f"noalloc {M}x{N}x{K}")
        assert_a8w4_close(y_np, y_lib.cpu().numpy(), f"noalloc vs library {M}x{N}x{K}")
    assert lib.qg_device_status(True) == 0


def test_noalloc_rejects_sizes_beyond_its_scratch(lib, cuda):
    # Every buffer is as large as the rejected call claims, so even a call
    # that wrongly went ahead would stay inside its buffers; the rejection
    # shows as a status code and an untouched y.
    f = _fn(lib)
    packed = torch.zeros(lib.pack_w4_g32_bytes(64, 1024), dtype=torch.uint8, device="cuda")
    # 8192 rows x 1024 codes = 8 MiB > 4 MiB of scratch
    x = torch.zeros((8192, 1024), dtype=torch.float32, device="cuda")
    y = torch.zeros((8192, 64), dtype=torch.float32, device="cuda")
    assert f(8192, 64, 1024, _p(x), 1024, _p(packed), None, -1.0, 1.0, _p(y), 64, None) == QG_ERR_WORKSPACE
    # 8193 rows > 8192 row parameters
    x = torch.zeros((8193, 32), dtype=torch.float32, device="cuda")
    y = torch.zeros((8193, 64), dtype=torch.float32, device="cuda")
    assert f(8193, 64, 32, _p(x), 32, _p(packed), None, -1.0, 1.0, _p(y), 64, None) == QG_ERR_WORKSPACE
    # K beyond the shared-memory rows of the CUDA-core GEMM (M > 1)
    x2 = torch.zeros((2, 25632), dtype=torch.float32, device="cuda")
    y2 = torch.zeros((2, 64), dtype=torch.float32, device="cuda")
    packed2 = torch.zeros(lib.pack_w4_g32_bytes(64, 25632), dtype=torch.uint8, device="cuda")
    assert f(2, 64, 25632, _p(x2), 25632, _p(packed2), None, -1.0, 1.0, _p(y2), 64, None) == QG_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert (y == 0).all() and (y2 == 0).all()
