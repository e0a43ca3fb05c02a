"""The allocation-free A8W4 entry point, called through the C ABI.

qgemm_a8w4_f32_noalloc serves callers that cannot give the library a
workspace (a plugin whose host framework owns the device allocator, or a
serving loop that must not call cudaMalloc after start-up).  Its scratch is
a fixed device array inside the library.  Two calls in a row, with different
inputs and row counts, must each match the workspace-taking entry point
qgemm_a8w4_f32 within the A8W4 tolerance used everywhere in these tests.
This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest

import workloads

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")

TOL = 1e-4
QG_ERR_WORKSPACE = -7


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


def _close(y, y_ref):
    err = np.abs(y.astype(np.float64) - y_ref.astype(np.float64)) / np.maximum(np.abs(y_ref), 1.0)
    assert err.max() <= TOL, err.max()


def test_noalloc_matches_workspace_entry_point_twice(lib, cuda):
    f = _fn(lib)
    lib.qg_device_status(True)
    N, K = 384, 1024
    w = workloads.a8w4(32, N, K, seed=4242, clamp=(-np.inf, np.inf))
    packed = lib.pack_w4_g32(_dev(w["qw"]), _dev(w["sw"]))
    bias = _dev(w["bias"])
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # second call: fewer rows and different activations, so stale scratch
    # from the first call would show up in its result
    x2 = np.random.default_rng(7).standard_normal((8, K)).astype(np.float32) * 3.0
    for x in (w["x"], x2):
        M = x.shape[0]
        xd = _dev(x)
        y = torch.full((M, N), 123.0, dtype=torch.float32, device="cuda")
        rc = f(M, N, K, _p(xd), K, _p(packed), _p(bias), float("-inf"), float("inf"), _p(y), N,
               stream)
        assert rc == 0, lib.lib.qg_status_string(rc)
        y_ref = torch.empty((M, N), dtype=torch.float32, device="cuda")
        lib.qgemm_a8w4_f32(xd, packed, N, bias, float("-inf"), float("inf"), y_ref)
        torch.cuda.synchronize()
        _close(y.cpu().numpy(), y_ref.cpu().numpy())
    assert lib.qg_device_status(True) == 0


def test_noalloc_rejects_sizes_beyond_its_scratch(lib, cuda):
    f = _fn(lib)
    y = torch.zeros((2, 64), dtype=torch.float32, device="cuda")
    x = torch.zeros((2, 1024), dtype=torch.float32, device="cuda")
    packed = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda")
    # 8192 rows x 1024 codes = 8 MiB > 4 MiB of scratch; 8193 rows > 8192
    assert f(8192, 64, 1024, _p(x), 1024, _p(packed), None, -1.0, 1.0, _p(y), 64, None) == QG_ERR_WORKSPACE
    assert f(8193, 64, 32, _p(x), 32, _p(packed), None, -1.0, 1.0, _p(y), 64, None) == QG_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert (y == 0).all()
