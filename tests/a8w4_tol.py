"""The A8W4 f32 output tolerance shared by every A8W4 parity test, and a
record of the error each comparison actually saw.

The Kleidi blockwise GEMV prototype (pytorch/ao PR #997) reports that its
kernels pass with a tolerance of 1e-4 and gives no formula.  A pure relative
error is undefined where y is near 0: y = sA * sum_g sw[n,g] * I[n,g] + bias
is a float32 sum of G group terms, and its rounding error is set by the size
of those terms (about G * 2^-24 * sA * sum_g |sw*I|), not by |y|.  The
reading used here: |y - y_ref| <= 1e-4 * max(|y_ref|, 1), i.e. relative 1e-4
for |y| >= 1 and absolute 1e-4 below, with y_ref the float64 oracle.  The
quantized activations (codes, scales, zero-points) are compared bit for bit
elsewhere; this helper covers only the float outputs.

Every call appends what it measured to OBSERVED; tests/conftest.py prints a
summary at the end of the run, so the margin each workload leaves under the
bound is visible in the test log.
"""
import numpy as np

TOL = 1e-4
FLOOR = 1.0
OBSERVED = []


def error_stats(y, y_ref):
    y = np.asarray(y, np.float64)
    y_ref = np.asarray(y_ref, np.float64)
    d = np.abs(y - y_ref)
    a = np.abs(y_ref)
    big = a >= 1.0
    return {
        "n": int(d.size),
        "max_abs": float(d.max(initial=0.0)),
        "max_rel_where_abs_ge_1": float((d[big] / a[big]).max(initial=0.0)),
        "max_scaled": float((d / np.maximum(a, FLOOR)).max(initial=0.0)),
        "max_scaled_floor_1e-3": float((d / np.maximum(a, 1e-3)).max(initial=0.0)),
        "max_scaled_floor_1e-2": float((d / np.maximum(a, 1e-2)).max(initial=0.0)),
    }


def assert_a8w4_close(y, y_ref, label=""):
    y = np.asarray(y)
    y_ref = np.asarray(y_ref)
    assert y.shape == y_ref.shape, (y.shape, y_ref.shape)
    st = error_stats(y, y_ref)
    OBSERVED.append((label, st))
    err = np.abs(y.astype(np.float64) - y_ref.astype(np.float64)) / np.maximum(np.abs(y_ref), FLOOR)
    i = int(np.argmax(err))
    assert err.flat[i] <= TOL, f"max err {err.flat[i]:.3e} at {np.unravel_index(i, y.shape)}: " \
                               f"{y.flat[i]} vs {y_ref.flat[i]}"
