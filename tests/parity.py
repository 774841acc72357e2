"""The parity bar shared by the GPU tests.

Floating point: each output must satisfy |y - y_ref| <= 2e-3 * B + 1e-5, where
y_ref = sum_k x[k] * w[k][n] and B = sum_k |x[k] * w[k][n]| are the fp64
oracle's values and y is the fp16 output widened to fp64.
Integer work (packing) is compared bit for bit.
"""
import numpy as np

RTOL_B = 2e-3
ATOL = 1e-5


def check_product(y_gpu, y_ref, bound, what=""):
    y = np.asarray(y_gpu, dtype=np.float16).astype(np.float64)
    err = np.abs(y - y_ref)
    lim = RTOL_B * bound + ATOL
    bad = err > lim
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {bad.size} outputs outside |y-y_ref| <= 2e-3*B + 1e-5; "
            f"first {idx.tolist()}: y={y[bad][:5]}, ref={y_ref[bad][:5]}, B={bound[bad][:5]}")
    return float((err / lim).max()) if err.size else 0.0
