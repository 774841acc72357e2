"""The parity bar shared by the GPU tests.

Floating point: each output must satisfy |y - y_ref| <= RTOL * B + 1e-5, where
y_ref = sum_k x[k] * w[k][n] (+ bias[n]) and B = sum_k |x[k] * w[k][n]|
(+ |bias[n]|) are the fp64 oracle's values and y is the device output widened
to fp64.  Integer work (packing) is compared bit for bit.

RTOL is 2e-3 for fp16 (the product's stated tolerance).  For bf16 it is derived
from the arithmetic, u = 2^-8 being bf16's unit roundoff: the batched kernel
rounds each weight to bf16 once in one FMA, (q - round(z)) * s plus
-(z - round(z)) * s rounded (at most 2u |w|, since |z - round(z)| <= |q - z|
for the clamped integer zero point), the fp32 accumulation adds at most
K 2^-24 <= 2^-10 of B for K <= 16384, and y is rounded to bf16 once (u |y|
<= u B): RTOL_BF16 = 3u + 2^-10.  The decode kernel keeps q - round(z) exact
and needs only the last two terms.
"""
import numpy as np

RTOL_B = 2e-3
RTOL_BF16 = 3 * 2.0 ** -8 + 2.0 ** -10
ATOL = 1e-5


def widen_output(y_gpu):
    """fp64 values of a device output: a torch tensor (fp16 / bf16), or a host
    array already widened (float32 / float64) or still float16."""
    if hasattr(y_gpu, "float"):
        return y_gpu.float().cpu().numpy().astype(np.float64)
    return np.asarray(y_gpu).astype(np.float64)


def check_product(y_gpu, y_ref, bound, what="", dtype="fp16"):
    y = widen_output(y_gpu)
    rtol = RTOL_BF16 if dtype == "bf16" else RTOL_B
    err = np.abs(y - y_ref)
    lim = rtol * bound + ATOL
    bad = err > lim
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {bad.size} outputs outside |y-y_ref| <= {rtol:.4g}*B + 1e-5; "
            f"first {idx.tolist()}: y={y[bad][:5]}, ref={y_ref[bad][:5]}, B={bound[bad][:5]}")
    return float((err / lim).max()) if err.size else 0.0
