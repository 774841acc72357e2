"""Parity at the largest shapes the library is timed on, on sampled outputs.

The full fp64 product of these shapes would take the oracle minutes, so each
test checks a few thousand outputs (m, n), each computed on its own by the
oracle straight from the packed words (``wq_matmul_sampled``), plus every
output for finiteness.  The samples include the first and last token and
column and the boundaries of the 128-column tiles.
"""
import numpy as np
import pytest

import wq_inputs
from gpu_cases import to_dev
from parity import check_product, widen_output

pytestmark = pytest.mark.gpu


def _samples(M, N, count, seed):
    rng = np.random.default_rng(seed)
    ms = rng.integers(0, M, count)
    ns = rng.integers(0, N, count)
    edge_n = np.array([0, 1, 127, 128, N - 129, N - 128, N - 2, N - 1])
    edge_m = np.array([0, M - 1])
    em, en = np.meshgrid(edge_m, edge_n, indexing="ij")
    return np.concatenate([ms, em.ravel()]), np.concatenate([ns, en.ravel()])


def _check_sampled(orc, case, y, what, count=3000, seed=0):
    M, N = case.wl.M, case.wl.N
    yh = widen_output(y)
    assert np.isfinite(yh).all(), what
    ms, ns = _samples(M, N, count, seed)
    wq, wlo = orc.pack(case.codes, case.wl.bits)
    y_ref, b = orc.wq_matmul_sampled(case.x, wq, wlo, case.scales, case.zeros, case.wl.bits,
                                     case.wl.group_size, ms, ns, dtype=case.dtype)
    check_product(yh[ms, ns], y_ref, b, what, dtype=case.dtype)


@pytest.mark.parametrize("dtype", ["fp16"])
def test_gemm_large(cuda, libwq, orc, dtype):
    """M=256 x K=16384 x N=18944, 4-bit group 128: 64 k blocks per CTA, 148 tiles, no split."""
    import torch
    case = wq_inputs.custom(256, 16384, 18944, 4, 128, seed=21, dtype=dtype)
    d = to_dev(case, cuda)
    w_q, w_lo = libwq.pack_kmajor(d["codes"], 4)
    del d["codes"]
    y = libwq.gemm(d["x"], w_q, w_lo, d["scales"], d["zeros"], 4, 128)
    torch.cuda.synchronize()
    assert libwq.device_status() == 0
    _check_sampled(orc, case, y, f"gemm 256x16384x18944 {dtype}")


@pytest.mark.parametrize("M,K,N,bits,G,dtype", [(16, 16384, 16384, 4, 128, "bf16"),
                                               (1, 16384, 8192, 3, 128, "fp16"),
                                               (8, 4096, 65536, 2, 64, "bf16"),
                                               (3, 32768, 4096, 8, -1, "fp16")])
def test_gemv_large(cuda, libwq, orc, M, K, N, bits, G, dtype):
    """Long K (up to 32768), wide N (up to 65536) and all 16 tokens on the decode kernel."""
    import torch
    case = wq_inputs.custom(M, K, N, bits, G, seed=M + K // 1024 + bits, dtype=dtype)
    d = to_dev(case, cuda)
    w_q, w_lo = libwq.pack_kmajor(d["codes"], bits)
    del d["codes"]
    y = libwq.gemv(d["x"], w_q, w_lo, d["scales"], d["zeros"], bits, G)
    torch.cuda.synchronize()
    assert libwq.device_status() == 0
    _check_sampled(orc, case, y, f"gemv {M}x{K}x{N} {bits}-bit G{G} {dtype}", count=2000)
