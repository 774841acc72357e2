"""The GPTQModel packed format on the GPU: conversion bit for bit against the
oracle, and the README's product computed through it against the oracle's
dequantize-then-matmul of the GPTQModel operands."""
import numpy as np
import pytest

import oracle.gptqmodel_format as gf
import oracle.numpy_oracle as no
import wq_inputs
from guard import Guarded
from parity import check_product

pytestmark = pytest.mark.gpu


def operands(M, K, N, bits, G, seed):
    rng = np.random.default_rng(seed)
    case = wq_inputs.custom(M, K, N, bits, G, seed=seed)
    groups = K // (K if G == -1 else G)
    zq = rng.integers(0, 1 << bits, size=(groups, N)).astype(np.uint8)
    return case, gf.pack_rows(case.codes, bits), gf.pack_zeros(zq, bits), zq


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
@pytest.mark.parametrize("K,N,G", [(256, 72, 64), (1024, 100 * 8, 128), (96 * 32 // 3 * 3, 40, -1)])
def test_conversion_bit_exact(cuda, libwq, bits, K, N, G):
    import torch
    if bits == 3 and K % 32:
        pytest.skip("3-bit planes need K % 32 == 0")
    if K % (32 // bits if bits != 3 else 32):
        pytest.skip("K not a multiple of the word width")
    case, qw, qz, zq = operands(1, K, N, bits, G, seed=K + N + bits)
    t = lambda a: torch.from_numpy(a.view(np.int32)).to(cuda)
    w_q, w_lo, zeros = libwq.from_gptqmodel(t(qw), t(qz), bits, G, K)
    torch.cuda.synchronize()
    ref_q, ref_lo = no.pack(case.codes, bits)
    assert np.array_equal(w_q.cpu().numpy().view(np.uint32), ref_q)
    if bits == 3:
        assert np.array_equal(w_lo.cpu().numpy().view(np.uint32), ref_lo)
    assert np.array_equal(zeros.float().cpu().numpy(), zq.astype(np.float32))
    zb = libwq.from_gptqmodel(t(qw), t(qz), bits, G, K, dtype=torch.bfloat16)[2]
    assert np.array_equal(zb.float().cpu().numpy(), zq.astype(np.float32))


@pytest.mark.parametrize("M,K,N,bits,G", [(1, 4096, 512, 4, 128), (5, 2048, 264, 3, 128),
                                          (64, 1024, 256, 2, 64), (300, 512, 136, 8, -1)])
def test_readme_product(cuda, libwq, M, K, N, bits, G):
    import torch
    case, qw, qz, zq = operands(M, K, N, bits, G, seed=M + K + N)
    t = lambda a: torch.from_numpy(a.view(np.int32)).to(cuda)
    x = torch.from_numpy(case.x).to(cuda)
    s = torch.from_numpy(case.scales).to(cuda)
    out = Guarded((M, N), torch.float16, cuda)
    y = libwq.gptqmodel_quantized_matmul(x, t(qw), t(qz), s, bits, G, out=out.view)
    torch.cuda.synchronize()
    assert out.intact()
    y_ref, b = gf.quantized_matmul(case.x, qw, qz, case.scales, bits, G)
    check_product(y.cpu().numpy(), y_ref, b, f"gptqmodel {(M, K, N, bits, G)}")


def test_rejected(cuda, libwq):
    import torch
    qw = torch.zeros((52, 8), dtype=torch.int32, device=cuda)   # ceil(512 / 10) rows: right for 3 bits
    qz = torch.zeros((4, 1), dtype=torch.int32, device=cuda)
    libwq.from_gptqmodel(qw, qz, 3, 128, 512)
    with pytest.raises(ValueError, match="qweight"):
        libwq.from_gptqmodel(qw[:51], qz, 3, 128, 512)
    with pytest.raises(ValueError, match="qzeros"):
        libwq.from_gptqmodel(qw, qz[:3], 3, 128, 512)
    with pytest.raises(ValueError):
        libwq.from_gptqmodel(qw, qz, 1, 128, 512)
