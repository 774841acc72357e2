"""The C oracle and its separately written NumPy twin agree on random small problems."""
import numpy as np
import pytest

import wq_inputs


@pytest.mark.parametrize("bits", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("G", [32, 64, 128, -1])
@pytest.mark.parametrize("M", [1, 3, 16])
def test_c_vs_numpy(orc, bits, G, M):
    K, N = 256, 40
    case = wq_inputs.custom(M, K, N, bits, G, seed=bits * 100 + M)
    tw = orc.numpy_oracle
    wq, wlo = orc.pack(case.codes, bits)
    wq2, wlo2 = tw.pack(case.codes, bits)
    assert np.array_equal(wq, wq2)
    if bits == 3:
        assert np.array_equal(wlo, wlo2)
    assert np.array_equal(orc.unpack(wq, wlo, K, N, bits), tw.unpack(wq, wlo, K, N, bits))
    y, b = orc.wq_matmul(case.x, wq, wlo, case.scales, case.zeros, bits, G)
    y2, b2 = tw.wq_matmul(case.x, wq, wlo, case.scales, case.zeros, bits, G)
    assert np.all(np.abs(y - y2) <= 1e-12 * b + 1e-300)
    assert np.allclose(b, b2, rtol=1e-12, atol=0)


def test_sampled_equals_full(orc):
    case = wq_inputs.custom(4, 512, 96, 4, 128, seed=11)
    wq, wlo = orc.pack(case.codes, 4)
    y, b = orc.wq_matmul(case.x, wq, wlo, case.scales, case.zeros, 4, 128)
    rng = np.random.default_rng(5)
    ms = rng.integers(0, 4, 50)
    ns = rng.integers(0, 96, 50)
    ys, bs = orc.wq_matmul_sampled(case.x, wq, wlo, case.scales, case.zeros, 4, 128, ms, ns)
    assert np.array_equal(ys, y[ms, ns])
    assert np.array_equal(bs, b[ms, ns])


@pytest.mark.parametrize("bits", [1, 3, 4, 8])
@pytest.mark.parametrize("G", [32, -1])
def test_c_vs_numpy_bf16(orc, bits, G):
    K, N, M = 256, 40, 5
    case = wq_inputs.custom(M, K, N, bits, G, seed=bits * 10 + 3, dtype="bf16")
    bias = wq_inputs.bias_vector(N, seed=bits, dtype="bf16")
    tw = orc.numpy_oracle
    wq, wlo = orc.pack(case.codes, bits)
    y, b = orc.wq_matmul(case.x, wq, wlo, case.scales, case.zeros, bits, G, bias=bias, dtype="bf16")
    y2, b2 = tw.wq_matmul(case.x, wq, wlo, case.scales, case.zeros, bits, G, bias=bias, dtype="bf16")
    assert np.all(np.abs(y - y2) <= 1e-12 * b + 1e-300)
    assert np.allclose(b, b2, rtol=1e-12, atol=0)


def test_sampled_equals_full_bf16(orc):
    case = wq_inputs.custom(4, 512, 96, 3, 64, seed=12, dtype="bf16")
    bias = wq_inputs.bias_vector(96, seed=2, dtype="bf16")
    wq, wlo = orc.pack(case.codes, 3)
    y, b = orc.wq_matmul(case.x, wq, wlo, case.scales, case.zeros, 3, 64, bias=bias, dtype="bf16")
    rng = np.random.default_rng(6)
    ms = rng.integers(0, 4, 50)
    ns = rng.integers(0, 96, 50)
    ys, bs = orc.wq_matmul_sampled(case.x, wq, wlo, case.scales, case.zeros, 3, 64, ms, ns,
                                   bias=bias, dtype="bf16")
    assert np.array_equal(ys, y[ms, ns])
    assert np.array_equal(bs, b[ms, ns])
