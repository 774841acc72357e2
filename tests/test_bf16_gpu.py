"""bf16 products (WQ_FLAG_BF16: x, scales, zeros, bias and y in bfloat16)
against the fp64 oracle on the same bf16 bytes, element by element.

The bar is the bf16 tolerance derived in parity.py (3u + 2^-10 of B); the
closed forms (q == z gives 0, a one-hot x gives bf16(w[k]) exactly) are
checked bit for bit.
"""
import numpy as np
import pytest

import wq_inputs
from gpu_cases import host, oracle_product, tensor, to_dev
from parity import check_product

pytestmark = pytest.mark.gpu

BF = "bf16"


def _run(libwq, fn, d, bits, G, **kw):
    w_q, w_lo = libwq.pack_kmajor(d["codes"], bits)
    return getattr(libwq, fn)(d["x"], w_q, w_lo, d["scales"], d["zeros"], bits, G, **kw)


@pytest.mark.parametrize("name", ["decode_gemv_m1", "decode_gemv_m16", "gemv_3bit", "sweep_1bit",
                                  "sweep_2bit", "sweep_8bit_perchannel"])
@pytest.mark.parametrize("ready", [False, True])
def test_gemv_workloads_full(cuda, libwq, orc, name, ready):
    """Every output of the decode workloads drawn in bf16, in both launch plans."""
    import torch
    case = wq_inputs.draw(wq_inputs.WORKLOADS[name], seed=0, dtype=BF)
    d = to_dev(case, cuda)
    torch.cuda.synchronize()
    y = _run(libwq, "gemv", d, case.wl.bits, case.wl.group_size, inputs_ready=ready)
    assert y.dtype == torch.bfloat16
    y_ref, b = oracle_product(orc, case)
    check_product(y, y_ref, b, name + " bf16", dtype=BF)
    assert libwq.device_status() == 0


def test_prefill_gemm_full(cuda, libwq, orc):
    """Every output of the M=512 x K=4096 x N=2048 4-bit product in bf16 (split-K cluster)."""
    case = wq_inputs.draw(wq_inputs.WORKLOADS["prefill_gemm"], seed=0, dtype=BF)
    d = to_dev(case, cuda)
    y = _run(libwq, "gemm", d, 4, 128)
    y_ref, b = oracle_product(orc, case)
    check_product(y, y_ref, b, "prefill_gemm bf16", dtype=BF)


GEMV_SHAPES = [
    # M, K, N, bits, G
    (1, 32, 8, 4, 32),
    (3, 40, 16, 4, -1),
    (2, 1024, 40, 8, 16),
    (8, 512, 128, 2, 64),
    (16, 1024, 136, 1, 128),
    (1, 1024, 200, 3, 64),
    (12, 2048, 56, 3, 128),
    (4, 8192, 16, 4, 128),
    (1, 8192, 128, 2, 128),   # 2-bit words on the lean kernel
    (11, 2048, 72, 2, -1),
    (1, 8192, 128, 1, 128),   # 1-bit words on the lean kernel
    (6, 4096, 64, 1, -1),
]


@pytest.mark.parametrize("M,K,N,bits,G", GEMV_SHAPES)
def test_gemv_shapes(cuda, libwq, orc, M, K, N, bits, G):
    case = wq_inputs.custom(M, K, N, bits, G, seed=M * 5 + K + N + bits, dtype=BF)
    y = _run(libwq, "gemv", to_dev(case, cuda), bits, G)
    y_ref, b = oracle_product(orc, case)
    check_product(y, y_ref, b, f"gemv bf16 {(M, K, N, bits, G)}", dtype=BF)


GEMM_SHAPES = [
    (1, 64, 8, 4, 64),
    (5, 128, 136, 4, 32),
    (16, 4096, 128, 4, 128),
    (33, 512, 264, 8, 16),
    (100, 1024, 256, 2, 64),
    (128, 256, 512, 1, 128),
    (200, 2048, 384, 3, 128),
    (300, 512, 128, 4, 64),
    (64, 8192, 136, 1, -1),
]


@pytest.mark.parametrize("M,K,N,bits,G", GEMM_SHAPES)
def test_gemm_shapes(cuda, libwq, orc, M, K, N, bits, G):
    case = wq_inputs.custom(M, K, N, bits, G, seed=3 * M + K + N + bits, dtype=BF)
    y = _run(libwq, "gemm", to_dev(case, cuda), bits, G)
    y_ref, b = oracle_product(orc, case)
    check_product(y, y_ref, b, f"gemm bf16 {(M, K, N, bits, G)}", dtype=BF)


@pytest.mark.parametrize("fn,M", [("gemv", 3), ("gemm", 48)])
@pytest.mark.parametrize("bits", [1, 2, 3, 4, 8])
def test_fractional_and_out_of_range_zero_points(cuda, libwq, orc, fn, M, bits):
    """Zero points anywhere in [-3, 2^bits + 3), most of them not integers:
    the integer part used by the exact conversion is clamped to [0, 2^bits - 1]
    and the rest applied separately."""
    K, N, G = 1024, 128, (128 if bits in (1, 2, 3) else 64)
    case = wq_inputs.custom(M, K, N, bits, G, seed=60 + bits, dtype=BF)
    rng = np.random.default_rng(100 + bits)
    case.zeros = wq_inputs.bf16_bits(rng.uniform(-3.0, (1 << bits) + 3.0, size=case.zeros.shape))
    y = _run(libwq, fn, to_dev(case, cuda), bits, G)
    y_ref, b = oracle_product(orc, case)
    check_product(y, y_ref, b, f"{fn} bf16 zeros, {bits}-bit", dtype=BF)


@pytest.mark.parametrize("fn,M", [("gemv", 1), ("gemv", 16), ("gemm", 40)])
@pytest.mark.parametrize("bits", [1, 2, 3, 4, 8])
def test_q_equals_z_gives_zero(cuda, libwq, fn, M, bits):
    K, N, G = 512, 64, 128
    case = wq_inputs.custom(M, K, N, bits, G, seed=8, dtype=BF)
    zq = np.random.default_rng(11).integers(0, 1 << bits, size=(K // G, N))
    case.codes = np.repeat(zq, G, axis=0).astype(np.uint8)
    case.zeros = wq_inputs.bf16_bits(zq)
    y = host(_run(libwq, fn, to_dev(case, cuda), bits, G))
    assert np.all(y == 0.0)


@pytest.mark.parametrize("fn", ["gemv", "gemm"])
@pytest.mark.parametrize("bits", [1, 2, 3, 4, 8])
def test_one_hot_rows_are_exact(cuda, libwq, fn, bits):
    """x = e_k gives bf16(w[k]) exactly: (q - z) * s has at most 16 significant
    bits, so it is exact in fp32 and rounds once, the same way on both sides."""
    import torch
    K, N, G = 512, 64, 128
    case = wq_inputs.custom(16, K, N, bits, G, seed=33, dtype=BF)
    ks = np.random.default_rng(4).choice(K, 16, replace=False)
    x = np.zeros((16, K), np.uint16)
    x[np.arange(16), ks] = 0x3F80  # 1.0
    case.x = x
    y = host(_run(libwq, fn, to_dev(case, cuda), bits, G))
    g = ks // G
    s = torch.from_numpy(case.scales.view(np.int16)).view(torch.bfloat16).double().numpy()
    z = torch.from_numpy(case.zeros.view(np.int16)).view(torch.bfloat16).double().numpy()
    w = (case.codes[ks].astype(np.float64) - z[g]) * s[g]
    expect = torch.from_numpy(w.astype(np.float32)).to(torch.bfloat16).double().numpy()
    assert np.array_equal(y, expect)


@pytest.mark.parametrize("fn,M", [("gemv", 4), ("gemm", 64)])
def test_values_beyond_fp16_range(cuda, libwq, orc, fn, M):
    """x around 2^40 and scales around 2^-50 (neither fits fp16): the product is
    computed in bf16's range, not through fp16."""
    K, N, G, bits = 1024, 256, 128, 4
    case = wq_inputs.custom(M, K, N, bits, G, seed=70, dtype=BF)
    rng = np.random.default_rng(71)
    case.x = wq_inputs.bf16_bits(rng.standard_normal((M, K)) * 2.0 ** 40)
    case.scales = wq_inputs.bf16_bits(rng.uniform(0.5, 1.0, size=case.scales.shape) * 2.0 ** -50)
    y = _run(libwq, fn, to_dev(case, cuda), bits, G)
    y_ref, b = oracle_product(orc, case)
    assert np.all(np.abs(y_ref) < 2.0 ** 8) and np.any(np.abs(y_ref) > 2.0 ** -12)
    check_product(y, y_ref, b, f"{fn} bf16 wide range", dtype=BF)


@pytest.mark.parametrize("fn,M,K,N,bits,G", [("gemv", 1, 4096, 4096, 4, 128), ("gemv", 16, 4096, 11008, 3, 128),
                                              ("gemm", 512, 4096, 2048, 4, 128), ("gemm", 33, 512, 264, 8, 16)])
def test_bias_matches_oracle(cuda, libwq, orc, fn, M, K, N, bits, G):
    import torch
    case = wq_inputs.custom(M, K, N, bits, G, seed=M + bits + 1, dtype=BF)
    bias = wq_inputs.bias_vector(N, seed=12, dtype=BF)
    d = to_dev(case, cuda)
    y = _run(libwq, fn, d, bits, G, bias=tensor(bias, cuda, BF))
    if fn == "gemm":
        w_q, w_lo = libwq.pack_kmajor(d["codes"], bits)
        y2 = torch.empty_like(y)
        libwq.gemm_noalloc(d["x"], w_q, w_lo, d["scales"], d["zeros"], bits, G, out=y2,
                           bias=tensor(bias, cuda, BF))
        torch.cuda.synchronize()
        assert torch.equal(y, y2)
    y_ref, b = oracle_product(orc, case, bias=bias)
    check_product(y, y_ref, b, f"{fn} bf16 + bias", dtype=BF)


@pytest.mark.parametrize("M", [1, 12, 16, 64])
def test_matmul_either_route(cuda, libwq, orc, M):
    K, N = 4096, 512
    case = wq_inputs.custom(M, K, N, 4, 128, seed=80 + M, dtype=BF)
    y = _run(libwq, "matmul", to_dev(case, cuda), 4, 128)
    y_ref, b = oracle_product(orc, case)
    check_product(y, y_ref, b, f"matmul bf16 M={M}", dtype=BF)


def test_pdl_chain(cuda, libwq):
    """WQ_FLAG_PDL in bf16: a chain where each x is the previous y gives the
    same bits as the same calls run one at a time."""
    import torch
    K = N = 1024
    case = wq_inputs.custom(4, K, N, 4, 128, seed=13, dtype=BF)
    d = to_dev(case, cuda)
    w_q, w_lo = libwq.pack_kmajor(d["codes"], 4)
    s = d["scales"] * 0.1

    def chain(one_at_a_time):
        ys, x = [], d["x"]
        for _ in range(4):
            x = libwq.gemv(x, w_q, w_lo, s, d["zeros"], 4, 128, pdl=True)
            ys.append(x)
            if one_at_a_time:
                torch.cuda.synchronize()
        torch.cuda.synchronize()
        return [host(y) for y in ys]

    for a, b in zip(chain(True), chain(False)):
        assert np.isfinite(a).all() and np.any(a != 0)
        assert np.array_equal(a, b)


def test_mixed_element_types_are_refused(cuda, libwq):
    import torch
    case = wq_inputs.custom(1, 512, 256, 4, 128, seed=1, dtype=BF)
    d = to_dev(case, cuda)
    w_q, _ = libwq.pack_kmajor(d["codes"], 4)
    with pytest.raises(TypeError, match="scales"):
        libwq.gemv(d["x"], w_q, None, d["scales"].half(), d["zeros"], 4, 128)
    with pytest.raises(TypeError, match="bias"):
        libwq.gemm(d["x"], w_q, None, d["scales"], d["zeros"], 4, 128,
                   bias=torch.zeros(256, dtype=torch.float16, device=cuda))
    with pytest.raises(TypeError, match="out"):
        libwq.gemv(d["x"], w_q, None, d["scales"], d["zeros"], 4, 128,
                   out=torch.empty((1, 256), dtype=torch.float16, device=cuda))
