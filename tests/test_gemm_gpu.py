"""wq_gemm (tcgen05 tensor cores) against the fp64 oracle, element by element."""
import numpy as np
import pytest

import wq_inputs
from gpu_cases import oracle_product, to_dev
from guard import Guarded, Guarded1D
from parity import check_product

pytestmark = pytest.mark.gpu


def run_gemm(libwq, d, bits, G, **kw):
    """The product into an output with sentinel rows around it, which must survive."""
    w_q, w_lo = libwq.pack_kmajor(d["codes"], bits)
    M, N = d["x"].shape[0], w_q.shape[1]
    out = Guarded((M, N), d["x"].dtype, d["x"].device)
    y = libwq.gemm(d["x"], w_q, w_lo, d["scales"], d["zeros"], bits, G, out=out.view, **kw)
    assert out.intact(), "a store landed outside y"
    return y.cpu().numpy()


def test_prefill_workload_full(cuda, libwq, orc):
    """Every output of the M=512 x K=4096 x N=2048 4-bit product, in the bench's launch configuration."""
    case = wq_inputs.draw(wq_inputs.WORKLOADS["prefill_gemm"], seed=0)
    d = to_dev(case, cuda)
    y = run_gemm(libwq, d, 4, 128)
    y_ref, b = oracle_product(orc, case)
    check_product(y, y_ref, b, "prefill_gemm")


@pytest.mark.parametrize("name", ["tiny_gemv", "decode_gemv_m16", "gemv_3bit", "sweep_1bit",
                                  "sweep_8bit_perchannel"])
def test_gemv_workloads_through_gemm(cuda, libwq, orc, name):
    """The GEMV workloads also go through the batched path (any M)."""
    case = wq_inputs.draw(wq_inputs.WORKLOADS[name], seed=0)
    d = to_dev(case, cuda)
    y = run_gemm(libwq, d, case.wl.bits, case.wl.group_size)
    y_ref, b = oracle_product(orc, case)
    check_product(y, y_ref, b, name)


SHAPES = [
    # M, K, N, bits, G
    (1, 64, 8, 4, 64),          # one k block, one ragged column tile
    (5, 128, 136, 4, 32),       # two groups per k block
    (16, 4096, 128, 4, 128),    # one tile, split over an 8-CTA cluster
    (33, 512, 264, 8, 16),      # 4 groups per k block, ragged tiles
    (100, 1024, 256, 2, 64),
    (128, 256, 512, 1, 128),
    (200, 2048, 384, 3, 128),
    (256, 192, 1024, 3, -1),
    (300, 512, 128, 4, 64),     # two balanced token tiles of 160
    (512, 128, 8192, 8, 128),   # many tiles, no split
    (64, 8192, 136, 1, -1),
    (7, 4096, 2048, 2, 32),
    # ragged last 64-deep block, and groups whose boundaries fall inside a block
    (48, 4160, 264, 4, -1),     # K = 65 blocks: a ragged block, K split over clusters
    (3, 544, 64, 4, -1),
    (40, 576, 136, 4, 96),      # group 96 straddles blocks
    (24, 3072, 128, 3, 96),     # 3-bit planes with group 96
    (9, 520, 64, 8, 40),        # 8-bit, K = 8 blocks + 8, group 40
    (96, 1088, 256, 2, 64),     # 17 blocks
    (2, 96, 64, 4, 32),         # one and a half blocks
]


@pytest.mark.parametrize("M,K,N,bits,G", SHAPES)
def test_shapes(cuda, libwq, orc, M, K, N, bits, G):
    case = wq_inputs.custom(M, K, N, bits, G, seed=3 * M + K + N + bits)
    d = to_dev(case, cuda)
    y = run_gemm(libwq, d, bits, G)
    y_ref, b = oracle_product(orc, case)
    check_product(y, y_ref, b, f"{(M, K, N, bits, G)}")


@pytest.mark.parametrize("bits", [1, 2, 3, 4, 8])
def test_fractional_zero_points(cuda, libwq, orc, bits):
    import torch
    M, K, N, G = 48, 1024, 128, 64
    case = wq_inputs.custom(M, K, N, bits, G, seed=40 + bits)
    rng = np.random.default_rng(bits)
    case.zeros = rng.uniform(-0.5, (1 << bits) - 0.5, size=case.zeros.shape).astype(np.float16)
    d = to_dev(case, cuda)
    d["zeros"] = torch.from_numpy(case.zeros).to(cuda)
    y = run_gemm(libwq, d, bits, G)
    y_ref, b = oracle_product(orc, case)
    check_product(y, y_ref, b, f"fractional z, {bits}-bit")


@pytest.mark.parametrize("bits", [1, 2, 3, 4, 8])
def test_q_equals_z_gives_zero(cuda, libwq, bits):
    import torch
    M, K, N, G = 64, 512, 128, 128
    case = wq_inputs.custom(M, K, N, bits, G, seed=8)
    zq = np.random.default_rng(2).integers(0, 1 << bits, size=(K // G, N))
    d = to_dev(case, cuda)
    d["codes"] = torch.from_numpy(np.repeat(zq, G, axis=0).astype(np.uint8)).to(cuda)
    d["zeros"] = torch.from_numpy(zq.astype(np.float16)).to(cuda)
    y = run_gemm(libwq, d, bits, G)
    assert np.all(y.astype(np.float64) == 0.0)


@pytest.mark.parametrize("bits", [1, 2, 3, 4, 8])
def test_one_hot_rows_are_exact(cuda, libwq, bits):
    """x = e_k for 64 rows k gives fp16(w[k]) exactly."""
    import torch
    K, N, G = 1024, 256, 128
    case = wq_inputs.custom(64, K, N, bits, G, seed=13)
    ks = np.random.default_rng(4).choice(K, 64, replace=False)
    x = np.zeros((64, K), np.float16)
    x[np.arange(64), ks] = 1.0
    d = to_dev(case, cuda)
    d["x"] = torch.from_numpy(x).to(cuda)
    y = run_gemm(libwq, d, bits, G)
    g = ks // G
    w = (case.codes[ks].astype(np.float64) - case.zeros[g].astype(np.float64)) * case.scales[g].astype(np.float64)
    assert np.array_equal(y, w.astype(np.float16))


def test_deterministic_and_status(cuda, libwq):
    case = wq_inputs.draw(wq_inputs.WORKLOADS["prefill_gemm"], seed=1)
    d = to_dev(case, cuda)
    a = run_gemm(libwq, d, 4, 128)
    b = run_gemm(libwq, d, 4, 128, pdl=True)
    assert np.array_equal(a, b)
    assert libwq.device_status() == 0


def test_rejected_calls(cuda, libwq):
    """x must come in 16-byte rows for the tensor-memory copy engine: 8-bit
    codes with K = 516 pass every format rule but are refused (WQ_ERR_ALIGNMENT)."""
    case = wq_inputs.custom(4, 516, 64, 8, -1, seed=1)
    d = to_dev(case, cuda)
    w_q, _ = libwq.pack_kmajor(d["codes"], 8)
    with pytest.raises(libwq.WQError) as e:
        libwq.gemm(d["x"], w_q, None, d["scales"], d["zeros"], 8, -1)
    assert e.value.status == 3


def test_workspace_guards(cuda, libwq, orc):
    """The split-K workspace: nothing is written outside the bytes the size query names."""
    import torch
    M, K, N, bits, G = 64, 4096, 512, 4, 128
    case = wq_inputs.custom(M, K, N, bits, G, seed=11)
    d = to_dev(case, cuda)
    need = libwq.gemm_workspace_size(M, K, N, bits, G)
    assert need > 0
    ws = Guarded1D(need, torch.uint8, cuda)
    y = run_gemm(libwq, d, bits, G, workspace=ws.view)
    assert ws.intact(), "a store landed outside the workspace"
    y_ref, b = oracle_product(orc, case)
    check_product(y, y_ref, b, "workspace_guards")


def test_pdl_flags(cuda, libwq):
    """WQ_FLAG_PDL on a chain where each x is the previous y, and
    WQ_FLAG_PDL_INPUTS_READY on calls that overwrite the previous call's input
    and output, give the same bits as plain calls."""
    import torch
    M, K = 96, 1024
    case = wq_inputs.custom(M, K, K, 4, 128, seed=5)
    d = to_dev(case, cuda)
    w_q, w_lo = libwq.pack_kmajor(d["codes"], 4)
    s = d["scales"] * 0.1

    def chain(pdl):
        ys, x = [], d["x"]
        for _ in range(4):
            x = libwq.gemm(x, w_q, w_lo, s, d["zeros"], 4, 128, pdl=pdl)
            ys.append(x)
        torch.cuda.synchronize()
        return [y.cpu().numpy() for y in ys]

    for a, b in zip(chain(False), chain(True)):
        assert np.isfinite(a).all()
        assert np.array_equal(a, b)

    other = to_dev(wq_inputs.custom(M, K, K, 4, 128, seed=6), cuda)
    w2, _ = libwq.pack_kmajor(other["codes"], 4)
    ref0 = libwq.gemm(d["x"], w_q, None, s, d["zeros"], 4, 128).cpu().numpy()
    ref1 = libwq.gemm(other["x"], w2, None, other["scales"], other["zeros"], 4, 128).cpu().numpy()
    buf = d["x"].clone()
    y0 = torch.empty((M, K), dtype=torch.float16, device=cuda)
    libwq.gemm(buf, w_q, None, s, d["zeros"], 4, 128, out=y0)
    libwq.gemm(other["x"], w2, None, other["scales"], other["zeros"], 4, 128, out=buf, inputs_ready=True)
    torch.cuda.synchronize()
    assert np.array_equal(y0.cpu().numpy(), ref0)
    assert np.array_equal(buf.cpu().numpy(), ref1)
    assert libwq.device_status() == 0


@pytest.mark.parametrize("M,K,N,bits,G", [(512, 4096, 2048, 4, 128), (33, 512, 264, 8, 16),
                                         (200, 2048, 384, 3, 128)])
def test_bias_matches_oracle(cuda, libwq, orc, M, K, N, bits, G):
    """y = x @ w + bias through the split-K and single-CTA epilogues, against the oracle;
    wq_gemm_noalloc gives the same bits."""
    import torch
    case = wq_inputs.custom(M, K, N, bits, G, seed=M + bits)
    d = to_dev(case, cuda)
    bias_np = wq_inputs.bias_vector(N, seed=9)
    bias = torch.from_numpy(bias_np).to(cuda)
    w_q, w_lo = libwq.pack_kmajor(d["codes"], bits)
    y = libwq.gemm(d["x"], w_q, w_lo, d["scales"], d["zeros"], bits, G, bias=bias)
    y2 = torch.empty_like(y)
    libwq.gemm_noalloc(d["x"], w_q, w_lo, d["scales"], d["zeros"], bits, G, out=y2, bias=bias)
    torch.cuda.synchronize()
    assert torch.equal(y, y2)
    wq_, wlo_ = orc.pack(case.codes, bits)
    y_ref, b = orc.wq_matmul(case.x, wq_, wlo_, case.scales, case.zeros, bits, G, bias=bias_np)
    check_product(y.cpu().numpy(), y_ref, b, f"gemm {M}x{K}x{N} + bias")


@pytest.mark.parametrize("M", [1, 12, 16, 64])
def test_matmul_either_route_matches_oracle(cuda, libwq, orc, M):
    """wq_matmul over the crossover: both routes against the oracle."""
    K, N = 4096, 512
    case = wq_inputs.custom(M, K, N, 4, 128, seed=40 + M)
    d = to_dev(case, cuda)
    w_q, w_lo = libwq.pack_kmajor(d["codes"], 4)
    y = libwq.matmul(d["x"], w_q, w_lo, d["scales"], d["zeros"], 4, 128).cpu().numpy()
    assert libwq.uses_gemv(M, K, N, 4, 128) == (M <= 16)
    y_ref, b = oracle_product(orc, case)
    check_product(y, y_ref, b, f"matmul M={M}")
