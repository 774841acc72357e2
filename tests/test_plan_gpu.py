"""wq_gemv_plan (weights bound once, x per call): the same bits as wq_gemv, and
the oracle's product."""
import numpy as np
import pytest

import wq_inputs
from gpu_cases import host, oracle_product, to_dev
from parity import check_product

pytestmark = pytest.mark.gpu

# (M, K, N, bits, G, dtype, flags): both GEMV kernels, their plans and flags
CASES = [
    (1, 4096, 4096, 4, 128, "fp16", {"inputs_ready": True}),   # the decode layer
    (1, 4096, 4096, 4, 128, "fp16", {"pdl": True}),            # x staged (a chain)
    (4, 4096, 1024, 8, 128, "bf16", {}),
    (16, 2048, 512, 4, -1, "fp16", {}),
    (3, 16384, 64, 4, 128, "fp16", {"inputs_ready": True}),    # a cluster along K
    (2, 1024, 200, 3, 64, "fp16", {}),                         # 3-bit: the table kernel
    (12, 512, 136, 1, 128, "bf16", {"pdl": True}),
]


@pytest.mark.parametrize("M,K,N,bits,G,dtype,flags", CASES)
def test_plan_equals_gemv(cuda, libwq, orc, M, K, N, bits, G, dtype, flags):
    import torch
    case = wq_inputs.custom(M, K, N, bits, G, seed=M + K + N + bits, dtype=dtype)
    d = to_dev(case, cuda)
    w_q, w_lo = libwq.pack_kmajor(d["codes"], bits)
    plan = libwq.GemvPlan(w_q, w_lo, d["scales"], d["zeros"], bits, G, M, **flags)
    y_plan = plan(d["x"])
    y_call = libwq.gemv(d["x"], w_q, w_lo, d["scales"], d["zeros"], bits, G, **flags)
    torch.cuda.synchronize()
    a = y_plan.view(torch.int16).cpu().numpy()
    b = y_call.view(torch.int16).cpu().numpy()
    assert np.array_equal(a, b)
    y_ref, bound = oracle_product(orc, case)
    check_product(host(y_plan), y_ref, bound, f"plan {(M, K, N, bits, G, dtype, flags)}", dtype=dtype)


def test_plan_takes_a_new_x_and_out_each_call(cuda, libwq):
    import torch
    M, K, N = 2, 4096, 512
    case = wq_inputs.custom(M, K, N, 4, 128, seed=3)
    d = to_dev(case, cuda)
    w_q, _ = libwq.pack_kmajor(d["codes"], 4)
    bias = torch.randn(N, device=cuda).half()
    plan = libwq.GemvPlan(w_q, None, d["scales"], d["zeros"], 4, 128, M, bias=bias)
    out = torch.empty((M, N), dtype=torch.float16, device=cuda)
    for seed in range(3):
        x = torch.randn((M, K), device=cuda).half()
        plan(x, out=out)
        ref = libwq.gemv(x, w_q, None, d["scales"], d["zeros"], 4, 128, bias=bias)
        torch.cuda.synchronize()
        assert torch.equal(out, ref)


def test_plan_rejects_bad_x(cuda, libwq):
    import torch
    M, K, N = 1, 1024, 256
    case = wq_inputs.custom(M, K, N, 4, 128, seed=4)
    d = to_dev(case, cuda)
    w_q, _ = libwq.pack_kmajor(d["codes"], 4)
    plan = libwq.GemvPlan(w_q, None, d["scales"], d["zeros"], 4, 128, M)
    with pytest.raises(ValueError):
        plan(torch.zeros((2, K), dtype=torch.float16, device=cuda))        # shape
    with pytest.raises(ValueError):
        plan(torch.zeros((M, K), dtype=torch.bfloat16, device=cuda))       # type
    flat = torch.zeros(M * K + 8, dtype=torch.float16, device=cuda)
    with pytest.raises(libwq.WQError):
        plan(flat[1:1 + M * K].view(M, K))                                 # 2-byte aligned only
    with pytest.raises(libwq.WQError):  # a group size that does not divide K
        libwq.GemvPlan(w_q, None, d["scales"], d["zeros"], 4, 96, M)
