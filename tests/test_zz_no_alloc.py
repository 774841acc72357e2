"""wq_gemm_noalloc: the batched product with the library's fixed split-K
scratch, against wq_gemm with a caller workspace (bit for bit) and the fp64
oracle (within the product tolerance).

The file name sorts last so that these tests also run after every other test
in one process; they must pass alone in a fresh process too.
"""
import ctypes

import numpy as np
import pytest

import wq_inputs
from gpu_cases import oracle_product, to_dev
from parity import check_product

SCRATCH_LIMIT = 7
SCRATCH_BYTES = 16 << 20
P = 0x10000  # 16-byte aligned fake device address, never dereferenced on a rejected call

# M, K, N, bits, G: every shape splits K, so the scratch is in use
SHAPES = [
    (512, 4096, 2048, 4, 128),   # the prefill workload: 16 MiB of scratch, the whole array
    (16, 4096, 4096, 4, 128),    # 32 tiles, 4-CTA clusters
    (100, 1024, 1000, 3, 128),   # ragged tokens and columns, 3-bit planes
    (64, 8192, 136, 8, -1),      # per-channel, 8-CTA clusters
]


def test_rejects_shapes_beyond_the_scratch(libwq):
    """Host-side: 74 column tiles x 2-CTA clusters x 8 slices of 16 KiB need
    19 MiB (148 SMs, also assumed without a device): rejected before launch."""
    L = libwq.lib()
    assert L.wq_gemm_workspace_size(256, 4096, 9472, 4, 128) > SCRATCH_BYTES
    st = L.wq_gemm_noalloc(P, P, None, P, P, None, P, 256, 4096, 9472, 4, 128, 0, None)
    assert st == SCRATCH_LIMIT
    assert L.wq_status_string(SCRATCH_LIMIT)


@pytest.mark.gpu
@pytest.mark.parametrize("M,K,N,bits,G", SHAPES)
def test_matches_wq_gemm_on_two_calls_in_a_row(cuda, libwq, orc, M, K, N, bits, G):
    import torch
    need = libwq.gemm_workspace_size(M, K, N, bits, G)
    assert 0 < need <= SCRATCH_BYTES
    case = wq_inputs.custom(M, K, N, bits, G, seed=7 * M + N + bits)
    d = to_dev(case, cuda)
    w_q, w_lo = libwq.pack_kmajor(d["codes"], bits)
    ws = torch.empty(need, dtype=torch.uint8, device=cuda)
    ref = libwq.gemm(d["x"], w_q, w_lo, d["scales"], d["zeros"], bits, G, workspace=ws)
    outs = []
    for _ in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.float16, device=cuda)
        libwq.gemm_noalloc(d["x"], w_q, w_lo, d["scales"], d["zeros"], bits, G, out=y)
        outs.append(y)
    torch.cuda.synchronize()
    for y in outs:
        assert torch.equal(y, ref)
    y_ref, b = oracle_product(orc, case)
    check_product(outs[1].cpu().numpy(), y_ref, b, f"noalloc {M}x{K}x{N} {bits}-bit G{G}")
    assert libwq.device_status() == 0


@pytest.mark.gpu
def test_no_device_memory_taken_per_call(cuda, libwq):
    """After the first call (which may load the library's device image), calls
    leave the device's free memory unchanged."""
    import torch
    M, K, N, bits, G = SHAPES[1]
    case = wq_inputs.custom(M, K, N, bits, G, seed=1)
    d = to_dev(case, cuda)
    w_q, w_lo = libwq.pack_kmajor(d["codes"], bits)
    y = torch.empty((M, N), dtype=torch.float16, device=cuda)
    libwq.gemm_noalloc(d["x"], w_q, w_lo, d["scales"], d["zeros"], bits, G, out=y)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info(cuda)[0]
    for _ in range(3):
        libwq.gemm_noalloc(d["x"], w_q, w_lo, d["scales"], d["zeros"], bits, G, out=y)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info(cuda)[0] == free0
    assert libwq.device_status() == 0


@pytest.mark.gpu
def test_rejected_on_the_device_too(cuda, libwq):
    """The scratch limit holds on a B200 (148 SMs): nothing is launched and y is untouched."""
    import torch
    if torch.cuda.get_device_properties(cuda).multi_processor_count != 148:
        pytest.skip("the split-K plan, and so which shapes exceed the scratch, follows the SM count")
    M, K, N = 256, 4096, 9472
    x = torch.zeros((M, K), dtype=torch.float16, device=cuda)
    w_q = torch.zeros((K // 8, N), dtype=torch.int32, device=cuda)
    s = torch.zeros((K // 128, N), dtype=torch.float16, device=cuda)
    y = torch.full((M, N), 3.0, dtype=torch.float16, device=cuda)
    with pytest.raises(libwq.WQError) as e:
        libwq.gemm_noalloc(x, w_q, None, s, s, 4, 128, out=y)
    assert e.value.status == SCRATCH_LIMIT
    torch.cuda.synchronize()
    assert bool((y == 3.0).all())
