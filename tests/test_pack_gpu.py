"""GPU packing and unpacking are bit-exact against the oracle."""
import numpy as np
import pytest

import wq_inputs
from _golden import read_cases, words
from gpu_cases import to_dev

pytestmark = pytest.mark.gpu


def _u32(t):
    return t.cpu().numpy().view(np.uint32)


@pytest.mark.parametrize("name", sorted(read_cases("pack_words.txt")))
def test_golden_words(cuda, libwq, name):
    import torch
    c = read_cases("pack_words.txt")[name]
    K, N, bits = c["K"], c["N"], c["bits"]
    codes = torch.tensor(c["codes"], dtype=torch.uint8).reshape(K, N).to(cuda)
    w_q, w_lo = libwq.pack_kmajor(codes, bits)
    assert np.array_equal(_u32(w_q), words(c, "wq", N))
    if bits == 3:
        assert np.array_equal(_u32(w_lo), words(c, "wlo", N))
    assert np.array_equal(libwq.unpack_kmajor(w_q, w_lo, K, bits).cpu().numpy(),
                          np.array(c["codes"], np.uint8).reshape(K, N))


@pytest.mark.parametrize("bits", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("K,N", [(32, 1), (64, 5), (96, 1000), (512, 256), (1024, 4104)])
def test_random_codes_bit_exact(cuda, libwq, orc, bits, K, N):
    case = wq_inputs.custom(1, K, N, bits, -1, seed=K + N + bits)
    codes = case.codes.copy()
    codes[:, 0] = (1 << bits) - 1          # every bit position set in column 0
    d = to_dev(case, cuda)
    import torch
    d["codes"] = torch.from_numpy(codes).to(cuda)
    w_q, w_lo = libwq.pack_kmajor(d["codes"], bits)
    ref_q, ref_lo = orc.pack(codes, bits)
    assert np.array_equal(_u32(w_q), ref_q)
    if bits == 3:
        assert np.array_equal(_u32(w_lo), ref_lo)
    back = libwq.unpack_kmajor(w_q, w_lo, K, bits).cpu().numpy()
    assert np.array_equal(back, codes)


@pytest.mark.parametrize("name", ["decode_gemv_m1", "gemv_3bit", "sweep_1bit", "sweep_2bit",
                                  "sweep_8bit", "prefill_gemm"])
def test_full_size_workloads_bit_exact(cuda, libwq, orc, name):
    case = wq_inputs.draw(wq_inputs.WORKLOADS[name], seed=0)
    d = to_dev(case, cuda)
    bits = case.wl.bits
    w_q, w_lo = libwq.pack_kmajor(d["codes"], bits)
    ref_q, ref_lo = orc.pack(case.codes, bits)
    assert np.array_equal(_u32(w_q), ref_q)
    if bits == 3:
        assert np.array_equal(_u32(w_lo), ref_lo)
    back = libwq.unpack_kmajor(w_q, w_lo, case.wl.K, bits)
    assert bool((back == d["codes"]).all())


@pytest.mark.parametrize("bits", [1, 2, 4])
def test_out_of_range_codes_are_reported(cuda, libwq, bits):
    import torch
    codes = torch.zeros((64, 8), dtype=torch.uint8, device=cuda)
    codes[5, 3] = 1 << bits
    with pytest.raises(libwq.WQError) as e:
        libwq.pack_kmajor(codes, bits)
    assert e.value.status == 4
    # without the check the code is masked: no neighbouring field changes
    w_q, _ = libwq.pack_kmajor(codes, bits, check_range=False)
    assert int(w_q.abs().sum().item()) == 0


def test_bad_arguments_raise_before_launch(cuda, libwq):
    import torch
    codes = torch.zeros((12, 8), dtype=torch.uint8, device=cuda)
    with pytest.raises(libwq.WQError) as e:
        libwq.pack_kmajor(codes, 4)
    assert e.value.status == 1


@pytest.mark.parametrize("bits", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("K,N", [(32, 1), (96, 1000), (64, 5)])
def test_packing_stays_inside_its_planes(cuda, libwq, orc, bits, K, N):
    """Pack and unpack through the C ABI into buffers with sentinel rows around
    them: every word and code lands inside its plane, none outside."""
    import torch
    from guard import Guarded
    case = wq_inputs.custom(1, K, N, bits, -1, seed=7 * K + N + bits)
    codes = torch.from_numpy(case.codes).to(cuda)
    hs, ls = libwq.words_shape(K, N, bits)
    gq = Guarded(hs, torch.int32, cuda)
    glo = Guarded(ls, torch.int32, cuda) if ls else None
    stream = torch.cuda.current_stream().cuda_stream
    st = libwq.lib().wq_pack_kmajor(codes.data_ptr(), K, N, bits, gq.view.data_ptr(),
                                    glo.view.data_ptr() if glo else None, None, stream)
    assert st == 0
    assert gq.intact() and (glo is None or glo.intact())
    ref_q, ref_lo = orc.pack(case.codes, bits)
    assert np.array_equal(_u32(gq.view), ref_q)
    if bits == 3:
        assert np.array_equal(_u32(glo.view), ref_lo)
    back = Guarded((K, N), torch.uint8, cuda)
    st = libwq.lib().wq_unpack_kmajor(gq.view.data_ptr(), glo.view.data_ptr() if glo else None, K, N, bits,
                                      back.view.data_ptr(), stream)
    assert st == 0
    assert back.intact()
    assert np.array_equal(back.view.cpu().numpy(), case.codes)
