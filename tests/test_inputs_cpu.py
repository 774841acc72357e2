"""The seeded input generator: bf16 rounding equals torch's, fp16 and bf16 problems share one
stream of draws, and the draws are deterministic and inside their stated ranges."""
import numpy as np
import torch

import wq_inputs


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    v = np.concatenate([rng.standard_normal(10000) * 10.0 ** rng.integers(-20, 20, 10000),
                        [0.0, -0.0, 1.0, 1.00390625, 1.01171875, -3.0, 65504.0, 1e30]])
    ours = wq_inputs.bf16_bits(v)
    ref = torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_same_stream_for_both_types():
    wl = wq_inputs.WORKLOADS["tiny_gemv"]
    a = wq_inputs.draw(wl, seed=4)
    b = wq_inputs.draw(wl, seed=4, dtype="bf16")
    assert np.array_equal(a.codes, b.codes)
    # the same draws, rounded to each type: zeros are integers (exact in both)
    zb = (b.zeros.astype(np.uint32) << 16).view(np.float32)
    assert np.array_equal(a.zeros.astype(np.float32), zb)
    xb = (b.x.astype(np.uint32) << 16).view(np.float32)
    assert np.all(np.abs(xb - a.x.astype(np.float32)) <= 2.0 ** -8 * np.abs(xb) + 2.0 ** -24)


def test_deterministic_and_in_range():
    for name, wl in wq_inputs.WORKLOADS.items():
        if wl.K * wl.N > 1 << 24:
            continue
        a = wq_inputs.draw(wl, seed=0)
        b = wq_inputs.draw(wl, seed=0)
        assert np.array_equal(a.codes, b.codes) and np.array_equal(a.x, b.x), name
        assert a.codes.max() <= (1 << wl.bits) - 1, name
        assert a.scales.min() >= np.float16(wl.s_lo) and a.scales.max() <= np.float16(wl.s_hi), name
        assert a.scales.shape == (wl.groups, wl.N) and a.x.shape == (wl.M, wl.K), name


def test_gptq_problem_recipe():
    """The GPTQ benchmark's problem: W inside +-1/sqrt(cols), H = A A^T + I
    symmetric with every eigenvalue at least 1 (up to fp32 rounding), the same
    bytes for the same seed."""
    W, H = wq_inputs.gptq_problem(16, 96, seed=3)
    assert W.dtype == np.float32 and H.dtype == np.float32
    assert W.shape == (16, 96) and H.shape == (96, 96)
    assert np.abs(W).max() <= 1 / np.sqrt(96)
    np.testing.assert_allclose(H, H.T, rtol=1e-6, atol=1e-4)
    assert np.linalg.eigvalsh(H.astype(np.float64)).min() > 1 - 1e-3
    W2, H2 = wq_inputs.gptq_problem(16, 96, seed=3)
    assert np.array_equal(W, W2) and np.array_equal(H, H2)
