"""wq_gptq_quantize against the GPTQ oracle (``oracle/gptq.py``).

Where no error reaches another column (diagonal Hessians, the hand-worked
cases) every code and every fake-quantised weight is decided by the same fp32
operations on both sides and must be equal bit for bit.  Elsewhere both sides
run the page's fp32 algorithm with a different order of summation (and the
CUDA path with one factorisation where the page has three), so the current
value of a column differs in the last bits between the two; a rounding
decision whose value ``w / s`` lies that close to a tie (k + 1/2) may go
either way, and from there on the row follows another trajectory (a different
code changes the error every later column receives).  Both are valid GPTQ
runs.  So the general case checks what is unique and that the rest is valid:

* row by row, the codes are the oracle's up to the end of the row, or up to a
  column at which the oracle's ``w / s`` lies within ``TIE`` of a tie (a
  wrong update or index would part the rows far from ties);
* the total loss equals the oracle's to 1e-2 (a parted row ends within a
  fraction of a percent of the oracle's loss);
* every row's loss equals the closed form ``0.5 (w - w_hat)^T H (w - w_hat)``
  of the row the CUDA path itself produced (the identity the oracle is pinned
  to; it fails for a wrong update, index or sign);
* every code is in range and the fake-quantised weights are exactly
  ``(q - z) s`` of the codes.

At 8192 columns about one sampled row in four parts (measured on B200; the
factor then agrees with an fp64 factorisation to 2e-6 relative).
"""
import numpy as np
import pytest

import _golden
import wq_inputs
from oracle import gptq

pytestmark = pytest.mark.gpu

TIE = 0.02  # |w/s - (k + 1/2)| of the oracle at the first differing code of a row


def _gpu(libwq, cuda, W, H, s, z, G, bits, blocksize=128, percdamp=0.01):
    import torch
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(cuda)
    out = libwq.gptq_quantize(t(W), t(H), t(s), t(z), G, bits, blocksize=blocksize, percdamp=percdamp)
    torch.cuda.synchronize()
    half = 1 << (bits - 1)
    return {"Q": out["Q"].cpu().numpy(),
            "codes": out["codes"].cpu().numpy().T.astype(np.int32) - half,  # (rows, cols), signed
            "losses": out["losses"].cpu().numpy()}


def _valid(g, W0, Hd, s, z, G, bits):
    """What holds for any GPTQ trajectory of the page's arithmetic."""
    qmin, qmax = gptq.qrange(bits)
    assert g["codes"].min() >= qmin and g["codes"].max() <= qmax
    sc = np.repeat(s, G, axis=1)[:, :W0.shape[1]].astype(np.float32)
    zc = np.repeat(z, G, axis=1)[:, :W0.shape[1]].astype(np.float32)
    np.testing.assert_array_equal(g["Q"], ((g["codes"].astype(np.float32) - zc) * sc).astype(np.float32))
    ident = gptq.gptq_loss_of(W0, g["Q"], Hd)
    np.testing.assert_allclose(g["losses"], ident, rtol=2e-3, atol=1e-30)


def _same_or_tie(g, ref):
    """Rows whose codes equal the oracle's, or part from it at a near tie;
    returns the number of parted rows."""
    parted = 0
    for r in range(ref["codes"].shape[0]):
        d = np.nonzero(g["codes"][r] != ref["codes"][r])[0]
        if len(d) == 0:
            continue
        t = float(ref["ratio"][r, d[0]])
        dist = abs(abs(t - np.floor(t)) - 0.5)
        assert dist < TIE, f"row {r} parts at column {d[0]}, w/s = {t}, {dist:.4f} from a tie"
        parted += 1
    return parted


def test_golden_cases(cuda, libwq):
    for name, c in _golden.read_cases("gptq_small.txt").items():
        r, k = int(c["rows"][0]), int(c["cols"][0])
        g = _gpu(libwq, cuda, np.array(c["W"]).reshape(r, k), np.array(c["H"]).reshape(k, k),
                 np.array(c["scale"]).reshape(r, -1), np.array(c["zero"]).reshape(r, -1), c["group"], c["bits"],
                 percdamp=c["percdamp"][0])
        assert g["codes"].ravel().tolist() == [int(v) for v in c["codes"]], name
        np.testing.assert_allclose(g["Q"].ravel(), c["Q"], rtol=1e-6, atol=1e-7, err_msg=name)
        np.testing.assert_allclose(g["losses"], c["losses"], rtol=1e-5, err_msg=name)


@pytest.mark.parametrize("rows,cols,G,bits,blocksize", [(96, 320, 64, 4, 128), (70, 200, 128, 8, 48),
                                                         (5, 33, 7, 2, 1)])
def test_diagonal_hessian_bit_exact(cuda, libwq, rows, cols, G, bits, blocksize):
    rng = np.random.default_rng(rows + cols)
    W = rng.uniform(-0.1, 0.1, (rows, cols)).astype(np.float32)
    h = rng.uniform(0.5, 4.0, cols).astype(np.float32)
    s, z = gptq.symmetric_group_qparams(W, G, bits)
    ref = gptq.quantize_weight(W, np.diag(h), s, z, G, bits, blocksize=blocksize)
    g = _gpu(libwq, cuda, W, np.diag(h), s, z, G, bits, blocksize)
    assert np.array_equal(g["codes"], ref["codes"])
    np.testing.assert_array_equal(g["Q"], ref["Q"])
    np.testing.assert_allclose(g["losses"], ref["losses"], rtol=1e-5)


GENERAL = [(128, 512, 128, 8, 128), (200, 700, 96, 4, 128), (64, 256, 32, 4, 32), (33, 130, 128, 3, 128),
           (1, 64, 64, 8, 128), (257, 129, 128, 8, 100)]


@pytest.mark.parametrize("rows,cols,G,bits,blocksize", GENERAL)
def test_general_hessian(cuda, libwq, rows, cols, G, bits, blocksize):
    W, H = wq_inputs.gptq_problem(rows, cols, seed=rows * 7 + cols)
    s, z = gptq.symmetric_group_qparams(W, G, bits)
    ref = gptq.quantize_weight(W, H, s, z, G, bits, blocksize=blocksize)
    g = _gpu(libwq, cuda, W, H, s, z, G, bits, blocksize)
    _same_or_tie(g, ref)
    assert abs(g["losses"].sum() - ref["loss"]) <= 1e-2 * ref["loss"]
    _valid(g, ref["W0"], ref["H"], s, z, G, bits)


def test_nonzero_zero_points(cuda, libwq):
    """Asymmetric parameters on the signed scale: z = -round(mn / s) - 2^(b-1)."""
    rows, cols, G, bits = 48, 256, 64, 4
    W, H = wq_inputs.gptq_problem(rows, cols, seed=11)
    blk = W.reshape(rows, cols // G, G)
    mn, mx = np.minimum(blk.min(-1), 0), np.maximum(blk.max(-1), 0)
    s = ((mx - mn) / np.float32(15)).astype(np.float32)
    z = (-np.rint(mn / s) - 8).astype(np.float32)
    ref = gptq.quantize_weight(W, H, s, z, G, bits)
    g = _gpu(libwq, cuda, W, H, s, z, G, bits)
    _same_or_tie(g, ref)
    _valid(g, ref["W0"], ref["H"], s, z, G, bits)


def test_dead_columns(cuda, libwq):
    rows, cols, G, bits = 40, 192, 64, 8
    W, H = wq_inputs.gptq_problem(rows, cols, seed=3)
    dead = [0, 63, 64, 191]
    H[dead, :] = 0
    H[:, dead] = 0
    s, z = gptq.symmetric_group_qparams(W, G, bits)
    ref = gptq.quantize_weight(W, H, s, z, G, bits)
    g = _gpu(libwq, cuda, W, H, s, z, G, bits)
    assert np.all(g["Q"][:, dead] == 0) and np.all(g["codes"][:, dead] == 0)
    _same_or_tie(g, ref)
    _valid(g, ref["W0"], ref["H"], s, z, G, bits)


def test_not_positive_definite_reported(cuda, libwq):
    rows, cols = 8, 96
    W = np.ones((rows, cols), np.float32)
    H = -np.eye(cols, dtype=np.float32)
    s = np.full((rows, 1), 0.1, np.float32)
    z = np.zeros((rows, 1), np.float32)
    libwq.device_status(reset=True)
    g = _gpu(libwq, cuda, W, H, s, z, 128, 8)
    assert libwq.device_status(reset=True) == 9
    assert np.isnan(g["losses"]).all()
    assert libwq.device_status(reset=True) == 0


def test_page_workload_sampled_rows(cuda, libwq):
    """The page's benchmark problem (8192 x 8192, symmetric 8-bit, groups of
    128, blocks of 128, percdamp 0.01): the whole matrix on the GPU, the
    oracle on sampled rows (rows are independent given the Hessian)."""
    rows = cols = 8192
    W, H = wq_inputs.gptq_problem(rows, cols, seed=42)
    s, z = gptq.symmetric_group_qparams(W, 128, 8)
    g = _gpu(libwq, cuda, W, H, s, z, 128, 8)
    pick = np.sort(np.random.default_rng(0).choice(rows, 16, replace=False))
    ref = gptq.quantize_weight(W[pick], H, s[pick], z[pick], 128, 8)
    sub = {k: v[pick] for k, v in g.items()}
    parted = _same_or_tie(sub, ref)
    assert parted <= len(pick) // 2, f"{parted} of {len(pick)} rows parted at a tie"
    np.testing.assert_allclose(sub["losses"].sum(), ref["losses"].sum(), rtol=1e-2)
    _valid(sub, ref["W0"], ref["H"], s[pick], z[pick], 128, 8)
    assert np.isfinite(g["losses"]).all()
