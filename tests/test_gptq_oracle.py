"""Pins of the GPTQ oracle (``oracle/gptq.py``) to facts other than itself.

* hand-worked quantisations (``tests/golden/gptq_small.txt``): codes, the
  fake-quantised weights and the per-row losses;
* the diagonal-Hessian special case: no error reaches another column, so the
  codes are plain round-to-nearest and each loss term is ``diff^2 h``;
* the closed-form loss identity: the loop's per-row loss equals
  ``0.5 (w - w_hat)^T H (w - w_hat)`` of the damped Hessian (each column's term
  is the rise of that quadratic form when the column is fixed while the later
  ones sit at their optimum), which a dropped, mis-signed or mis-indexed
  update breaks;
* the Hinv factor: upper triangular with ``Hinv^T Hinv H = I``;
* blocksize invariance: the block update reorganises the same column updates,
  so blocks of 1, 32 and 128 give the same codes;
* dead columns and the gain over round-to-nearest.

Each planted mistake in ``MUTANTS`` (a one-token change of the oracle's own
source, run on the CPU) fails at least one pin.
"""
import inspect
import types

import numpy as np
import pytest

import _golden
import wq_inputs
from oracle import gptq


def _run(m, c, precision=np.float32, blocksize=128):
    r, k = int(c["rows"][0]), int(c["cols"][0])
    return m.quantize_weight(np.array(c["W"]).reshape(r, k), np.array(c["H"]).reshape(k, k),
                             np.array(c["scale"]).reshape(r, -1), np.array(c["zero"]).reshape(r, -1),
                             c["group"], c["bits"], blocksize=blocksize,
                             percdamp=c["percdamp"][0], precision=precision)


def _problem(rows, cols, seed, G=128, bits=8):
    W, H = wq_inputs.gptq_problem(rows, cols, seed)
    s, z = gptq.symmetric_group_qparams(W, G, bits)
    return W, H, s, z


# ---- the pins, each taking a module-like object with quantize_weight ----

def pin_golden(m):
    for name, c in _golden.read_cases("gptq_small.txt").items():
        for ft in (np.float32, np.float64):
            out = _run(m, c, ft)
            assert out["codes"].ravel().tolist() == [int(v) for v in c["codes"]], name
            np.testing.assert_allclose(out["Q"].ravel(), c["Q"], rtol=1e-6, atol=1e-7, err_msg=name)
            np.testing.assert_allclose(out["losses"], c["losses"], rtol=1e-5, err_msg=name)


def pin_diagonal(m):
    rng = np.random.default_rng(5)
    rows, cols, G = 16, 96, 32
    W = rng.uniform(-0.1, 0.1, (rows, cols)).astype(np.float32)
    h = rng.uniform(0.5, 4.0, cols).astype(np.float32)
    s, z = gptq.symmetric_group_qparams(W, G, 4)
    out = m.quantize_weight(W, np.diag(h), s, z, G, 4, percdamp=0.01)
    damp = np.float32(0.01) * np.mean(h, dtype=np.float32)
    sc = np.repeat(s, G, axis=1)
    q = np.clip(np.rint(W / sc), -8, 7)
    assert np.array_equal(out["codes"], q.astype(np.int32))
    what = (q * sc).astype(np.float32)
    np.testing.assert_array_equal(out["Q"], what)
    loss = 0.5 * np.sum((W.astype(np.float64) - what) ** 2 * (h.astype(np.float64) + damp), axis=1)
    np.testing.assert_allclose(out["losses"], loss, rtol=1e-5)


def pin_loss_identity(m):
    for (rows, cols, bits, seed) in [(24, 256, 8, 1), (16, 320, 4, 2)]:
        W, H, s, z = _problem(rows, cols, seed, bits=bits)
        for ft, tol in ((np.float64, 1e-9), (np.float32, 2e-4)):
            out = m.quantize_weight(W, H, s, z, 128, bits, precision=ft)
            ident = gptq.gptq_loss_of(out["W0"], out["Q"], out["H"])
            np.testing.assert_allclose(out["losses"], ident, rtol=tol)


def pin_hinv(m):
    W, H, s, z = _problem(4, 200, 3)
    out = m.quantize_weight(W, H, s, z, 128, 8, precision=np.float64)
    U = out["Hinv"]
    assert np.array_equal(U, np.triu(U)) and np.all(np.diag(U) > 0)
    np.testing.assert_allclose(U.T @ U @ out["H"], np.eye(200), atol=1e-9)


def pin_blocksize(m):
    W, H, s, z = _problem(16, 384, 4)
    ref = m.quantize_weight(W, H, s, z, 128, 8, blocksize=128, precision=np.float64)
    for bs in (1, 32, 100):
        out = m.quantize_weight(W, H, s, z, 128, 8, blocksize=bs, precision=np.float64)
        assert np.array_equal(out["codes"], ref["codes"]), bs
        np.testing.assert_allclose(out["losses"], ref["losses"], rtol=1e-9)


def pin_dead_columns(m):
    W, H, s, z = _problem(8, 160, 6)
    dead = [3, 77, 159]
    H = H.copy()
    H[dead, :] = 0
    H[:, dead] = 0
    out = m.quantize_weight(W, H, s, z, 128, 8)
    assert np.all(out["Q"][:, dead] == 0) and np.all(out["codes"][:, dead] == 0)
    assert np.all(out["W0"][:, dead] == 0)
    hd = np.diag(H).astype(np.float32).copy()
    hd[dead] = 1
    damp = np.float32(0.01) * np.mean(hd, dtype=np.float32)
    np.testing.assert_allclose(np.diag(out["H"])[dead], 1 + damp, rtol=1e-6)
    ident = gptq.gptq_loss_of(out["W0"], out["Q"], out["H"])
    np.testing.assert_allclose(out["losses"], ident, rtol=2e-4)


def pin_beats_round_to_nearest(m):
    W, H, s, z = _problem(32, 256, 7)
    out = m.quantize_weight(W, H, s, z, 128, 4)
    sc = np.repeat(s, 128, axis=1)
    rtn = (np.clip(np.rint(W / sc), -8, 7) * sc).astype(np.float32)
    loss_rtn = gptq.gptq_loss_of(out["W0"], rtn, out["H"])
    assert np.all(out["losses"] < loss_rtn)
    assert out["loss"] < loss_rtn.sum()


PINS = [pin_golden, pin_diagonal, pin_loss_identity, pin_hinv, pin_blocksize, pin_dead_columns,
        pin_beats_round_to_nearest]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_oracle_meets_pin(pin):
    pin(gptq)


# ---- planted mistakes: (function, original text, mutated text) ----
MUTANTS = {
    "no_block_update": ("quantize_weight", "W[:, i2:] -= (Err1", "W[:, i2:] -= 0 * (Err1"),
    "block_update_sign": ("quantize_weight", "W[:, i2:] -= (Err1", "W[:, i2:] += (Err1"),
    "inner_update_sign": ("quantize_weight", "W1[:, i:] -= np.outer", "W1[:, i:] += np.outer"),
    "no_inner_update": ("quantize_weight", "W1[:, i:] -= np.outer(err1", "W1[:, i:] -= 0 * np.outer(err1"),
    "lower_factor": ("quantize_weight", "Err1 @ Hinv[i1:i2, i2:]", "Err1 @ Hinv.T[i1:i2, i2:]"),
    "first_pivot": ("quantize_weight", "d = Hinv1[i, i]", "d = Hinv1[0, 0]"),
    "loss_not_halved": ("quantize_weight", "/ ft(2)", "/ ft(1)"),
    "floor_not_round": ("quantize_weight", "np.rint(t)", "np.floor(t)"),
    "group_modulo": ("quantize_weight", "(i1 + i) // group_size", "(i1 + i) % group_size"),
    "error_not_scaled": ("quantize_weight", "err1 = ((w - q) / d)", "err1 = ((w - q) * 1)"),
    "no_damp": ("prepare", "H[idx, idx] += damp", "H[idx, idx] += 0 * damp"),
    "dead_kept": ("prepare", "W[:, dead] = 0", "W[:, dead] = W[:, dead]"),
    "factor_not_inverse": ("prepare", "np.linalg.cholesky(inv).T", "np.linalg.cholesky(H).T"),
    "no_clamp": ("quantize_weight", "ft(qmin), ft(qmax)", "ft(-1e9), ft(1e9)"),
}


def _mutant(fn_name, old, new):
    """Both functions recompiled in one namespace, so that quantize_weight
    calls the (possibly mutated) prepare."""
    ns = dict(vars(gptq))
    for f in ("prepare", "quantize_weight"):
        src = inspect.getsource(getattr(gptq, f))
        if f == fn_name:
            assert src.count(old) == 1, (fn_name, old)
            src = src.replace(old, new)
        exec(compile(src, f"<mutant {f}>", "exec"), ns)
    return types.SimpleNamespace(quantize_weight=ns["quantize_weight"], prepare=ns["prepare"])


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_fails_a_pin(name):
    m = _mutant(*MUTANTS[name])
    failed = []
    for pin in PINS:
        try:
            with np.errstate(all="ignore"):
                pin(m)
        except (AssertionError, np.linalg.LinAlgError, ValueError, FloatingPointError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"mutant {name} passes every pin"
