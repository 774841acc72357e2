"""Pins for the MSE-observer search oracle (``oracle/mse_observer.py``), CPU only.

Expected values come from the hand-worked cases in ``tests/golden/mse_search.txt``
and from facts the method fixes: a group already on the grid of its own
min-max parameters is reproduced exactly by the first candidate; scaling W by
a power of two scales s and the errors and changes nothing else; the
exhaustive result is NumPy's first-occurrence argmin of the candidate errors;
a patience longer than the grid changes nothing.  The mutants at the end
each plant one plausible mistake; every one must fail a pin.
"""
import types

import numpy as np
import pytest

from _golden import read_cases

import oracle.mse_observer as mo


def _cases():
    return read_cases("mse_search.txt")


def pin_golden(impl):
    for name, c in _cases().items():
        G = c["group"]
        w = np.array(c["values"], np.float32).reshape(1, -1)
        patience = int(c["patience"][0]) if "patience" in c else None
        kw = {"symmetric": True} if "symmetric" in c and int(c["symmetric"][0]) else {}
        r = impl.search(w, c["bits"], G, maxshrink=c["maxshrink"][0], grid=int(c["grid"][0]),
                        norm=c["norm"][0], patience=patience, **kw)
        assert r["steps_evaluated"] == int(c["evaluated"][0]), name
        assert np.array_equal(r["step"][0], np.array(c["steps"], np.int32)), (name, r["step"])
        assert np.array_equal(r["scale"][0], np.array(c["scale"], np.float32)), (name, r["scale"])
        assert np.array_equal(r["zero"][0], np.array(c["zero"], np.float32)), (name, r["zero"])
        assert np.array_equal(r["errors"][0].ravel(), np.array(c["errors"])), (name, r["errors"])


def _on_grid(bits, rows, groups, G, seed):
    """W whose groups are exactly (q - z) s with q spanning [0, qmax], s = 2^-e, integer z."""
    rng = np.random.default_rng(seed)
    qmax = (1 << bits) - 1
    q = rng.integers(0, qmax + 1, size=(rows, groups, G))
    q[..., 0] = 0
    q[..., 1] = qmax
    z = rng.integers(0, qmax + 1, size=(rows, groups, 1))
    s = 2.0 ** -rng.integers(2, 9, size=(rows, groups, 1))
    w = ((q - z) * s).astype(np.float32).reshape(rows, groups * G)
    return w, s[..., 0].astype(np.float32), z[..., 0].astype(np.float32)


def pin_on_grid_is_exact(impl):
    for bits in (1, 2, 3, 4, 8):
        G = 16 if bits < 8 else 260
        w, s, z = _on_grid(bits, 3, 5, G, bits)
        r = impl.search(w, bits, G, maxshrink=0.2, grid=100, norm=2.4)
        assert np.all(r["step"] == 0), bits
        assert np.all(r["err"] == 0.0), bits
        assert np.array_equal(r["scale"], s), bits
        assert np.array_equal(r["zero"], z), bits


def pin_power_of_two_scaling(impl):
    rng = np.random.default_rng(7)
    w = rng.standard_normal((4, 256)).astype(np.float32)
    base = impl.search(w, 4, 64, maxshrink=0.3, grid=50, norm=2.4)
    for k in (-3, 2):
        r = impl.search(w * np.float32(2.0 ** k), 4, 64, maxshrink=0.3, grid=50, norm=2.4)
        assert np.array_equal(r["step"], base["step"]), k
        assert np.array_equal(r["scale"], base["scale"] * np.float32(2.0 ** k)), k
        assert np.array_equal(r["zero"], base["zero"]), k
        assert np.allclose(r["errors"], base["errors"] * 2.0 ** (k * 2.4), rtol=1e-12, atol=0), k


def pin_exhaustive_is_first_argmin(impl):
    rng = np.random.default_rng(8)
    for bits, G in ((2, 32), (4, 128), (8, 64)):
        w = (rng.standard_normal((6, 4 * G)) * rng.uniform(0.1, 3.0, size=(6, 1))).astype(np.float32)
        r = impl.search(w, bits, G, maxshrink=0.25, grid=40, norm=2.4)
        assert r["steps_evaluated"] == 10
        assert np.array_equal(r["step"], np.argmin(r["errors"], axis=-1)), bits
        assert np.array_equal(r["err"], np.min(r["errors"], axis=-1)), bits


def pin_long_patience_changes_nothing(impl):
    rng = np.random.default_rng(9)
    w = rng.standard_normal((5, 128)).astype(np.float32)
    a = impl.search(w, 3, 32, maxshrink=0.2, grid=100, norm=2.0)
    b = impl.search(w, 3, 32, maxshrink=0.2, grid=100, norm=2.0, patience=20)
    assert b["steps_evaluated"] == 20
    for key in ("step", "scale", "zero", "err"):
        assert np.array_equal(a[key], b[key]), key


def pin_zero_group(impl):
    w = np.zeros((2, 64), np.float32)
    r = impl.search(w, 4, 32, maxshrink=0.2, grid=100, norm=2.4)
    assert np.all(r["step"] == 0)
    assert np.all(r["scale"] == np.float32(2.0 ** -23))
    assert np.all(r["zero"] == 0) and np.all(r["err"] == 0)


def pin_symmetric_range_matches_asymmetric(impl):
    """A group whose range is symmetric, mn = -mx with mx = (2^b - 1)/2 * 2^-e, and one
    candidate (p = 1): the asymmetric rule gives the same scale 2^-e and zero point
    2^(b-1), so the symmetric search must give the same scale, errors and, stored in
    the product's unsigned format, zero point 2^(b-1)."""
    rng = np.random.default_rng(10)
    for bits in (2, 3, 4, 8):
        half = ((1 << bits) - 1) / 2.0
        G = 32
        e = rng.integers(2, 8, size=(3, 4, 1))
        mx = half * 2.0 ** -e
        w = rng.uniform(-1.0, 1.0, size=(3, 4, G)) * mx
        w[..., 0] = -mx[..., 0]
        w[..., 1] = mx[..., 0]
        w = w.astype(np.float32).reshape(3, 4 * G)
        a = impl.search(w, bits, G, maxshrink=1.0, grid=1, norm=2.4)
        b = impl.search(w, bits, G, maxshrink=1.0, grid=1, norm=2.4, symmetric=True)
        assert np.array_equal(b["scale"], (2.0 ** -e[..., 0]).astype(np.float32)), bits
        assert np.array_equal(a["scale"], b["scale"]), bits
        assert np.array_equal(a["errors"], b["errors"]), bits
        assert np.all(b["zero"] == 0), bits
        _, zu = mo.to_unsigned(np.zeros_like(b["step"]), b["zero"], bits)
        assert np.array_equal(zu, a["zero"]), bits


def pin_symmetric_invariants(impl):
    """Power-of-two scaling and the first-argmin rule hold for the symmetric form too."""
    rng = np.random.default_rng(11)
    w = rng.standard_normal((4, 256)).astype(np.float32)
    base = impl.search(w, 4, 32, maxshrink=0.3, grid=50, norm=2.4, symmetric=True)
    assert np.all(base["zero"] == 0)
    assert np.array_equal(base["step"], np.argmin(base["errors"], axis=-1))
    r = impl.search(w * np.float32(0.25), 4, 32, maxshrink=0.3, grid=50, norm=2.4, symmetric=True)
    assert np.array_equal(r["step"], base["step"])
    assert np.array_equal(r["scale"], base["scale"] * np.float32(0.25))


PINS = [pin_golden, pin_on_grid_is_exact, pin_power_of_two_scaling, pin_exhaustive_is_first_argmin,
        pin_long_patience_changes_nothing, pin_zero_group, pin_symmetric_range_matches_asymmetric,
        pin_symmetric_invariants]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(mo)


def test_rejects_bad_arguments():
    with pytest.raises(ValueError):
        mo.search(np.zeros((2, 10), np.float32), 4, 4)        # cols % group_size
    with pytest.raises(ValueError):
        mo.search(np.zeros((2, 8), np.float32), 9, 4)         # bits
    with pytest.raises(ValueError):
        mo.search(np.zeros((2, 8), np.float32), 4, 4, maxshrink=0.001, grid=100)  # no candidate
    with pytest.raises(ValueError):
        mo.search(np.zeros((2, 8), np.float32), 4, 4, patience=0)


# ------------------------------------------------------------------ mutants
def _module_with(**over):
    """A copy of the oracle's search whose helper functions are replaced."""
    src_search = mo.search
    g = dict(src_search.__globals__)
    g.update(over)
    search = types.FunctionType(src_search.__code__, g, "search", src_search.__defaults__,
                                src_search.__closure__)
    search.__kwdefaults__ = src_search.__kwdefaults__
    return types.SimpleNamespace(search=search)


def _qparams_no_zero(lo, hi, bits):          # range not widened to contain 0
    qmin, qmax = mo.qrange(bits)
    lo = np.asarray(lo, np.float32)
    hi = np.asarray(hi, np.float32)
    s = ((hi - lo) / np.float32(qmax - qmin)).astype(np.float32)
    s = np.where(s == 0, np.float32(mo.EPS32), s).astype(np.float32)
    z = np.clip(np.float32(qmin) - np.rint(lo / s), qmin, qmax).astype(np.float32)
    return s, z


def _qparams_zero_sign(lo, hi, bits):        # z = qmin + round(lo / s)
    s, _ = mo.qparams(lo, hi, bits)
    lo = np.minimum(np.asarray(lo, np.float32), 0)
    qmin, qmax = mo.qrange(bits)
    return s, np.clip(np.float32(qmin) + np.rint(lo / s), qmin, qmax).astype(np.float32)


def _fake_quant_floor(w, s, z, bits, symmetric=False):   # floor instead of round to nearest
    qmin, qmax = mo.qrange(bits, symmetric)
    q = np.clip(np.floor((np.asarray(w, np.float32) / s + z).astype(np.float32)), qmin, qmax).astype(np.float32)
    return q.astype(np.int32), ((q - z) * s).astype(np.float32)


def _qparams_ties_up(lo, hi, bits):          # round(lo / s) with ties up instead of to even
    s, _ = mo.qparams(lo, hi, bits)
    lo = np.minimum(np.asarray(lo, np.float32), 0)
    qmin, qmax = mo.qrange(bits)
    r = np.floor((lo / s).astype(np.float32) + np.float32(0.5))
    return s, np.clip(np.float32(qmin) - r, qmin, qmax).astype(np.float32)


def _error_abs(w, w_hat, norm):              # norm ignored
    return mo.group_error(w, w_hat, 1.0)


def _candidates_wrong(maxshrink, grid):      # p_i = 1 - i * maxshrink / grid
    n = int(maxshrink * grid)
    return np.array([1.0 - i * maxshrink / grid for i in range(n)]).astype(np.float32)


def _search_ties_move(w, bits, group_size, maxshrink=0.2, grid=100, norm=2.4, patience=None, symmetric=False):
    r = mo.search(w, bits, group_size, maxshrink, grid, norm, patience, symmetric)
    e = r["errors"]
    last = e.shape[-1] - 1 - np.argmin(e[..., ::-1], axis=-1)   # the last smallest error wins
    r = dict(r)
    r["step"] = last.astype(np.int32)
    p = mo.candidates(maxshrink, grid)[last]
    grp = np.asarray(w, np.float32).reshape(w.shape[0], -1, group_size)
    qp = mo.qparams_symmetric if symmetric else mo.qparams
    r["scale"], r["zero"] = qp((grp.min(-1) * p).astype(np.float32), (grp.max(-1) * p).astype(np.float32), bits)
    return r


def _search_patience_per_group(w, bits, group_size, maxshrink=0.2, grid=100, norm=2.4, patience=None,
                               symmetric=False):
    if patience is None:
        return mo.search(w, bits, group_size, maxshrink, grid, norm, symmetric=symmetric)
    r = dict(mo.search(w, bits, group_size, maxshrink, grid, norm, symmetric=symmetric))
    e = r["errors"]
    steps = np.zeros(e.shape[:-1], np.int32)
    for idx in np.ndindex(*e.shape[:-1]):
        best, stale = np.inf, 0
        for i, v in enumerate(e[idx]):
            if v < best:
                best, steps[idx], stale = v, i, 0
            else:
                stale += 1
                if stale >= patience:
                    break
    r["step"] = steps
    p = mo.candidates(maxshrink, grid)[steps]
    grp = np.asarray(w, np.float32).reshape(w.shape[0], -1, group_size)
    r["scale"], r["zero"] = mo.qparams((grp.min(-1) * p).astype(np.float32),
                                       (grp.max(-1) * p).astype(np.float32), bits)
    r["steps_evaluated"] = e.shape[-1]
    return r


def _qparams_sym_denominator(lo, hi, bits):   # symmetric scale over qmax = 2^(b-1) - 1
    qmin, qmax = mo.qrange(bits, symmetric=True)
    a = np.maximum(np.abs(np.asarray(lo, np.float32)), np.abs(np.asarray(hi, np.float32)))
    s = (a / np.float32(qmax)).astype(np.float32)
    return np.where(s == 0, np.float32(mo.EPS32), s).astype(np.float32), np.zeros_like(s)


def _fake_quant_sym_unsigned(w, s, z, bits, symmetric=False):   # symmetric codes clipped to [0, 2^b - 1]
    return mo.fake_quant(w, s, z, bits, False)


MUTANTS = {
    "symmetric_scale_over_qmax": _module_with(qparams_symmetric=_qparams_sym_denominator),
    "symmetric_unsigned_clip": _module_with(fake_quant=_fake_quant_sym_unsigned),
    "range_without_zero": _module_with(qparams=_qparams_no_zero),
    "zero_point_sign": _module_with(qparams=_qparams_zero_sign),
    "floor_rounding": _module_with(fake_quant=_fake_quant_floor),
    "zero_point_ties_up": _module_with(qparams=_qparams_ties_up),
    "norm_ignored": _module_with(group_error=_error_abs),
    "shrink_steps_scaled": _module_with(candidates=_candidates_wrong),
    "ties_move_to_later_candidate": types.SimpleNamespace(search=_search_ties_move),
    "patience_per_group": types.SimpleNamespace(search=_search_patience_per_group),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_some_pin_catches_mutant(name):
    failed = []
    for pin in PINS:
        try:
            pin(MUTANTS[name])
        except (AssertionError, ValueError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"mutant {name} passed every pin"
