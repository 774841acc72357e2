"""CPU oracle for the MSE-observer search of per-group scales and zero points.

TEST INFRASTRUCTURE: only ``tests/``, ``__graft_entry__.smoke()`` and the
bench's CPU-baseline / reference arm may import this module.

What it computes follows the "Benchmark for MSE observer grid search" page
(gist ``mse_bench.py``): ``grid_search_eager`` and
``grid_search_eager_no_patience`` for the steps, ``_fused_grid_search_kernel``
for the fake quantisation, ``calculate_range`` for the code range.  For each
group of ``group_size`` consecutive values of a row of W:

* ``mn, mx`` = the group's minimum and maximum;
* candidate ``i`` (``i < int(maxshrink * grid)``) shrinks them by
  ``p_i = 1 - i / grid``: ``lo = mn * p_i``, ``hi = mx * p_i``;
* ``(s, z)`` = the affine min-max parameters of ``[lo, hi]`` for unsigned
  codes ``[0, 2**bits - 1]`` (see ``qparams``);
* fake quantisation: ``q = clamp(round(w / s + z), 0, 2**bits - 1)``,
  ``w_hat = (q - z) * s``;
* ``err_i = sum |w_hat - w| ** norm`` over the group;
* the best candidate is the first with the smallest error (a later candidate
  replaces it only when strictly smaller);
* with ``patience``, the search stops after ``patience`` consecutive
  candidates in which no group of the whole tensor improved
  (``grid_search_eager``); without, every candidate is evaluated
  (``grid_search_eager_no_patience``).

Precision: the page works in the dtype of W; here W is fp32 and every step
up to ``w_hat`` is done in IEEE fp32 (NumPy float32 arithmetic, round half
to even), so candidate parameters and codes are exactly what an fp32
implementation computes.  The error terms are then evaluated in fp64 from
the fp32 difference ``w_hat - w`` and summed in ascending order.

The page imports the parameter function (``calculate_qparams``) instead of
printing it.  ``qparams`` restates the standard affine ("asymmetric")
min-max quantisation of Jacob et al. 2018, *Quantization and Training of
Neural Networks for Efficient Integer-Arithmetic-Only Inference*, section
2.1: the range is widened to contain 0, ``s = (hi - lo) / (qmax - qmin)``,
and ``z = qmin - round(lo / s)`` clamped to the code range, so that 0 is
exactly representable.  A zero scale becomes the fp32 machine epsilon, the
replacement the page's kernels use (``_scale_round_config``, ``scale_eps``).

Symmetric integers.  The page's search also takes symmetric arguments
(``args.symmetric``: codes ``[-2**(bits-1), 2**(bits-1) - 1]`` in the fused
kernel's launch, no zero point in its fake quantisation).  The page does not
print their parameter rule either; ``qparams_symmetric`` takes the standard
symmetric (absolute-maximum) rule: ``s = max(|lo|, |hi|) / ((qmax - qmin) / 2)``
with the same zero-scale replacement, and ``z = 0``.  On the product's
unsigned format a symmetric code ``q`` is stored as ``q + 2**(bits-1)`` with
zero point ``2**(bits-1)`` (``to_unsigned``), which dequantises to the same
``q * s``.

Parity pins: ``tests/test_mse_oracle.py`` (a hand-worked example in
``tests/golden/mse_search.txt``, closed forms, invariants, special cases).
"""
from __future__ import annotations

import numpy as np

F32 = np.float32
EPS32 = np.finfo(np.float32).eps  # 2**-23


def qrange(bits: int, symmetric: bool = False):
    """Code range of ``bits``-bit integers: unsigned [0, 2^b - 1], or signed
    [-2^(b-1), 2^(b-1) - 1] for the symmetric form."""
    if not 1 <= bits <= 8:
        raise ValueError(f"bits must be in 1..8, got {bits}")
    if symmetric:
        return -(1 << (bits - 1)), (1 << (bits - 1)) - 1
    return 0, (1 << bits) - 1


def candidates(maxshrink: float, grid: int) -> np.ndarray:
    """Shrink factors p_i = 1 - i / grid, i < int(maxshrink * grid), as fp32."""
    n = int(maxshrink * grid)
    if n < 1:
        raise ValueError("maxshrink * grid must be at least 1")
    return np.array([1.0 - i / grid for i in range(n)], dtype=np.float64).astype(F32)


def qparams(lo, hi, bits: int):
    """fp32 (scale, zero point) of the range [lo, hi] (arrays of fp32)."""
    qmin, qmax = qrange(bits)
    lo = np.minimum(np.asarray(lo, F32), F32(0))
    hi = np.maximum(np.asarray(hi, F32), F32(0))
    s = ((hi - lo) / F32(qmax - qmin)).astype(F32)
    s = np.where(s == F32(0), F32(EPS32), s).astype(F32)
    z = (F32(qmin) - np.rint((lo / s).astype(F32))).astype(F32)
    z = np.clip(z, F32(qmin), F32(qmax)).astype(F32)
    return s, z


def qparams_symmetric(lo, hi, bits: int):
    """fp32 (scale, zero point = 0) of the range [lo, hi] for signed codes:
    s = max(|lo|, |hi|) / ((qmax - qmin) / 2), a zero scale replaced by 2^-23."""
    qmin, qmax = qrange(bits, symmetric=True)
    a = np.maximum(np.abs(np.asarray(lo, F32)), np.abs(np.asarray(hi, F32))).astype(F32)
    s = (a / F32((qmax - qmin) / 2)).astype(F32)
    s = np.where(s == F32(0), F32(EPS32), s).astype(F32)
    return s, np.zeros_like(s, dtype=F32)


def to_unsigned(codes, zero, bits: int):
    """Signed symmetric codes and zero points as the product's unsigned format:
    q + 2^(bits-1) and z + 2^(bits-1) (the same (q - z) * s)."""
    off = 1 << (bits - 1)
    return (np.asarray(codes) + off).astype(np.int32), (np.asarray(zero, F32) + F32(off)).astype(F32)


def fake_quant(w, s, z, bits: int, symmetric: bool = False):
    """(codes, w_hat): q = clamp(round(w / s + z)), w_hat = (q - z) * s, fp32.

    ``s`` and ``z`` broadcast against ``w`` (one value per group: shape (..., 1))."""
    qmin, qmax = qrange(bits, symmetric)
    w = np.asarray(w, F32)
    t = ((w / s).astype(F32) + z).astype(F32)
    q = np.clip(np.rint(t), F32(qmin), F32(qmax)).astype(F32)
    w_hat = ((q - z).astype(F32) * s).astype(F32)
    return q.astype(np.int32), w_hat


def group_error(w, w_hat, norm: float) -> np.ndarray:
    """sum over the last axis of |w_hat - w| ** norm, fp64, ascending order."""
    d = np.abs((np.asarray(w_hat, F32) - np.asarray(w, F32)).astype(F32)).astype(np.float64)
    terms = d ** float(norm)
    out = np.zeros(terms.shape[:-1], dtype=np.float64)
    for k in range(terms.shape[-1]):
        out += terms[..., k]
    return out


def search(w, bits: int, group_size: int, maxshrink: float = 0.2, grid: int = 100,
           norm: float = 2.4, patience: int | None = None, symmetric: bool = False) -> dict:
    """The grid search for every group of W (rows x cols, fp32; cols % group_size == 0).

    Defaults are the page's benchmark CLI (maxshrink 0.20, grid 100, norm 2.4);
    its patience default, 5, is passed explicitly, since None means every
    candidate is evaluated.

    ``symmetric``: signed codes and the symmetric parameter rule
    (``qparams_symmetric``); the zero points returned are then 0 (signed).

    Returns a dict of arrays of shape (rows, cols // group_size):
    ``step`` (best candidate index), ``err`` (its error), ``scale``, ``zero``
    (fp32, the parameters of that candidate), ``min``, ``max`` (the group's
    shrunk range for that candidate: mn * p, mx * p), and ``errors`` of shape
    (rows, groups, steps evaluated), plus ``steps_evaluated``.
    """
    w = np.asarray(w, F32)
    if w.ndim != 2:
        raise ValueError("W must be 2-D (rows, cols)")
    R, C = w.shape
    if group_size < 1 or C % group_size != 0:
        raise ValueError("cols must be a multiple of group_size")
    if patience is not None and patience < 1:
        raise ValueError("patience must be at least 1")
    grp = w.reshape(R, C // group_size, group_size)
    mn = grp.min(axis=-1)
    mx = grp.max(axis=-1)
    ps = candidates(maxshrink, grid)
    params = (lambda lo, hi: qparams_symmetric(lo, hi, bits)) if symmetric else (lambda lo, hi: qparams(lo, hi, bits))
    best_err = np.full(mn.shape, np.inf)
    best_step = np.zeros(mn.shape, dtype=np.int32)
    errors = []
    stale = 0
    for i, p in enumerate(ps):
        lo = (mn * p).astype(F32)
        hi = (mx * p).astype(F32)
        s, z = params(lo, hi)
        _, w_hat = fake_quant(grp, s[..., None], z[..., None], bits, symmetric)
        err = group_error(grp, w_hat, norm)
        errors.append(err)
        improved = err < best_err
        best_err = np.where(improved, err, best_err)
        best_step = np.where(improved, i, best_step).astype(np.int32)
        if patience is not None:
            stale = 0 if improved.any() else stale + 1
            if stale >= patience:
                break
    p_best = ps[best_step]
    lo = (mn * p_best).astype(F32)
    hi = (mx * p_best).astype(F32)
    s, z = params(lo, hi)
    return {"step": best_step, "err": best_err, "scale": s, "zero": z, "min": lo, "max": hi,
            "errors": np.stack(errors, axis=-1), "steps_evaluated": len(errors)}
