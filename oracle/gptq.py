"""CPU oracle for GPTQ block quantisation of a weight matrix.

TEST INFRASTRUCTURE: only ``tests/``, ``__graft_entry__.smoke()`` and the
bench's CPU-baseline / reference arm may import this module.

What it computes follows the "benchmark GPTQ implementations" page:
``_prepare_weight_and_hessian`` for the set-up, ``quantize_weight_eager``
(GROUP strategy) for the column loop, and ``_quantize_block_triton_kernel``
for the inline fake quantisation.  For W (rows x cols, one row per output
channel) and the Hessian H (cols x cols):

* set-up: columns with ``H[c, c] == 0`` are dead: ``H[c, c] = 1`` and
  ``W[:, c] = 0``; then ``damp = percdamp * mean(diag H)`` is added to the
  diagonal; ``Hinv`` = the upper Cholesky factor of the inverse of that
  matrix (Cholesky factor, then the inverse from the factor, then the upper
  factor of the inverse);
* columns are taken in blocks of ``blocksize``; inside a block, column ``i``
  (current, already updated values ``w``) is fake-quantised with its group's
  ``(s, zp)``: ``q = clamp(nearbyint(w / s) + zp, -2**(b-1), 2**(b-1) - 1)``,
  ``w_hat = (q - zp) * s``; its loss term is ``(w - w_hat)**2 / d**2`` with
  ``d = Hinv[i, i]``; the error ``err = (w - w_hat) / d`` is taken out of the
  block's later columns: ``W1[:, i:] -= err * Hinv[i, i:]``;
* after a block, the quantised block replaces W's columns and the block's
  errors update every later column: ``W[:, i2:] -= Err1 @ Hinv[i1:i2, i2:]``;
* the loss is half the sum of the loss terms; the result is the fake-quantised
  W (``w_hat`` everywhere), plus, here, the integer codes ``q``.

Precision: the page fixes it (``GPTQ_PRECISION = float32``).  Every step is
NumPy float32 arithmetic; the Cholesky factors come from LAPACK in single
precision (``numpy.linalg.cholesky``, ``scipy.linalg.lapack.spotri`` for the
inverse from the factor) and the block update from a float32 matrix product.
These library primitives are steps of the page's own algorithm, called in its
order.  ``precision=np.float64`` runs the same steps in double precision (used
by the pins only).

Scales and zero points are inputs, as on the page (they come from the
module's observer before the loop starts).  ``symmetric_group_qparams`` gives
the plainest observer for the page's benchmark arguments (``symmetric=True``,
GROUP strategy, ``group_size`` 128): per row and group, the symmetric
absolute-maximum rule of ``mse_observer.qparams_symmetric`` with no shrink.

Parity pins: ``tests/test_gptq_oracle.py`` (a hand-worked two-column case in
``tests/golden/gptq_small.txt``, the diagonal-Hessian special case, the
closed-form loss identity, blocksize invariance, dead columns, and the
quantisation gain over round-to-nearest).
"""
from __future__ import annotations

import numpy as np

from . import mse_observer


def qrange(bits: int):
    """The signed code range of the page's block kernel: [-2^(b-1), 2^(b-1) - 1]."""
    return -(1 << (bits - 1)), (1 << (bits - 1)) - 1


def symmetric_group_qparams(W, group_size: int, bits: int):
    """(scale, zero point), each (rows, ceil(cols / group_size)) fp32: the
    absolute-maximum symmetric rule over each row's groups (zero point 0)."""
    W = np.asarray(W, np.float32)
    rows, cols = W.shape
    ng = -(-cols // group_size)
    lo = np.empty((rows, ng), np.float32)
    hi = np.empty((rows, ng), np.float32)
    for g in range(ng):
        blk = W[:, g * group_size:(g + 1) * group_size]
        lo[:, g] = blk.min(axis=1)
        hi[:, g] = blk.max(axis=1)
    return mse_observer.qparams_symmetric(lo, hi, bits)


def prepare(W, H, percdamp: float = 0.01, precision=np.float32):
    """The set-up of ``_prepare_weight_and_hessian``: (W with dead columns
    zeroed, the damped Hessian, Hinv = upper Cholesky factor of its inverse)."""
    from scipy.linalg import lapack

    ft = precision
    W = np.array(W, dtype=ft, copy=True)
    H = np.array(H, dtype=ft, copy=True)
    n = H.shape[0]
    dead = np.diag(H) == 0
    H[dead, dead] = 1
    W[:, dead] = 0
    damp = ft(percdamp) * np.mean(np.diag(H), dtype=ft)
    idx = np.arange(n)
    H[idx, idx] += damp
    L = np.linalg.cholesky(H)                      # H = L L^T
    potri = lapack.spotri if ft == np.float32 else lapack.dpotri
    inv, info = potri(L, lower=1)                  # (L L^T)^-1 from L, lower triangle
    if info != 0:
        raise np.linalg.LinAlgError(f"potri info {info}")
    inv = np.tril(inv) + np.tril(inv, -1).T
    Hinv = np.linalg.cholesky(inv).T.astype(ft)    # upper: inv = Hinv^T Hinv
    return W, H, Hinv


def quantize_weight(W, H, scale, zero, group_size: int, bits: int, blocksize: int = 128,
                    percdamp: float = 0.01, precision=np.float32):
    """GPTQ of W (rows x cols) with the Hessian H, GROUP strategy.

    ``scale`` / ``zero``: (rows, ceil(cols / group_size)); column c uses group
    ``c // group_size``.  Returns a dict: ``loss`` (float), ``losses`` (per
    row, half the sum of its loss terms), ``Q`` (fake-quantised W, rows x cols),
    ``codes`` (signed integer codes, int32), ``ratio`` (each column's current
    value over its scale, the number that is rounded), ``W0`` (W with dead
    columns zeroed), ``H`` (the damped Hessian) and ``Hinv``."""
    ft = precision
    W, Hd, Hinv = prepare(W, H, percdamp, ft)
    W0 = W.copy()
    rows, cols = W.shape
    s_all = np.asarray(scale, ft)
    z_all = np.asarray(zero, ft)
    qmin, qmax = qrange(bits)
    codes = np.zeros((rows, cols), np.int32)
    ratio = np.zeros((rows, cols), ft)
    losses = np.zeros(rows, ft)
    for i1 in range(0, cols, blocksize):
        i2 = min(i1 + blocksize, cols)
        count = i2 - i1
        W1 = W[:, i1:i2].copy()
        Q1 = np.zeros_like(W1)
        Err1 = np.zeros_like(W1)
        losses1 = np.zeros_like(W1)
        Hinv1 = Hinv[i1:i2, i1:i2]
        for i in range(count):
            w = W1[:, i].copy()
            d = Hinv1[i, i]
            g = (i1 + i) // group_size
            s = s_all[:, g]
            zp = z_all[:, g]
            t = (w / s).astype(ft)
            ratio[:, i1 + i] = t
            qi = np.clip(np.rint(t) + zp, ft(qmin), ft(qmax)).astype(ft)
            q = ((qi - zp).astype(ft) * s).astype(ft)
            codes[:, i1 + i] = qi.astype(np.int32)
            Q1[:, i] = q
            losses1[:, i] = ((w - q) ** 2 / d ** 2).astype(ft)
            err1 = ((w - q) / d).astype(ft)
            W1[:, i:] -= np.outer(err1, Hinv1[i, i:]).astype(ft)
            Err1[:, i] = err1
        W[:, i1:i2] = Q1
        losses += (np.sum(losses1, axis=1, dtype=ft) / ft(2)).astype(ft)
        W[:, i2:] -= (Err1 @ Hinv[i1:i2, i2:]).astype(ft)
    return {"loss": float(np.sum(losses, dtype=ft)), "losses": losses, "Q": W, "codes": codes,
            "ratio": ratio, "W0": W0, "H": Hd, "Hinv": Hinv}


def gptq_loss_of(W, Q, Hd):
    """Half the quadratic form of the damped Hessian per row, in fp64:
    0.5 (w - q)^T H (w - q).  For exact GPTQ arithmetic this equals the
    per-row loss the column loop accumulates (each column's term is the
    increase of this quadratic form when that column is fixed while the later
    columns stay at their optimum)."""
    D = np.asarray(W, np.float64) - np.asarray(Q, np.float64)
    return 0.5 * np.einsum("ri,ij,rj->r", D, np.asarray(Hd, np.float64), D)
