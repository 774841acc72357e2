"""CPU oracle for the GPTQModel packed format (qweight, qzeros).

TEST INFRASTRUCTURE: only ``tests/``, ``__graft_entry__.smoke()`` and the
bench's CPU-baseline / reference arm may import this module.

What it follows: the "GPTQModel-Compatible Triton Kernel" README, sections
"API Reference" (``gptqmodel_quantized_matmul(x, qweight, qzeros, scales,
bits, group_size)``: qweight of shape (K_packed, N), packed zero points,
scales of shape (num_groups, N)), "Quantization Format" (2-bit: 16 values
per int32, 3-bit: 10 values per int32 with padding, 4-bit: 8, 8-bit: 4) and
"Dequantization Formula" (``scales * (quantized_weight - quantized_zero)``).

The README does not give the bit order or the orientation of qzeros.
Readings (stated here, pinned by hand-worked words in
``tests/golden/gptqmodel_words.txt``):

* V values per word (V = 16, 10, 8, 4 for 2, 3, 4, 8 bits).  Code k of a
  column lives in word k // V of that column at bit ``bits * (k % V)``, the
  lowest bits first -- the order of ``dashq_kernel.py``'s ``_pack_kmajor``.
  For 2, 4 and 8 bits (V = 32 / bits) qweight is therefore bit for bit the
  K-major word array this library's product reads.
* 3-bit words hold 10 codes in bits 0-29; bits 30 and 31 are padding, zero.
  K_packed = ceil(K / 10); a last word with fewer codes is zero above them.
* qzeros has shape (num_groups, ceil(N / V)): the zero point of group g,
  column n is the code in word n // V of row g at bit ``bits * (n % V)`` --
  packed along N the same way.
* No offset is added to the zero points (the README formula has none).
"""
from __future__ import annotations

import numpy as np

VALUES_PER_WORD = {2: 16, 3: 10, 4: 8, 8: 4}


def values_per_word(bits: int) -> int:
    if bits not in VALUES_PER_WORD:
        raise ValueError(f"the GPTQModel format takes 2, 3, 4 or 8 bits, not {bits}")
    return VALUES_PER_WORD[bits]


def pack_rows(codes_kn, bits: int) -> np.ndarray:
    """(K, N) codes -> (ceil(K / V), N) uint32 words, code k at bit bits * (k % V) of word k // V."""
    V = values_per_word(bits)
    q = np.asarray(codes_kn, dtype=np.uint64)
    if q.size and int(q.max()) >= (1 << bits):
        raise ValueError("code out of range")
    K, N = q.shape
    words = np.zeros(((K + V - 1) // V, N), dtype=np.uint64)
    for k in range(K):
        words[k // V] |= q[k] << np.uint64(bits * (k % V))
    return words.astype(np.uint32)


def unpack_rows(words, bits: int, K: int) -> np.ndarray:
    """The inverse of ``pack_rows``: (K, N) uint8 codes."""
    V = values_per_word(bits)
    w = np.asarray(words, dtype=np.uint32)
    out = np.zeros((K, w.shape[1]), dtype=np.uint8)
    for k in range(K):
        out[k] = (w[k // V] >> np.uint32(bits * (k % V))) & np.uint32((1 << bits) - 1)
    return out


def pack_zeros(zeros_gn, bits: int) -> np.ndarray:
    """(groups, N) integer zero points -> (groups, ceil(N / V)) uint32 words packed along N."""
    return pack_rows(np.asarray(zeros_gn).T, bits).T.copy()


def unpack_zeros(qzeros, bits: int, N: int) -> np.ndarray:
    """(groups, ceil(N / V)) words -> (groups, N) uint8 zero points."""
    return unpack_rows(np.asarray(qzeros).T, bits, N).T.copy()


def dequant(qweight, qzeros, scales, K: int, N: int, bits: int, group_size: int, dtype: str = "fp16"):
    """w[k][n] = s[g][n] * (q[k][n] - z[g][n]), g = k // G (G = K for -1), fp64."""
    from .numpy_oracle import widen
    G = K if group_size == -1 else group_size
    q = unpack_rows(qweight, bits, K).astype(np.float64)
    z = unpack_zeros(qzeros, bits, N).astype(np.float64)
    s = widen(scales, dtype)
    g = np.arange(K) // G
    return s[g] * (q - z[g])


def quantized_matmul(x, qweight, qzeros, scales, bits: int, group_size: int, dtype: str = "fp16"):
    """``gptqmodel_quantized_matmul``: y = x @ dequantize(qweight), and the bound sum |x w|, fp64."""
    from .numpy_oracle import widen
    xd = widen(x, dtype)
    K = xd.shape[1]
    N = np.asarray(qweight).shape[1]
    w = dequant(qweight, qzeros, scales, K, N, bits, group_size, dtype)
    return xd @ w, np.abs(xd) @ np.abs(w)
