"""NumPy twin of the C oracle (fp64).

TEST INFRASTRUCTURE, written separately from ``wq_oracle.c`` so the two can
check each other.  It follows the same passages:

* ``dashq_kernel.py`` module docstring and ``_pack_kmajor``: row k of a
  ``(K, N)`` code matrix goes to word ``k // eps`` at bit ``bits * (k % eps)``,
  ``eps = 32 // bits``;
* ``_unpack_kmajor``: ``(word >> bits*j) & (2**bits - 1)``;
* ``TritonQuantLinear.__init__`` / ``dequantize_weight``: 3-bit codes are a
  2-bit plane of ``q >> 1`` and a 1-bit plane of ``q & 1``;
  ``w = (q - z) * s`` with ``s, z`` repeated over each group of rows;
* "GPTQModel-Compatible Triton Kernel" README, "API Reference" and
  "Group Quantization": ``y = x @ dequantize(qweight)``, ``group_size = -1``
  is one group per output channel.

The matmul step is NumPy's fp64 matmul (a library primitive).

Floating-point inputs are fp16 (NumPy ``float16``) or bf16 (``uint16`` bit
patterns): a bf16 value is the upper half of the binary32 with the same top 16
bits, so it widens through NumPy's ``float32``.
"""
from __future__ import annotations

import numpy as np


def _eps(bits: int) -> int:
    return 32 // bits


def pack_plane(v_kn: np.ndarray, bits: int) -> np.ndarray:
    v = np.asarray(v_kn, dtype=np.uint64)
    K, N = v.shape
    eps = _eps(bits)
    assert K % eps == 0
    parts = v.reshape(K // eps, eps, N)
    shifts = (np.arange(eps, dtype=np.uint64) * np.uint64(bits)).reshape(1, eps, 1)
    words = np.bitwise_or.reduce(parts << shifts, axis=1)
    return words.astype(np.uint32)


def pack(codes_kn: np.ndarray, bits: int):
    codes = np.asarray(codes_kn, dtype=np.uint8)
    if bits not in (1, 2, 3, 4, 8):
        raise ValueError(f"unsupported bits {bits}")
    if codes.size and int(codes.max()) >= (1 << bits):
        raise ValueError("code out of range")
    if bits == 3:
        assert codes.shape[0] % 32 == 0
        return pack_plane(codes >> 1, 2), pack_plane(codes & 1, 1)
    return pack_plane(codes, bits), None


def unpack_plane(words: np.ndarray, bits: int) -> np.ndarray:
    w = np.asarray(words, dtype=np.uint32)
    WK, N = w.shape
    eps = _eps(bits)
    shifts = (np.arange(eps, dtype=np.uint32) * np.uint32(bits)).reshape(1, eps, 1)
    q = (w.reshape(WK, 1, N) >> shifts) & np.uint32((1 << bits) - 1)
    return q.reshape(WK * eps, N)


def unpack(wq, wlo, K: int, N: int, bits: int) -> np.ndarray:
    if bits == 3:
        hi = unpack_plane(wq, 2)[:K]
        lo = unpack_plane(wlo, 1)[:K]
        return ((hi << 1) | lo).astype(np.uint8)
    return unpack_plane(wq, bits)[:K].astype(np.uint8)


def widen(a, dtype: str = "fp16") -> np.ndarray:
    """fp16 / bf16 values as fp64."""
    if dtype == "bf16":
        u = np.asarray(a)
        if u.dtype != np.uint16:
            raise ValueError("bf16 arrays are passed as uint16 bit patterns")
        return (u.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    if dtype != "fp16":
        raise ValueError(f"unsupported dtype {dtype}")
    return np.asarray(a, dtype=np.float16).astype(np.float64)


def dequant(wq, wlo, scales, zeros, K: int, N: int, bits: int, group_size: int,
            dtype: str = "fp16") -> np.ndarray:
    G = K if group_size == -1 else group_size
    q = unpack(wq, wlo, K, N, bits).astype(np.float64)
    s = np.repeat(widen(scales, dtype), G, axis=0)
    z = np.repeat(widen(zeros, dtype), G, axis=0)
    return (q - z) * s


def wq_matmul(x, wq, wlo, scales, zeros, bits: int, group_size: int, N: int | None = None, bias=None,
              dtype: str = "fp16"):
    """y = x @ w (+ bias[n], one value per output column, as the module's
    forward adds it), and the bound sum |x w| (+ |bias|)."""
    x = widen(x, dtype)
    K = x.shape[1]
    N = np.asarray(wq).shape[1] if N is None else N
    w = dequant(wq, wlo, scales, zeros, K, N, bits, group_size, dtype)
    y, b = x @ w, np.abs(x) @ np.abs(w)
    if bias is not None:
        bv = widen(bias, dtype).reshape(1, N)
        y, b = y + bv, b + np.abs(bv)
    return y, b
