"""CPU oracle for ``y = x @ dequant(W_q)``.

TEST INFRASTRUCTURE: only ``tests/``, ``__graft_entry__.smoke()`` and the
bench's CPU-baseline / reference arm may import this package.  The product
(``gemm_wq_gemv_b200``) never imports it and never falls back to it.

Two independent restatements of the same plain definition live here:

* ``wq_oracle.c`` (plain C, fp64, loaded with ctypes) -- the oracle proper;
* ``numpy_oracle`` (NumPy, fp64) -- a twin written separately, used to
  cross-check the C file on small shapes.

Both follow ``dashq_kernel.py`` (module docstring, ``_pack_kmajor``,
``_unpack_kmajor``, ``TritonQuantLinear.__init__``, ``dequantize_weight``,
``forward``) and the "GPTQModel-Compatible Triton Kernel" README (sections
"API Reference", "Dequantization Formula", "Group Quantization").

Floating-point inputs (x, scales, zeros, bias) are all fp16 or all bf16
(``dtype="fp16"`` or ``"bf16"``; the module's ``out_dtype``): fp16 arrays as
NumPy ``float16``, bf16 arrays as ``uint16`` bit patterns (NumPy has no
bfloat16).

``mse_observer`` (NumPy) is the oracle of the MSE-observer search of
per-group scales and zero points (the "Benchmark for MSE observer grid
search" page), pinned by ``tests/test_mse_oracle.py``.

Parity pins: every function here is pinned by ``tests/test_oracle_pins.py``
(hand-derived golden words and products, closed forms, brute force, library
special cases); none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

from . import numpy_oracle  # noqa: F401  (re-exported twin)

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "wq_oracle.c"
_LIB = _HERE / "liboracle.so"
_lib = None


class OracleError(RuntimeError):
    pass


def build(force: bool = False) -> Path:
    """Compile ``wq_oracle.c`` into ``liboracle.so`` (gcc -O2, OpenMP, no fast-math)."""
    if force or not _LIB.exists() or _LIB.stat().st_mtime < _SRC.stat().st_mtime:
        tmp = _LIB.with_suffix(f".so.tmp{os.getpid()}")
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall",
               "-o", str(tmp), str(_SRC), "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(str(_LIB))
        p = ctypes.c_void_p
        i = ctypes.c_int
        L.orc_threads.restype = i
        L.orc_set_threads.argtypes = [i]
        L.orc_set_threads.restype = None
        for f in ("orc_half_to_double", "orc_bf16_to_double"):
            getattr(L, f).argtypes = [ctypes.c_uint16]
            getattr(L, f).restype = ctypes.c_double
        L.orc_widen.argtypes = [p, i, i, p]
        L.orc_pack_kmajor.argtypes = [p, i, i, i, p, p]
        L.orc_unpack_kmajor.argtypes = [p, p, i, i, i, p]
        L.orc_dequant.argtypes = [p, p, p, p, i, i, i, i, p, i]
        L.orc_matmul.argtypes = [p, p, i, i, i, p, p, i]
        L.orc_wq_matmul.argtypes = [p, p, p, p, p, i, i, i, i, i, p, p, i]
        L.orc_wq_matmul_sampled.argtypes = [p, p, p, p, p, i, i, i, i, i, p, p, i, p, p, i]
        L.orc_add_bias.argtypes = [p, p, p, i, i, i]
        for f in ("orc_widen", "orc_pack_kmajor", "orc_unpack_kmajor", "orc_dequant", "orc_matmul",
                  "orc_wq_matmul", "orc_wq_matmul_sampled", "orc_add_bias"):
            getattr(L, f).restype = i
        _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _check(rc, what):
    if rc != 0:
        raise OracleError(f"{what} failed with code {rc}")


_DT = {"fp16": 0, "bf16": 1}


def _dt(dtype: str) -> int:
    if dtype not in _DT:
        raise OracleError(f"dtype must be 'fp16' or 'bf16', not {dtype!r}")
    return _DT[dtype]


def _bits(a, dtype: str) -> np.ndarray:
    """The stored 16-bit patterns of an fp16 (float16) or bf16 (uint16) array."""
    if dtype == "bf16":
        a = np.asarray(a)
        if a.dtype != np.uint16:
            raise OracleError("bf16 arrays are passed as uint16 bit patterns")
        return np.ascontiguousarray(a)
    _dt(dtype)
    return np.ascontiguousarray(a, dtype=np.float16).view(np.uint16)


def words_shape(K: int, N: int, bits: int):
    """Shapes of the packed planes: (hi/only plane, lo plane or None)."""
    if bits == 3:
        return (K // 16, N), (K // 32, N)
    return (K // (32 // bits), N), None


def threads() -> int:
    return int(lib().orc_threads())


def set_threads(n: int) -> None:
    """Threads of the OpenMP loops from now on (for timing; results do not depend on it)."""
    lib().orc_set_threads(int(n))


def half_to_double(h: int) -> float:
    return float(lib().orc_half_to_double(int(h) & 0xFFFF))


def bf16_to_double(h: int) -> float:
    return float(lib().orc_bf16_to_double(int(h) & 0xFFFF))


def widen(a, dtype: str = "fp16") -> np.ndarray:
    """The values of an fp16 / bf16 array as fp64 (same shape)."""
    v = _bits(a, dtype)
    out = np.zeros(v.shape, dtype=np.float64)
    _check(lib().orc_widen(_ptr(v), v.size, _dt(dtype), _ptr(out)), "widen")
    return out


def pack(codes_kn: np.ndarray, bits: int):
    """``(K, N)`` uint8 codes -> ``(wq, wlo)`` uint32 words (``wlo`` is None unless 3-bit)."""
    codes = np.ascontiguousarray(codes_kn, dtype=np.uint8)
    K, N = codes.shape
    hs, ls = words_shape(K, N, bits)
    wq = np.zeros(hs, dtype=np.uint32)
    wlo = np.zeros(ls, dtype=np.uint32) if ls else None
    _check(lib().orc_pack_kmajor(_ptr(codes), K, N, bits, _ptr(wq), _ptr(wlo)), "pack")
    return wq, wlo


def unpack(wq: np.ndarray, wlo, K: int, N: int, bits: int) -> np.ndarray:
    wq = np.ascontiguousarray(wq, dtype=np.uint32)
    wlo = None if wlo is None else np.ascontiguousarray(wlo, dtype=np.uint32)
    out = np.zeros((K, N), dtype=np.uint8)
    _check(lib().orc_unpack_kmajor(_ptr(wq), _ptr(wlo), K, N, bits, _ptr(out)), "unpack")
    return out


def dequant(wq, wlo, scales, zeros, K: int, N: int, bits: int, group_size: int,
            dtype: str = "fp16") -> np.ndarray:
    wq = np.ascontiguousarray(wq, dtype=np.uint32)
    wlo = None if wlo is None else np.ascontiguousarray(wlo, dtype=np.uint32)
    s = _bits(scales, dtype)
    z = _bits(zeros, dtype)
    w = np.zeros((K, N), dtype=np.float64)
    _check(lib().orc_dequant(_ptr(wq), _ptr(wlo), _ptr(s), _ptr(z), K, N, bits, group_size,
                             _ptr(w), _dt(dtype)), "dequant")
    return w


def matmul(x, w_kn, dtype: str = "fp16"):
    x = _bits(x, dtype)
    w = np.ascontiguousarray(w_kn, dtype=np.float64)
    M, K = x.shape
    N = w.shape[1]
    y = np.zeros((M, N), dtype=np.float64)
    b = np.zeros((M, N), dtype=np.float64)
    _check(lib().orc_matmul(_ptr(x), _ptr(w), M, K, N, _ptr(y), _ptr(b), _dt(dtype)), "matmul")
    return y, b


def wq_matmul(x, wq, wlo, scales, zeros, bits: int, group_size: int, N: int | None = None, bias=None,
              dtype: str = "fp16"):
    """``(y_ref, bound)`` in fp64 for the packed problem (unpack, dequant, matmul,
    then the optional ``bias`` of shape (N,))."""
    x = _bits(x, dtype)
    M, K = x.shape
    wq = np.ascontiguousarray(wq, dtype=np.uint32)
    N = wq.shape[1] if N is None else N
    wlo = None if wlo is None else np.ascontiguousarray(wlo, dtype=np.uint32)
    s = _bits(scales, dtype)
    z = _bits(zeros, dtype)
    y = np.zeros((M, N), dtype=np.float64)
    b = np.zeros((M, N), dtype=np.float64)
    _check(lib().orc_wq_matmul(_ptr(x), _ptr(wq), _ptr(wlo), _ptr(s), _ptr(z), M, K, N, bits,
                               group_size, _ptr(y), _ptr(b), _dt(dtype)), "wq_matmul")
    if bias is not None:
        add_bias(y, b, bias, dtype)
    return y, b


def add_bias(y, bound, bias, dtype: str = "fp16"):
    """In place: ``y[m][n] += bias[n]``, ``bound[m][n] += |bias[n]|`` (fp64)."""
    bias = _bits(bias, dtype)
    M, N = y.shape
    if bias.shape != (N,) or y.dtype != np.float64 or not y.flags.c_contiguous:
        raise OracleError("add_bias: y (M, N) fp64 contiguous and bias (N,) expected")
    _check(lib().orc_add_bias(_ptr(y), _ptr(bound), _ptr(bias), M, N, _dt(dtype)), "add_bias")


def wq_matmul_sampled(x, wq, wlo, scales, zeros, bits: int, group_size: int, ms, ns, bias=None,
                      dtype: str = "fp16"):
    """``(y_ref, bound)`` for the single outputs ``(ms[i], ns[i])`` (+ ``bias[ns[i]]``)."""
    x = _bits(x, dtype)
    M, K = x.shape
    wq = np.ascontiguousarray(wq, dtype=np.uint32)
    N = wq.shape[1]
    wlo = None if wlo is None else np.ascontiguousarray(wlo, dtype=np.uint32)
    s = _bits(scales, dtype)
    z = _bits(zeros, dtype)
    ms = np.ascontiguousarray(ms, dtype=np.int32)
    ns = np.ascontiguousarray(ns, dtype=np.int32)
    y = np.zeros(len(ms), dtype=np.float64)
    b = np.zeros(len(ms), dtype=np.float64)
    _check(lib().orc_wq_matmul_sampled(_ptr(x), _ptr(wq), _ptr(wlo), _ptr(s), _ptr(z), M, K, N,
                                       bits, group_size, _ptr(ms), _ptr(ns), len(ms), _ptr(y),
                                       _ptr(b), _dt(dtype)), "wq_matmul_sampled")
    if bias is not None:
        bv = widen(bias, dtype)[ns]
        y += bv
        b += np.abs(bv)
    return y, b
