"""Seeded synthetic inputs for the weight-only quantized matrix product.

This module draws random numbers and nothing else: it holds none of the
method's arithmetic (no packing, no dequantisation, no product).  Both the CPU
oracle (through the tests) and the CUDA path (through the tests and the bench)
take their inputs from here, so the two sides see byte-identical data.

Shapes and distributions follow the workloads the method is described on
(``dashq_kernel.py``: K-major codes ``(K, N)``, per-group ``s, z`` of shape
``(K // group_size, N)``; "GPTQModel-Compatible Triton Kernel" README, section
"API Reference": ``x`` of shape ``(M, K)``, ``group_size = -1`` meaning one
group per output channel).

Recipe (one ``numpy.random.default_rng(seed)`` stream, PCG64, drawn in this
order): ``x`` ~ N(0, 1) rounded to fp16; codes uniform integers in
``[0, 2**bits - 1]``; scales uniform in ``[s_lo, s_hi]`` rounded to fp16;
zeros uniform integers in ``[0, 2**bits - 1]`` stored as fp16.

bf16 problems (``dtype="bf16"``) take the same draws from the same stream and
round x and the scales to bfloat16 instead (round to nearest, ties to even);
their x, scales, zeros and bias are ``uint16`` bit patterns, NumPy having no
bfloat16 type.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np


@dataclass(frozen=True)
class Workload:
    """One synthetic problem: ``y (M, N) = x (M, K) @ dequant(codes (K, N))``."""

    name: str
    M: int
    K: int
    N: int
    bits: int
    group_size: int  # -1: one group spanning all of K
    s_lo: float = 0.005
    s_hi: float = 0.02

    @property
    def groups(self) -> int:
        return 1 if self.group_size == -1 else self.K // self.group_size


@dataclass
class Case:
    """Host arrays of one drawn problem (numpy, C-contiguous)."""

    wl: Workload
    x: np.ndarray        # (M, K) float16
    codes: np.ndarray    # (K, N) uint8, values in [0, 2**bits - 1]
    scales: np.ndarray   # (groups, N) float16
    zeros: np.ndarray    # (groups, N) float16, integer-valued
    seed: int = 0
    extra: dict = field(default_factory=dict)
    dtype: str = "fp16"  # "bf16": x, scales, zeros hold bfloat16 bit patterns (uint16)


# The named workloads: the small parity case, the decode GEMV at three token
# counts, the 3-bit two-plane GEMV, the bit-width sweep and the batched GEMM.
WORKLOADS = {
    "tiny_gemv": Workload("tiny_gemv", 1, 512, 256, 4, 128),
    "decode_gemv_m1": Workload("decode_gemv_m1", 1, 4096, 4096, 4, 128),
    "decode_gemv_m4": Workload("decode_gemv_m4", 4, 4096, 4096, 4, 128),
    "decode_gemv_m16": Workload("decode_gemv_m16", 16, 4096, 4096, 4, 128),
    "gemv_3bit": Workload("gemv_3bit", 1, 4096, 11008, 3, 128, 0.01, 0.04),
    "sweep_1bit": Workload("sweep_1bit", 1, 8192, 8192, 1, 128),
    "sweep_2bit": Workload("sweep_2bit", 1, 8192, 8192, 2, 128),
    "sweep_8bit": Workload("sweep_8bit", 1, 8192, 8192, 8, 128),
    "sweep_8bit_perchannel": Workload("sweep_8bit_perchannel", 1, 8192, 8192, 8, -1),
    "prefill_gemm": Workload("prefill_gemm", 512, 4096, 2048, 4, 128),
}


def bf16_bits(a) -> np.ndarray:
    """Finite values rounded to bfloat16 (nearest, ties to even), as uint16 bit patterns."""
    u = np.ascontiguousarray(np.asarray(a, dtype=np.float64).astype(np.float32)).view(np.uint32)
    u = u.astype(np.uint64)
    r = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return np.ascontiguousarray(r.astype(np.uint16))


def _as(a, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return bf16_bits(a)
    if dtype != "fp16":
        raise ValueError(f"dtype must be 'fp16' or 'bf16', not {dtype!r}")
    return np.ascontiguousarray(np.asarray(a).astype(np.float16))


def draw(wl: Workload, seed: int = 0, dtype: str = "fp16") -> Case:
    """Draw one problem for workload ``wl`` from ``default_rng(seed)``."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((wl.M, wl.K))
    qmax = (1 << wl.bits) - 1
    codes = rng.integers(0, qmax + 1, size=(wl.K, wl.N), dtype=np.int64).astype(np.uint8)
    scales = rng.uniform(wl.s_lo, wl.s_hi, size=(wl.groups, wl.N))
    zeros = rng.integers(0, qmax + 1, size=(wl.groups, wl.N), dtype=np.int64)
    return Case(wl, _as(x, dtype), np.ascontiguousarray(codes), _as(scales, dtype),
                _as(zeros, dtype), seed, dtype=dtype)


def custom(M: int, K: int, N: int, bits: int, group_size: int, seed: int = 0,
           s_lo: float = 0.005, s_hi: float = 0.02, name: str = "custom",
           dtype: str = "fp16") -> Case:
    """Draw a problem of arbitrary shape with the same distributions."""
    return draw(Workload(name, M, K, N, bits, group_size, s_lo, s_hi), seed, dtype)


def x_batch(M: int, K: int, seed: int, dtype: str = "fp16") -> np.ndarray:
    """A fresh ``(M, K)`` activation block ~ N(0, 1)."""
    rng = np.random.default_rng(seed)
    return _as(rng.standard_normal((M, K)), dtype)


def bias_vector(N: int, seed: int, dtype: str = "fp16") -> np.ndarray:
    """A fused-bias vector ``(N,)`` ~ U[-1, 1]."""
    rng = np.random.default_rng(seed)
    return _as(rng.uniform(-1.0, 1.0, size=N), dtype)


def gptq_problem(rows: int, cols: int, seed: int = 42):
    """The GPTQ benchmark's synthetic problem ("benchmark GPTQ implementations"
    page, ``make_inputs``): W (rows x cols) fp32 drawn as a linear layer's
    default initialisation, U[-1/sqrt(cols), 1/sqrt(cols)], and the positive
    definite Hessian H = A A^T + I (cols x cols, fp32) with A ~ N(0, 1).

    One ``default_rng(seed)`` stream: W first, then A.  H is formed in fp32,
    as on the page (the bytes may differ between BLAS builds in the last
    place; both sides of a comparison are given the same array)."""
    rng = np.random.default_rng(seed)
    bound = 1.0 / np.sqrt(cols)
    W = rng.uniform(-bound, bound, size=(rows, cols)).astype(np.float32)
    A = rng.standard_normal((cols, cols)).astype(np.float32)
    H = A @ A.T
    H[np.arange(cols), np.arange(cols)] += np.float32(1.0)
    return W, H
