"""The pins are strong enough: each plausible oracle mistake fails at least one.

Each mutant below is a copy of the NumPy twin with one planted mistake (run on
the CPU only).  A mutant that passed every pin would mean the pins could not
tell that mistake from the right answer.
"""
import types

import numpy as np
import pytest

import oracle_pins
from oracle import numpy_oracle as tw


def _mutant(**overrides):
    m = types.SimpleNamespace(pack=tw.pack, unpack=tw.unpack, wq_matmul=tw.wq_matmul)
    for k, v in overrides.items():
        setattr(m, k, v)
    return m


def _with_bias(y, b, bias, N, sign=1.0, by_row=False, dtype="fp16", widen=tw.widen):
    if bias is None:
        return y, b
    bv = widen(bias, dtype)
    if by_row:  # indexed by the token instead of the output column
        bv = np.resize(bv, y.shape[0]).reshape(-1, 1)
    else:
        bv = bv.reshape(1, N)
    return y + sign * bv, b + np.abs(bv)


def _matmul_with(dequant_fn, bias_sign=1.0, bias_by_row=False, bias_used=True, widen=tw.widen):
    def wq_matmul(x, wq, wlo, s, z, bits, G, N=None, bias=None, dtype="fp16"):
        x = widen(x, dtype)
        K = x.shape[1]
        N = np.asarray(wq).shape[1] if N is None else N
        w = dequant_fn(wq, wlo, s, z, K, N, bits, G, dtype)
        return _with_bias(x @ w, np.abs(x) @ np.abs(w), bias if bias_used else None, N,
                          bias_sign, bias_by_row, dtype, widen)
    return wq_matmul


def _transposed(x, wq, wlo, s, z, bits, G, N=None, bias=None, dtype="fp16"):
    xx = tw.widen(x, dtype)
    N = np.asarray(wq).shape[1] if N is None else N
    w = tw.dequant(wq, wlo, s, z, xx.shape[1], N, bits, G, dtype)
    y = xx @ (w.T if w.shape[0] == w.shape[1] else w[::-1])
    return _with_bias(y, np.abs(xx) @ np.abs(w), bias, N, dtype=dtype)


def _bf16_as_fp16(a, dtype="fp16"):  # bf16 patterns read as binary16
    if dtype == "bf16":
        return np.asarray(a, np.uint16).view(np.float16).astype(np.float64)
    return tw.widen(a, dtype)


def _bf16_bias_126(a, dtype="fp16"):  # bf16 exponent bias off by one
    return tw.widen(a, dtype) * (2.0 if dtype == "bf16" else 1.0)


def _bf16_fraction_8(a, dtype="fp16"):  # bf16 split as 7 exponent + 8 fraction bits
    if dtype != "bf16":
        return tw.widen(a, dtype)
    u = np.asarray(a, np.uint16).astype(np.int64)
    e, f = (u >> 8) & 0x7F, u & 0xFF
    v = np.where(e == 0, f * 2.0 ** -70, (256 + f) * 2.0 ** (e - 63 - 8))
    return np.where(u & 0x8000, -v, v)


def _dq(q_fn=None, combine=lambda q, z, s: (q - z) * s, expand=np.repeat, widen=tw.widen):
    def dequant(wq, wlo, s, z, K, N, bits, G, dtype="fp16"):
        Gr = K if G == -1 else G
        q = (q_fn or tw.unpack)(wq, wlo, K, N, bits).astype(np.float64)
        s64 = widen(s, dtype)
        z64 = widen(z, dtype)
        if expand is np.repeat:
            s64, z64 = np.repeat(s64, Gr, axis=0), np.repeat(z64, Gr, axis=0)
        else:
            s64, z64 = expand(s64, Gr, K), expand(z64, Gr, K)
        return combine(q, z64, s64)
    return dequant


def _tile(a, Gr, K):  # row k takes group k % groups instead of k // G
    return np.stack([a[k % a.shape[0]] for k in range(K)])


def _shifted(a, Gr, K):  # off-by-one group
    return np.stack([a[min(k // Gr + 1, a.shape[0] - 1)] for k in range(K)])


def _pack_reversed(codes, bits):
    codes = np.asarray(codes, np.uint8)
    if bits == 3:
        return tw.pack(codes, 3)
    K, N = codes.shape
    eps = 32 // bits
    v = codes.astype(np.uint64).reshape(K // eps, eps, N)
    sh = (np.arange(eps)[::-1].astype(np.uint64) * np.uint64(bits)).reshape(1, eps, 1)
    return np.bitwise_or.reduce(v << sh, axis=1).astype(np.uint32), None


def _pack_planes_swapped(codes, bits):
    if bits != 3:
        return tw.pack(codes, bits)
    codes = np.asarray(codes, np.uint8)
    return tw.pack_plane((codes & 1) * 1 + 0, 2), tw.pack_plane(codes >> 2, 1)


def _unpack_no_mask(wq, wlo, K, N, bits):
    if bits == 3:
        return tw.unpack(wq, wlo, K, N, bits)
    w = np.asarray(wq, np.uint32).view(np.int32)
    eps = 32 // bits
    q = np.stack([(w >> (bits * j)) for j in range(eps)], axis=1)  # arithmetic shift, no mask
    q = np.where(np.arange(eps).reshape(1, eps, 1) == eps - 1, q, q & ((1 << bits) - 1))
    return q.reshape(-1, N)[:K].astype(np.uint8)


def _unpack_3bit_lo_index(wq, wlo, K, N, bits):
    if bits != 3:
        return tw.unpack(wq, wlo, K, N, bits)
    hi = tw.unpack_plane(wq, 2)[:K]
    lo = tw.unpack_plane(wlo, 1)
    lo = np.stack([lo[(k % 16) + 16 * (k // 32)] for k in range(K)])  # wrong bit of the lo word
    return ((hi << 1) | lo).astype(np.uint8)


MUTANTS = {
    "zero_point_dropped": _mutant(wq_matmul=_matmul_with(_dq(combine=lambda q, z, s: q * s))),
    "sign_flipped": _mutant(wq_matmul=_matmul_with(_dq(combine=lambda q, z, s: (z - q) * s))),
    "scale_missing": _mutant(wq_matmul=_matmul_with(_dq(combine=lambda q, z, s: q - z))),
    "group_index_modulo": _mutant(wq_matmul=_matmul_with(_dq(expand=_tile))),
    "group_index_off_by_one": _mutant(wq_matmul=_matmul_with(_dq(expand=_shifted))),
    "shift_order_reversed": _mutant(pack=_pack_reversed),
    "planes_swapped_3bit": _mutant(pack=_pack_planes_swapped),
    "top_field_sign_extended": _mutant(unpack=_unpack_no_mask,
                                       wq_matmul=_matmul_with(_dq(q_fn=_unpack_no_mask))),
    "lo_plane_bit_index_3bit": _mutant(unpack=_unpack_3bit_lo_index,
                                       wq_matmul=_matmul_with(_dq(q_fn=_unpack_3bit_lo_index))),
    "operand_transposed": _mutant(wq_matmul=_transposed),
    "bias_dropped": _mutant(wq_matmul=_matmul_with(tw.dequant, bias_used=False)),
    "bias_sign_flipped": _mutant(wq_matmul=_matmul_with(tw.dequant, bias_sign=-1.0)),
    "bias_indexed_by_token": _mutant(wq_matmul=_matmul_with(tw.dequant, bias_by_row=True)),
    "bf16_read_as_fp16": _mutant(wq_matmul=_matmul_with(_dq(widen=_bf16_as_fp16), widen=_bf16_as_fp16)),
    "bf16_exponent_bias_126": _mutant(wq_matmul=_matmul_with(_dq(widen=_bf16_bias_126),
                                                             widen=_bf16_bias_126)),
    "bf16_fraction_width_8": _mutant(wq_matmul=_matmul_with(_dq(widen=_bf16_fraction_8),
                                                            widen=_bf16_fraction_8)),
    "bf16_scale_read_as_fp16": _mutant(wq_matmul=_matmul_with(_dq(widen=_bf16_as_fp16))),
    "bound_signed": _mutant(
        wq_matmul=lambda *a, **k: (lambda r: (r[0], np.abs(r[0])))(tw.wq_matmul(*a, **k))),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_some_pin_catches_mutant(name):
    impl = MUTANTS[name]
    failed = []
    for pin in oracle_pins.PINS:
        try:
            pin(impl)
        except (AssertionError, ValueError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"mutant {name} passed every pin"


def test_unmutated_twin_passes_every_pin():
    for pin in oracle_pins.PINS:
        pin(_mutant())
