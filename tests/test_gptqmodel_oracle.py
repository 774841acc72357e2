"""Pins for the GPTQModel packed-format oracle (``oracle/gptqmodel_format.py``), CPU only.

The README fixes the number of values per word and the dequantisation formula
but not the bit order; the hand-worked words in
``tests/golden/gptqmodel_words.txt`` pin the reading, the round trips pin
every bit position, and for 2, 4 and 8 bits the format must coincide with the
K-major words this library's product reads (the same rule)."""
import numpy as np
import pytest

import oracle.gptqmodel_format as gf
import oracle.numpy_oracle as no
from _golden import read_cases

CASES = read_cases("gptqmodel_words.txt")


@pytest.mark.parametrize("name", sorted(CASES))
def test_golden_words(name):
    c = CASES[name]
    bits = c["bits"]
    if "qz" in c:
        z = np.array(c["zeros"], np.uint8).reshape(1, -1)
        w = gf.pack_zeros(z, bits)
        assert np.array_equal(w.ravel(), np.array(c["qz"], np.uint32)), name
        assert np.array_equal(gf.unpack_zeros(w, bits, c["N"]), z), name
    else:
        codes = np.array(c["codes"], np.uint8).reshape(c["K"], c["N"])
        w = gf.pack_rows(codes, bits)
        assert np.array_equal(w.ravel(), np.array(c["wq"], np.uint32)), name
        assert np.array_equal(gf.unpack_rows(w, bits, c["K"]), codes), name


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_every_code_at_every_position(bits):
    """A single nonzero code at each row (and each column for qzeros) lands in
    exactly its own field and comes back; 3-bit padding bits stay zero."""
    V = gf.values_per_word(bits)
    K = 3 * V + 1
    top = (1 << bits) - 1
    for k in range(K):
        codes = np.zeros((K, 2), np.uint8)
        codes[k, 1] = top
        w = gf.pack_rows(codes, bits)
        assert w.shape == ((K + V - 1) // V, 2)
        assert np.count_nonzero(w) == 1 and w[k // V, 1] == np.uint32(top << (bits * (k % V)))
        assert np.array_equal(gf.unpack_rows(w, bits, K), codes)
    if bits == 3:
        rng = np.random.default_rng(0)
        w = gf.pack_rows(rng.integers(0, 8, size=(40, 5)), 3)
        assert not np.any(w >> np.uint32(30))


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_same_words_as_the_kmajor_format(bits):
    """For V = 32 / bits the reading gives the product's own K-major words."""
    rng = np.random.default_rng(bits)
    codes = rng.integers(0, 1 << bits, size=(256, 12)).astype(np.uint8)
    assert np.array_equal(gf.pack_rows(codes, bits), no.pack(codes, bits)[0])


def test_dequant_formula():
    """s * (q - z) with g = k // G, per-channel G = K: a small case worked out directly."""
    codes = np.array([[1, 5], [3, 0], [2, 7], [0, 4]], np.uint8)          # K = 4, N = 2
    zeros = np.array([[1, 2], [3, 3]], np.uint8)                            # G = 2
    scales = np.array([[0.5, 2.0], [0.25, 1.0]], np.float16)
    w = gf.dequant(gf.pack_rows(codes, 4), gf.pack_zeros(zeros, 4), scales, 4, 2, 4, 2)
    expect = np.array([[0.0, 6.0], [1.0, -4.0], [-0.25, 4.0], [-0.75, 1.0]])
    assert np.array_equal(w, expect)
    w1 = gf.dequant(gf.pack_rows(codes, 4), gf.pack_zeros(zeros[:1], 4), scales[:1], 4, 2, 4, -1)
    assert np.array_equal(w1, np.array([[0.0, 6.0], [1.0, -4.0], [0.5, 10.0], [-0.5, 4.0]]))


def test_rejects():
    with pytest.raises(ValueError):
        gf.values_per_word(1)
    with pytest.raises(ValueError):
        gf.pack_rows(np.full((4, 1), 8, np.uint8), 3)
