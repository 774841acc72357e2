"""Pins for the CPU oracle: facts fixed by the pages and by mathematics.

Each ``pin_*`` takes an implementation ``impl`` with ``pack``, ``unpack`` and
``wq_matmul`` (the C oracle, its NumPy twin, or a deliberately broken copy of
the twin) and raises ``AssertionError`` when the implementation disagrees with
the fact.  None of the expected values below comes from the implementation
under test or from the CUDA library:

* golden words and products were worked out by hand (``tests/golden/``);
* closed forms: all ``q == z`` gives ``y = 0``; a one-hot ``x = e_k`` gives
  row ``k`` of the dequantised matrix; the product is linear in ``x``;
* special cases: 8-bit with ``s = 1, z = 0`` is a plain integer matmul (checked
  with NumPy's matmul); per-channel equals grouped when all groups share
  ``s, z``; ``group_size = -1`` equals ``group_size = K``;
* brute force: every single-code matrix of a tiny shape packs to the one word
  the layout rule predicts;
* bf16 inputs: values that fp16 and bf16 both hold exactly give the same
  product as fp16; powers of two beyond fp16's range (bit patterns written
  from the bfloat16 field layout) give products known in closed form.
"""
from __future__ import annotations

import numpy as np

from _golden import read_cases, words

BITS = (1, 2, 3, 4, 8)


def _kdiv(bits):
    return 32 if bits == 3 else 32 // bits


def _rng(seed):
    return np.random.default_rng(1000 + seed)


def pin_golden_pack(impl):
    """Hand-derived words (dashq_kernel.py `_pack_kmajor`, 3-bit planes)."""
    for name, c in read_cases("pack_words.txt").items():
        K, N, bits = c["K"], c["N"], c["bits"]
        codes = np.array(c["codes"], dtype=np.uint8).reshape(K, N)
        wq, wlo = impl.pack(codes, bits)
        assert np.array_equal(np.asarray(wq, np.uint32), words(c, "wq", N)), name
        if bits == 3:
            assert np.array_equal(np.asarray(wlo, np.uint32), words(c, "wlo", N)), name
        back = impl.unpack(words(c, "wq", N), words(c, "wlo", N), K, N, bits)
        assert np.array_equal(back, codes), name


def pin_golden_products(impl):
    """Hand-computed products (README "Dequantization Formula", "API Reference")."""
    for name, c in read_cases("products.txt").items():
        M, K, N, bits, G = c["M"], c["K"], c["N"], c["bits"], c["group"]
        groups = 1 if G == -1 else K // G
        x = np.array(c["x"], dtype=np.float16).reshape(M, K)
        s = np.array(c["scales"], dtype=np.float16).reshape(groups, N)
        z = np.array(c["zeros"], dtype=np.float16).reshape(groups, N)
        codes = np.array(c["codes"], dtype=np.uint8).reshape(K, N)
        wq, wlo = impl.pack(codes, bits)
        assert np.array_equal(np.asarray(wq, np.uint32), words(c, "wq", N)), name
        y, b = impl.wq_matmul(x, words(c, "wq", N), words(c, "wlo", N), s, z, bits, G)
        assert np.array_equal(y, np.array(c["y"]).reshape(M, N)), (name, y)
        assert np.array_equal(b, np.array(c["bound"]).reshape(M, N)), (name, b)


def pin_roundtrip(impl):
    """unpack(pack(q)) == q bit for bit, with 0 and 2**bits-1 at every bit position."""
    for bits in BITS:
        kd = _kdiv(bits)
        K, N = 2 * kd, 5
        rng = _rng(bits)
        codes = rng.integers(0, 1 << bits, size=(K, N)).astype(np.uint8)
        codes[:, 0] = (1 << bits) - 1
        codes[:, 1] = 0
        codes[::2, 2] = (1 << bits) - 1
        wq, wlo = impl.pack(codes, bits)
        assert np.array_equal(impl.unpack(wq, wlo, K, N, bits), codes), bits
        assert np.all(np.asarray(wq, np.uint32)[:, 0] == 0xFFFFFFFF), bits
        assert np.all(np.asarray(wq, np.uint32)[:, 1] == 0), bits


def pin_single_code_bruteforce(impl):
    """Every single nonzero code at every row lands at the predicted bits."""
    for bits in (1, 2, 4, 8):
        eps = 32 // bits
        K = 2 * eps
        for v in range(1, 1 << bits):
            for k in range(K):
                codes = np.zeros((K, 2), dtype=np.uint8)
                codes[k, 1] = v
                wq, _ = impl.pack(codes, bits)
                expect = np.zeros((K // eps, 2), dtype=np.uint32)
                expect[k // eps, 1] = np.uint32(v) << np.uint32(bits * (k % eps))
                assert np.array_equal(np.asarray(wq, np.uint32), expect), (bits, v, k)
    for v in range(1, 8):
        for k in range(32):
            codes = np.zeros((32, 1), dtype=np.uint8)
            codes[k, 0] = v
            wq, wlo = impl.pack(codes, 3)
            hi = np.zeros((2, 1), dtype=np.uint32)
            lo = np.zeros((1, 1), dtype=np.uint32)
            hi[k // 16, 0] = np.uint32(v >> 1) << np.uint32(2 * (k % 16))
            lo[0, 0] = np.uint32(v & 1) << np.uint32(k)
            assert np.array_equal(np.asarray(wq, np.uint32), hi), (3, v, k)
            assert np.array_equal(np.asarray(wlo, np.uint32), lo), (3, v, k)


def _problem(bits, M, K, N, G, seed, int_zeros=True):
    rng = _rng(seed)
    groups = 1 if G == -1 else K // G
    x = rng.standard_normal((M, K)).astype(np.float16)
    codes = rng.integers(0, 1 << bits, size=(K, N)).astype(np.uint8)
    s = rng.uniform(0.005, 0.05, size=(groups, N)).astype(np.float16)
    if int_zeros:
        z = rng.integers(0, 1 << bits, size=(groups, N)).astype(np.float16)
    else:
        z = rng.uniform(0, (1 << bits) - 1, size=(groups, N)).astype(np.float16)
    return x, codes, s, z


def pin_zero_when_q_equals_z(impl):
    """All q == z gives y = 0 exactly, whatever x and s."""
    for bits in BITS:
        kd = _kdiv(bits)
        for G in (kd * 2, -1):
            K, N, M = kd * 4, 6, 3
            groups = 1 if G == -1 else K // G
            x, _, s, _ = _problem(bits, M, K, N, G, bits)
            zq = _rng(bits + 50).integers(0, 1 << bits, size=(groups, N))
            Gr = K if G == -1 else G
            codes = np.repeat(zq, Gr, axis=0).astype(np.uint8)
            wq, wlo = impl.pack(codes, bits)
            y, b = impl.wq_matmul(x, wq, wlo, s, zq.astype(np.float16), bits, G)
            assert np.all(y == 0.0), (bits, G)
            assert np.all(b == 0.0), (bits, G)


def pin_one_hot_row(impl):
    """x = e_k picks row k of w = (q - z[k // G]) * s[k // G], exactly."""
    for bits in BITS:
        kd = _kdiv(bits)
        for G in (kd, 2 * kd, -1):
            K, N = 4 * kd, 7
            groups = 1 if G == -1 else K // G
            Gr = K if G == -1 else G
            _, codes, s, z = _problem(bits, 1, K, N, G, 7 * bits, int_zeros=False)
            wq, wlo = impl.pack(codes, bits)
            x = np.eye(K, dtype=np.float16)
            y, _ = impl.wq_matmul(x, wq, wlo, s, z, bits, G)
            for k in range(K):
                g = k // Gr
                expect = (codes[k].astype(np.float64) - z[g].astype(np.float64)) * s[g].astype(np.float64)
                assert np.array_equal(y[k], expect), (bits, G, k)
            assert groups >= 1


def pin_linearity(impl):
    """y(x1 + x2) == y(x1) + y(x2); exact for small integer x and power-of-two s."""
    for bits in BITS:
        kd = _kdiv(bits)
        K, N, G = 4 * kd, 5, 2 * kd
        rng = _rng(200 + bits)
        codes = rng.integers(0, 1 << bits, size=(K, N)).astype(np.uint8)
        s = (2.0 ** rng.integers(-6, -2, size=(K // G, N))).astype(np.float16)
        z = rng.integers(0, 1 << bits, size=(K // G, N)).astype(np.float16)
        x1 = rng.integers(-8, 9, size=(2, K)).astype(np.float16)
        x2 = rng.integers(-8, 9, size=(2, K)).astype(np.float16)
        wq, wlo = impl.pack(codes, bits)
        y1, _ = impl.wq_matmul(x1, wq, wlo, s, z, bits, G)
        y2, _ = impl.wq_matmul(x2, wq, wlo, s, z, bits, G)
        y12, _ = impl.wq_matmul((x1 + x2).astype(np.float16), wq, wlo, s, z, bits, G)
        assert np.array_equal(y12, y1 + y2), bits


def pin_integer_matmul_special_case(impl):
    """8-bit, s = 1, z = 0: the product is x @ codes (NumPy's matmul)."""
    rng = _rng(300)
    K, N, M = 64, 9, 3
    codes = rng.integers(0, 256, size=(K, N)).astype(np.uint8)
    x = rng.standard_normal((M, K)).astype(np.float16)
    wq, wlo = impl.pack(codes, 8)
    for G in (-1, 16):
        groups = 1 if G == -1 else K // G
        ones = np.ones((groups, N), dtype=np.float16)
        zero = np.zeros((groups, N), dtype=np.float16)
        y, _ = impl.wq_matmul(x, wq, wlo, ones, zero, 8, G)
        ref = x.astype(np.float64) @ codes.astype(np.float64)
        assert np.allclose(y, ref, rtol=1e-13, atol=1e-10), G


def pin_group_equivalences(impl):
    """group -1 == group K; groups sharing (s, z) == one group."""
    for bits in BITS:
        kd = _kdiv(bits)
        K, N, M = 4 * kd, 6, 2
        x, codes, s1, z1 = _problem(bits, M, K, N, -1, 400 + bits)
        wq, wlo = impl.pack(codes, bits)
        ya, _ = impl.wq_matmul(x, wq, wlo, s1, z1, bits, -1)
        yb, _ = impl.wq_matmul(x, wq, wlo, s1, z1, bits, K)
        assert np.array_equal(ya, yb), bits
        G = kd
        s4 = np.repeat(s1, K // G, axis=0)
        z4 = np.repeat(z1, K // G, axis=0)
        yc, _ = impl.wq_matmul(x, wq, wlo, s4, z4, bits, G)
        assert np.array_equal(ya, yc), bits


def pin_group_index(impl):
    """Distinct per-group scales: row k must use group k // G, not k % G."""
    bits, K, N, G = 4, 64, 3, 16
    codes = np.full((K, N), 9, dtype=np.uint8)
    s = np.array([[1.0] * N, [2.0] * N, [4.0] * N, [8.0] * N], dtype=np.float16)
    z = np.array([[1.0] * N, [2.0] * N, [3.0] * N, [5.0] * N], dtype=np.float16)
    wq, wlo = impl.pack(codes, bits)
    x = np.zeros((K // G, K), dtype=np.float16)
    for g in range(K // G):
        x[g, g * G:(g + 1) * G] = 1.0
    y, _ = impl.wq_matmul(x, wq, wlo, s, z, bits, G)
    expect = np.array([16 * 8 * 1.0, 16 * 7 * 2.0, 16 * 6 * 4.0, 16 * 4 * 8.0])
    assert np.array_equal(y[:, 0], expect), y[:, 0]


def pin_bias(impl):
    """The fused bias (one fp16 value per output column, added after the
    product): with x = 0, or with every q == z, y is the bias exactly in every
    row and the bound is |bias|; with x = e_k, row k is w[k] + bias, exact in
    fp64 since both addends are exact."""
    for bits in (1, 3, 4, 8):
        kd = _kdiv(bits)
        K, N, M, G = 4 * kd, 9, 3, 2 * kd
        x, codes, s, z = _problem(bits, M, K, N, G, 300 + bits, int_zeros=False)
        bias = _rng(400 + bits).uniform(-3, 3, size=N).astype(np.float16)
        bias64 = bias.astype(np.float64)
        wq, wlo = impl.pack(codes, bits)
        y, b = impl.wq_matmul(np.zeros_like(x), wq, wlo, s, z, bits, G, bias=bias)
        assert np.array_equal(y, np.tile(bias64, (M, 1))), (bits, "x = 0")
        assert np.array_equal(b, np.tile(np.abs(bias64), (M, 1))), (bits, "bound, x = 0")
        zq = _rng(bits + 60).integers(0, 1 << bits, size=(K // G, N))
        wq0, wlo0 = impl.pack(np.repeat(zq, G, axis=0).astype(np.uint8), bits)
        y, _ = impl.wq_matmul(x, wq0, wlo0, s, zq.astype(np.float16), bits, G, bias=bias)
        assert np.array_equal(y, np.tile(bias64, (M, 1))), (bits, "q == z")
        y, _ = impl.wq_matmul(np.eye(K, dtype=np.float16), wq, wlo, s, z, bits, G, bias=bias)
        for k in range(K):
            g = k // G
            row = (codes[k].astype(np.float64) - z[g].astype(np.float64)) * s[g].astype(np.float64)
            assert np.array_equal(y[k], row + bias64), (bits, "one-hot", k)


def _bf16_exact(a):
    """bf16 bit patterns of values that bfloat16 holds exactly (checked)."""
    f = np.asarray(a, dtype=np.float64).astype(np.float32)
    u = f.view(np.uint32)
    assert np.all((u & np.uint32(0xFFFF)) == 0), "value not exact in bf16"
    return (u >> np.uint32(16)).astype(np.uint16)


def _bf16_pow2(e):
    """bf16 pattern of 2**e from the field layout: exponent field e + 127 at bit 7
    (normal), or fraction bit e + 133 (subnormal, e in [-133, -127))."""
    if e >= -126:
        return np.uint16((e + 127) << 7)
    return np.uint16(1 << (e + 133))


def pin_bf16_same_values_as_fp16(impl):
    """Values that both formats hold exactly (8 significant bits, inside fp16's
    normal range) give the same y and bound whether passed as fp16 or bf16."""
    for bits in BITS:
        kd = _kdiv(bits)
        K, N, M, G = 4 * kd, 7, 3, 2 * kd
        rng = _rng(500 + bits)
        x = rng.integers(-255, 256, size=(M, K)) * 2.0 ** rng.integers(-9, 3, size=(M, K))
        s = rng.integers(1, 256, size=(K // G, N)) * 2.0 ** -14
        z = rng.integers(0, 2 * min(1 << bits, 128), size=(K // G, N)) / 2.0 - 0.5  # 8 bits
        bias = rng.integers(-255, 256, size=N) * 2.0 ** -5
        codes = rng.integers(0, 1 << bits, size=(K, N)).astype(np.uint8)
        wq, wlo = impl.pack(codes, bits)
        y16, b16 = impl.wq_matmul(x.astype(np.float16), wq, wlo, s.astype(np.float16),
                                  z.astype(np.float16), bits, G, bias=bias.astype(np.float16))
        yb, bb = impl.wq_matmul(_bf16_exact(x), wq, wlo, _bf16_exact(s), _bf16_exact(z), bits, G,
                                bias=_bf16_exact(bias), dtype="bf16")
        assert np.array_equal(y16, yb), bits
        assert np.array_equal(b16, bb), bits
        assert np.any(y16 != 0), bits


def pin_bf16_beyond_fp16_range(impl):
    """x = 2**e1 e_k, s = 2**e2 with e1, e2 outside fp16's range (one of them a
    bf16 subnormal): row k is (q - z) * 2**(e1 + e2) exactly, plus the bias."""
    bits, K, N, G = 4, 16, 5, 8
    rng = _rng(600)
    codes = rng.integers(0, 16, size=(K, N)).astype(np.uint8)
    zq = rng.integers(0, 16, size=(K // G, N))
    wq, wlo = impl.pack(codes, bits)
    for e1, e2 in ((100, -110), (-120, 30), (60, -130), (-20, -20)):
        x = np.zeros((K, K), dtype=np.uint16)
        x[np.arange(K), np.arange(K)] = _bf16_pow2(e1)
        s = np.full((K // G, N), _bf16_pow2(e2), dtype=np.uint16)
        z = _bf16_exact(zq)
        bias = np.full(N, _bf16_pow2(-3) | np.uint16(0x8000), dtype=np.uint16)  # -1/8
        y, b = impl.wq_matmul(x, wq, wlo, s, z, bits, G, bias=bias, dtype="bf16")
        for k in range(K):
            row = (codes[k].astype(np.float64) - zq[k // G]) * 2.0 ** (e1 + e2)
            assert np.array_equal(y[k], row - 0.125), (e1, e2, k)
            assert np.array_equal(b[k], np.abs(row) + 0.125), (e1, e2, k)


PINS = [
    pin_golden_pack,
    pin_golden_products,
    pin_roundtrip,
    pin_single_code_bruteforce,
    pin_zero_when_q_equals_z,
    pin_one_hot_row,
    pin_linearity,
    pin_integer_matmul_special_case,
    pin_group_equivalences,
    pin_group_index,
    pin_bias,
    pin_bf16_same_values_as_fp16,
    pin_bf16_beyond_fp16_range,
]
