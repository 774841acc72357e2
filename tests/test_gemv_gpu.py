"""wq_gemv (M <= 16) against the fp64 oracle, element by element."""
import numpy as np
import pytest

import wq_inputs
from gpu_cases import oracle_product, to_dev
from guard import Guarded
from parity import check_product

pytestmark = pytest.mark.gpu


def run_gemv(libwq, d, bits, G, **kw):
    """The product into an output with sentinel rows around it, which must survive."""
    w_q, w_lo = libwq.pack_kmajor(d["codes"], bits)
    M, N = d["x"].shape[0], w_q.shape[1]
    out = Guarded((M, N), d["x"].dtype, d["x"].device)
    y = libwq.gemv(d["x"], w_q, w_lo, d["scales"], d["zeros"], bits, G, out=out.view, **kw)
    assert out.intact(), "a store landed outside y"
    return y.cpu().numpy()


FULL = ["tiny_gemv", "decode_gemv_m1", "decode_gemv_m4", "decode_gemv_m16", "gemv_3bit",
        "sweep_1bit", "sweep_2bit", "sweep_8bit", "sweep_8bit_perchannel"]


@pytest.mark.parametrize("name", FULL)
def test_workloads_full(cuda, libwq, orc, name):
    """Every output of each GEMV workload, at full size, in the bench's launch configuration."""
    case = wq_inputs.draw(wq_inputs.WORKLOADS[name], seed=0)
    d = to_dev(case, cuda)
    y = run_gemv(libwq, d, case.wl.bits, case.wl.group_size)
    y_ref, b = oracle_product(orc, case)
    check_product(y, y_ref, b, name)


SHAPES = [
    # M, K, N, bits, G
    (1, 32, 8, 4, 32),        # one quad, one ragged column block
    (3, 40, 16, 4, -1),       # ragged last quad (5 word rows)
    (1, 512, 264, 4, 64),
    (2, 1024, 40, 8, 16),
    (5, 2048, 72, 8, -1),
    (8, 512, 128, 2, 64),
    (9, 768, 96, 2, 256),
    (16, 1024, 136, 1, 128),
    (7, 4096, 64, 1, -1),
    (1, 1024, 200, 3, 64),
    (12, 2048, 56, 3, 128),
    (16, 3072, 48, 3, -1),
    (4, 8192, 16, 4, 128),    # long K per column block: many quads per warp
    (16, 256, 4096, 4, 128),  # wide N, short K
    (16, 8192, 64, 4, 128),   # two token tiles, K split over a cluster
    (13, 4096, 128, 8, 256),  # 8-bit, two token tiles, ragged token count
    (16, 2048, 96, 8, -1),    # 8-bit per channel, two token tiles
    (9, 1056, 40, 4, 32),     # 33 quads over 8 warps, G = 32: one group per quad
    (1, 4096, 4104, 4, 128),  # the one-token decode kernel, ragged last column block
    (1, 2048, 4096, 4, 128),  # the one-token decode kernel, 8 quads per warp
    (1, 8192, 256, 2, 128),   # 2-bit words on the lean kernel: one token, aligned plan
    (16, 2048, 96, 2, 128),   # 2-bit, two token tiles
    (4, 4096, 136, 2, -1),    # 2-bit per channel, ragged column block
    (5, 1088, 40, 2, 64),     # 2-bit, 17 quads over 8 warps (ragged range)
    (1, 8192, 512, 1, 128),   # 1-bit words on the lean kernel
    (8, 4096, 72, 1, -1),     # 1-bit per channel, 8 tokens, ragged column block
    (3, 2176, 40, 1, 128),    # 1-bit, 17 quads (ragged range)
    (12, 2048, 64, 1, 128),   # 1-bit with 12 tokens: the table kernel
]


@pytest.mark.parametrize("M,K,N,bits,G", SHAPES)
def test_small_shapes(cuda, libwq, orc, M, K, N, bits, G):
    case = wq_inputs.custom(M, K, N, bits, G, seed=M * 7 + K + N + bits)
    d = to_dev(case, cuda)
    y = run_gemv(libwq, d, bits, G)
    y_ref, b = oracle_product(orc, case)
    check_product(y, y_ref, b, f"{(M, K, N, bits, G)}")


@pytest.mark.parametrize("bits", [1, 2, 3, 4, 8])
def test_fractional_zero_points(cuda, libwq, orc, bits):
    """Zero points that are not integers (any fp16 value is allowed)."""
    import torch
    K, N, M, G = 1024, 96, 3, (128 if bits in (1, 2, 3) else 64)
    case = wq_inputs.custom(M, K, N, bits, G, seed=77 + bits)
    rng = np.random.default_rng(bits)
    case.zeros = rng.uniform(-0.5, (1 << bits) - 0.5, size=case.zeros.shape).astype(np.float16)
    d = to_dev(case, cuda)
    d["zeros"] = torch.from_numpy(case.zeros).to(cuda)
    y = run_gemv(libwq, d, bits, G)
    y_ref, b = oracle_product(orc, case)
    check_product(y, y_ref, b, f"fractional z, {bits}-bit")


@pytest.mark.parametrize("bits", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("M", [1, 16])
def test_q_equals_z_gives_zero(cuda, libwq, bits, M):
    import torch
    K, N = 512, 64
    G = 128
    case = wq_inputs.custom(M, K, N, bits, G, seed=5)
    zq = np.random.default_rng(9).integers(0, 1 << bits, size=(K // G, N))
    codes = np.repeat(zq, G, axis=0).astype(np.uint8)
    d = to_dev(case, cuda)
    d["codes"] = torch.from_numpy(codes).to(cuda)
    d["zeros"] = torch.from_numpy(zq.astype(np.float16)).to(cuda)
    y = run_gemv(libwq, d, bits, G)
    assert np.all(y.astype(np.float64) == 0.0)


@pytest.mark.parametrize("bits", [1, 2, 3, 4, 8])
def test_one_hot_rows_are_exact(cuda, libwq, orc, bits):
    """x = e_k gives fp16(w[k]) exactly, for 16 rows k at once."""
    import torch
    K, N, G = 512, 64, 128
    case = wq_inputs.custom(16, K, N, bits, G, seed=31)
    ks = np.random.default_rng(3).choice(K, 16, replace=False)
    x = np.zeros((16, K), np.float16)
    x[np.arange(16), ks] = 1.0
    d = to_dev(case, cuda)
    d["x"] = torch.from_numpy(x).to(cuda)
    y = run_gemv(libwq, d, bits, G)
    q = case.codes.astype(np.float64)
    g = ks // G
    w = (q[ks] - case.zeros[g].astype(np.float64)) * case.scales[g].astype(np.float64)
    assert np.array_equal(y, w.astype(np.float16))


def test_pdl_flag_same_result(cuda, libwq, orc):
    """The launch flags may pick another kernel (x written by the previous kernel
    takes the one that stages x), so the flag changes at most the rounding
    order: both results match the oracle."""
    case = wq_inputs.draw(wq_inputs.WORKLOADS["tiny_gemv"], seed=0)
    d = to_dev(case, cuda)
    y_ref, b = oracle_product(orc, case)
    for kw in ({}, {"pdl": True}, {"inputs_ready": True}):
        check_product(run_gemv(libwq, d, 4, 128, **kw), y_ref, b, f"tiny_gemv {kw}")


@pytest.mark.parametrize("M", [1, 4, 16])
def test_pdl_chain_where_each_input_is_the_previous_output(cuda, libwq, M):
    """WQ_FLAG_PDL: x of each call is y of the one before; the overlapped chain
    must give the same bits as the same calls run one at a time."""
    import torch
    K = N = 1024
    case = wq_inputs.custom(M, K, N, 4, 128, seed=11)
    d = to_dev(case, cuda)
    w_q, w_lo = libwq.pack_kmajor(d["codes"], 4)
    s = d["scales"] * 0.1  # keeps the chained values in range

    def chain(one_at_a_time):
        ys, x = [], d["x"]
        for _ in range(4):
            x = libwq.gemv(x, w_q, w_lo, s, d["zeros"], 4, 128, pdl=True)
            ys.append(x)
            if one_at_a_time:
                torch.cuda.synchronize()
        torch.cuda.synchronize()
        return [y.cpu().numpy() for y in ys]

    for a, b in zip(chain(True), chain(False)):
        assert np.isfinite(a).all()
        assert np.array_equal(a, b)


def test_inputs_ready_orders_the_writes_of_y(cuda, libwq):
    """WQ_FLAG_PDL_INPUTS_READY: inputs are read at once, y is written only after
    the previous kernel completes -- so a call may overwrite the previous call's
    input (write after read) and its output (write after write)."""
    import torch
    cases = [wq_inputs.custom(4, 4096, 4096, 4, 128, seed=20 + i) for i in range(3)]
    ds = [to_dev(c, cuda) for c in cases]
    packed = [libwq.pack_kmajor(d["codes"], 4) for d in ds]
    ref = []
    for d, (w_q, _) in zip(ds, packed):  # same launch flag as below, so the same plan
        torch.cuda.synchronize()
        ref.append(libwq.gemv(d["x"], w_q, None, d["scales"], d["zeros"], 4, 128,
                              inputs_ready=True).cpu().numpy())
    buf = ds[0]["x"].clone()                       # call 0 reads buf ...
    y0 = torch.empty((4, 4096), dtype=torch.float16, device=cuda)
    out = torch.empty((4, 4096), dtype=torch.float16, device=cuda)
    for _ in range(3):
        buf.copy_(ds[0]["x"])
        libwq.gemv(buf, packed[0][0], None, ds[0]["scales"], ds[0]["zeros"], 4, 128, out=y0)
        # ... call 1 writes buf (its output, 4 x 4096 like x of call 0)
        libwq.gemv(ds[1]["x"], packed[1][0], None, ds[1]["scales"], ds[1]["zeros"], 4, 128,
                   out=buf, inputs_ready=True)
        # calls 2 and 3 write the same output; the last one must win
        libwq.gemv(ds[2]["x"], packed[2][0], None, ds[2]["scales"], ds[2]["zeros"], 4, 128,
                   out=out, inputs_ready=True)
        libwq.gemv(ds[1]["x"], packed[1][0], None, ds[1]["scales"], ds[1]["zeros"], 4, 128,
                   out=out, inputs_ready=True)
        torch.cuda.synchronize()
        assert np.array_equal(y0.cpu().numpy(), ref[0])
        assert np.array_equal(buf.cpu().numpy(), ref[1])
        assert np.array_equal(out.cpu().numpy(), ref[1])


@pytest.mark.parametrize("name", ["decode_gemv_m1", "decode_gemv_m4", "decode_gemv_m16", "gemv_3bit",
                                  "sweep_1bit", "sweep_8bit_perchannel"])
def test_inputs_ready_plan_matches_oracle(cuda, libwq, orc, name):
    """WQ_FLAG_PDL_INPUTS_READY selects its own CTA shape; every output against the oracle."""
    import torch
    case = wq_inputs.draw(wq_inputs.WORKLOADS[name], seed=0)
    d = to_dev(case, cuda)
    w_q, w_lo = libwq.pack_kmajor(d["codes"], case.wl.bits)
    torch.cuda.synchronize()
    y = libwq.gemv(d["x"], w_q, w_lo, d["scales"], d["zeros"], case.wl.bits, case.wl.group_size,
                   inputs_ready=True).cpu().numpy()
    y_ref, b = oracle_product(orc, case)
    check_product(y, y_ref, b, name)
    assert libwq.device_status() == 0


@pytest.mark.parametrize("name,ready", [("tiny_gemv", False), ("decode_gemv_m1", True),
                                        ("decode_gemv_m16", False), ("gemv_3bit", True)])
def test_bias_matches_oracle(cuda, libwq, orc, name, ready):
    """y = x @ w + bias, every output against the oracle (bound includes |bias|)."""
    import torch
    case = wq_inputs.draw(wq_inputs.WORKLOADS[name], seed=0)
    d = to_dev(case, cuda)
    bias = wq_inputs.bias_vector(case.wl.N, seed=5)
    w_q, w_lo = libwq.pack_kmajor(d["codes"], case.wl.bits)
    torch.cuda.synchronize()
    y = libwq.gemv(d["x"], w_q, w_lo, d["scales"], d["zeros"], case.wl.bits, case.wl.group_size,
                   bias=torch.from_numpy(bias).to(cuda), inputs_ready=ready).cpu().numpy()
    wq_, wlo_ = orc.pack(case.codes, case.wl.bits)
    y_ref, b = orc.wq_matmul(case.x, wq_, wlo_, case.scales, case.zeros, case.wl.bits,
                             case.wl.group_size, bias=bias)
    check_product(y, y_ref, b, name + " + bias")


def test_deterministic(cuda, libwq):
    case = wq_inputs.draw(wq_inputs.WORKLOADS["decode_gemv_m4"], seed=1)
    d = to_dev(case, cuda)
    a = run_gemv(libwq, d, 4, 128)
    b = run_gemv(libwq, d, 4, 128)
    assert np.array_equal(a, b)


def test_rejected_calls(cuda, libwq):
    import torch
    case = wq_inputs.draw(wq_inputs.WORKLOADS["tiny_gemv"], seed=0)
    d = to_dev(case, cuda)
    w_q, _ = libwq.pack_kmajor(d["codes"], 4)
    x17 = torch.zeros((17, 512), dtype=torch.float16, device=cuda)
    with pytest.raises(libwq.WQError) as e:
        libwq.gemv(x17, w_q, None, d["scales"], d["zeros"], 4, 128)
    assert e.value.status == 1
    # group 16 is a legal 4-bit group size but not one wq_gemv takes (it needs a
    # multiple of 4 * eps = 32): the library, not the binding, refuses it
    s16 = torch.zeros((512 // 16, 256), dtype=torch.float16, device=cuda)
    with pytest.raises(libwq.WQError) as e:
        libwq.gemv(d["x"], w_q, None, s16, s16, 4, 16)
    assert e.value.status == 2
    # tensors whose shapes disagree with K, N and the group size never reach the library
    with pytest.raises(ValueError, match="scales"):
        libwq.gemv(d["x"], w_q, None, d["scales"][:2], d["zeros"], 4, 128)
    with pytest.raises(ValueError, match="out"):
        libwq.gemv(d["x"], w_q, None, d["scales"], d["zeros"], 4, 128,
                   out=torch.empty((1, 128), dtype=torch.float16, device=cuda))


# Shapes whose plan gives every warp one box covering its whole range, with all
# groups starting on 4-quad blocks (the group-by-group main loop of the 4/8-bit
# kernel): 4-bit K = 16384 and 8-bit K = 8192 over N = 64 split K over a cluster
# of 8 CTAs, 8 quads per warp; 4096 x 4096 takes one CTA per column block, 16
# quads per warp (G = 256: two 4-quad blocks per group).  G = -1 is one group
# across the range.
ALIGNED = [(3, 16384, 64, 4, 128), (1, 16384, 64, 4, -1), (2, 8192, 64, 8, 128), (1, 4096, 4096, 4, 256),
           (1, 8192, 512, 2, 128), (6, 8192, 64, 2, 128), (1, 8192, 512, 1, 128), (4, 16384, 64, 1, 128),
           (1, 4096, 4096, 4, 64), (1, 8192, 8192, 2, 128),
           (1, 4096, 4096, 4, 128), (1, 2048, 2560, 4, 128)]  # the last two: the one-token decode kernel


@pytest.mark.parametrize("M,K,N,bits,G", ALIGNED)
def test_aligned_plan_fractional_zero_points(cuda, libwq, orc, M, K, N, bits, G):
    import torch
    case = wq_inputs.custom(M, K, N, bits, G, seed=K + N + bits)
    rng = np.random.default_rng(K + bits)
    case.zeros = rng.uniform(-0.5, (1 << bits) - 0.5, size=case.zeros.shape).astype(np.float16)
    d = to_dev(case, cuda)
    d["zeros"] = torch.from_numpy(case.zeros).to(cuda)
    y = run_gemv(libwq, d, bits, G)
    y_ref, b = oracle_product(orc, case)
    check_product(y, y_ref, b, f"aligned plan, fractional z, {(M, K, N, bits, G)}")


@pytest.mark.parametrize("M,K,N,bits,G", ALIGNED)
def test_aligned_plan_q_equals_z_gives_zero(cuda, libwq, M, K, N, bits, G):
    import torch
    case = wq_inputs.custom(M, K, N, bits, G, seed=11)
    Gr = K if G == -1 else G
    zq = np.random.default_rng(13).integers(0, 1 << bits, size=(K // Gr, N))
    d = to_dev(case, cuda)
    d["codes"] = torch.from_numpy(np.repeat(zq, Gr, axis=0).astype(np.uint8)).to(cuda)
    d["zeros"] = torch.from_numpy(zq.astype(np.float16)).to(cuda)
    y = run_gemv(libwq, d, bits, G)
    assert np.all(y.astype(np.float64) == 0.0)


@pytest.mark.parametrize("M,K,N,bits,G", ALIGNED)
def test_aligned_plan_one_hot_rows_are_exact(cuda, libwq, M, K, N, bits, G):
    import torch
    Mh = 8
    case = wq_inputs.custom(Mh, K, N, bits, G, seed=17)
    ks = np.random.default_rng(K).choice(K, Mh, replace=False)
    x = np.zeros((Mh, K), np.float16)
    x[np.arange(Mh), ks] = 1.0
    d = to_dev(case, cuda)
    d["x"] = torch.from_numpy(x).to(cuda)
    y = run_gemv(libwq, d, bits, G)
    Gr = K if G == -1 else G
    q = case.codes.astype(np.float64)
    g = ks // Gr
    w = (q[ks] - case.zeros[g].astype(np.float64)) * case.scales[g].astype(np.float64)
    assert np.array_equal(y, w.astype(np.float16))


@pytest.mark.parametrize("bits", [1, 2, 4, 8])
def test_pdl_chain_at_decode_size(cuda, libwq, orc, bits):
    """WQ_FLAG_PDL on the 4096 x 4096 decode shape (the staged-x plan of the lean
    kernel): the first product matches the oracle, and the overlapped chain gives
    the same bits as the same calls run one at a time."""
    import torch
    K = N = 4096
    case = wq_inputs.custom(1, K, N, bits, 128, seed=40 + bits)
    d = to_dev(case, cuda)
    w_q, w_lo = libwq.pack_kmajor(d["codes"], bits)
    y0 = libwq.gemv(d["x"], w_q, w_lo, d["scales"], d["zeros"], bits, 128, pdl=True)
    y_ref, b = oracle_product(orc, case)
    check_product(y0.cpu().numpy(), y_ref, b, f"decode size, {bits}-bit, pdl")
    s = d["scales"] * 0.05  # keeps the chained values in range

    def chain(one_at_a_time):
        ys, x = [], d["x"]
        for _ in range(3):
            x = libwq.gemv(x, w_q, w_lo, s, d["zeros"], bits, 128, pdl=True)
            ys.append(x)
            if one_at_a_time:
                torch.cuda.synchronize()
        torch.cuda.synchronize()
        return [y.cpu().numpy() for y in ys]

    for a, c in zip(chain(True), chain(False)):
        assert np.isfinite(a).all() and np.any(a != 0)
        assert np.array_equal(a, c)
