"""The binding's shape and device checks, which run before any C call.

The library sizes its copies and stores from the scalars K, N, M and bits, so
a tensor of another shape would be read or written out of its bounds; the
binding refuses every such mismatch with ValueError.  The checks look only at
shapes and devices, so they run here on CPU tensors."""
import pytest
import torch


def planes(K, N, bits):
    eps = 16 if bits == 3 else 32 // bits
    w_q = torch.zeros((K // eps, N), dtype=torch.int32)
    w_lo = torch.zeros((K // 32, N), dtype=torch.int32) if bits == 3 else None
    return w_q, w_lo


def args(M=2, K=256, N=64, bits=4, G=128):
    x = torch.zeros((M, K), dtype=torch.float16)
    w_q, w_lo = planes(K, N, bits)
    g = K if G == -1 else G
    s = torch.zeros((K // g, N), dtype=torch.float16)
    return dict(x=x, w_q=w_q, w_lo=w_lo, scales=s, zeros=s.clone(),
                bias=torch.zeros(N, dtype=torch.float16), out=torch.zeros((M, N), dtype=torch.float16),
                bits=bits, group_size=G)


@pytest.mark.parametrize("bits,G", [(1, 128), (2, 64), (3, 128), (4, 128), (8, -1), (4, -1)])
def test_consistent_shapes_pass(libwq, bits, G):
    libwq._check_product(**args(bits=bits, G=G))
    a = args(bits=bits, G=G)
    libwq._check_product(**dict(a, bias=None, out=None))


@pytest.mark.parametrize("field,bad", [
    ("w_q", torch.zeros((31, 64), dtype=torch.int32)),       # one word row short
    ("w_q", torch.zeros((64, 64), dtype=torch.int32)),       # 2-bit rows for 4-bit codes
    ("w_lo", torch.zeros((8, 64), dtype=torch.int32)),       # a lo plane for 4-bit words
    ("scales", torch.zeros((1, 64), dtype=torch.float16)),   # per-channel rows for group 128
    ("zeros", torch.zeros((2, 32), dtype=torch.float16)),    # half the columns
    ("bias", torch.zeros(32, dtype=torch.float16)),
    ("out", torch.zeros((2, 32), dtype=torch.float16)),
    ("out", torch.zeros((1, 64), dtype=torch.float16)),      # fewer tokens than x
])
def test_each_mismatch_is_refused(libwq, field, bad):
    a = args()
    a[field] = bad
    with pytest.raises(ValueError, match=field if field != "w_lo" else "w_lo"):
        libwq._check_product(**a)


def test_three_bit_planes(libwq):
    a = args(bits=3)
    libwq._check_product(**a)
    with pytest.raises(ValueError, match="lo plane"):
        libwq._check_product(**dict(a, w_lo=None))
    with pytest.raises(ValueError, match="w_lo"):
        libwq._check_product(**dict(a, w_lo=torch.zeros((4, 64), dtype=torch.int32)))
    with pytest.raises(ValueError, match="w_q"):
        libwq._check_product(**dict(a, w_q=torch.zeros((8, 64), dtype=torch.int32)))


def test_rules_the_library_names_are_left_to_it(libwq):
    """Bit widths and group sizes the C rules reject keep their WQ_ERR status:
    the shape check does not pre-empt them."""
    a = args()
    libwq._check_product(**dict(a, bits=5))
    libwq._check_product(**dict(a, group_size=96))


def test_devices_must_match(libwq):
    a = args()
    a["bias"] = torch.zeros(64, dtype=torch.float16, device="meta")
    with pytest.raises(ValueError, match="device"):
        libwq._check_product(**a)
    w_q, _ = planes(256, 64, 4)
    with pytest.raises(ValueError, match="device"):
        libwq._same_device(w_q, w_lo=torch.zeros((8, 64), dtype=torch.int32, device="meta"))


def test_unpack_plane_shapes(libwq):
    w_q, w_lo = planes(256, 64, 3)
    libwq._check_planes(w_q, w_lo, 256, 3)
    with pytest.raises(ValueError, match="w_q"):
        libwq._check_planes(w_q, w_lo, 512, 3)
    w4, _ = planes(256, 64, 4)
    with pytest.raises(ValueError, match="w_q"):
        libwq._check_planes(w4, None, 128, 4)
