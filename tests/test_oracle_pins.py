"""The oracle (C and its NumPy twin) against facts fixed by the pages and mathematics."""
import pytest

import oracle_pins

IMPLS = ["c_oracle", "numpy_twin"]


def _impl(name):
    import oracle
    if name == "c_oracle":
        oracle.build()
        return oracle
    return oracle.numpy_oracle


@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("pin", oracle_pins.PINS, ids=lambda f: f.__name__)
def test_pin(impl, pin):
    pin(_impl(impl))


def test_half_to_double_definition(orc):
    """binary16 widening: normal, subnormal, signed zero, inf, nan, max."""
    import math
    assert orc.half_to_double(0x3C00) == 1.0
    assert orc.half_to_double(0xC000) == -2.0
    assert orc.half_to_double(0x0001) == 2.0 ** -24
    assert orc.half_to_double(0x03FF) == 1023 * 2.0 ** -24
    assert orc.half_to_double(0x0400) == 2.0 ** -14
    assert orc.half_to_double(0x7BFF) == 65504.0
    assert orc.half_to_double(0x3555) == 0.25 + 0x155 / 4096
    assert orc.half_to_double(0x7C00) == math.inf
    assert math.isnan(orc.half_to_double(0x7E00))
    assert math.copysign(1.0, orc.half_to_double(0x8000)) == -1.0


def test_half_to_double_matches_numpy_everywhere(orc):
    """Every one of the 65536 binary16 patterns widens as NumPy's float16 does."""
    import numpy as np
    bits = np.arange(1 << 16, dtype=np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([orc.half_to_double(int(h)) for h in bits])
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all()
    assert np.array_equal(np.signbit(got[~np.isnan(got)]), np.signbit(ref[~np.isnan(ref)]))


def test_bf16_to_double_definition(orc):
    """bfloat16 widening: normal, subnormal, signed zero, inf, nan, extremes."""
    import math
    assert orc.bf16_to_double(0x3F80) == 1.0
    assert orc.bf16_to_double(0xC000) == -2.0
    assert orc.bf16_to_double(0x4049) == 3.140625
    assert orc.bf16_to_double(0x0001) == 2.0 ** -133
    assert orc.bf16_to_double(0x007F) == 127 * 2.0 ** -133
    assert orc.bf16_to_double(0x0080) == 2.0 ** -126
    assert orc.bf16_to_double(0x7F7F) == 255 * 2.0 ** 120
    assert orc.bf16_to_double(0x7F80) == math.inf
    assert math.isnan(orc.bf16_to_double(0x7FC0))
    assert math.copysign(1.0, orc.bf16_to_double(0x8000)) == -1.0


@pytest.mark.parametrize("impl", IMPLS)
def test_bf16_widening_matches_torch_everywhere(impl):
    """Every one of the 65536 bfloat16 patterns widens as torch's bfloat16 does."""
    import numpy as np
    import torch
    bits = np.arange(1 << 16, dtype=np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    got = _impl(impl).widen(bits, "bf16")
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all()
    assert np.array_equal(np.signbit(got[~np.isnan(got)]), np.signbit(ref[~np.isnan(ref)]))


def test_oracle_rejects_bad_input(orc):
    import numpy as np
    with pytest.raises(orc.OracleError):
        orc.pack(np.full((8, 1), 16, np.uint8), 4)      # code does not fit 4 bits
    with pytest.raises(orc.OracleError):
        orc.pack(np.zeros((12, 1), np.uint8), 4)        # K not a multiple of 8
    with pytest.raises(orc.OracleError):
        orc.pack(np.zeros((16, 1), np.uint8), 3)        # 3-bit needs K % 32 == 0
    with pytest.raises(orc.OracleError):
        orc.pack(np.zeros((8, 1), np.uint8), 5)         # unsupported width
    with pytest.raises(orc.OracleError):
        orc.widen(np.zeros(4, np.float16), "bf16")     # bf16 comes as uint16 patterns
    with pytest.raises(orc.OracleError):
        orc.widen(np.zeros(4, np.float16), "fp32")     # not a supported dtype
