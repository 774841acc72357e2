"""Helpers for the -m gpu parity tests: move a drawn case to the device and run
the oracle on the same bytes."""
from __future__ import annotations

import numpy as np


def tensor(a, dev, dtype="fp16"):
    """A host array on the device: fp16 / uint8 as they are, bf16 bit patterns
    (uint16) as torch.bfloat16."""
    import torch
    if dtype == "bf16" and a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev)


def to_dev(case, dev):
    dt = getattr(case, "dtype", "fp16")
    return dict(
        x=tensor(case.x, dev, dt),
        codes=tensor(case.codes, dev),
        scales=tensor(case.scales, dev, dt),
        zeros=tensor(case.zeros, dev, dt),
    )


def host(y):
    """A device result as fp64 on the host (bf16 and fp16 widen exactly)."""
    return y.float().cpu().numpy().astype(np.float64)


def oracle_product(orc, case, bias=None):
    wq, wlo = orc.pack(case.codes, case.wl.bits)
    return orc.wq_matmul(case.x, wq, wlo, case.scales, case.zeros, case.wl.bits, case.wl.group_size,
                         bias=bias, dtype=getattr(case, "dtype", "fp16"))


def gpu_pack(wq_mod, d, bits):
    return wq_mod.pack_kmajor(d["codes"], bits)
