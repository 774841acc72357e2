"""Helpers for the -m gpu parity tests: move a drawn case to the device and run
the oracle on the same bytes."""
from __future__ import annotations

import numpy as np


def to_dev(case, dev):
    import torch
    return dict(
        x=torch.from_numpy(case.x).to(dev),
        codes=torch.from_numpy(case.codes).to(dev),
        scales=torch.from_numpy(case.scales).to(dev),
        zeros=torch.from_numpy(case.zeros).to(dev),
    )


def oracle_product(orc, case):
    wq, wlo = orc.pack(case.codes, case.wl.bits)
    return orc.wq_matmul(case.x, wq, wlo, case.scales, case.zeros, case.wl.bits, case.wl.group_size)


def gpu_pack(wq_mod, d, bits):
    return wq_mod.pack_kmajor(d["codes"], bits)
