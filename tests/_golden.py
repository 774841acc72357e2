"""Reader for the hand-derived fixtures under ``tests/golden/``."""
from __future__ import annotations

from pathlib import Path

import numpy as np

GOLDEN = Path(__file__).resolve().parent / "golden"


def read_cases(name: str) -> dict:
    """Parse ``case ... end`` blocks into dicts of ints, floats and word lists."""
    cases, cur = {}, None
    for raw in (GOLDEN / name).read_text().splitlines():
        line = raw.split("#", 1)[0].strip()
        if not line:
            continue
        key, _, rest = line.partition(" ")
        if key == "case":
            cur = {"name": rest.strip()}
        elif key == "end":
            cases[cur["name"]] = cur
            cur = None
        else:
            toks = rest.split()
            if key in ("wq", "wlo", "qz"):
                cur[key] = [int(t, 16) for t in toks]
            elif key in ("bits", "K", "N", "M", "group"):
                cur[key] = int(toks[0])
            elif key == "codes":
                cur[key] = [int(t) for t in toks]
            else:
                cur[key] = [float(t) for t in toks]
    return cases


def words(case: dict, key: str, N: int):
    if key not in case:
        return None
    return np.array(case[key], dtype=np.uint32).reshape(-1, N)
