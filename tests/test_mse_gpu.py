"""wq_mse_search (the MSE-observer search kernel) against the oracle.

What is unique is compared bit for bit: for every group the kernel's scale and
zero point must be exactly the oracle's parameters of the candidate the kernel
chose.  Which candidate wins can differ only where two candidates' errors are
within rounding of each other: the kernel sums |w_hat - w|^norm in fp32 (and
takes the power with the library's powf), the oracle in fp64, from the same
fp32 differences.  So the chosen candidate's exact error must lie within that
rounding of the smallest exact error: per term at most 4 fp32 ulp for the
power, plus G additions of 2^-24, relative -- bounded here by
(G + 8) * 2^-23 of the error, with a floor of 1e-30 for zero errors.  Where no
near-tie exists the choice is the oracle's.  Patience is checked on the
hand-worked golden cases (exact values) and on random tensors where the stop
the kernel found is compared with the oracle's."""
import numpy as np
import pytest

import oracle.mse_observer as mo
from _golden import read_cases

pytestmark = pytest.mark.gpu


def rel_bound(G):
    return (G + 8) * 2.0 ** -23


def check_choice(r, ref, w, bits, G, symmetric, what, maxshrink, grid):
    step = r["step"].cpu().numpy()
    errs = ref["errors"]
    best = errs.min(axis=-1)
    chosen = np.take_along_axis(errs, step[..., None].astype(np.int64), axis=-1)[..., 0]
    assert np.all(step >= 0) and np.all(step < errs.shape[-1]), what
    assert np.all(chosen <= best * (1 + rel_bound(G)) + 1e-30), what
    # the parameters of the chosen candidate, bit for bit
    grp = np.asarray(w, np.float32).reshape(w.shape[0], -1, G)
    p = mo.candidates(maxshrink, grid)[step]
    lo = (grp.min(-1) * p).astype(np.float32)
    hi = (grp.max(-1) * p).astype(np.float32)
    s, z = (mo.qparams_symmetric if symmetric else mo.qparams)(lo, hi, bits)
    assert np.array_equal(r["scale"].cpu().numpy(), s), what
    assert np.array_equal(r["zero"].cpu().numpy(), z), what
    # the reported error is the chosen candidate's, summed in fp32
    e = r["err"].cpu().numpy().astype(np.float64)
    assert np.all(np.abs(e - chosen) <= chosen * rel_bound(G) + 1e-30), what
    # where every other candidate's exact error exceeds the best by more than the
    # rounding bound (relative to the larger), the choice is the oracle's
    others = np.where(np.arange(errs.shape[-1]) == ref["step"][..., None], np.inf, errs)
    clear = others.min(axis=-1) > best * (1 + 2 * rel_bound(G)) + 1e-30
    assert np.array_equal(step[clear], ref["step"][clear]), what
    assert clear.mean() > 0.5, (what, float(clear.mean()))  # the test data leaves most groups clear


CASES = [
    # rows, cols, G, bits, norm, symmetric
    (64, 1024, 16, 4, 2.4, False),   # the page's defaults: group 16, 4-bit, norm 2.4
    (32, 512, 32, 3, 2.0, False),
    (16, 768, 8, 2, 1.0, False),
    (24, 640, 128, 8, 2.4, False),   # generic path (group 128)
    (40, 960, 48, 4, 3.0, False),    # generic path, group not a power of two
    (64, 1024, 16, 4, 2.4, True),    # symmetric codes
    (16, 512, 64, 3, 2.0, True),
]


@pytest.mark.parametrize("rows,cols,G,bits,norm,symmetric", CASES)
def test_exhaustive_search(cuda, libwq, rows, cols, G, bits, norm, symmetric):
    import torch
    rng = np.random.default_rng(rows + cols + G + bits)
    w = (rng.standard_normal((rows, cols)) * rng.uniform(0.02, 2.0, size=(rows, 1))).astype(np.float32)
    r = libwq.mse_search(torch.from_numpy(w).to(cuda), bits, G, maxshrink=0.2, grid=100, norm=norm,
                         symmetric=symmetric)
    torch.cuda.synchronize()
    ref = mo.search(w, bits, G, maxshrink=0.2, grid=100, norm=norm, symmetric=symmetric)
    check_choice(r, ref, w, bits, G, symmetric, f"{(rows, cols, G, bits, norm, symmetric)}", 0.2, 100)


def test_golden_cases(cuda, libwq):
    """The hand-worked searches (exhaustive and with patience): every value exact."""
    import torch
    for name, c in read_cases("mse_search.txt").items():
        G = c["group"]
        w = np.array(c["values"], np.float32).reshape(1, -1)
        patience = int(c["patience"][0]) if "patience" in c else None
        symmetric = "symmetric" in c and bool(int(c["symmetric"][0]))
        r = libwq.mse_search(torch.from_numpy(w).to(cuda), c["bits"], G, maxshrink=c["maxshrink"][0],
                             grid=int(c["grid"][0]), norm=c["norm"][0], patience=patience, symmetric=symmetric)
        torch.cuda.synchronize()
        assert np.array_equal(r["step"].cpu().numpy()[0], np.array(c["steps"], np.int32)), name
        assert np.array_equal(r["scale"].cpu().numpy()[0], np.array(c["scale"], np.float32)), name
        assert np.array_equal(r["zero"].cpu().numpy()[0], np.array(c["zero"], np.float32)), name


@pytest.mark.parametrize("patience", [1, 2, 5])
def test_patience_on_structured_tensor(cuda, libwq, patience):
    """Groups on the grid of their own first candidate (exact, error 0 at step 0):
    no candidate after the first improves any group, so the search stops after
    1 + patience candidates and every group keeps candidate 0, in both the
    oracle and the kernel."""
    import torch
    rng = np.random.default_rng(patience)
    bits, G, rows, groups = 4, 16, 8, 32
    q = rng.integers(0, 16, size=(rows, groups, G))
    q[..., 0], q[..., 1] = 0, 15
    zp = rng.integers(0, 16, size=(rows, groups, 1))
    s = 2.0 ** -rng.integers(2, 8, size=(rows, groups, 1))
    w = ((q - zp) * s).astype(np.float32).reshape(rows, groups * G)
    ref = mo.search(w, bits, G, maxshrink=0.2, grid=100, norm=2.4, patience=patience)
    assert ref["steps_evaluated"] == 1 + patience
    r = libwq.mse_search(torch.from_numpy(w).to(cuda), bits, G, norm=2.4, patience=patience)
    torch.cuda.synchronize()
    assert np.all(r["step"].cpu().numpy() == 0)
    assert np.array_equal(r["scale"].cpu().numpy(), ref["scale"])
    assert np.array_equal(r["zero"].cpu().numpy(), ref["zero"])
    assert np.all(r["err"].cpu().numpy() == 0)


def test_patience_random_matches_exhaustive_prefix(cuda, libwq):
    """On random data some group improves at nearly every candidate, so patience 5
    stops late or never; the kernel's choice then equals its own exhaustive
    choice restricted to the evaluated prefix, and the parity rules above hold."""
    import torch
    rng = np.random.default_rng(3)
    w = rng.standard_normal((32, 512)).astype(np.float32)
    wt = torch.from_numpy(w).to(cuda)
    a = libwq.mse_search(wt, 4, 16, patience=5)
    b = libwq.mse_search(wt, 4, 16)
    ref = mo.search(w, 4, 16, maxshrink=0.2, grid=100, norm=2.4, patience=5)
    torch.cuda.synchronize()
    if ref["steps_evaluated"] == 20:   # no stop: patience changes nothing
        for k in ("step", "scale", "zero", "err"):
            assert torch.equal(a[k], b[k]), k
    check_choice(a, ref, w, 4, 16, False, "patience 5", 0.2, 100)


def test_rejected_arguments(cuda, libwq):
    import torch
    w = torch.zeros((4, 64), dtype=torch.float32, device=cuda)
    with pytest.raises(ValueError):
        libwq.mse_search(w, 4, 24)                      # cols % group_size
    with pytest.raises(libwq.WQError) as e:
        libwq.mse_search(w, 9, 16)
    assert e.value.status == 2
    with pytest.raises(libwq.WQError) as e:
        libwq.mse_search(w, 4, 16, maxshrink=0.5, grid=100)   # 50 candidates > 32
    assert e.value.status == 1
    with pytest.raises(libwq.WQError) as e:
        libwq.mse_search(w, 4, 16, norm=float("nan"))
    assert e.value.status == 1
