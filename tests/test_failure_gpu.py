"""Failure detection on the GPU without a fault: a bounded wait that runs out.

``wq_selftest_wait_timeout`` makes one CTA wait, with the products' bounded
mbarrier wait, on a barrier that nothing completes.  The wait must give up
after its limit, the kernel must record WQ_ERR_TIMEOUT and exit, and the
context must stay usable: the products' own status words stay clear and a
product launched afterwards is still correct.
"""
import time

import pytest

import wq_inputs
from gpu_cases import oracle_product, to_dev
from parity import check_product

pytestmark = pytest.mark.gpu

TIMEOUT = 5


def test_wait_runs_out_and_reports_timeout(cuda, libwq):
    for limit_ns in (1_000_000, 20_000_000):
        t0 = time.perf_counter()
        st = libwq.selftest_wait_timeout(limit_ns)
        elapsed = time.perf_counter() - t0
        assert st == TIMEOUT, libwq.describe(st)
        assert elapsed >= limit_ns * 1e-9          # it waited at least its limit
        assert elapsed < 1.0                       # and then gave up
    assert libwq.device_status() == 0              # the products' status words are untouched


def test_context_usable_after_the_timeout(cuda, libwq, orc):
    for _ in range(3):
        assert libwq.selftest_wait_timeout(2_000_000) == TIMEOUT
    case = wq_inputs.draw(wq_inputs.WORKLOADS["tiny_gemv"], seed=3)
    d = to_dev(case, cuda)
    w_q, w_lo = libwq.pack_kmajor(d["codes"], 4)
    y = libwq.gemv(d["x"], w_q, w_lo, d["scales"], d["zeros"], 4, 128)
    g = libwq.gemm(d["x"], w_q, w_lo, d["scales"], d["zeros"], 4, 128)
    y_ref, b = oracle_product(orc, case)
    check_product(y, y_ref, b, "gemv after the self-test")
    check_product(g, y_ref, b, "gemm after the self-test")
    assert libwq.device_status() == 0
