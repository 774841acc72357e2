"""The checked build (libwq_checked.so, WQ_CHECKS): the GPU parity suites of
the products run again with every kernel checking the index of each access it
computes itself; the results must match the oracle as before and no check may
fire (the stand-in for a memory checker on this hardware)."""
import os
import subprocess
import sys
from pathlib import Path

import pytest

pytestmark = pytest.mark.gpu
ROOT = Path(__file__).resolve().parents[1]


def test_checked_build_runs_the_parity_suites(cuda):
    if os.environ.get("WQ_LIB") == "checked":
        pytest.skip("already running under the checked build")
    from gemm_wq_gemv_b200 import build
    build.build(checks=True)
    env = dict(os.environ, WQ_LIB="checked")
    suites = ["tests/test_gemv_gpu.py", "tests/test_gemm_gpu.py", "tests/test_bf16_gpu.py",
              "tests/test_plan_gpu.py", "tests/test_pack_gpu.py"]
    r = subprocess.run([sys.executable, "-m", "pytest", *suites, "-m", "gpu", "-x", "-q", "-p", "no:cacheprovider"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=1800)
    tail = "\n".join((r.stdout + r.stderr).splitlines()[-30:])
    assert r.returncode == 0, tail
    assert " passed" in r.stdout, tail


def test_checked_build_reports_itself(cuda):
    code = "import gemm_wq_gemv_b200 as wq; print(int(wq.checked_build()))"
    out = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=dict(os.environ, WQ_LIB="checked"),
                         capture_output=True, text=True, timeout=300).stdout.strip()
    assert out == "1"
    import gemm_wq_gemv_b200 as wq
    assert wq.checked_build() == (os.environ.get("WQ_LIB") == "checked")
