"""Shared pytest set-up: the ``gpu`` marker and the built oracle."""
import pytest


def pytest_configure(config):
    config.addinivalue_line(
        "markers", "gpu: needs an sm_100a GPU and the built CUDA library (libwq.so)")


@pytest.fixture(scope="session")
def orc():
    """The C oracle (built on first use)."""
    import oracle
    oracle.build()
    return oracle


@pytest.fixture(scope="session")
def libwq():
    """libwq.so, built in-tree if it is missing or older than its sources
    (with WQ_LIB=checked: the checked build, libwq_checked.so)."""
    import os
    from gemm_wq_gemv_b200 import build
    build.build(checks=os.environ.get("WQ_LIB") == "checked")
    import gemm_wq_gemv_b200 as wq
    return wq


@pytest.fixture(autouse=True)
def no_bounds_check_fired(request):
    """Under the checked build, every GPU test ends with no bounds check fired."""
    import os
    yield
    if os.environ.get("WQ_LIB") == "checked" and request.node.get_closest_marker("gpu"):
        import gemm_wq_gemv_b200 as wq
        st = wq.device_status(reset=True)
        assert st in (0, 5), f"a bounds check of the checked build fired (status {st})"


@pytest.fixture(scope="session")
def cuda(libwq):
    """The CUDA device for the -m gpu tests (fails loudly if there is none)."""
    import torch
    if not torch.cuda.is_available():
        pytest.fail("the -m gpu tests need a CUDA device")
    major, minor = torch.cuda.get_device_capability()
    assert (major, minor) == (10, 0), f"libwq.so holds sm_100a code only, device is sm_{major}{minor}"
    return torch.device("cuda:0")
