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
    """libwq.so, built in-tree if it is missing or older than its sources."""
    from gemm_wq_gemv_b200 import build
    build.build()
    import gemm_wq_gemv_b200 as wq
    return wq


@pytest.fixture(scope="session")
def cuda(libwq):
    """The CUDA device for the -m gpu tests (fails loudly if there is none)."""
    import torch
    if not torch.cuda.is_available():
        pytest.fail("the -m gpu tests need a CUDA device")
    major, minor = torch.cuda.get_device_capability()
    assert (major, minor) == (10, 0), f"libwq.so holds sm_100a code only, device is sm_{major}{minor}"
    return torch.device("cuda:0")
