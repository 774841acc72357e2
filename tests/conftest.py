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
