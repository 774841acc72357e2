"""Host-side behaviour of the Python binding that needs no GPU: it refuses CPU
tensors (there is no CPU path) and fails loudly when libwq.so is missing."""
from pathlib import Path

import pytest
import torch


def test_cpu_tensors_are_refused(libwq):
    x = torch.zeros((1, 64), dtype=torch.float16)
    w = torch.zeros((8, 8), dtype=torch.int32)
    s = torch.zeros((1, 8), dtype=torch.float16)
    for fn in (libwq.gemv, libwq.gemm, libwq.matmul):
        with pytest.raises(ValueError, match="CUDA tensor"):
            fn(x, w, None, s, s, 4, 64)


def test_cpu_tensors_are_refused_in_bf16_too(libwq):
    x = torch.zeros((1, 64), dtype=torch.bfloat16)
    w = torch.zeros((8, 8), dtype=torch.int32)
    s = torch.zeros((1, 8), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        libwq.gemv(x, w, None, s, s, 4, 64)


def test_element_types(libwq):
    """x must be float16 or bfloat16; scales, zeros and bias must match it."""
    w = torch.zeros((8, 8), dtype=torch.int32)
    x32 = torch.zeros((1, 64), dtype=torch.float32)
    with pytest.raises(TypeError, match="float16 or torch.bfloat16"):
        libwq.gemv(x32, w, None, x32, x32, 4, 64)
    assert libwq._elem_type(torch.zeros(1, dtype=torch.bfloat16)) is torch.bfloat16
    assert libwq._elem_type(torch.zeros(1, dtype=torch.float16)) is torch.float16


def test_non_tensor_is_refused(libwq):
    with pytest.raises(TypeError, match="torch.Tensor"):
        libwq.gemv([[0.0]], None, None, None, None, 4, 64)


def test_missing_library_fails_loudly(libwq, monkeypatch):
    monkeypatch.setattr(libwq, "_lib", None)
    monkeypatch.setattr(libwq, "LIB_PATH", Path("/nonexistent/libwq.so"))
    with pytest.raises(RuntimeError, match="missing"):
        libwq.lib()


def test_status_names(libwq):
    assert libwq.STATUS[7] == "WQ_ERR_SCRATCH_LIMIT"
    assert "scratch" in libwq.describe(7)
    err = libwq.WQError("wq_gemv", 3)
    assert err.status == 3 and "WQ_ERR_ALIGNMENT" in str(err)


def test_gptq_refuses_cpu_tensors(libwq):
    W = torch.zeros((4, 64), dtype=torch.float32)
    H = torch.eye(64, dtype=torch.float32)
    s = torch.ones((4, 1), dtype=torch.float32)
    with pytest.raises(ValueError, match="CUDA tensor"):
        libwq.gptq_quantize(W, H, s, s * 0, 64, 8)


def test_gptq_status_name(libwq):
    assert libwq.STATUS[9] == "WQ_ERR_NOT_POSITIVE_DEFINITE"
    assert "positive definite" in libwq.describe(9)
