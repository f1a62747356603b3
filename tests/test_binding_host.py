"""The Python binding on the CPU: argument checks happen before any call into
the library, and a missing library fails loudly (there is no fallback)."""
import pytest
import torch

import w8a8_quantized_matmul_b200 as m
from w8a8_quantized_matmul_b200 import _lib


def test_host_tensors_are_refused_before_any_call():
    X = torch.zeros((4, 64), dtype=torch.float16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        m.int8_quantize_weight_rows(X)
    with pytest.raises(ValueError, match="CUDA tensor"):
        m.int8_rotate_quantize_rows(X, 16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        m.int4_rotate_quantize_groups(X, 16)


def test_non_tensor_argument_is_refused():
    import numpy as np
    with pytest.raises(TypeError, match="torch.Tensor"):
        m.int8_quantize_weight_rows(np.zeros((4, 64), np.float16))


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "libint8mm.so"))
    monkeypatch.setattr(_lib, "_lib", None)
    with pytest.raises(ImportError, match="missing"):
        _lib.load()


def test_status_strings_through_the_binding():
    assert "invalid" in _lib.status_string(_lib.I8MM_ERR_INVALID_ARG).lower()
    assert "time" in _lib.status_string(_lib.I8MM_ERR_TIMEOUT).lower()
    err = _lib.Int8mmError("int8_mixed_matmul", _lib.I8MM_ERR_WORKSPACE)
    assert "int8_mixed_matmul" in str(err) and err.status == _lib.I8MM_ERR_WORKSPACE
