"""The Python binding on a machine without a GPU: it fails loudly instead of
falling back to any CPU computation."""

import pytest
import torch

from matrix_aware_optimizers_02_b200 import _lib as L
from matrix_aware_optimizers_02_b200 import api


def test_missing_library_raises(monkeypatch):
    monkeypatch.setattr(L, "_lib", None)
    with pytest.raises(ImportError, match="not built"):
        L.load("/nonexistent/libmao.so")


def _cpu(m, n, dtype=torch.float32):
    return torch.zeros((m, n), dtype=dtype)


def test_muon_rejects_host_tensors():
    with pytest.raises(ValueError, match="CUDA tensor"):
        api.MuonBatch([(_cpu(8, 16), _cpu(8, 16), _cpu(8, 16))], mu=0.95, lr=0.02)


def test_soap_rejects_host_tensors():
    d = {"W": _cpu(8, 16), "G": _cpu(8, 16), "M": _cpu(8, 16), "V": _cpu(8, 16), "L": _cpu(8, 8),
         "R": _cpu(16, 16), "QL": _cpu(8, 8), "QR": _cpu(16, 16)}
    with pytest.raises(ValueError, match="CUDA tensor"):
        api.SoapBatch([d], beta1=0.95, beta2=0.95, eps=1e-8, lr=3e-3)


def test_foam_rejects_host_tensors():
    d = {"W": _cpu(8, 16), "G": _cpu(8, 16), "M": _cpu(8, 16), "r": torch.zeros(8), "c": torch.zeros(16),
         "R": _cpu(16, 16), "QR": _cpu(16, 16)}
    with pytest.raises(ValueError, match="CUDA tensor"):
        api.FoamBatch([d], beta1=0.95, beta2=0.95, eps=1e-8, lr=3e-3)


def test_gemm_rejects_host_tensors():
    A = torch.zeros((1, 128, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        api.gemm(A, A)
