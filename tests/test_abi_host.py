"""Host-side checks of the C ABI: the library loads, exports every declared
symbol, counts state like the printed figures, and rejects bad arguments
before touching a GPU (these run on a machine without one)."""

import ctypes
import json
import os
import re

import pytest

from matrix_aware_optimizers_02_b200 import _lib as L
from oracle import mao_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    names = set()
    for h in ("mao.h", "mao_testing.h"):
        text = open(os.path.join(ROOT, "include", h)).read()
        names.update(re.findall(r"^MAO_API\s+[\w\s\*]+?\b(mao_\w+)\s*\(", text, flags=re.M))
    return names


@pytest.fixture(scope="module")
def lib():
    return L.load()


def test_library_exports_every_declared_symbol(lib):
    declared = _declared_symbols()
    assert len(declared) >= 15
    for name in declared:
        assert hasattr(lib, name), name
    assert set(L.SIGNATURES) == declared


def test_version_and_strings(lib):
    assert lib.mao_version() == 4
    for s in range(0, 11):
        assert len(lib.mao_status_string(s)) > 0
    assert lib.mao_status_string(999) == b"unknown status"


def test_state_counts_match_oracle_and_printed_memory(lib):
    with open(os.path.join(ROOT, "tests", "golden", "state_bytes_gpt2_large.json")) as f:
        g = json.load(f)
    d, layers = g["d_model"], g["layers"]
    shapes = [(d, d)] * 4 + [(d, 4 * d), (4 * d, d)]
    soap = sum(lib.mao_soap_state_elems(m, n) for m, n in shapes) * layers * 4 / 2 ** 30
    foam = sum(lib.mao_foam_state_elems(m, n) for m, n in shapes) * layers * 4 / 2 ** 30
    assert round(soap, 2) == g["soap_gib"] and round(foam, 2) == g["foam_gib"]
    for m, n in [(3, 5), (768, 2304), (14336, 4096)]:
        assert lib.mao_soap_state_elems(m, n) == O.soap_state_elems(m, n)
        assert lib.mao_foam_state_elems(m, n) == O.foam_state_elems(m, n)
        assert lib.mao_muon_state_elems(m, n) == m * n
    assert lib.mao_soap_state_elems(0, 5) == 0


# fake, never-dereferenced device addresses
A16 = 0x10000
MIS = 0x10004


def _muon(lib, mats, params=None, ws=A16, ws_bytes=1 << 40, stats=None):
    n = len(mats)
    arr = (L.MuonMat * max(n, 1))(*mats)
    p = params or L.MuonParams(0.95, 0.02, 0.0, 1e-7, 5, None, 0)
    return lib.mao_muon_step(arr, n, ctypes.byref(p), ws, ws_bytes, stats, None)


def test_muon_validation_errors(lib):
    ok = L.MuonMat(16, 32, A16, A16, L.MAO_F32, A16)
    assert _muon(lib, []) == L.MAO_OK  # count 0: nothing to do
    assert lib.mao_muon_step(None, 1, None, A16, 1, None, None) == L.MAO_ERR_INVALID_ARG
    assert _muon(lib, [L.MuonMat(0, 32, A16, A16, 0, A16)]) == L.MAO_ERR_SHAPE
    assert _muon(lib, [L.MuonMat(16, 30, A16, A16, 0, A16)]) == L.MAO_ERR_SHAPE  # 30 % 4 != 0
    assert _muon(lib, [L.MuonMat(16, 36, A16, A16, L.MAO_BF16, A16)]) == L.MAO_ERR_SHAPE  # bf16 rows
    assert _muon(lib, [L.MuonMat(16, 32, A16, A16, 7, A16)]) == L.MAO_ERR_DTYPE
    assert _muon(lib, [L.MuonMat(16, 32, None, A16, 0, A16)]) == L.MAO_ERR_INVALID_ARG
    assert _muon(lib, [L.MuonMat(16, 32, MIS, A16, 0, A16)]) == L.MAO_ERR_ALIGN
    assert _muon(lib, [ok], params=L.MuonParams(0.95, 0.02, 0.0, 1e-7, 17, None, 0)) == L.MAO_ERR_INVALID_ARG
    assert _muon(lib, [ok], params=L.MuonParams(0.95, 0.02, 0.0, 1e-7, 5, None, 9)) == L.MAO_ERR_INVALID_ARG
    assert _muon(lib, [ok], params=L.MuonParams(float("nan"), 0.02, 0.0, 1e-7, 5, None, 0)) == L.MAO_ERR_INVALID_ARG
    assert _muon(lib, [ok], ws=None) == L.MAO_ERR_WORKSPACE
    assert _muon(lib, [ok], ws_bytes=100) == L.MAO_ERR_WORKSPACE
    assert _muon(lib, [ok], ws=A16 + 16) == L.MAO_ERR_ALIGN  # workspace must be 256-byte aligned


def test_muon_workspace_size_grows_with_batch(lib):
    p = L.MuonParams(0.95, 0.02, 0.0, 1e-7, 5, None, 3)
    sizes = []
    for n in (1, 2, 8):
        arr = (L.MuonMat * n)(*[L.MuonMat(768, 2304, A16, A16, 1, A16)] * n)
        b = ctypes.c_size_t(0)
        assert lib.mao_muon_workspace_size(arr, n, ctypes.byref(p), ctypes.byref(b)) == L.MAO_OK
        sizes.append(b.value)
    assert sizes[0] < sizes[1] < sizes[2]
    # bf16 operands: at least X twice (ping-pong) plus A and B
    assert sizes[0] >= 2 * (2 * 768 * 2304 + 2 * 768 * 768)
    b = ctypes.c_size_t(0)
    assert lib.mao_muon_workspace_size(None, 1, ctypes.byref(p), ctypes.byref(b)) == L.MAO_ERR_INVALID_ARG


def test_soap_foam_validation(lib):
    rf = L.Refresh(L.REFRESH_EVERY_K, 1, 10, 0.1, 1)
    sp = L.SoapParams(0.95, 0.95, 1e-8, 3e-3, 0.0, 1, rf)
    mat = L.SoapMat(16, 32, A16, A16, 0, A16, A16, A16, A16, A16, A16, None, None)
    arr = (L.SoapMat * 1)(mat)
    b = ctypes.c_size_t(0)
    assert lib.mao_soap_workspace_size(arr, 1, ctypes.byref(sp), ctypes.byref(b)) == L.MAO_OK
    bad = L.SoapParams(0.95, 0.95, 1e-8, 3e-3, 0.0, 0, rf)  # t < 1
    assert lib.mao_soap_workspace_size(arr, 1, ctypes.byref(bad), ctypes.byref(b)) == L.MAO_ERR_INVALID_ARG
    bad_rf = L.SoapParams(0.95, 0.95, 1e-8, 3e-3, 0.0, 1, L.Refresh(L.REFRESH_EVERY_K, 0, 10, 0.1, 1))
    assert lib.mao_soap_workspace_size(arr, 1, ctypes.byref(bad_rf), ctypes.byref(b)) == L.MAO_ERR_INVALID_ARG
    fp = L.FoamParams(0.95, 0.95, 1e-8, 3e-3, 0.0, 1, L.Refresh(L.REFRESH_ADAPTIVE, 1, 10, 0.1, 1), 0)
    fmat = L.FoamMat(16, 30, A16, A16, 0, A16, A16, A16, A16, A16, None)
    farr = (L.FoamMat * 1)(fmat)
    assert lib.mao_foam_workspace_size(farr, 1, ctypes.byref(fp), ctypes.byref(b)) == L.MAO_ERR_SHAPE


def test_gemm_entry_validation(lib):
    b = ctypes.c_size_t(0)
    assert lib.mao_test_gemm_workspace_size(0, 1, 0, 8, 8, ctypes.byref(b)) == L.MAO_ERR_SHAPE
    assert lib.mao_test_gemm_workspace_size(6, 1, 8, 8, 8, ctypes.byref(b)) == L.MAO_ERR_INVALID_ARG
    for kind in range(6):
        assert lib.mao_test_gemm_workspace_size(kind, 1, 8, 8, 8, ctypes.byref(b)) == L.MAO_OK
    assert lib.mao_test_gemm_workspace_size(1, 2, 64, 64, 32, ctypes.byref(b)) == L.MAO_OK
    assert b.value >= 2 * 3 * 2 * (2 * 64 * 32)  # three bf16 planes of A and of B
    assert lib.mao_test_gemm(0, 0, 0, A16, A16, A16, 1, 8, 8, 12, A16, 1 << 20, None) == L.MAO_ERR_SHAPE
    assert lib.mao_test_gemm(0, 2, 0, A16, A16, A16, 1, 8, 8, 16, A16, 1 << 20, None) == L.MAO_ERR_INVALID_ARG


@pytest.mark.parametrize("kind,k,pf", [(L.REFRESH_EVERY_K, 3, 10), (L.REFRESH_ADAPTIVE, 1, 4), (L.REFRESH_NEVER, 1, 10)])
def test_precond_workspace_size_is_independent_of_t(lib, kind, k, pf):
    """One workspace serves every step: plain, refresh and check steps alike."""
    rf = L.Refresh(kind, k, pf, 0.1, 1)
    mats = [L.SoapMat(m, n, A16, A16, 1, A16, A16, A16, A16, A16, A16, None, None)
            for (m, n) in [(256, 512), (1024, 136), (8, 8)]]
    arr = (L.SoapMat * 3)(*mats)
    fm = [L.FoamMat(m, n, A16, A16, 1, A16, A16, A16, A16, A16, None) for (m, n) in [(256, 512), (1024, 136)]]
    farr = (L.FoamMat * 2)(*fm)
    sizes, fsizes = set(), set()
    for t in range(1, 9):
        b = ctypes.c_size_t(0)
        sp = L.SoapParams(0.95, 0.95, 1e-8, 3e-3, 0.0, t, rf)
        assert lib.mao_soap_workspace_size(arr, 3, ctypes.byref(sp), ctypes.byref(b)) == L.MAO_OK
        sizes.add(b.value)
        fp = L.FoamParams(0.95, 0.95, 1e-8, 3e-3, 0.0, t, rf, 0)
        assert lib.mao_foam_workspace_size(farr, 2, ctypes.byref(fp), ctypes.byref(b)) == L.MAO_OK
        fsizes.add(b.value)
    assert len(sizes) == 1 and len(fsizes) == 1


def test_pair_kernel_flag_validation(lib):
    b = ctypes.c_size_t(0)
    assert lib.mao_test_gemm_workspace_size(1 | 32, 1, 8, 8, 8, ctypes.byref(b)) == L.MAO_OK
    assert lib.mao_test_gemm_workspace_size(2 | 32, 1, 8, 8, 8, ctypes.byref(b)) == L.MAO_OK
    assert lib.mao_test_gemm_workspace_size(5 | 32, 1, 8, 8, 8, ctypes.byref(b)) == L.MAO_OK
    assert lib.mao_test_gemm_workspace_size(0 | 16, 1, 8, 8, 8, ctypes.byref(b)) == L.MAO_OK  # bf16 on one CTA
    assert lib.mao_test_gemm_workspace_size(0 | 32, 1, 8, 8, 8, ctypes.byref(b)) == L.MAO_OK  # bf16 on CTA pairs
    assert lib.mao_test_gemm_workspace_size(1 | 64, 1, 8, 8, 8, ctypes.byref(b)) == L.MAO_ERR_INVALID_ARG
    assert lib.mao_test_gemm_workspace_size(0 | 64, 1, 8, 8, 8, ctypes.byref(b)) == L.MAO_ERR_INVALID_ARG


def _muon_size(lib, mat, params=None):
    p = params or L.MuonParams(0.95, 0.02, 0.0, 1e-7, 5, None, 0)
    size = ctypes.c_size_t(0)
    st = lib.mao_muon_workspace_size((L.MuonMat * 1)(mat), 1, ctypes.byref(p), ctypes.byref(size))
    return st, size.value


def test_muon_split_and_polar_validation(lib):
    """A split matrix must divide into equal blocks whose widths keep 16-byte rows (a
    multiple of 4 fp32, of 8 for a bf16 G); the polar method must be a known one."""
    F32, BF16 = L.MAO_F32, L.MAO_BF16
    st, split = _muon_size(lib, L.MuonMat(16, 96, A16, A16, F32, A16, 1, 3))
    assert st == L.MAO_OK
    st, whole = _muon_size(lib, L.MuonMat(16, 96, A16, A16, F32, A16))
    assert st == L.MAO_OK and split != whole  # three 16 x 32 logical matrices, not one 16 x 96
    assert _muon_size(lib, L.MuonMat(16, 24, A16, A16, F32, A16, 1, 6))[0] == L.MAO_OK     # width 4
    assert _muon_size(lib, L.MuonMat(16, 48, A16, A16, BF16, A16, 1, 3))[0] == L.MAO_OK    # bf16 width 16
    assert _muon_size(lib, L.MuonMat(16, 96, A16, A16, F32, A16, 1, 5))[0] == L.MAO_ERR_SHAPE   # 96 % 5
    assert _muon_size(lib, L.MuonMat(16, 30, A16, A16, F32, A16, 1, 3))[0] == L.MAO_ERR_SHAPE   # width 10
    assert _muon_size(lib, L.MuonMat(16, 48, A16, A16, BF16, A16, 1, 4))[0] == L.MAO_ERR_SHAPE  # bf16 width 12
    assert _muon_size(lib, L.MuonMat(15, 32, A16, A16, F32, A16, 2, 1))[0] == L.MAO_ERR_SHAPE   # 15 % 2
    assert _muon_size(lib, L.MuonMat(16, 32, A16, A16, F32, A16, -1, 1))[0] == L.MAO_ERR_INVALID_ARG
    assert _muon_size(lib, L.MuonMat(16, 32, A16, A16, F32, A16),
                      L.MuonParams(0.95, 0.02, 0.0, 1e-7, 5, None, 0, 2))[0] == L.MAO_ERR_INVALID_ARG
    # the step validates the same way before anything is enqueued
    assert _muon(lib, [L.MuonMat(16, 96, A16, A16, F32, A16, 1, 5)]) == L.MAO_ERR_SHAPE


def test_refresh_lag_validation(lib):
    m = n = 16
    mats = (L.SoapMat * 1)(L.SoapMat(m, n, A16, A16, L.MAO_F32, A16, A16, A16, A16, A16, A16, None, None))
    size = ctypes.c_size_t(0)
    good = L.SoapParams(0.95, 0.95, 1e-8, 3e-3, 0.0, 1, L.Refresh(L.REFRESH_EVERY_K, 1, 10, 0.1, 1, 1))
    assert lib.mao_soap_workspace_size(mats, 1, ctypes.byref(good), ctypes.byref(size)) == L.MAO_OK
    bad = L.SoapParams(0.95, 0.95, 1e-8, 3e-3, 0.0, 1, L.Refresh(L.REFRESH_EVERY_K, 1, 10, 0.1, 1, 2))
    assert lib.mao_soap_workspace_size(mats, 1, ctypes.byref(bad), ctypes.byref(size)) == L.MAO_ERR_INVALID_ARG
