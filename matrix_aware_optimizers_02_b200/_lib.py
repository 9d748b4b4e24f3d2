"""ctypes declarations of the libmao C ABI (include/mao.h, include/mao_testing.h).

Loading fails loudly when the shared library is missing: there is no fallback
implementation of any step.
"""

from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_float, c_int32, c_int64, c_size_t, c_uint64, c_void_p

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmao.so")

# status codes
MAO_OK = 0
MAO_ERR_INVALID_ARG = 1
MAO_ERR_SHAPE = 2
MAO_ERR_DTYPE = 3
MAO_ERR_ALIGN = 4
MAO_ERR_WORKSPACE = 5
MAO_ERR_CUDA = 6
MAO_ERR_NONFINITE = 7
MAO_ERR_TIMEOUT = 8
MAO_ERR_UNSUPPORTED = 9
MAO_ERR_NOT_INITIALIZED = 10

MAO_F32, MAO_BF16 = 0, 1
NORM_MODES = {"none": 0, "row": 1, "col": 2, "col_row": 3, "row_col": 4}
REFRESH_EVERY_K, REFRESH_ADAPTIVE, REFRESH_NEVER = 0, 1, 2
POLAR_NS, POLAR_EXACT = 0, 1


class Refresh(ctypes.Structure):
    _fields_ = [("kind", c_int32), ("k", c_int32), ("pf", c_int32), ("tol", c_float), ("sort", c_int32),
                ("lag", c_int32)]


class Stats(ctypes.Structure):
    _fields_ = [("update_rms", c_float), ("offdiag_ratio", c_float), ("refreshed", c_int32),
                ("nonfinite", c_int32)]


class MuonMat(ctypes.Structure):
    _fields_ = [("m", c_int32), ("n", c_int32), ("W", c_void_p), ("G", c_void_p), ("g_dtype", c_int32),
                ("M", c_void_p), ("split_rows", c_int32), ("split_cols", c_int32)]


class MuonParams(ctypes.Structure):
    _fields_ = [("mu", c_float), ("lr", c_float), ("wd", c_float), ("eps", c_float), ("ns_steps", c_int32),
                ("ns_coef", POINTER(c_float)), ("norm", c_int32), ("polar", c_int32)]


class SoapMat(ctypes.Structure):
    _fields_ = [("m", c_int32), ("n", c_int32), ("W", c_void_p), ("G", c_void_p), ("g_dtype", c_int32),
                ("M", c_void_p), ("V", c_void_p), ("L", c_void_p), ("R", c_void_p), ("QL", c_void_p),
                ("QR", c_void_p), ("perm_L", c_void_p), ("perm_R", c_void_p)]


class SoapParams(ctypes.Structure):
    _fields_ = [("beta1", c_float), ("beta2", c_float), ("eps", c_float), ("lr", c_float), ("wd", c_float),
                ("t", c_int64), ("refresh", Refresh)]


class FoamMat(ctypes.Structure):
    _fields_ = [("m", c_int32), ("n", c_int32), ("W", c_void_p), ("G", c_void_p), ("g_dtype", c_int32),
                ("M", c_void_p), ("r", c_void_p), ("c", c_void_p), ("R", c_void_p), ("QR", c_void_p),
                ("perm_R", c_void_p)]


class FoamParams(ctypes.Structure):
    _fields_ = [("beta1", c_float), ("beta2", c_float), ("eps", c_float), ("lr", c_float), ("wd", c_float),
                ("t", c_int64), ("refresh", Refresh), ("tau_raw_trace", c_int32)]


class LaunchInfo(ctypes.Structure):
    _fields_ = [("kernel", c_int32), ("pad", c_int32), ("flops", ctypes.c_double), ("bytes", ctypes.c_double),
                ("tc_flops", ctypes.c_double), ("exec_flops", ctypes.c_double), ("exec_tc_flops", ctypes.c_double)]


KERNEL_NAMES = {1: "muon_prep", 2: "muon_scale", 3: "ns_gram", 4: "ns_poly", 5: "ns_axpy", 6: "muon_colsq",
                7: "muon_colscale", 8: "muon_rowscale", 9: "muon_update", 10: "muon_stats", 11: "split3",
                12: "gemm_test", 13: "pc_elementwise", 14: "pc_factor", 15: "pc_check", 16: "pc_power",
                17: "pc_sort", 18: "pc_qr", 19: "pc_rotate", 20: "pc_update", 21: "pc_panel", 22: "pc_chol",
                23: "pc_qr_apply", 24: "pc_qr_reduce", 25: "pc_stats", 26: "mop_init"}

# name -> (restype, argtypes)
SIGNATURES = {
    "mao_muon_workspace_size": (c_int32, [POINTER(MuonMat), c_int32, POINTER(MuonParams), POINTER(c_size_t)]),
    "mao_muon_step": (c_int32, [POINTER(MuonMat), c_int32, POINTER(MuonParams), c_void_p, c_size_t, c_void_p,
                                c_void_p]),
    "mao_muon_step_noalloc": (c_int32, [POINTER(MuonMat), c_int32, POINTER(MuonParams), c_void_p, c_void_p]),
    "mao_muon_noalloc_status": (c_int32, [c_void_p, POINTER(c_int32)]),
    "mao_soap_workspace_size": (c_int32, [POINTER(SoapMat), c_int32, POINTER(SoapParams), POINTER(c_size_t)]),
    "mao_soap_step": (c_int32, [POINTER(SoapMat), c_int32, POINTER(SoapParams), c_void_p, c_size_t, c_void_p,
                                c_void_p]),
    "mao_foam_workspace_size": (c_int32, [POINTER(FoamMat), c_int32, POINTER(FoamParams), POINTER(c_size_t)]),
    "mao_foam_step": (c_int32, [POINTER(FoamMat), c_int32, POINTER(FoamParams), c_void_p, c_size_t, c_void_p,
                                c_void_p]),
    "mao_muon_state_elems": (c_uint64, [c_int32, c_int32]),
    "mao_soap_state_elems": (c_uint64, [c_int32, c_int32]),
    "mao_foam_state_elems": (c_uint64, [c_int32, c_int32]),
    "mao_status_string": (ctypes.c_char_p, [c_int32]),
    "mao_workspace_status": (c_int32, [c_void_p, c_void_p, POINTER(c_int32)]),
    "mao_version": (c_int32, []),
    "mao_profile_start": (c_int32, [POINTER(c_void_p), POINTER(LaunchInfo), c_int32]),
    "mao_profile_stop": (c_int32, []),
    "mao_device_check": (c_int32, []),
    "mao_test_gemm_workspace_size": (c_int32, [c_int32, c_int32, c_int32, c_int32, c_int32, POINTER(c_size_t)]),
    "mao_test_wait_timeout": (c_int32, [c_void_p, c_size_t, c_void_p]),
    "mao_test_set_table_kernel": (c_int32, [c_int32]),
    "mao_test_gemm": (c_int32, [c_int32, c_int32, c_int32, c_void_p, c_void_p, c_void_p, c_int32, c_int32, c_int32,
                                c_int32, c_void_p, c_size_t, c_void_p]),
}

_lib = None


class MaoError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        msg = status_string(status) if _lib is not None else str(status)
        super().__init__(f"{what}: {msg} (status {status})" if what else f"{msg} (status {status})")


def load(path: str = LIB_PATH):
    """Load libmao.so and declare every exported signature (raises if absent)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libmao.so not built at {path}; run `python -m matrix_aware_optimizers_02_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def status_string(s: int) -> str:
    return load().mao_status_string(s).decode()


def check(status: int, what: str = ""):
    if status != MAO_OK:
        raise MaoError(status, what)
