"""Thin Python binding over libmao: builds the C descriptors from torch tensors
and calls the library on the current CUDA stream.  Argument marshalling only;
every arithmetic step runs in the library's kernels.

    from matrix_aware_optimizers_02_b200 import api
    step = api.MuonBatch([(W, G, M), ...], mu=0.95, lr=0.02, norm="col_row")
    step()            # one optimizer step on torch.cuda.current_stream()
"""

from __future__ import annotations

import ctypes
from typing import Iterable, Optional, Sequence, Tuple

import torch

from . import _lib as L


def _stream_handle(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


def _g_dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return L.MAO_F32
    if t.dtype == torch.bfloat16:
        return L.MAO_BF16
    raise TypeError(f"gradient dtype {t.dtype} not supported (float32 or bfloat16)")


def _check_mat(name: str, t: torch.Tensor, shape, dtype=torch.float32):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _alloc_workspace(nbytes: int, device) -> torch.Tensor:
    # 256-byte alignment: the caching allocator returns 512-byte aligned blocks
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


class MuonBatch:
    """One Muon / Muon+ step over a fixed list of (W, G, M) matrices.

    W, M: float32 (m, n) contiguous CUDA tensors updated in place; G: float32 or
    bfloat16 (m, n).  The descriptors and the workspace are built once; calling
    the object enqueues one step on the given (or current) stream.
    """

    def __init__(self, mats: Sequence[Tuple[torch.Tensor, torch.Tensor, torch.Tensor]], *, mu: float, lr: float,
                 wd: float = 0.0, eps: float = 1e-7, ns_steps: int = 5,
                 ns_coef: Optional[Sequence[Sequence[float]]] = None, norm: str = "none",
                 split: Optional[Sequence[Tuple[int, int]]] = None, polar: str = "ns",
                 workspace: Optional[torch.Tensor] = None, with_stats: bool = False, allocate: bool = True):
        self.lib = L.load()
        self.mats = list(mats)
        n = len(self.mats)
        arr = (L.MuonMat * max(n, 1))()
        dev = None
        if split is not None and len(split) != n:
            raise ValueError("split must give one (split_rows, split_cols) pair per matrix")
        for i, (W, G, M) in enumerate(self.mats):
            m_, n_ = W.shape
            _check_mat("W", W, (m_, n_))
            _check_mat("G", G, (m_, n_), None)
            _check_mat("M", M, (m_, n_))
            sr, sc = split[i] if split is not None else (1, 1)
            arr[i] = L.MuonMat(m_, n_, W.data_ptr(), G.data_ptr(), _g_dtype(G), M.data_ptr(), int(sr), int(sc))
            dev = W.device
        self.arr = arr
        self.count = n
        self._coef = None
        coef_ptr = None
        if ns_coef is not None:
            flat = [float(x) for triple in ns_coef for x in triple]
            if len(flat) != 3 * ns_steps:
                raise ValueError("ns_coef must hold ns_steps (a, b, c) triples")
            self._coef = (ctypes.c_float * len(flat))(*flat)
            coef_ptr = ctypes.cast(self._coef, ctypes.POINTER(ctypes.c_float))
        if norm not in L.NORM_MODES:
            raise ValueError(f"norm must be one of {sorted(L.NORM_MODES)}")
        polars = {"ns": L.POLAR_NS, "exact": L.POLAR_EXACT}
        if polar not in polars:
            raise ValueError(f"polar must be one of {sorted(polars)}")
        self.params = L.MuonParams(mu, lr, wd, eps, ns_steps, coef_ptr, L.NORM_MODES[norm], polars[polar])
        nbytes = ctypes.c_size_t(0)
        L.check(self.lib.mao_muon_workspace_size(arr, n, ctypes.byref(self.params), ctypes.byref(nbytes)),
                "mao_muon_workspace_size")
        self.ws_bytes = nbytes.value
        dev = dev if dev is not None else torch.device("cuda")
        self.workspace = None
        if workspace is not None or allocate:
            self.attach_workspace(workspace if workspace is not None else _alloc_workspace(self.ws_bytes, dev))
        self.stats = None
        if with_stats:
            self.stats = torch.zeros((max(n, 1), 4), dtype=torch.float32, device=dev)

    def attach_workspace(self, workspace: torch.Tensor) -> None:
        """Use `workspace` (uint8 CUDA tensor of at least ws_bytes) from now on; several
        batches run on one stream may share one workspace."""
        if workspace.numel() * workspace.element_size() < self.ws_bytes:
            raise ValueError("workspace too small")
        self.workspace = workspace

    def __call__(self, stream: Optional[torch.cuda.Stream] = None) -> None:
        with torch.cuda.nvtx.range("mao.muon_step"):  # names the step's launches in a trace
            st = self.lib.mao_muon_step(self.arr, self.count, ctypes.byref(self.params), self.workspace.data_ptr(),
                                        self.ws_bytes, self.stats.data_ptr() if self.stats is not None else None,
                                        _stream_handle(stream))
        L.check(st, "mao_muon_step")

    def device_status(self, stream: Optional[torch.cuda.Stream] = None) -> int:
        """Status word recorded on the device by the last step (synchronises the stream)."""
        where = ctypes.c_int32(0)
        return self.lib.mao_workspace_status(self.workspace.data_ptr(), _stream_handle(stream), ctypes.byref(where))

    def stats_dict(self):
        """Per-matrix diagnostics of the last step (update_rms, nonfinite)."""
        if self.stats is None:
            return None
        s = self.stats[: self.count].cpu()
        nonfinite = s[:, 3].contiguous().view(torch.int32)
        return {"update_rms": s[:, 0].tolist(), "nonfinite": nonfinite.tolist()}


def muon_step(mats, **kw) -> None:
    """Functional form: build a MuonBatch and run one step."""
    MuonBatch(mats, **kw)()


def gemm(A: torch.Tensor, B: torch.Tensor, *, kind: str = "bf16", a_mn_major: bool = False,
         b_mn_major: bool = False, kernel: str = "auto",
         stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Verification entry: D[b] = A[b] @ B[b]^T through the tensor-core GEMM core.

    A is (batch, M, K) (or (batch, K, M) when a_mn_major); B is (batch, N, K)
    (or (batch, K, N) when b_mn_major).  Kinds:
      "bf16"        bf16 operands, accumulated over all of K in the tensor memory;
      "split3"      fp32 operands held as three bf16 planes, fp32-faithful;
      "bf16_fold"   bf16 operands, partial sums over 256 of K folded in fp32;
      "split3_bf16" fp32 A (three planes) times bf16 B;
      "bf16_split3" bf16 A times fp32 B (three planes);
      "split2"      fp32 operands held as two bf16 planes each, three products.
    kernel ("auto", "one_cta", "cta_pair") picks the one-CTA or the CTA-pair kernel.
    Returns fp32 (batch, M, N).
    """
    lib = L.load()
    k = {"bf16": 0, "split3": 1, "bf16_fold": 2, "split3_bf16": 3, "bf16_split3": 4, "split2": 5}[kind]
    a_dt, b_dt = {"bf16": ("bf16", "bf16"), "split3": ("f32", "f32"), "bf16_fold": ("bf16", "bf16"),
                  "split3_bf16": ("f32", "bf16"), "bf16_split3": ("bf16", "f32"), "split2": ("f32", "f32")}[kind]
    dts = {"bf16": torch.bfloat16, "f32": torch.float32}
    for name, X, dt in (("A", A, dts[a_dt]), ("B", B, dts[b_dt])):
        if X.dim() != 3:
            raise ValueError(f"{name} must be 3-D (batch, rows, cols), got {tuple(X.shape)}")
        _check_mat(name, X, tuple(X.shape), dt)
    if A.shape[0] != B.shape[0] or (A.shape[1] if a_mn_major else A.shape[2]) != (B.shape[1] if b_mn_major
                                                                                   else B.shape[2]):
        raise ValueError(f"A {tuple(A.shape)} and B {tuple(B.shape)} do not share batch and K")
    k |= {"auto": 0, "one_cta": 16, "cta_pair": 32}[kernel]
    batch = A.shape[0]
    M = A.shape[2] if a_mn_major else A.shape[1]
    K = A.shape[1] if a_mn_major else A.shape[2]
    N = B.shape[2] if b_mn_major else B.shape[1]
    D = torch.empty((batch, M, N), dtype=torch.float32, device=A.device)
    nbytes = ctypes.c_size_t(0)
    L.check(lib.mao_test_gemm_workspace_size(k, batch, M, N, K, ctypes.byref(nbytes)), "gemm workspace")
    ws = _alloc_workspace(nbytes.value, A.device)
    L.check(lib.mao_test_gemm(k, int(a_mn_major), int(b_mn_major), A.data_ptr(), B.data_ptr(), D.data_ptr(), batch,
                              M, N, K, ws.data_ptr(), nbytes.value, _stream_handle(stream)), "mao_test_gemm")
    where = ctypes.c_int32(0)
    st = lib.mao_workspace_status(ws.data_ptr(), _stream_handle(stream), ctypes.byref(where))
    L.check(st, f"gemm device status (site {where.value})")
    return D


def set_table_kernel(kernel: str = "auto") -> None:
    """Verification switch: run every fp32-faithful table-mode product of this process on
    the library's choice ("auto"), the one-CTA kernel ("one_cta") or the CTA-pair kernel
    wherever it applies ("cta_pair")."""
    L.check(L.load().mao_test_set_table_kernel({"auto": 0, "one_cta": 1, "cta_pair": 2}[kernel]),
            "mao_test_set_table_kernel")


def _refresh(kind: str, k: int, pf: int, tol: float, sort: bool, lag: bool = False) -> "L.Refresh":
    kinds = {"every_k": L.REFRESH_EVERY_K, "adaptive": L.REFRESH_ADAPTIVE, "never": L.REFRESH_NEVER}
    if kind not in kinds:
        raise ValueError(f"refresh must be one of {sorted(kinds)}")
    return L.Refresh(kinds[kind], int(k), int(pf), float(tol), int(bool(sort)), int(bool(lag)))


class _PrecondBatch:
    """Shared plumbing of SoapBatch / FoamBatch."""

    def _finish(self, size_fn, n, device, workspace, with_stats, allocate=True):
        nbytes = ctypes.c_size_t(0)
        L.check(size_fn(self.arr, n, ctypes.byref(self.params), ctypes.byref(nbytes)), size_fn.__name__)
        self.ws_bytes = nbytes.value
        self.workspace = None
        if workspace is not None or allocate:
            self.attach_workspace(workspace if workspace is not None else _alloc_workspace(self.ws_bytes, device))
        self.stats = torch.zeros((max(n, 1), 4), dtype=torch.float32, device=device) if with_stats else None

    def attach_workspace(self, workspace: torch.Tensor) -> None:
        """Use `workspace` (uint8 CUDA tensor of at least ws_bytes); several batches run on
        one stream may share one workspace."""
        if workspace.numel() * workspace.element_size() < self.ws_bytes:
            raise ValueError("workspace too small")
        self.workspace = workspace

    def device_status(self, stream: Optional[torch.cuda.Stream] = None) -> int:
        where = ctypes.c_int32(0)
        return self.lib.mao_workspace_status(self.workspace.data_ptr(), _stream_handle(stream), ctypes.byref(where))

    def stats_dict(self):
        """Per-matrix diagnostics of the last step."""
        if self.stats is None:
            return None
        s = self.stats[: self.count].cpu()
        return {"update_rms": s[:, 0].tolist(), "offdiag_ratio": s[:, 1].tolist(),
                "refreshed": s[:, 2].contiguous().view(torch.int32).tolist(),
                "nonfinite": s[:, 3].contiguous().view(torch.int32).tolist()}


class SoapBatch(_PrecondBatch):
    """One two-sided SOAP step over a fixed list of matrices.

    Each entry is a dict with CUDA tensors W (m, n) fp32, G (m, n) fp32/bf16 and
    the state M, V (m, n), L, QL (m, m), R, QR (n, n) fp32; optional int32
    perm_L (m) / perm_R (n) receive the basis permutations of the step.
    Call with the 1-based step number t.
    """

    def __init__(self, mats, *, beta1: float, beta2: float, eps: float, lr: float, wd: float = 0.0,
                 refresh: str = "every_k", k: int = 1, pf: int = 10, tol: float = 0.1, sort: bool = True,
                 lag: bool = False, workspace: Optional[torch.Tensor] = None, with_stats: bool = False, t: int = 1,
                 allocate: bool = True):
        self.lib = L.load()
        self.mats = list(mats)
        n = len(self.mats)
        self.arr = (L.SoapMat * max(n, 1))()
        dev = None
        for i, d in enumerate(self.mats):
            W = d["W"]
            m_, n_ = W.shape
            for name, shape in (("W", (m_, n_)), ("M", (m_, n_)), ("V", (m_, n_)), ("L", (m_, m_)),
                                ("QL", (m_, m_)), ("R", (n_, n_)), ("QR", (n_, n_))):
                _check_mat(name, d[name], shape)
            _check_mat("G", d["G"], (m_, n_), None)
            pl, pr = d.get("perm_L"), d.get("perm_R")
            self.arr[i] = L.SoapMat(m_, n_, W.data_ptr(), d["G"].data_ptr(), _g_dtype(d["G"]), d["M"].data_ptr(),
                                    d["V"].data_ptr(), d["L"].data_ptr(), d["R"].data_ptr(), d["QL"].data_ptr(),
                                    d["QR"].data_ptr(), pl.data_ptr() if pl is not None else None,
                                    pr.data_ptr() if pr is not None else None)
            dev = W.device
        self.count = n
        self.params = L.SoapParams(beta1, beta2, eps, lr, wd, int(t), _refresh(refresh, k, pf, tol, sort, lag))
        self._finish(self.lib.mao_soap_workspace_size, n, dev if dev is not None else "cuda", workspace, with_stats,
                     allocate)

    def __call__(self, t: int, stream: Optional[torch.cuda.Stream] = None) -> None:
        self.params.t = int(t)
        with torch.cuda.nvtx.range("mao.soap_step"):
            st = self.lib.mao_soap_step(self.arr, self.count, ctypes.byref(self.params), self.workspace.data_ptr(),
                                        self.ws_bytes, self.stats.data_ptr() if self.stats is not None else None,
                                        _stream_handle(stream))
        L.check(st, "mao_soap_step")


class FoamBatch(_PrecondBatch):
    """One FOAM step over a fixed list of matrices.

    Each entry is a dict with W (m, n), G (m, n), M (m, n), r (m), c (n), R and
    QR (n, n); optional int32 perm_R (n).  Call with the 1-based step number t.
    """

    def __init__(self, mats, *, beta1: float, beta2: float, eps: float, lr: float, wd: float = 0.0,
                 refresh: str = "adaptive", k: int = 1, pf: int = 10, tol: float = 0.1, sort: bool = True,
                 lag: bool = False, tau_raw_trace: bool = False, workspace: Optional[torch.Tensor] = None,
                 with_stats: bool = False, t: int = 1, allocate: bool = True):
        self.lib = L.load()
        self.mats = list(mats)
        n = len(self.mats)
        self.arr = (L.FoamMat * max(n, 1))()
        dev = None
        for i, d in enumerate(self.mats):
            W = d["W"]
            m_, n_ = W.shape
            for name, shape in (("W", (m_, n_)), ("M", (m_, n_)), ("r", (m_,)), ("c", (n_,)), ("R", (n_, n_)),
                                ("QR", (n_, n_))):
                _check_mat(name, d[name], shape)
            _check_mat("G", d["G"], (m_, n_), None)
            pr = d.get("perm_R")
            self.arr[i] = L.FoamMat(m_, n_, W.data_ptr(), d["G"].data_ptr(), _g_dtype(d["G"]), d["M"].data_ptr(),
                                    d["r"].data_ptr(), d["c"].data_ptr(), d["R"].data_ptr(), d["QR"].data_ptr(),
                                    pr.data_ptr() if pr is not None else None)
            dev = W.device
        self.count = n
        self.params = L.FoamParams(beta1, beta2, eps, lr, wd, int(t), _refresh(refresh, k, pf, tol, sort, lag),
                                   int(bool(tau_raw_trace)))
        self._finish(self.lib.mao_foam_workspace_size, n, dev if dev is not None else "cuda", workspace, with_stats,
                     allocate)

    def __call__(self, t: int, stream: Optional[torch.cuda.Stream] = None) -> None:
        self.params.t = int(t)
        with torch.cuda.nvtx.range("mao.foam_step"):
            st = self.lib.mao_foam_step(self.arr, self.count, ctypes.byref(self.params), self.workspace.data_ptr(),
                                        self.ws_bytes, self.stats.data_ptr() if self.stats is not None else None,
                                        _stream_handle(stream))
        L.check(st, "mao_foam_step")
