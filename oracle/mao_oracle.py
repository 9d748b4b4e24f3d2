"""Float64 CPU oracle for the per-matrix Muon / Muon+ / SOAP / FOAM optimizer step.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the C-ABI library, its
Python binding, the kernels) may import or call this module.  It exists so that
the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
can check the CUDA path against a plain, slow, obviously correct statement of
what the method computes.

Everything here is NumPy in float64, one matrix at a time, in the order the
source pages give.  Library primitives used as single steps: ``@`` (matmul),
``numpy.linalg.qr`` (Householder QR), ``numpy.linalg.svd`` (MOP's exact polar
factor, which the pages define by the SVD), and, only in the self-check helpers
at the bottom, ``numpy.linalg.eigh``.

Sources (cited by page title and section):
  [SMB-review]  "SOAP, Muon and Beyond" (Korean review): §1-1 Problem definition
                (AdamW and Shampoo factor equations), §2-1 Main contribution
                (polar factor, Shampoo=Muon identity, RMS matching), §3-2 Module
                breakdown (Muon recipe, SOAP rotation, real-time eigenbasis update).
  [SMB-summary] "SOAP, Muon, and Beyond" (English summary): eq. (1) SOAP update,
                "Update-RMS Matching", "SOAP Instability Diagnosis".
  [FOAM-review] "Factored One-sided Adam-Moment for Practical and Scalable SOAP"
                (Korean review): §1 Key Terms & Definitions, §3 Method & Key Results.
  [MuonPlus]    "Muon+: Towards Better Muon via One Additional Normalization Step":
                technical summary §2 Methodology.

Readings taken where the pages are silent:
  * Newton-Schulz form: the quintic X <- aX + (bA + cA^2)X with A = X X^T, run on
    the wide orientation (transposed when m > n); default (a,b,c) =
    (3.4445, -4.7750, 2.0315) each iteration.  The pages name Newton-Schulz only.
  * Pre-normalisation X0 = M / (||M||_F + 1e-7) (recipe epsilon, [SMB-review] §3-2).
  * Muon+ Norm^(d): l2 normalisation of each row / column, denominator norm+1e-7,
    Col-Row = column first then row; applied before the lr*sqrt(m/n) scale.
  * Decoupled weight decay W <- W(1 - lr*wd) (recipe value only on the pages).
  * SOAP/FOAM Adam: bias-corrected, eps outside the square root; V is not
    re-projected when the basis changes (only permuted with it).
  * Eigenbasis refresh: one power step P = L Q then Q = qr(P) with a positive
    diagonal in the triangular factor; optional sort of the basis by the
    Rayleigh quotients diag(Q^T L Q), descending, stable, before the power step.
  * FOAM tau uses the bias-corrected trace tr(R / (1 - beta2^t)); adaptive check:
    on steps with (t-1) % pf == 0, rho = ||offdiag(Q^T R Q)||_F / ||Q^T R Q||_F,
    refresh iff rho > tol.

Parity pins for every function are in tests/test_oracle_*.py.  No function here
is "parity unpinned".
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

# Default quintic Newton-Schulz coefficients (a, b, c), one triple per iteration.
NS_DEFAULT_COEF = (3.4445, -4.7750, 2.0315)
NS_EPS = 1e-7          # Frobenius pre-normalisation epsilon ([SMB-review] §3-2 recipe)
NORM_EPS = 1e-7        # Muon+ row/column normalisation epsilon (reading)

NORM_NONE, NORM_ROW, NORM_COL, NORM_COL_ROW, NORM_ROW_COL = 0, 1, 2, 3, 4
REFRESH_EVERY_K, REFRESH_ADAPTIVE, REFRESH_NEVER = 0, 1, 2


def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


# Working precision of the SOAP / FOAM functions below.  float64 is the oracle;
# float32 runs the same steps in single precision and serves only to measure the
# inherent fp32 rounding floor of a case (the tests' tolerance for quantities the
# method amplifies).
def _w(a, dtype):
    return np.asarray(a, dtype=dtype)


# --------------------------------------------------------------------------
# Muon  ([MuonPlus] §2 Methodology; [SMB-review] §2-1 (2), §3-2 (2))
# --------------------------------------------------------------------------

def newton_schulz(M, coefs=None, steps: int = 5, eps: float = NS_EPS, dtype=np.float64):
    """Approximate the polar factor U V^T of M (M = U S V^T) by Newton-Schulz.

    [SMB-review] §2-1 (2): Muon approximates Polar(M) = U V^T by a Newton-Schulz
    iteration.  Steps: X0 = M / (||M||_F + eps); if M has more rows than
    columns, iterate on X0^T; each iteration with coefficients (a, b, c):
        A = X X^T ;  B = b A + c A A ;  X = a X + B X.
    The result is returned in M's orientation.
    """
    X = np.asarray(M, dtype=dtype)
    if coefs is None:
        coefs = [NS_DEFAULT_COEF] * steps
    transposed = X.shape[0] > X.shape[1]
    X = X / (np.sqrt(np.sum(X * X)) + dtype(eps))
    if transposed:
        X = X.T
    for (a, b, c) in coefs:
        A = X @ X.T
        B = dtype(b) * A + dtype(c) * (A @ A)
        X = dtype(a) * X + B @ X
    return X.T if transposed else X


def muon_plus_norm(O, mode: int, eps: float = NORM_EPS):
    """Muon+ normalisation Norm^(d) applied to the orthogonalised update.

    [MuonPlus] §2 Methodology: O_t = Norm^(d)(Ortho(M_t)) with d = row, column,
    Col-Row or Row-Col.  Reading: each row (column) is divided by its l2 norm
    plus eps; the combined modes apply the first-named direction first.
    """
    O = _f64(O)

    def rows(X):
        return X / (np.sqrt(np.sum(X * X, axis=1, keepdims=True)) + eps)

    def cols(X):
        return X / (np.sqrt(np.sum(X * X, axis=0, keepdims=True)) + eps)

    if mode == NORM_NONE:
        return O.copy()
    if mode == NORM_ROW:
        return rows(O)
    if mode == NORM_COL:
        return cols(O)
    if mode == NORM_COL_ROW:
        return rows(cols(O))
    if mode == NORM_ROW_COL:
        return cols(rows(O))
    raise ValueError(f"unknown norm mode {mode}")


def polar_exact(M):
    """Exact polar factor U V^T of M = U S V^T from the thin SVD.

    [SMB-summary] "Muon vs SOAP Comparison": MOP is Muon with the Newton-Schulz
    approximation replaced by the exact polar decomposition computed by SVD.
    """
    U, _, Vt = np.linalg.svd(_f64(M), full_matrices=False)
    return U @ Vt


def muon_step(W, G, M, *, mu: float, lr: float, wd: float = 0.0, ns_coefs=None,
              ns_steps: int = 5, norm: int = NORM_NONE, split=(1, 1), polar: str = "ns"):
    """One Muon (or Muon+, or MOP) step on one m x n matrix.

    [MuonPlus] §2 Methodology: M <- mu M + (1-mu) G; O = Ortho(M) (Newton-Schulz);
    optionally O <- Norm^(d)(O); W <- W - lr sqrt(m/n) O.  Decoupled weight decay
    W(1 - lr wd) is the reading of the recipe's weight decay ([SMB-review] §3-2).

    split = (sr, sc): the stored matrix holds sr x sc logical matrices of equal
    size (a fused QKV projection is (1, 3) when q, k, v are column blocks).  The
    recipe of [SMB-review] §3-2 (2) and §4-4 (2) orthogonalises each logical
    matrix on its own; reading: every per-matrix quantity (the Frobenius
    pre-normalisation, Newton-Schulz, Norm^(d) and the sqrt(m/n) scale) is that
    of the logical block.
    polar = "ns" (Newton-Schulz) or "exact" (MOP: the SVD polar factor).
    Returns (W_new, M_new, O) with O the final (normalised) direction.
    """
    W, G, M = _f64(W), _f64(G), _f64(M)
    m, n = W.shape
    sr, sc = split
    if m % sr or n % sc:
        raise ValueError(f"{m}x{n} does not split into {sr}x{sc} equal blocks")
    mb, nb = m // sr, n // sc
    M_new = mu * M + (1.0 - mu) * G                                   # M1
    O = np.empty_like(M_new)
    for i in range(sr):
        for j in range(sc):
            blk = M_new[i * mb:(i + 1) * mb, j * nb:(j + 1) * nb]
            if polar == "exact":
                ob = polar_exact(blk)                                 # MOP
            elif polar == "ns":
                ob = newton_schulz(blk, ns_coefs, ns_steps)           # M2 + M3
            else:
                raise ValueError(f"unknown polar method {polar}")
            ob = muon_plus_norm(ob, norm)                             # M4
            O[i * mb:(i + 1) * mb, j * nb:(j + 1) * nb] = ob
    W_new = W * (1.0 - lr * wd) - lr * np.sqrt(mb / nb) * O          # M5 (every block has the same shape)
    return W_new, M_new, O


# --------------------------------------------------------------------------
# Shared SOAP / FOAM pieces
# --------------------------------------------------------------------------

def qr_positive(P, dtype=np.float64):
    """Q factor of P = Q R with diag(R) > 0 (unique for full-rank P).

    The per-step QR orthogonalisation of the eigenbasis ([SMB-review] §3-2 (4),
    [SMB-summary] "SOAP Instability Diagnosis").  numpy's Householder QR is
    sign-fixed so that every diagonal entry of R is positive.
    """
    Q, R = np.linalg.qr(_w(P, dtype))
    s = np.sign(np.diag(R))
    s[s == 0] = 1.0
    return Q * s[None, :]


def rayleigh_keys(F, Q):
    """key_i = Q[:, i]^T F Q[:, i], i.e. diag(Q^T F Q)."""
    F, Q = _f64(F), _f64(Q)
    return np.einsum("ki,ki->i", Q, F @ Q)


def sort_perm(keys):
    """Stable descending argsort (ties keep the lower index first)."""
    keys = _f64(keys)
    return np.argsort(-keys, kind="stable").astype(np.int32)


def refresh_basis(F, Q, sort: bool, dtype=np.float64, perm=None):
    """One eigenbasis refresh of the factor F from the current basis Q.

    [SMB-review] §3-2 (4): refresh the basis from the updated factor, then QR.
    Reading: optional stable descending sort of Q's columns by diag(Q^T F Q),
    then one power step P = F Q and Q <- qr(P) (positive diagonal).
    Returns (Q_new, perm) where perm[i] is the old column placed at i.
    `perm`, when given, replaces the sort (replay of an ordering decided
    elsewhere, e.g. at near-equal keys; tests only).
    """
    F, Q = _w(F, dtype), _w(Q, dtype)
    k = Q.shape[1]
    if perm is not None:
        perm = np.asarray(perm, dtype=np.int32)
    else:
        perm = sort_perm(rayleigh_keys(F, Q)) if sort else np.arange(k, dtype=np.int32)
    Qp = Q[:, perm]
    P = F @ Qp
    return qr_positive(P, dtype), perm


def offdiag_ratio(D):
    """rho = ||D - diag(D)||_F / ||D||_F."""
    D = _f64(D)
    off = D - np.diag(np.diag(D))
    den = np.sqrt(np.sum(D * D))
    return float(np.sqrt(np.sum(off * off)) / den) if den > 0 else 0.0


def refresh_decision(kind: int, t: int, k: int = 1, pf: int = 10, tol: float = 0.1,
                     F=None, Q=None, dtype=np.float64):
    """Whether a basis refresh happens at step t (1-based), and the check ratio.

    EVERY_K: (t-1) % k == 0 ([SMB-summary] "SOAP Instability Diagnosis": every
    step, or every 10 steps for the stale baseline).  ADAPTIVE ([FOAM-review] §3,
    the Purifying-Shampoo tolerance criterion with pf=10, tol=0.1; the criterion
    itself is not printed -- reading): on steps with (t-1) % pf == 0, compute
    D = Q^T F Q and refresh iff ||offdiag D||_F / ||D||_F > tol.
    Returns (refresh, rho) with rho = -1.0 when no check ran.
    """
    if kind == REFRESH_NEVER:
        return False, -1.0
    if kind == REFRESH_EVERY_K:
        return ((t - 1) % k) == 0, -1.0
    if kind == REFRESH_ADAPTIVE:
        if (t - 1) % pf != 0:
            return False, -1.0
        D = _w(Q, dtype).T @ _w(F, dtype) @ _w(Q, dtype)
        rho = offdiag_ratio(D)
        return rho > tol, rho
    raise ValueError(f"unknown refresh kind {kind}")


# --------------------------------------------------------------------------
# SOAP  ([SMB-review] §1-1, §3-2 (3)(4); [SMB-summary] eq. (1))
# --------------------------------------------------------------------------

@dataclass
class SoapState:
    M: np.ndarray
    V: np.ndarray
    L: np.ndarray
    R: np.ndarray
    QL: np.ndarray
    QR: np.ndarray

    @staticmethod
    def init(m: int, n: int, eps_init: float = 1e-6) -> "SoapState":
        """L = R = eps_init * I, Q = I, M = V = 0 (initial state reading)."""
        return SoapState(np.zeros((m, n)), np.zeros((m, n)), eps_init * np.eye(m),
                         eps_init * np.eye(n), np.eye(m), np.eye(n))

    def copy(self, dtype=np.float64) -> "SoapState":
        return SoapState(*(np.array(x, dtype=dtype, copy=True) for x in
                           (self.M, self.V, self.L, self.R, self.QL, self.QR)))


@dataclass
class SoapResult:
    W: np.ndarray
    state: SoapState
    U: np.ndarray
    perm_L: np.ndarray
    perm_R: np.ndarray
    refreshed_L: bool
    refreshed_R: bool
    rho_L: float = -1.0
    rho_R: float = -1.0


def soap_factors(L, R, G, beta2: float, dtype=np.float64):
    """S1: L <- b2 L + (1-b2) G G^T ;  R <- b2 R + (1-b2) G^T G  ([SMB-review] §1-1)."""
    G = _w(G, dtype)
    return (beta2 * _w(L, dtype) + (1.0 - beta2) * (G @ G.T),
            beta2 * _w(R, dtype) + (1.0 - beta2) * (G.T @ G))


def soap_precondition(W, G, M, V, QL, QR, *, t: int, beta1: float, beta2: float, eps: float,
                      lr: float, wd: float = 0.0, dtype=np.float64):
    """S5-S8 in a given pair of bases ([SMB-summary] eq. (1), [SMB-review] §3-2 (3)):
      S5  M <- b1 M + (1-b1) G
      S6  Gh = QL^T G QR ;  Mh = QL^T M QR
      S7  V <- b2 V + (1-b2) Gh^2 ;  N = (Mh/(1-b1^t)) / (sqrt(V/(1-b2^t)) + eps)
      S8  U = QL N QR^T ;  W <- W(1 - lr wd) - lr U
    Returns (W_new, M_new, V_new, U).  V is the second moment already expressed in
    these bases (after any permutation of the refresh).
    """
    W, G, M, V, QL, QR = (_w(x, dtype) for x in (W, G, M, V, QL, QR))
    M = beta1 * M + (1.0 - beta1) * G                      # S5
    Gh = QL.T @ G @ QR                                     # S6
    Mh = QL.T @ M @ QR
    V = beta2 * V + (1.0 - beta2) * Gh * Gh                # S7
    mhat = Mh / (1.0 - beta1 ** t)
    vhat = V / (1.0 - beta2 ** t)
    N = mhat / (np.sqrt(vhat) + eps)
    U = QL @ N @ QR.T                                      # S8
    W_new = W * (1.0 - lr * wd) - lr * U
    return W_new, M, V, U


def soap_step(W, G, state: SoapState, *, t: int, beta1: float, beta2: float,
              eps: float, lr: float, wd: float = 0.0, refresh_kind: int = REFRESH_EVERY_K,
              k: int = 1, pf: int = 10, tol: float = 0.1, sort: bool = True, lag: bool = False,
              dtype=np.float64, force_perm_L=None, force_perm_R=None) -> SoapResult:
    """One two-sided SOAP step with the real-time eigenbasis refresh.

    Order ([SMB-review] §3-2 (4)): the current gradient enters the factors first,
    then the basis is refreshed from them (power step + QR), then the momentum is
    preconditioned in the refreshed basis:
      S1  factor EMAs (soap_factors)
      S2  refresh decision
      S3  sort keys diag(Q^T F Q), permutation, power step P = F Q
      S4  Q <- qr(P)
      S5-S8  soap_precondition
    lag=True takes the order of the standard implementation that [SMB-summary]
    ("SOAP Instability Diagnosis") and [SMB-review] §2-1 (3) blame for the
    slingshot instability: the refresh (S2-S4) runs on the factors as they were
    before this step's gradient entered them, and S1 follows it.
    """
    W, G = _w(W, dtype), _w(G, dtype)
    s = state.copy(dtype)
    m, n = W.shape
    if not lag:
        s.L, s.R = soap_factors(s.L, s.R, G, beta2, dtype)                  # S1
    refL, rhoL = refresh_decision(refresh_kind, t, k, pf, tol, s.L, s.QL, dtype)  # S2
    refR, rhoR = refresh_decision(refresh_kind, t, k, pf, tol, s.R, s.QR, dtype)
    permL = np.arange(m, dtype=np.int32)
    permR = np.arange(n, dtype=np.int32)
    # S3 + S4 (V follows the permutation of its basis; no re-projection)
    if refL:
        s.QL, permL = refresh_basis(s.L, s.QL, sort, dtype, force_perm_L)
        s.V = s.V[permL, :]
    if refR:
        s.QR, permR = refresh_basis(s.R, s.QR, sort, dtype, force_perm_R)
        s.V = s.V[:, permR]
    if lag:
        s.L, s.R = soap_factors(s.L, s.R, G, beta2, dtype)                  # S1 after the refresh
    W_new, s.M, s.V, U = soap_precondition(W, G, s.M, s.V, s.QL, s.QR, t=t, beta1=beta1, beta2=beta2,
                                           eps=eps, lr=lr, wd=wd, dtype=dtype)
    return SoapResult(W_new, s, U, permL, permR, refL, refR, rhoL, rhoR)


# --------------------------------------------------------------------------
# FOAM  ([FOAM-review] §1 Key Terms, §3 Method)
# --------------------------------------------------------------------------

@dataclass
class FoamState:
    M: np.ndarray
    r: np.ndarray
    c: np.ndarray
    R: np.ndarray
    QR: np.ndarray

    @staticmethod
    def init(m: int, n: int, eps_init: float = 1e-6) -> "FoamState":
        """R = eps_init * I, Q_R = I, M = r = c = 0 (initial state reading)."""
        return FoamState(np.zeros((m, n)), np.zeros(m), np.zeros(n), eps_init * np.eye(n), np.eye(n))

    def copy(self, dtype=np.float64) -> "FoamState":
        return FoamState(*(np.array(x, dtype=dtype, copy=True) for x in
                           (self.M, self.r, self.c, self.R, self.QR)))


@dataclass
class FoamResult:
    W: np.ndarray
    state: FoamState
    U: np.ndarray
    perm_R: np.ndarray
    refreshed: bool
    rho: float
    tau: float


def foam_tau(R, r, c, t: int, beta2: float, raw_trace: bool = False) -> float:
    """Trace normalisation tau = tr(R^) / (||r^||_1 ||c^||_1).

    [FOAM-review] §1 (Factored Adam-Moment).  Reading: every statistic carries the
    Adam bias correction 1/(1-b2^t); raw_trace=True uses the literal tr(R).
    """
    bc = 1.0 - beta2 ** t
    tr = float(np.trace(_f64(R)))
    if not raw_trace:
        tr = tr / bc
    rn = float(np.sum(np.abs(_f64(r)))) / bc
    cn = float(np.sum(np.abs(_f64(c)))) / bc
    return tr / (rn * cn)


def foam_precondition(W, G, M, r, c, R, QR, *, t: int, beta1: float, beta2: float, eps: float,
                      lr: float, wd: float = 0.0, raw_trace: bool = False, dtype=np.float64):
    """F4-F6 in a given input-side basis QR ([FOAM-review] §1, §3):
      F4  M <- b1 M + (1-b1) G ;  Gr = G QR ;  Mr = M QR
      F5  r <- b2 r + (1-b2) rowmean(Gr^2) ; c <- b2 c + (1-b2) colmean(Gr^2) ;
          v^_ij = tau r^_i c^_j ;  N = (Mr/(1-b1^t)) / (sqrt(v^) + eps)
      F6  U = N QR^T ;  W <- W(1 - lr wd) - lr U
    c is the column EMA already in QR's column order.  Returns
    (W_new, M_new, r_new, c_new, U, tau).
    """
    W, G, M, r, c, QR = (_w(x, dtype) for x in (W, G, M, r, c, QR))
    M = beta1 * M + (1.0 - beta1) * G                      # F4
    Gr = G @ QR
    Mr = M @ QR
    G2 = Gr * Gr                                           # F5
    r = beta2 * r + (1.0 - beta2) * np.mean(G2, axis=1)
    c = beta2 * c + (1.0 - beta2) * np.mean(G2, axis=0)
    tau = foam_tau(R, r, c, t, beta2, raw_trace)
    bc2 = 1.0 - beta2 ** t
    vhat = tau * np.outer(r / bc2, c / bc2)
    N = (Mr / (1.0 - beta1 ** t)) / (np.sqrt(vhat) + eps)
    U = N @ QR.T                                           # F6
    W_new = W * (1.0 - lr * wd) - lr * U
    return W_new, M, r, c, U, tau


def foam_step(W, G, state: FoamState, *, t: int, beta1: float, beta2: float, eps: float,
              lr: float, wd: float = 0.0, refresh_kind: int = REFRESH_ADAPTIVE, k: int = 1,
              pf: int = 10, tol: float = 0.1, sort: bool = True, lag: bool = False,
              raw_trace: bool = False, dtype=np.float64, force_perm=None) -> FoamResult:
    """One FOAM step (input-only preconditioning, factored Adam moment).

    [FOAM-review] §1, §3:
      F1  R <- b2 R + (1-b2) G^T G             (input-side factor only; L dropped)
      F2  refresh decision (adaptive criterion, pf, tol)
      F3  refresh Q_R as in SOAP; the permutation also permutes c
      F4-F6  foam_precondition
    lag=True refreshes from R as it was before this step's gradient entered it
    (F2-F3 before F1), as soap_step's lag does.
    """
    W, G = _w(W, dtype), _w(G, dtype)
    s = state.copy(dtype)
    n = W.shape[1]
    if not lag:
        s.R = beta2 * s.R + (1.0 - beta2) * (G.T @ G)          # F1
    ref, rho = refresh_decision(refresh_kind, t, k, pf, tol, s.R, s.QR, dtype)  # F2
    perm = np.arange(n, dtype=np.int32)
    if ref:                                                    # F3
        s.QR, perm = refresh_basis(s.R, s.QR, sort, dtype, force_perm)
        s.c = s.c[perm]
    if lag:
        s.R = beta2 * s.R + (1.0 - beta2) * (G.T @ G)          # F1 after the refresh
    W_new, s.M, s.r, s.c, U, tau = foam_precondition(W, G, s.M, s.r, s.c, s.R, s.QR, t=t, beta1=beta1,
                                                     beta2=beta2, eps=eps, lr=lr, wd=wd, raw_trace=raw_trace,
                                                     dtype=dtype)
    return FoamResult(W_new, s, U, perm, ref, rho, tau)


# --------------------------------------------------------------------------
# State accounting ([FOAM-review] §1 Key Terms, §3 Method)
# --------------------------------------------------------------------------

def soap_state_elems(m: int, n: int) -> int:
    """SOAP state: M, V (m x n each), L, Q_L (m x m), R, Q_R (n x n) = 2mn+2m^2+2n^2."""
    return 2 * m * n + 2 * m * m + 2 * n * n


def foam_state_elems(m: int, n: int) -> int:
    """FOAM state: M (m x n), R, Q_R (n x n), r (m), c (n) = mn+2n^2+m+n."""
    return m * n + 2 * n * n + m + n


# --------------------------------------------------------------------------
# Self-check helpers (used only by the oracle's own pins)
# --------------------------------------------------------------------------

def polar_svd(M):
    """Exact polar factor (self-check helper; the same as polar_exact)."""
    return polar_exact(M)


def _inv_quarter_root_psd(S, rtol: float = 1e-12):
    """S^{-1/4} on the range of a symmetric PSD matrix (pseudo-inverse root)."""
    w, V = np.linalg.eigh(_f64(S))
    keep = w > rtol * max(w.max(), 0.0)
    wr = np.zeros_like(w)
    wr[keep] = w[keep] ** -0.25
    return (V * wr[None, :]) @ V.T


def shampoo_update(G, L, R):
    """Shampoo preconditioned update L^{-1/4} G R^{-1/4} ([SMB-review] §1-1)."""
    return _inv_quarter_root_psd(L) @ _f64(G) @ _inv_quarter_root_psd(R)
