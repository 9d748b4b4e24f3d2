"""Pins for the oracle's Muon / Muon+ functions against facts other than the oracle.

Each pin is a closed form, an invariant or a brute-force computation, chosen so
that a dropped term, a wrong sign, a transposed operand or swapped coefficients
fails at least one test.
"""

import numpy as np
import pytest

from oracle import mao_oracle as O
from matrix_aware_optimizers_02_b200 import synth

SHAPES = [(6, 9), (9, 6), (8, 8), (1, 5), (5, 1), (17, 40)]


def _phi_chain(x, coefs):
    # scalar odd polynomial applied to singular values, written out per entry
    out = np.array(x, dtype=np.float64)
    for (a, b, c) in coefs:
        out = np.array([a * v + b * v ** 3 + c * v ** 5 for v in out])
    return out


@pytest.mark.parametrize("shape", SHAPES)
def test_ns_matches_singular_value_closed_form(shape):
    """NS_k(M) = U phi^k(S/(||M||_F+eps)) V^T with U, S, V built first (no SVD call)."""
    m, n = shape
    rng = np.random.default_rng(1)
    k = min(m, n)
    U = synth.random_orthogonal(rng, m)[:, :k]
    V = synth.random_orthogonal(rng, n)[:, :k]
    S = rng.uniform(0.05, 3.0, size=k)
    M = (U * S) @ V.T
    coefs = [O.NS_DEFAULT_COEF] * 5
    got = O.newton_schulz(M, coefs)
    fro = np.sqrt(np.sum(S ** 2))
    want = (U * _phi_chain(S / (fro + O.NS_EPS), coefs)) @ V.T
    assert np.allclose(got, want, rtol=0, atol=1e-10)


def test_ns_distinct_coefficients_per_step():
    """Per-iteration coefficients are applied in order (reordering them changes the result)."""
    rng = np.random.default_rng(2)
    U = synth.random_orthogonal(rng, 7)[:, :5]
    V = synth.random_orthogonal(rng, 5)
    S = np.array([1.0, 0.5, 0.2, 0.1, 0.05])
    M = (U * S) @ V.T
    coefs = [(3.0, -3.2, 1.2), (2.0, -1.5, 0.5), (1.5, -0.5, 0.0)]
    got = O.newton_schulz(M, coefs)
    want = (U * _phi_chain(S / (np.sqrt(np.sum(S ** 2)) + O.NS_EPS), coefs)) @ V.T
    assert np.allclose(got, want, atol=1e-12)
    rev = O.newton_schulz(M, coefs[::-1])
    assert not np.allclose(rev, want, atol=1e-6)


@pytest.mark.parametrize("shape", [(4, 4), (5, 8), (8, 5), (3, 11)])
def test_cubic_ns_converges_to_svd_polar_factor(shape):
    """Polar(M) = U V^T: the convergent cubic (1.5, -0.5, 0) reaches the SVD polar factor."""
    m, n = shape
    rng = np.random.default_rng(3)
    M = synth.matrix_with_spectrum(rng, m, n, rng.uniform(0.3, 2.0, size=min(m, n)))
    got = O.newton_schulz(M, [(1.5, -0.5, 0.0)] * 60)
    assert np.allclose(got, O.polar_svd(M), atol=1e-9)


def test_polar_svd_is_semi_orthogonal_and_nearest():
    rng = np.random.default_rng(4)
    M = rng.standard_normal((5, 9))
    P = O.polar_svd(M)
    assert np.allclose(P @ P.T, np.eye(5), atol=1e-12)
    # P = (M M^T)^{-1/2} M, computed through eigh
    w, Vv = np.linalg.eigh(M @ M.T)
    assert np.allclose(P, (Vv * w ** -0.5) @ Vv.T @ M, atol=1e-10)


def test_quintic_is_not_polar():
    """The quintic's fixed output band is not U V^T: only the closed form may be compared tightly."""
    rng = np.random.default_rng(5)
    M = rng.standard_normal((16, 32))
    out = O.newton_schulz(M)
    err = np.linalg.norm(out - O.polar_svd(M)) / np.linalg.norm(O.polar_svd(M))
    assert 1e-3 < err < 0.5


# ---------------------------------------------------------------- Muon step

@pytest.mark.parametrize("shape,wd", [((6, 10), 0.0), ((10, 6), 0.1), ((7, 7), 0.05)])
def test_muon_step_closed_form(shape, wd):
    """M and G sharing singular vectors: every step of M1..M5 in closed form."""
    m, n = shape
    rng = np.random.default_rng(6)
    k = min(m, n)
    U = synth.random_orthogonal(rng, m)[:, :k]
    V = synth.random_orthogonal(rng, n)[:, :k]
    s_m = rng.uniform(0.1, 1.0, size=k)
    s_g = rng.uniform(0.1, 1.0, size=k)
    M = (U * s_m) @ V.T
    G = (U * s_g) @ V.T
    W = rng.standard_normal((m, n))
    mu, lr = 0.95, 0.02
    W1, M1, O1 = O.muon_step(W, G, M, mu=mu, lr=lr, wd=wd)
    s_new = mu * s_m + (1 - mu) * s_g
    assert np.allclose(M1, (U * s_new) @ V.T, atol=1e-14)
    x = s_new / (np.sqrt(np.sum(s_new ** 2)) + O.NS_EPS)
    orth = (U * _phi_chain(x, [O.NS_DEFAULT_COEF] * 5)) @ V.T
    assert np.allclose(O1, orth, atol=1e-10)
    scale = np.sqrt(m / n)
    assert np.allclose(W1, W * (1 - lr * wd) - lr * scale * orth, atol=1e-10)


# ---------------------------------------------------------------- Muon+

def _brute_row_norm(X, eps):
    out = np.empty_like(X)
    for i in range(X.shape[0]):
        s = 0.0
        for j in range(X.shape[1]):
            s += X[i, j] * X[i, j]
        for j in range(X.shape[1]):
            out[i, j] = X[i, j] / (np.sqrt(s) + eps)
    return out


def _brute_col_norm(X, eps):
    return _brute_row_norm(X.T, eps).T


def test_muon_plus_modes_brute_force():
    rng = np.random.default_rng(7)
    X = rng.standard_normal((4, 6))
    e = O.NORM_EPS
    assert np.allclose(O.muon_plus_norm(X, O.NORM_ROW), _brute_row_norm(X, e), atol=1e-14)
    assert np.allclose(O.muon_plus_norm(X, O.NORM_COL), _brute_col_norm(X, e), atol=1e-14)
    assert np.allclose(O.muon_plus_norm(X, O.NORM_COL_ROW), _brute_row_norm(_brute_col_norm(X, e), e), atol=1e-14)
    assert np.allclose(O.muon_plus_norm(X, O.NORM_ROW_COL), _brute_col_norm(_brute_row_norm(X, e), e), atol=1e-14)
    assert np.array_equal(O.muon_plus_norm(X, O.NORM_NONE), X)
    # the two combined orders differ on a generic matrix
    assert not np.allclose(O.muon_plus_norm(X, O.NORM_COL_ROW), O.muon_plus_norm(X, O.NORM_ROW_COL), atol=1e-6)


def test_muon_plus_identity_on_semi_orthogonal():
    """Rows of U V^T (m <= n) already have unit norm; so do the columns when m >= n."""
    rng = np.random.default_rng(8)
    wide = O.polar_svd(rng.standard_normal((5, 9)))
    tall = O.polar_svd(rng.standard_normal((9, 5)))
    sq = O.polar_svd(rng.standard_normal((6, 6)))
    tol = 1e-6  # the 1e-7 epsilon in the denominator
    assert np.allclose(O.muon_plus_norm(wide, O.NORM_ROW), wide, atol=tol)
    assert np.allclose(O.muon_plus_norm(tall, O.NORM_COL), tall, atol=tol)
    for mode in (O.NORM_COL_ROW, O.NORM_ROW_COL, O.NORM_ROW, O.NORM_COL):
        assert np.allclose(O.muon_plus_norm(sq, mode), sq, atol=tol)


def test_muon_plus_last_direction_is_unit():
    rng = np.random.default_rng(9)
    X = rng.standard_normal((7, 12))
    cr = O.muon_plus_norm(X, O.NORM_COL_ROW)
    rc = O.muon_plus_norm(X, O.NORM_ROW_COL)
    assert np.allclose(np.linalg.norm(cr, axis=1), 1.0, atol=1e-6)
    assert np.allclose(np.linalg.norm(rc, axis=0), 1.0, atol=1e-6)


# ------------------------------------------------------------------ MOP and the logical-matrix split

@pytest.mark.parametrize("shape", [(6, 9), (9, 6), (7, 7)])
def test_mop_exact_polar_from_constructed_svd(shape):
    """MOP ([SMB-summary] "Muon vs SOAP Comparison"): the direction is U V^T of the momentum,
    built from a constructed SVD (no SVD call in the expected value), and the update is
    W - lr sqrt(m/n) U V^T."""
    m, n = shape
    rng = np.random.default_rng(31)
    k = min(m, n)
    U = synth.random_orthogonal(rng, m)[:, :k]
    V = synth.random_orthogonal(rng, n)[:, :k]
    S = rng.uniform(0.01, 5.0, size=k)
    G = (U * S) @ V.T
    W = rng.standard_normal((m, n))
    lr, mu = 0.03, 0.9
    Wn, Mn, Od = O.muon_step(W, G, np.zeros((m, n)), mu=mu, lr=lr, polar="exact")
    assert np.allclose(Od, U @ V.T, atol=1e-12)
    assert np.allclose(Wn, W - lr * np.sqrt(m / n) * (U @ V.T), atol=1e-12)
    assert np.allclose(Mn, (1 - mu) * G, atol=1e-15)


def _block_orthogonal(rng, b, count, scales):
    return [s * synth.random_orthogonal(rng, b) for s in scales[:count]]


def test_split_columns_orthogonalises_each_logical_matrix():
    """A fused [q | k | v] matrix (split (1, 3)) with blocks s_i Q_i, Q_i orthogonal: each block
    alone has every singular value s_i, so MOP gives [Q_1 Q_2 Q_3] and Newton-Schulz gives
    phi^k(s_i / (s_i sqrt(b) + eps)) Q_i per block, each with sqrt(b/b) = 1 as the scale.  The
    unsplit matrix (8 x 24) gives neither."""
    rng = np.random.default_rng(32)
    b = 8
    Qs = [synth.random_orthogonal(rng, b) for _ in range(3)]
    sc = [0.3, 1.7, 4.0]
    M = np.concatenate([s * Q for s, Q in zip(sc, Qs)], axis=1)
    W = np.zeros_like(M)
    _, _, O_mop = O.muon_step(W, M, np.zeros_like(M), mu=0.0, lr=1.0, polar="exact", split=(1, 3))
    assert np.allclose(O_mop, np.concatenate(Qs, axis=1), atol=1e-12)
    coefs = [O.NS_DEFAULT_COEF] * 5
    Wn, _, O_ns = O.muon_step(W, M, np.zeros_like(M), mu=0.0, lr=1.0, split=(1, 3))
    want = np.concatenate([_phi_chain([s / (s * np.sqrt(b) + O.NS_EPS)], coefs)[0] * Q for s, Q in zip(sc, Qs)],
                          axis=1)
    assert np.allclose(O_ns, want, atol=1e-10)
    assert np.allclose(Wn, -want, atol=1e-10)  # lr = 1, sqrt(8/8) = 1
    _, _, O_whole = O.muon_step(W, M, np.zeros_like(M), mu=0.0, lr=1.0, polar="exact")
    assert not np.allclose(O_whole, O_mop, atol=1e-3)


def test_split_rows_uses_block_shape_for_scale_and_norm():
    """Split (2, 1) of a 12 x 6 matrix into two 6 x 6 blocks: the scale is sqrt(6/6) = 1, not
    sqrt(12/6); Muon+ row normalisation of an exact orthogonal block is the identity."""
    rng = np.random.default_rng(33)
    Q1, Q2 = synth.random_orthogonal(rng, 6), synth.random_orthogonal(rng, 6)
    M = np.concatenate([2.0 * Q1, 0.5 * Q2], axis=0)
    W = rng.standard_normal((12, 6))
    lr = 0.1
    Wn, _, Od = O.muon_step(W, M, np.zeros_like(M), mu=0.0, lr=lr, polar="exact", split=(2, 1),
                            norm=O.NORM_ROW)
    want = np.concatenate([Q1, Q2], axis=0)
    assert np.allclose(Od, want, atol=1e-12)
    assert np.allclose(Wn, W - lr * want, atol=1e-12)
    with pytest.raises(ValueError):
        O.muon_step(W, M, np.zeros_like(M), mu=0.0, lr=lr, split=(5, 1))
