"""Pins for the oracle's SOAP pieces (factor EMAs, refresh, QR, Adam in the eigenbasis)."""

import numpy as np
import pytest

from oracle import mao_oracle as O
from matrix_aware_optimizers_02_b200 import synth


def _brute_gram_rows(G):
    m, n = G.shape
    out = np.zeros((m, m))
    for i in range(m):
        for j in range(m):
            out[i, j] = sum(G[i, k] * G[j, k] for k in range(n))
    return out


def _brute_rotate(QL, X, QR):
    """QL^T X QR by explicit sums."""
    m, n = X.shape
    out = np.zeros((m, n))
    for a in range(m):
        for b in range(n):
            s = 0.0
            for i in range(m):
                for j in range(n):
                    s += QL[i, a] * X[i, j] * QR[j, b]
            out[a, b] = s
    return out


def test_shampoo_beta0_equals_polar_square():
    """(G G^T)^{-1/4} G (G^T G)^{-1/4} = U V^T for full-rank square G."""
    rng = np.random.default_rng(10)
    G = rng.standard_normal((6, 6))
    assert np.allclose(O.shampoo_update(G, G @ G.T, G.T @ G), O.polar_svd(G), atol=1e-10)


@pytest.mark.parametrize("shape", [(4, 7), (7, 4)])
def test_shampoo_beta0_equals_polar_rectangular(shape):
    """Same identity for rectangular G, with the roots taken on the nonzero spectrum."""
    rng = np.random.default_rng(11)
    G = rng.standard_normal(shape)
    assert np.allclose(O.shampoo_update(G, G @ G.T, G.T @ G), O.polar_svd(G), atol=1e-9)


def test_qr_positive_properties():
    rng = np.random.default_rng(12)
    P = rng.standard_normal((8, 8))
    Q = O.qr_positive(P)
    R = Q.T @ P
    assert np.allclose(Q.T @ Q, np.eye(8), atol=1e-13)
    assert np.allclose(np.tril(R, -1), 0.0, atol=1e-12)
    assert np.all(np.diag(R) > 0)
    assert np.allclose(Q @ R, P, atol=1e-12)


def test_qr_positive_gram_schmidt_brute_force():
    """Classical Gram-Schmidt in explicit loops gives the same positive-diagonal Q."""
    rng = np.random.default_rng(13)
    P = rng.standard_normal((5, 5))
    Q = np.zeros_like(P)
    for j in range(5):
        v = P[:, j].copy()
        for i in range(j):
            v -= (Q[:, i] @ P[:, j]) * Q[:, i]
        Q[:, j] = v / np.sqrt(v @ v)
    assert np.allclose(O.qr_positive(P), Q, atol=1e-12)


def test_refresh_converges_to_sorted_eigenvectors():
    """Repeated power step + QR on a fixed factor is subspace iteration: it reaches
    the eigh eigenvectors, ordered by descending eigenvalue (up to sign)."""
    rng = np.random.default_rng(14)
    n = 6
    eig = np.array([0.3, 5.0, 0.05, 1.4, 12.0, 0.8])
    F = synth.symmetric_with_spectrum(rng, n, eig)
    Q = np.eye(n)
    for _ in range(200):
        Q, _perm = O.refresh_basis(F, Q, sort=True)
    w, Vv = np.linalg.eigh(F)
    order = np.argsort(-w)
    C = np.abs(Q.T @ Vv[:, order])
    assert np.allclose(C, np.eye(n), atol=1e-8)


def test_sort_permutation_recovers_descending_order():
    """With Q = eigenvectors in a shuffled order, the sort permutation is exactly the
    permutation that orders their eigenvalues descending (an integer decision)."""
    rng = np.random.default_rng(15)
    n = 7
    eig = np.array([3.0, 0.5, 9.0, 1.0, 0.1, 4.0, 2.0])
    Vv = synth.random_orthogonal(rng, n)
    F = (Vv * eig) @ Vv.T
    shuffle = rng.permutation(n)
    Qs = Vv[:, shuffle]
    Qn, perm = O.refresh_basis(F, Qs, sort=True)
    expected = np.argsort(-eig[shuffle], kind="stable")
    assert np.array_equal(perm, expected)
    # F Q = Q Lambda, so the QR leaves the sorted eigenvectors (signs made positive)
    assert np.allclose(np.abs(Qn.T @ Vv[:, shuffle[expected]]), np.eye(n), atol=1e-10)


def test_sort_ties_keep_lower_index():
    assert np.array_equal(O.sort_perm([1.0, 2.0, 2.0, 0.5, 2.0]), [1, 2, 4, 0, 3])


def test_factor_ema_brute_force():
    rng = np.random.default_rng(16)
    m, n = 3, 4
    G = rng.standard_normal((m, n))
    st = O.SoapState.init(m, n)
    b2 = 0.9
    res = O.soap_step(np.zeros((m, n)), G, st, t=1, beta1=0.9, beta2=b2, eps=1e-8, lr=0.0,
                      refresh_kind=O.REFRESH_NEVER)
    assert np.allclose(res.state.L, b2 * 1e-6 * np.eye(m) + (1 - b2) * _brute_gram_rows(G), atol=1e-15)
    assert np.allclose(res.state.R, b2 * 1e-6 * np.eye(n) + (1 - b2) * _brute_gram_rows(G.T), atol=1e-15)


def test_identity_basis_is_elementwise_adam():
    """With Q = I and no refresh, SOAP is elementwise Adam (bias-corrected, eps outside sqrt)."""
    rng = np.random.default_rng(17)
    m, n = 3, 4
    b1, b2, eps, lr = 0.9, 0.99, 1e-8, 1e-2
    st = O.SoapState.init(m, n)
    W = rng.standard_normal((m, n))
    Wb = W.copy()
    mb = np.zeros((m, n))
    vb = np.zeros((m, n))
    for t in range(1, 4):
        G = rng.standard_normal((m, n))
        res = O.soap_step(W, G, st, t=t, beta1=b1, beta2=b2, eps=eps, lr=lr, refresh_kind=O.REFRESH_NEVER)
        W, st = res.W, res.state
        for i in range(m):
            for j in range(n):
                mb[i, j] = b1 * mb[i, j] + (1 - b1) * G[i, j]
                vb[i, j] = b2 * vb[i, j] + (1 - b2) * G[i, j] ** 2
                mh = mb[i, j] / (1 - b1 ** t)
                vh = vb[i, j] / (1 - b2 ** t)
                Wb[i, j] = Wb[i, j] - lr * mh / (np.sqrt(vh) + eps)
        assert np.allclose(W, Wb, atol=1e-12)


def test_fixed_basis_first_step_sign_map_and_norm():
    """t = 1, M = V = 0, fixed orthogonal bases: N = Gh/(|Gh|+eps) with Gh = QL^T G QR,
    U = QL N QR^T and ||U||_F = ||N||_F (rotations preserve the Frobenius norm)."""
    rng = np.random.default_rng(18)
    m, n = 4, 5
    QL = synth.random_orthogonal(rng, m)
    QR = synth.random_orthogonal(rng, n)
    st = O.SoapState.init(m, n)
    st.QL, st.QR = QL, QR
    G = rng.standard_normal((m, n))
    eps = 1e-8
    res = O.soap_step(np.zeros((m, n)), G, st, t=1, beta1=0.95, beta2=0.95, eps=eps, lr=1.0,
                      refresh_kind=O.REFRESH_NEVER)
    Gh = _brute_rotate(QL, G, QR)
    N = Gh / (np.abs(Gh) + eps)
    assert np.allclose(res.U, QL @ N @ QR.T, atol=1e-12)
    assert np.isclose(np.linalg.norm(res.U), np.linalg.norm(N), rtol=1e-12)
    assert np.allclose(res.W, -res.U, atol=1e-15)


def test_refresh_uses_current_gradient():
    """The basis refreshed at step t is built from factors that already hold G_t:
    from L = 1e-6 I and a rank-one G = u v^T, the first left basis vector becomes +-u/||u||."""
    rng = np.random.default_rng(19)
    m, n = 6, 5
    u = rng.standard_normal(m)
    v = rng.standard_normal(n)
    G = np.outer(u, v)
    st = O.SoapState.init(m, n)
    res = O.soap_step(np.zeros((m, n)), G, st, t=1, beta1=0.95, beta2=0.95, eps=1e-8, lr=0.0,
                      refresh_kind=O.REFRESH_EVERY_K, k=1, sort=True)
    q0 = res.state.QL[:, 0]
    assert abs(abs(q0 @ u) / np.linalg.norm(u) - 1.0) < 1e-6
    r0 = res.state.QR[:, 0]
    assert abs(abs(r0 @ v) / np.linalg.norm(v) - 1.0) < 1e-6
    assert res.refreshed_L and res.refreshed_R


def test_every_k_schedule_and_v_permutation():
    rng = np.random.default_rng(20)
    m, n = 4, 3
    st = O.SoapState.init(m, n)
    st.V = rng.uniform(0.1, 1.0, size=(m, n))
    st.L = synth.symmetric_with_spectrum(rng, m, [0.1, 4.0, 2.0, 1.0])
    st.QL = np.eye(m)
    G = np.zeros((m, n))
    flags = [O.soap_step(np.zeros((m, n)), G, st, t=t, beta1=0.9, beta2=0.9, eps=1e-8, lr=0.0,
                         refresh_kind=O.REFRESH_EVERY_K, k=3).refreshed_L for t in range(1, 8)]
    assert flags == [True, False, False, True, False, False, True]
    res = O.soap_step(np.zeros((m, n)), G, st, t=1, beta1=0.9, beta2=0.9, eps=1e-8, lr=0.0,
                      refresh_kind=O.REFRESH_EVERY_K, k=1)
    keys = np.diag(0.9 * st.L)
    perm = np.argsort(-keys, kind="stable")
    assert np.array_equal(res.perm_L, perm)
    # G = 0: V' = b2 * V[perm_L][:, perm_R]
    assert np.allclose(res.state.V, 0.9 * st.V[perm][:, res.perm_R], atol=1e-15)


def test_forced_permutation_replays_the_sort():
    """Handing the sort's own permutation back reproduces the step exactly; another
    permutation changes the basis (so a replayed decision is really used)."""
    rng = np.random.default_rng(21)
    m, n = 5, 4
    st = O.SoapState.init(m, n)
    G = rng.standard_normal((m, n))
    a = O.soap_step(np.zeros((m, n)), G, st, t=1, beta1=0.9, beta2=0.9, eps=1e-8, lr=1.0)
    b = O.soap_step(np.zeros((m, n)), G, st, t=1, beta1=0.9, beta2=0.9, eps=1e-8, lr=1.0,
                    force_perm_L=a.perm_L, force_perm_R=a.perm_R)
    assert np.array_equal(a.W, b.W) and np.array_equal(a.state.QL, b.state.QL)
    c = O.soap_step(np.zeros((m, n)), G, st, t=1, beta1=0.9, beta2=0.9, eps=1e-8, lr=1.0,
                    force_perm_L=a.perm_L[::-1].copy(), force_perm_R=a.perm_R)
    assert not np.allclose(c.state.QL, a.state.QL)


def test_weight_decay_is_decoupled():
    """The recipe's weight decay acts on W alone: the steps with and without it differ
    by exactly -lr wd W, whatever the gradient (a decay folded into the gradient or the
    moments would change the Adam part too)."""
    rng = np.random.default_rng(41)
    m, n = 6, 5
    W = rng.standard_normal((m, n))
    G = rng.standard_normal((m, n)) * 0.1
    kw = dict(t=1, beta1=0.9, beta2=0.95, eps=1e-8, lr=0.01)
    a = O.soap_step(W, G, O.SoapState.init(m, n), wd=0.0, **kw)
    b = O.soap_step(W, G, O.SoapState.init(m, n), wd=0.3, **kw)
    np.testing.assert_allclose(b.W - a.W, -0.01 * 0.3 * W, rtol=0, atol=1e-15)
    np.testing.assert_array_equal(a.state.M, b.state.M)
    np.testing.assert_array_equal(a.state.V, b.state.V)


# ------------------------------------------------------------------ lagged refresh (stale basis)

def _diag_grad(d, m, n):
    G = np.zeros((m, n))
    for i, v in enumerate(d):
        G[i, i] = v
    return G


def test_lagged_refresh_sees_the_previous_gradient_only():
    """lag=True: the refresh runs on the factors before the current gradient enters them
    ([SMB-summary] "SOAP Instability Diagnosis": the current gradient is left out of the
    recalculation).  With beta2 = 0 and diagonal gradients the factors are diagonal, so the
    refreshed basis is a permutation matrix in closed form:
      t = 1: the old factors are 1e-6 I (all keys equal), so the basis stays I and the step is
             elementwise Adam, U = G/(|G|+eps);
      t = 2: the basis sorts the diagonal of G_1 G_1^T (not of G_2 G_2^T) in descending order.
    Without lag, t = 2 sorts G_2's diagonal instead."""
    m, n = 4, 5
    G1 = _diag_grad([1.0, 3.0, 2.0, 0.5], m, n)
    G2 = _diag_grad([2.0, 0.5, 1.0, 4.0], m, n)
    kw = dict(beta1=0.9, beta2=0.0, eps=1e-8, lr=1.0)
    st = O.SoapState.init(m, n)
    r1 = O.soap_step(np.zeros((m, n)), G1, st, t=1, lag=True, **kw)
    assert np.array_equal(r1.state.QL, np.eye(m)) and np.array_equal(r1.state.QR, np.eye(n))
    assert np.allclose(r1.U, G1 / (np.abs(G1) + 1e-8), atol=1e-15)
    r2 = O.soap_step(np.zeros((m, n)), G2, r1.state, t=2, lag=True, **kw)
    order1 = [1, 2, 0, 3]  # G1's squared diagonal, descending
    assert np.array_equal(r2.perm_L, order1)
    assert np.allclose(r2.state.QL, np.eye(m)[:, order1], atol=1e-15)
    # the factors still take in the current gradient, after the refresh
    assert np.allclose(r2.state.L, G2 @ G2.T, atol=1e-15)
    fresh = O.soap_step(np.zeros((m, n)), G2, r1.state, t=2, lag=False, **kw)
    assert np.array_equal(fresh.perm_L, [3, 0, 2, 1])
