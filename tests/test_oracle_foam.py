"""Pins for the oracle's FOAM step: factored moment, trace normalisation, adaptive check."""

import json
import os

import numpy as np
import pytest

from oracle import mao_oracle as O
from matrix_aware_optimizers_02_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_factored_moment_equals_dense_under_kronecker_structure():
    """With (G_s Q_R)^2 = k_s^2 a b^T every step and R_0 = 0, tau r^ c^T equals the
    dense rotated second moment V^ of one-sided SOAP, and the updates agree."""
    rng = np.random.default_rng(30)
    m, n, steps = 5, 4, 5
    Q = synth.random_orthogonal(rng, n)
    Gs, a, b, ks = synth.kronecker_gradients(rng, m, n, Q, steps)
    b1, b2, eps = 0.9, 0.95, 1e-8
    st = O.FoamState.init(m, n)
    st.R = np.zeros((n, n))
    st.QR = Q
    Vd = np.zeros((m, n))
    Md = np.zeros((m, n))
    for t in range(1, steps + 1):
        G = Gs[t - 1]
        res = O.foam_step(np.zeros((m, n)), G, st, t=t, beta1=b1, beta2=b2, eps=eps, lr=1.0,
                          refresh_kind=O.REFRESH_NEVER)
        st = res.state
        # dense one-sided reference, explicit loops over entries
        Gr = G @ Q
        for i in range(m):
            for j in range(n):
                Vd[i, j] = b2 * Vd[i, j] + (1 - b2) * Gr[i, j] ** 2
                Md[i, j] = b1 * Md[i, j] + (1 - b1) * G[i, j]
        bc2 = 1 - b2 ** t
        vfac = res.tau * np.outer(st.r / bc2, st.c / bc2)
        assert np.allclose(vfac, Vd / bc2, rtol=1e-12, atol=0)
        Nd = ((Md @ Q) / (1 - b1 ** t)) / (np.sqrt(Vd / bc2) + eps)
        assert np.allclose(res.U, Nd @ Q.T, rtol=1e-10, atol=1e-12)


def test_rank_one_identity_basis_sign_map():
    """Q_R = I, R_0 = 0, t = 1, G = u v^T: v^ = G^2 exactly, so U = G/(|G| + eps)."""
    rng = np.random.default_rng(31)
    m, n = 6, 4
    G = np.outer(rng.standard_normal(m), rng.standard_normal(n))
    st = O.FoamState.init(m, n)
    st.R = np.zeros((n, n))
    eps = 1e-8
    res = O.foam_step(np.zeros((m, n)), G, st, t=1, beta1=0.9, beta2=0.95, eps=eps, lr=1.0,
                      refresh_kind=O.REFRESH_NEVER)
    assert np.allclose(res.U, G / (np.abs(G) + eps), atol=1e-10)
    # bias-corrected trace ||G||_F^2 over ||r^||_1 ||c^||_1 = ||G||_F^4 / (m n)
    assert np.isclose(res.tau, m * n / np.sum(G * G), rtol=1e-12)


@pytest.mark.parametrize("x,expect", [(0.05, False), (0.2, True)])
def test_adaptive_check_threshold(x, expect):
    """D = [[1, x], [x, 1]] gives rho = |x|/sqrt(1+x^2); refresh iff rho > 0.1."""
    R = np.array([[1.0, x], [x, 1.0]])
    ref, rho = O.refresh_decision(O.REFRESH_ADAPTIVE, t=1, pf=10, tol=0.1, F=R, Q=np.eye(2))
    assert np.isclose(rho, abs(x) / np.sqrt(1 + x * x), rtol=1e-14)
    assert ref is expect


def test_adaptive_check_only_every_pf_steps():
    R = np.array([[1.0, 0.5], [0.5, 1.0]])
    fired = [O.refresh_decision(O.REFRESH_ADAPTIVE, t=t, pf=10, tol=0.1, F=R, Q=np.eye(2))[0]
             for t in range(1, 23)]
    assert [t for t, f in zip(range(1, 23), fired) if f] == [1, 11, 21]


def test_foam_refresh_permutes_c_and_sorts_basis():
    """Q_R = shuffled eigenvectors of R, G = 0: the refresh sorts them by eigenvalue and
    carries c along (c' = b2 c[perm]); r just decays."""
    rng = np.random.default_rng(32)
    m, n = 3, 5
    eig = np.array([1.0, 5.0, 0.2, 3.0, 0.7])
    Vv = synth.random_orthogonal(rng, n)
    st = O.FoamState.init(m, n)
    st.R = (Vv * eig) @ Vv.T
    shuffle = rng.permutation(n)
    st.QR = Vv[:, shuffle]
    st.c = rng.uniform(0.5, 1.5, size=n)
    st.r = rng.uniform(0.5, 1.5, size=m)
    b2 = 0.9
    res = O.foam_step(np.zeros((m, n)), np.zeros((m, n)), st, t=1, beta1=0.9, beta2=b2, eps=1e-8,
                      lr=1.0, refresh_kind=O.REFRESH_EVERY_K, k=1)
    expected = np.argsort(-eig[shuffle], kind="stable")
    assert np.array_equal(res.perm_R, expected)
    assert np.allclose(res.state.c, b2 * st.c[expected], atol=1e-15)
    assert np.allclose(res.state.r, b2 * st.r, atol=1e-15)
    assert np.allclose(np.abs(res.state.QR.T @ Vv[:, shuffle[expected]]), np.eye(n), atol=1e-10)


def test_foam_first_step_fires_on_non_diagonal_R():
    """At t = 1 with Q_R = I the check sees D = R; any G with correlated columns fires it."""
    rng = np.random.default_rng(33)
    m, n = 8, 6
    G = rng.standard_normal((m, n))
    st = O.FoamState.init(m, n)
    res = O.foam_step(np.zeros((m, n)), G, st, t=1, beta1=0.95, beta2=0.95, eps=1e-8, lr=1e-3,
                      refresh_kind=O.REFRESH_ADAPTIVE, pf=10, tol=0.1)
    assert res.refreshed and res.rho > 0.1
    QR = res.state.QR
    assert np.allclose(QR.T @ QR, np.eye(n), atol=1e-12)


def test_state_sizes_reproduce_printed_memory():
    """SOAP 2mn+2m^2+2n^2 and FOAM mn+2n^2+m+n in fp32 over the GPT-2-large shape set
    give the printed 23.73 GiB and 11.87 GiB."""
    with open(os.path.join(GOLDEN, "state_bytes_gpt2_large.json")) as f:
        g = json.load(f)
    d, L, bpe = g["d_model"], g["layers"], g["bytes_per_elem"]
    shapes = [(d, d)] * 4 + [(d, 4 * d), (4 * d, d)]
    soap = sum(O.soap_state_elems(m, n) for m, n in shapes) * L * bpe / 2 ** 30
    foam = sum(O.foam_state_elems(m, n) for m, n in shapes) * L * bpe / 2 ** 30
    assert round(soap, g["printed_digits"]) == g["soap_gib"]
    assert round(foam, g["printed_digits"]) == g["foam_gib"]
    # a plausible slip (counting one factor instead of factor + basis) misses the figure
    assert round(sum(m * n * 2 + m * m + n * n for m, n in shapes) * L * bpe / 2 ** 30, 2) != g["soap_gib"]


def test_weight_decay_is_decoupled():
    rng = np.random.default_rng(42)
    m, n = 6, 5
    W = rng.standard_normal((m, n))
    G = rng.standard_normal((m, n)) * 0.1
    kw = dict(t=1, beta1=0.9, beta2=0.95, eps=1e-8, lr=0.01)
    a = O.foam_step(W, G, O.FoamState.init(m, n), wd=0.0, **kw)
    b = O.foam_step(W, G, O.FoamState.init(m, n), wd=0.3, **kw)
    np.testing.assert_allclose(b.W - a.W, -0.01 * 0.3 * W, rtol=0, atol=1e-15)
    # the decay touches W only: every moment, the factor and the basis are unchanged
    for name in ("M", "r", "c", "R", "QR"):
        np.testing.assert_array_equal(getattr(a.state, name), getattr(b.state, name))


@pytest.mark.parametrize("t", [1, 2, 7])
def test_raw_trace_differs_by_the_bias_correction(t):
    """tau uses the bias-corrected trace tr(R / (1 - b2^t)); the literal tr(R) variant
    gives exactly (1 - b2^t) times it, for any state."""
    rng = np.random.default_rng(43 + t)
    n, m = 4, 6
    A = rng.standard_normal((n, n))
    R = A @ A.T
    r = np.abs(rng.standard_normal(m)) + 0.1
    c = np.abs(rng.standard_normal(n)) + 0.1
    b2 = 0.95
    bc = O.foam_tau(R, r, c, t, b2)
    raw = O.foam_tau(R, r, c, t, b2, raw_trace=True)
    assert np.isclose(raw, bc * (1.0 - b2 ** t), rtol=1e-13)
    # against the definition: tr(R^) / (||r^||_1 ||c^||_1) with every hat 1/(1 - b2^t)
    h = 1.0 / (1.0 - b2 ** t)
    assert np.isclose(bc, (np.trace(R) * h) / (np.sum(r) * h * np.sum(c) * h), rtol=1e-13)


def test_foam_lagged_refresh_sorts_previous_gradient_columns():
    """FOAM with lag=True (refresh before the current gradient enters R), beta2 = 0 and
    diagonal gradients: the t = 2 basis is the permutation that sorts G_1's squared column
    norms in descending order, and c follows that permutation."""
    m, n = 5, 4
    G1 = np.zeros((m, n))
    G2 = np.zeros((m, n))
    for i, (a, b) in enumerate(zip([1.0, 3.0, 2.0, 0.5], [2.0, 0.5, 1.0, 4.0])):
        G1[i, i] = a
        G2[i, i] = b
    kw = dict(beta1=0.9, beta2=0.0, eps=1e-8, lr=1.0, refresh_kind=O.REFRESH_EVERY_K, k=1)
    st = O.FoamState.init(m, n)
    r1 = O.foam_step(np.zeros((m, n)), G1, st, t=1, lag=True, **kw)
    assert np.array_equal(r1.state.QR, np.eye(n))
    r2 = O.foam_step(np.zeros((m, n)), G2, r1.state, t=2, lag=True, **kw)
    assert np.array_equal(r2.perm_R, [1, 2, 0, 3])
    assert np.allclose(r2.state.QR, np.eye(n)[:, [1, 2, 0, 3]], atol=1e-15)
    assert np.allclose(r2.state.R, G2.T @ G2, atol=1e-15)
    fresh = O.foam_step(np.zeros((m, n)), G2, r1.state, t=2, lag=False, **kw)
    assert np.array_equal(fresh.perm_R, [3, 0, 2, 1])
