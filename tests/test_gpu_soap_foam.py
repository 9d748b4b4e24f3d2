"""SOAP and FOAM through the C ABI against the float64 oracle on the same seeded
inputs.

Tolerances (relative Frobenius error unless stated):
  * states L, R, M, V, r, c and the bases Q: 1e-4 (fp32-faithful split-bf16 products);
  * the weight update: max(1e-4, 2x the oracle's own float32-mode floor on the
    same input).  SOAP's Adam in the eigenbasis is a near-sign map Gh/(|Gh|+eps)
    while V is small, which amplifies any fp32-level error in the basis; the
    float32 run of the same oracle measures that inherent floor;
  * basis permutations: identical wherever the oracle's consecutive sorted keys
    differ by more than 1e-5 relative; refresh decisions identical when
    |rho - tol| > 1e-5, and rho^2 within 1e-5 absolute (the device derives it from
    the power product and the sort keys, exact for an orthogonal basis).
Gradients use the configs' scales (N(0, 1e-3^2) .. N(0, 1e-2^2)), so the 1e-6 I
ridge keeps the factors well conditioned.  Where two sort keys are closer than
fp32 can resolve, the oracle replays the GPU's ordering (the decision is checked
at the well-separated positions; the states then follow that ordering).
"""

import numpy as np
import pytest
import torch

from matrix_aware_optimizers_02_b200 import synth
from oracle import mao_oracle as O

pytestmark = pytest.mark.gpu

STATE_TOL = 1e-4


@pytest.fixture(scope="module")
def api():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from matrix_aware_optimizers_02_b200 import api as A
    return A


def _rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def _t(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()


def _np(x):
    return x.double().cpu().numpy()


def _basis_rel(Qg, Qo):
    """Relative error of a basis, ignoring nothing (sign convention is fixed by the QR)."""
    return _rel(Qg, Qo)


def _perm_check(perm_gpu, perm_or, keys_sorted):
    """Positions whose neighbouring sorted keys are well separated must agree exactly."""
    k = len(perm_or)
    rel_gap = np.abs(np.diff(keys_sorted)) / np.maximum(np.abs(keys_sorted[:-1]), 1e-300)
    safe = np.ones(k, dtype=bool)
    close = np.where(rel_gap <= 1e-5)[0]
    safe[close] = False
    safe[close + 1] = False
    assert np.array_equal(perm_gpu[safe], perm_or[safe]), (perm_gpu[safe][:10], perm_or[safe][:10])
    return int((~safe).sum())


def _unsafe_positions(keys_sorted):
    rel_gap = np.abs(np.diff(keys_sorted)) / np.maximum(np.abs(keys_sorted[:-1]), 1e-300)
    close = np.where(rel_gap <= 1e-5)[0]
    return set(close.tolist()) | set((close + 1).tolist())


def _soap_oracle(W, G, st, t, eps, lr, refresh, k, sort, perm_gpu_L, perm_gpu_R, dtype=np.float64):
    """Oracle step; near-tie orderings replayed from the GPU after checking the rest."""
    kind = {"every_k": O.REFRESH_EVERY_K, "never": O.REFRESH_NEVER}[refresh]
    kw = dict(t=t, beta1=0.95, beta2=0.95, eps=eps, lr=lr, refresh_kind=kind, k=k, sort=sort)
    res = O.soap_step(W, G, st, **kw)
    fl = fr = None
    if res.refreshed_L and sort:
        keys = np.sort(O.rayleigh_keys(res.state.L, st.QL))[::-1]
        _perm_check(perm_gpu_L, res.perm_L, keys)
        if not np.array_equal(perm_gpu_L, res.perm_L):
            fl = perm_gpu_L
    if res.refreshed_R and sort:
        keys = np.sort(O.rayleigh_keys(res.state.R, st.QR))[::-1]
        _perm_check(perm_gpu_R, res.perm_R, keys)
        if not np.array_equal(perm_gpu_R, res.perm_R):
            fr = perm_gpu_R
    if fl is not None or fr is not None:
        res = O.soap_step(W, G, st, force_perm_L=fl, force_perm_R=fr, **kw)
    if dtype != np.float64:
        # the fp32 run keeps the fp64 run's orderings, so its error measures rounding, not ties
        pl = res.perm_L if res.refreshed_L and sort else None
        pr = res.perm_R if res.refreshed_R and sort else None
        res = O.soap_step(W, G, st, dtype=dtype, force_perm_L=pl, force_perm_R=pr, **kw)
    return res


def _grad(rng, shape, scale, g_bf16):
    """Seeded gradient; a bf16 gradient is bf16-rounded so both sides see the same values."""
    G = (rng.standard_normal(shape) * scale).astype(np.float32)
    return synth.bf16_round(G).astype(np.float32) if g_bf16 else G


def _gdev(G, g_bf16):
    return _t(G).to(torch.bfloat16) if g_bf16 else _t(G)


def _soap_case(api, shapes, steps, seed, eps=1e-8, g_scale=1e-3, lr=3e-3, refresh="every_k", k=1, sort=True,
               g_bf16=False, kernel="auto"):
    api.set_table_kernel(kernel)
    try:
        _soap_run(api, shapes, steps, seed, eps, g_scale, lr, refresh, k, sort, g_bf16)
    finally:
        api.set_table_kernel("auto")


def _soap_run(api, shapes, steps, seed, eps, g_scale, lr, refresh, k, sort, g_bf16):
    rng = np.random.default_rng(seed)
    b1 = b2 = 0.95
    dev, ora, Ws = [], [], []
    for (m, n) in shapes:
        W = (rng.standard_normal((m, n)) * 0.02).astype(np.float32)
        st = O.SoapState.init(m, n)
        d = {"W": _t(W), "G": _gdev(np.zeros((m, n), np.float32), g_bf16), "M": _t(st.M), "V": _t(st.V),
             "L": _t(st.L), "R": _t(st.R),
             "QL": _t(st.QL), "QR": _t(st.QR),
             "perm_L": torch.zeros(m, dtype=torch.int32, device="cuda"),
             "perm_R": torch.zeros(n, dtype=torch.int32, device="cuda")}
        dev.append(d)
        ora.append(st)
        Ws.append(W.astype(np.float64))
    batch = api.SoapBatch(dev, beta1=b1, beta2=b2, eps=eps, lr=lr, refresh=refresh, k=k, sort=sort)
    for t in range(1, steps + 1):
        Gs = [_grad(rng, s, g_scale, g_bf16) for s in shapes]
        for d, G in zip(dev, Gs):
            d["G"].copy_(_gdev(G, g_bf16))
        batch(t)
        assert batch.device_status() == 0
        torch.cuda.synchronize()
        for i, (m, n) in enumerate(shapes):
            d = dev[i]
            pl, pr = d["perm_L"].cpu().numpy(), d["perm_R"].cpu().numpy()
            res = _soap_oracle(Ws[i], Gs[i].astype(np.float64), ora[i], t, eps, lr, refresh, k, sort, pl, pr)
            for name in ("M", "L", "R", "V"):
                e = _rel(_np(d[name]), getattr(res.state, name))
                assert e < STATE_TOL, (t, i, name, e)
            r32 = _soap_oracle(Ws[i], Gs[i], ora[i], t, eps, lr, refresh, k, sort, pl, pr, dtype=np.float32)
            for name in ("QL", "QR"):
                # a basis is as well conditioned as its factor: where fp32 rounding alone moves it
                # by more than the state tolerance (a 4096-row factor of rank 256), the gate is
                # twice what an fp32 evaluation of the same steps reaches
                ref_q = getattr(res.state, name)
                e = _basis_rel(_np(d[name]), ref_q)
                gate = max(STATE_TOL, 2 * _basis_rel(getattr(r32.state, name).astype(np.float64), ref_q))
                assert e < gate, (t, i, name, e, gate)
            dW = _np(d["W"]) - Ws[i]
            ref = res.W - Ws[i]
            e = _rel(dW, ref)
            gate = max(STATE_TOL, 2 * _rel(r32.W.astype(np.float64) - Ws[i], ref))
            assert e < gate, (t, i, "dW", e, gate)
            # next step starts from the GPU's own state (replay), so decisions are checked per step
            ora[i] = O.SoapState(_np(d["M"]), _np(d["V"]), _np(d["L"]), _np(d["R"]), _np(d["QL"]), _np(d["QR"]))
            Ws[i] = _np(d["W"])


def test_soap_square_multistep(api):
    _soap_case(api, [(128, 128), (192, 192), (64, 64)], steps=3, seed=1)


def test_soap_ragged_shapes(api):
    """Rectangular shapes (one factor of each pair is rank deficient before the ridge)."""
    _soap_case(api, [(200, 136), (136, 200), (260, 260)], steps=2, seed=2, g_scale=1e-2)


def test_soap_no_sort_and_refresh_schedule(api):
    _soap_case(api, [(96, 96)], steps=3, seed=3, sort=False)
    _soap_case(api, [(96, 96)], steps=4, seed=4, refresh="every_k", k=2)
    _soap_case(api, [(96, 96)], steps=2, seed=5, refresh="never")


def test_soap_single_1024_spiked(api):
    """The single-weight SOAP case: 1024x1024, G ~ N(0, 1e-3^2) + rank-16 spike, L = R = 1e-6 I,
    b1 = b2 = 0.95, eps = 1e-8, QR power-iteration refresh every step, t = 1."""
    W, Gs = synth.soap_single_inputs(0, steps=1)
    m = n = 1024
    st = O.SoapState.init(m, n)
    d = {"W": _t(W), "G": _t(Gs[0]), "M": _t(st.M), "V": _t(st.V), "L": _t(st.L), "R": _t(st.R), "QL": _t(st.QL),
         "QR": _t(st.QR), "perm_L": torch.zeros(m, dtype=torch.int32, device="cuda"),
         "perm_R": torch.zeros(n, dtype=torch.int32, device="cuda")}
    batch = api.SoapBatch([d], beta1=0.95, beta2=0.95, eps=1e-8, lr=3e-3)
    batch(1)
    assert batch.device_status() == 0
    torch.cuda.synchronize()
    pl, pr = d["perm_L"].cpu().numpy(), d["perm_R"].cpu().numpy()
    res = _soap_oracle(W.astype(np.float64), Gs[0].astype(np.float64), st, 1, 1e-8, 3e-3, "every_k", 1, True, pl, pr)
    for name in ("M", "L", "R", "V", "QL", "QR"):
        e = _rel(_np(d[name]), getattr(res.state, name))
        assert e < STATE_TOL, (name, e)
    r32 = _soap_oracle(W, Gs[0], st, 1, 1e-8, 3e-3, "every_k", 1, True, pl, pr, dtype=np.float32)
    ref = res.W - W
    gate = max(STATE_TOL, 2 * _rel(r32.W.astype(np.float64) - W, ref))
    e = _rel(_np(d["W"]) - W, ref)
    assert e < gate, (e, gate)


# ------------------------------------------------------------------ FOAM

def _foam_case(api, shapes, steps, seed, refresh="adaptive", pf=10, tol=0.1, eps=1e-8, lr=3e-3, k=1,
               raw_trace=False, g_bf16=False, kernel="auto"):
    api.set_table_kernel(kernel)
    try:
        _foam_run(api, shapes, steps, seed, refresh, pf, tol, eps, lr, k, raw_trace, g_bf16)
    finally:
        api.set_table_kernel("auto")


def _foam_run(api, shapes, steps, seed, refresh, pf, tol, eps, lr, k, raw_trace, g_bf16):
    rng = np.random.default_rng(seed)
    b1 = b2 = 0.95
    dev, ora, Ws = [], [], []
    for (m, n) in shapes:
        W = (rng.standard_normal((m, n)) * 0.02).astype(np.float32)
        st = O.FoamState.init(m, n)
        dev.append({"W": _t(W), "G": _gdev(np.zeros((m, n), np.float32), g_bf16), "M": _t(st.M), "r": _t(st.r),
                    "c": _t(st.c),
                    "R": _t(st.R), "QR": _t(st.QR), "perm_R": torch.zeros(n, dtype=torch.int32, device="cuda")})
        ora.append(st)
        Ws.append(W.astype(np.float64))
    kind = {"adaptive": O.REFRESH_ADAPTIVE, "every_k": O.REFRESH_EVERY_K, "never": O.REFRESH_NEVER}[refresh]
    batch = api.FoamBatch(dev, beta1=b1, beta2=b2, eps=eps, lr=lr, refresh=refresh, pf=pf, tol=tol, k=k,
                          tau_raw_trace=raw_trace, with_stats=True)
    for t in range(1, steps + 1):
        Gs = [_grad(rng, s, 0.01, g_bf16) for s in shapes]
        for d, G in zip(dev, Gs):
            d["G"].copy_(_gdev(G, g_bf16))
        batch(t)
        assert batch.device_status() == 0
        torch.cuda.synchronize()
        stats = batch.stats_dict()
        for i, (m, n) in enumerate(shapes):
            d = dev[i]
            kw = dict(t=t, beta1=b1, beta2=b2, eps=eps, lr=lr, refresh_kind=kind, pf=pf, tol=tol, k=k,
                      raw_trace=raw_trace)
            res = O.foam_step(Ws[i], Gs[i].astype(np.float64), ora[i], **kw)
            pg = d["perm_R"].cpu().numpy()
            if res.refreshed and not np.array_equal(pg, res.perm_R):
                keys = np.sort(O.rayleigh_keys(res.state.R, ora[i].QR))[::-1]
                _perm_check(pg, res.perm_R, keys)
                res = O.foam_step(Ws[i], Gs[i].astype(np.float64), ora[i], force_perm=pg, **kw)
            if res.rho >= 0 and abs(res.rho - tol) > 1e-5:
                assert bool(stats["refreshed"][i] & 1) == res.refreshed, (t, i, res.rho)
                # the device forms rho^2 = 1 - sum diag(D)^2 / ||F Q||_F^2, exact for an
                # orthogonal Q: its absolute error is bounded by the fp32 basis's
                # ||Q^T Q - I||, about 1e-6 at these sizes
                assert abs(stats["offdiag_ratio"][i] ** 2 - res.rho ** 2) < 1e-5, (t, i, res.rho)
            for name in ("M", "R", "QR", "r", "c"):
                e = _rel(_np(d[name]), getattr(res.state, name))
                assert e < STATE_TOL, (t, i, name, e)
            e = _rel(_np(d["W"]) - Ws[i], res.W - Ws[i])
            assert e < STATE_TOL, (t, i, "dW", e)
            ora[i] = O.FoamState(_np(d["M"]), _np(d["r"]), _np(d["c"]), _np(d["R"]), _np(d["QR"]))
            Ws[i] = _np(d["W"])


def test_foam_tall_adaptive_multistep(api):
    """Tall shapes (full-rank input factor), adaptive check every 2 steps."""
    _foam_case(api, [(256, 128), (320, 192), (192, 192)], steps=4, seed=11, pf=2)


def test_foam_every_step_and_raw_trace(api):
    _foam_case(api, [(200, 136)], steps=2, seed=12, refresh="every_k", raw_trace=True)
    _foam_case(api, [(128, 64)], steps=2, seed=13, refresh="never")


def test_foam_kronecker_structure_matches_dense(api):
    """Gradients with rank-one rotated square (fixed Q_R, R_0 = 0): the factored
    second moment equals the dense one, so U equals the dense one-sided update."""
    rng = np.random.default_rng(14)
    m, n, steps = 96, 64, 3
    Q = synth.random_orthogonal(rng, n)
    Gs, a, b, ks = synth.kronecker_gradients(rng, m, n, Q, steps)
    st = O.FoamState.init(m, n)
    st.R = np.zeros((n, n))
    st.QR = Q
    W = np.zeros((m, n), np.float32)
    d = {"W": _t(W), "G": _t(np.zeros((m, n))), "M": _t(st.M), "r": _t(st.r), "c": _t(st.c), "R": _t(st.R),
         "QR": _t(Q)}
    batch = api.FoamBatch([d], beta1=0.9, beta2=0.95, eps=1e-8, lr=1.0, refresh="never")
    Vd = np.zeros((m, n))
    Md = np.zeros((m, n))
    Wd = np.zeros((m, n))
    for t in range(1, steps + 1):
        G = Gs[t - 1].astype(np.float32).astype(np.float64)
        d["G"].copy_(_t(G))
        batch(t)
        torch.cuda.synchronize()
        Gr = G @ Q
        Vd = 0.95 * Vd + 0.05 * Gr ** 2
        Md = 0.9 * Md + 0.1 * G
        Nd = ((Md @ Q) / (1 - 0.9 ** t)) / (np.sqrt(Vd / (1 - 0.95 ** t)) + 1e-8)
        Wd = Wd - Nd @ Q.T
        assert _rel(_np(d["W"]), Wd) < 1e-4, t


@pytest.mark.parametrize("kernel", ["one_cta", "cta_pair"])
def test_soap_bf16_gradients_each_kernel(api, kernel):
    """bf16 gradients (one exact plane: G G^T one product, Q_L^T G three) on each table
    kernel for every product that has a three-plane operand."""
    _soap_case(api, [(256, 384), (384, 256), (264, 136)], steps=2, seed=21, g_scale=1e-2, g_bf16=True,
               kernel=kernel)


def test_soap_fp32_gradients_cta_pair(api):
    _soap_case(api, [(200, 136), (136, 200), (260, 260)], steps=2, seed=22, g_scale=1e-2, kernel="cta_pair")


@pytest.mark.parametrize("kernel", ["one_cta", "cta_pair"])
def test_foam_bf16_gradients_each_kernel(api, kernel):
    _foam_case(api, [(384, 256), (256, 128), (200, 136)], steps=3, seed=23, pf=2, g_bf16=True, kernel=kernel)


def test_soap_large_factor_split_coefficients(api):
    """A 4096-row factor: the panel projections split their coefficient products over K
    (deterministic reduction) and the panel Grams over more slices; the QR sweeps 32 panels."""
    _soap_case(api, [(4096, 256)], steps=1, seed=24, g_scale=1e-2, g_bf16=True)
