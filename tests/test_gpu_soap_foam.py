"""SOAP and FOAM through the C ABI against the float64 oracle on the same seeded
inputs.

Gates (relative Frobenius error unless stated; every comparison also checks the
largest elementwise error in units of the reference's RMS, and every (error,
gate) pair is recorded in tests/gates.py):
  * states L, R, M, V, r, c: 1e-4 (fp32-faithful split-bf16 products);
  * the bases Q: 1e-4 where the factor has full rank.  Where it does not yet (a
    factor of k rows that has seen fewer than k gradient columns), the directions
    of its null space carry only the 1e-6 I ridge and are rounding noise in any
    fp32 arithmetic: the gate is then twice what an fp32 evaluation of the same
    steps by the oracle reaches, or 1e-4 if that is larger;
  * the weight update (SOAP and FOAM): max(1e-4, 2x the oracle's own float32-mode
    error on the same input), at every step.  Adam in the eigenbasis divides Mh by
    sqrt(V): wherever the rotated gradient has been small on every step so far, both
    are small and the ratio amplifies rounding; the float32 run of the oracle
    measures that inherent floor (SOAP: 2.5e-4 on a full-rank 192 x 192 weight at
    t = 2; FOAM: 4.5e-3 on a 1536 x 4608 weight at t = 1, whose 4608-column factor
    has rank 1536, so c is rounding noise in the null-space columns);
  * elementwise: max |err| / RMS(ref) below ten times the Frobenius gate, or below
    twice the oracle's float32-mode value where that is larger (the same
    amplification acts on single coordinates, of the update and of V);
  * basis permutations: identical wherever the oracle's consecutive sorted keys
    differ by more than 1e-5 relative; refresh decisions identical when
    |rho - tol| > 1e-5, and rho^2 within 1e-5 absolute (the device derives it from
    the power product and the sort keys, exact for an orthogonal basis).
Where two sort keys are closer than fp32 can resolve, the oracle replays the GPU's
ordering (the decision is checked at the well-separated positions; the states
then follow that ordering).  Multi-step runs come in two forms: replayed (each
step starts the oracle from the GPU's state, so decisions are checked per step)
and free-running (the oracle keeps its own float64 trajectory).
"""

import numpy as np
import pytest
import torch

from matrix_aware_optimizers_02_b200 import synth
from oracle import mao_oracle as O
from tests import gates

pytestmark = pytest.mark.gpu

STATE_TOL = 1e-4
ELEM_FACTOR = 10.0


@pytest.fixture(scope="module")
def api():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from matrix_aware_optimizers_02_b200 import api as A
    return A


def _t(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()


def _np(x):
    return x.double().cpu().numpy()


def _compare(label, name, got, ref, gate, ref32=None):
    """Frobenius and elementwise checks of one quantity.  With `ref32` (the oracle's
    float32 evaluation of the same steps) the elementwise gate is at least twice what
    that evaluation reaches."""
    gates.check(label, name, gates.rel(got, ref), gate)
    egate = ELEM_FACTOR * gate
    if ref32 is not None:
        egate = max(egate, 2.0 * gates.max_over_rms(ref32, ref))
    gates.check(label, name + " max/rms", gates.max_over_rms(got, ref), egate)


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


KINDS = {"every_k": O.REFRESH_EVERY_K, "adaptive": O.REFRESH_ADAPTIVE, "never": O.REFRESH_NEVER}


def _soap_oracle(W, G, st, kw, perm_gpu_L, perm_gpu_R, dtype=np.float64, force=None):
    """Oracle step; near-tie orderings replayed from the GPU after checking the rest.
    `force` = (perm_L, perm_R) skips the checks and uses those orderings."""
    if force is not None:
        return O.soap_step(W, G, st, dtype=dtype, force_perm_L=force[0], force_perm_R=force[1], **kw)
    res = O.soap_step(W, G, st, **kw)
    sort = kw["sort"]
    fl = fr = None
    # the keys come from the factors the refresh used: before this step's gradient under lag
    src_L = st.L if kw.get("lag") else res.state.L
    src_R = st.R if kw.get("lag") else res.state.R
    if res.refreshed_L and sort:
        keys = np.sort(O.rayleigh_keys(src_L, st.QL))[::-1]
        _perm_check(perm_gpu_L, res.perm_L, keys)
        if not np.array_equal(perm_gpu_L, res.perm_L):
            fl = perm_gpu_L
    if res.refreshed_R and sort:
        keys = np.sort(O.rayleigh_keys(src_R, st.QR))[::-1]
        _perm_check(perm_gpu_R, res.perm_R, keys)
        if not np.array_equal(perm_gpu_R, res.perm_R):
            fr = perm_gpu_R
    if fl is not None or fr is not None:
        res = O.soap_step(W, G, st, force_perm_L=fl, force_perm_R=fr, **kw)
    return res


def _grad(rng, shape, scale, g_bf16):
    """Seeded gradient; a bf16 gradient is bf16-rounded so both sides see the same values."""
    G = (rng.standard_normal(shape) * scale).astype(np.float32)
    return synth.bf16_round(G).astype(np.float32) if g_bf16 else G


def _gdev(G, g_bf16):
    return _t(G).to(torch.bfloat16) if g_bf16 else _t(G)


def _soap_case(api, shapes, steps, seed, eps=1e-8, g_scale=1e-3, lr=3e-3, refresh="every_k", k=1, sort=True,
               g_bf16=False, kernel="auto", wd=0.0, replay=True, pf=10, tol=0.1, lag=False, grads=None,
               label=None, probe=None):
    """`grads(t)` (optional) gives the step's gradients; `probe(t, dev)` (optional) sees the
    device tensors after each step."""
    api.set_table_kernel(kernel)
    try:
        _soap_run(api, shapes, steps, seed, eps, g_scale, lr, refresh, k, sort, g_bf16, wd, replay, pf, tol, lag,
                  grads, label or f"soap{shapes}s{seed}", probe)
    finally:
        api.set_table_kernel("auto")


def _soap_run(api, shapes, steps, seed, eps, g_scale, lr, refresh, k, sort, g_bf16, wd, replay, pf, tol, lag,
              grads, label, probe=None):
    rng = np.random.default_rng(seed)
    b1 = b2 = 0.95
    dev, ora, ora32, Ws, Ws32 = [], [], [], [], []
    # per matrix and side: gradients the factor had taken in when its basis was last
    # refreshed (None: never refreshed, the basis is still the exact identity)
    seen_at = [{"QL": None, "QR": None} for _ in shapes]
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
        ora32.append(st.copy(np.float32))
        Ws.append(W.astype(np.float64))
        Ws32.append(W.copy())
    batch = api.SoapBatch(dev, beta1=b1, beta2=b2, eps=eps, lr=lr, wd=wd, refresh=refresh, k=k, sort=sort, pf=pf,
                          tol=tol, lag=lag, with_stats=True)
    kw = dict(beta1=b1, beta2=b2, eps=eps, lr=lr, wd=wd, refresh_kind=KINDS[refresh], k=k, pf=pf, tol=tol,
              sort=sort, lag=lag)
    gpu_prev = [w.copy() for w in Ws]
    for t in range(1, steps + 1):
        Gs = grads(t) if grads is not None else [_grad(rng, s, g_scale, g_bf16) for s in shapes]
        for d, G in zip(dev, Gs):
            d["G"].copy_(_gdev(G, g_bf16))
        batch(t)
        assert batch.device_status() == 0
        torch.cuda.synchronize()
        if probe is not None:
            probe(t, dev)
        stats = batch.stats_dict()
        for i, (m, n) in enumerate(shapes):
            d = dev[i]
            lab = f"{label} t={t} #{i} {m}x{n}"
            pl, pr = d["perm_L"].cpu().numpy(), d["perm_R"].cpu().numpy()
            G64 = Gs[i].astype(np.float64)
            w_gpu_prev = gpu_prev[i]
            res = _soap_oracle(Ws[i], G64, ora[i], dict(kw, t=t), pl, pr)
            # the float32 evaluation of the same step keeps the float64 run's orderings
            force = (res.perm_L if res.refreshed_L and sort else None, res.perm_R if res.refreshed_R and sort else None)
            src32 = (ora[i].copy(np.float32), Ws[i].astype(np.float32)) if replay else (ora32[i], Ws32[i])
            r32 = _soap_oracle(src32[1], Gs[i], src32[0], dict(kw, t=t), None, None, np.float32, force)
            if refresh == "adaptive" and (t - 1) % pf == 0:
                for side, bit, rho, ref in (("L", 2, res.rho_L, res.refreshed_L), ("R", 1, res.rho_R, res.refreshed_R)):
                    if abs(rho - tol) > 1e-5:
                        assert bool(stats["refreshed"][i] & bit) == ref, (lab, side, rho)
                assert abs(stats["offdiag_ratio"][i] ** 2 - res.rho_R ** 2) < 1e-5, (lab, res.rho_R)
            for name in ("M", "L", "R", "V"):
                _compare(lab, "soap " + name, _np(d[name]), getattr(res.state, name), STATE_TOL,
                         getattr(r32.state, name).astype(np.float64))
            for name, rows, cols, refreshed in (("QL", m, n, res.refreshed_L), ("QR", n, m, res.refreshed_R)):
                if refreshed:
                    seen_at[i][name] = t - 1 if lag else t
                # a factor of `rows` rows has full rank once it has taken in `rows` gradient
                # columns (each m x n gradient brings n to the left factor, m to the right)
                full = seen_at[i][name] is None or seen_at[i][name] * cols >= rows
                ref_q = getattr(res.state, name)
                q32 = getattr(r32.state, name).astype(np.float64)
                gate = STATE_TOL if full else max(STATE_TOL, 2 * gates.rel(q32, ref_q))
                _compare(lab, "soap " + name + (" (full rank)" if full else " (rank-deficient)"), _np(d[name]),
                         ref_q, gate, q32)
            dW = _np(d["W"]) - w_gpu_prev
            ref = res.W - Ws[i]
            ref32 = r32.W.astype(np.float64) - (src32[1].astype(np.float64))
            gate = max(STATE_TOL, 2 * gates.rel(ref32, ref))
            _compare(lab, "soap dW", dW, ref, gate, ref32)
            rms_ref = float(np.linalg.norm(ref) / np.sqrt(m * n))
            gates.check(lab, "soap update_rms", abs(stats["update_rms"][i] - rms_ref) / rms_ref, gate)
            assert stats["nonfinite"][i] == 0
            gpu_prev[i] = _np(d["W"])
            if replay:
                # next step starts from the GPU's own state, so decisions are checked per step
                ora[i] = O.SoapState(_np(d["M"]), _np(d["V"]), _np(d["L"]), _np(d["R"]), _np(d["QL"]),
                                     _np(d["QR"]))
                Ws[i] = _np(d["W"])
            else:
                ora[i], Ws[i] = res.state, res.W
                ora32[i], Ws32[i] = r32.state, r32.W


def test_soap_square_multistep(api):
    _soap_case(api, [(128, 128), (192, 192), (64, 64)], steps=3, seed=1)


def test_soap_ragged_shapes(api):
    """Rectangular shapes (one factor of each pair is rank deficient before the ridge)."""
    _soap_case(api, [(200, 136), (136, 200), (260, 260)], steps=2, seed=2, g_scale=1e-2)


def test_soap_no_sort_and_refresh_schedule(api):
    _soap_case(api, [(96, 96)], steps=3, seed=3, sort=False)
    _soap_case(api, [(96, 96)], steps=4, seed=4, refresh="every_k", k=2)
    _soap_case(api, [(96, 96)], steps=2, seed=5, refresh="never")


def test_soap_adaptive_refresh(api):
    """SOAP with the adaptive check (pf = 2): the decision of each side is checked against
    the oracle's rho where |rho - tol| > 1e-5."""
    _soap_case(api, [(128, 96), (96, 160)], steps=5, seed=6, refresh="adaptive", pf=2, tol=0.1, g_scale=1e-2)


def test_soap_weight_decay(api):
    """Decoupled weight decay (wd = 0.1): the update product's epilogue scales W by 1 - lr wd."""
    _soap_case(api, [(128, 192), (192, 128)], steps=2, seed=7, wd=0.1, lr=1e-2, g_scale=1e-2)


def test_soap_lagged_refresh(api):
    """The standard implementation's order (refresh before the current gradient enters the
    factors), every 2 steps, against the oracle's lag=True."""
    _soap_case(api, [(96, 128), (128, 96)], steps=4, seed=8, k=2, lag=True, g_scale=1e-2)


@pytest.mark.parametrize("replay", [True, False])
def test_soap_single_1024_spiked_five_steps(api, replay):
    """The single-weight SOAP case: 1024x1024, G ~ N(0, 1e-3^2) + rank-16 spike, L = R = 1e-6 I,
    b1 = b2 = 0.95, eps = 1e-8, QR power-iteration refresh every step; steps 1-5 with a fresh
    gradient from seeds 1-4 after the first, replayed and free-running."""
    W0, Gs = synth.soap_single_inputs(0, steps=5)
    _soap_single(api, W0, lambda t: [Gs[t - 1]], 5, replay)


def _soap_single(api, W0, grads, steps, replay):
    m, n = W0.shape
    st = O.SoapState.init(m, n)
    d = {"W": _t(W0), "G": _t(np.zeros((m, n))), "M": _t(st.M), "V": _t(st.V), "L": _t(st.L), "R": _t(st.R),
         "QL": _t(st.QL), "QR": _t(st.QR), "perm_L": torch.zeros(m, dtype=torch.int32, device="cuda"),
         "perm_R": torch.zeros(n, dtype=torch.int32, device="cuda")}
    batch = api.SoapBatch([d], beta1=0.95, beta2=0.95, eps=1e-8, lr=3e-3, with_stats=True)
    kw = dict(beta1=0.95, beta2=0.95, eps=1e-8, lr=3e-3, refresh_kind=O.REFRESH_EVERY_K, k=1, sort=True)
    ora, W = st, W0.astype(np.float64)
    ora32, W32 = st.copy(np.float32), W0.copy()
    w_gpu = W0.astype(np.float64)
    for t in range(1, steps + 1):
        G = grads(t)[0]
        d["G"].copy_(_t(G))
        batch(t)
        assert batch.device_status() == 0
        torch.cuda.synchronize()
        lab = f"soap1024 {'replay' if replay else 'free'} t={t}"
        pl, pr = d["perm_L"].cpu().numpy(), d["perm_R"].cpu().numpy()
        res = _soap_oracle(W, G.astype(np.float64), ora, dict(kw, t=t), pl, pr)
        src = (ora.copy(np.float32), W.astype(np.float32)) if replay else (ora32, W32)
        r32 = _soap_oracle(src[1], G, src[0], dict(kw, t=t), None, None, np.float32, (res.perm_L, res.perm_R))
        for name in ("M", "L", "R", "V", "QL", "QR"):
            _compare(lab, "soap1024 " + name, _np(d[name]), getattr(res.state, name), STATE_TOL)
        ref = res.W - W
        ref32 = r32.W.astype(np.float64) - src[1].astype(np.float64)
        gate = max(STATE_TOL, 2 * gates.rel(ref32, ref))
        _compare(lab, "soap1024 dW", _np(d["W"]) - w_gpu, ref, gate, ref32)
        w_gpu = _np(d["W"])
        if replay:
            ora = O.SoapState(_np(d["M"]), _np(d["V"]), _np(d["L"]), _np(d["R"]), _np(d["QL"]), _np(d["QR"]))
            W = _np(d["W"])
        else:
            ora, W = res.state, res.W
            ora32, W32 = r32.state, r32.W


# ------------------------------------------------------------------ FOAM

def _foam_case(api, shapes, steps, seed, refresh="adaptive", pf=10, tol=0.1, eps=1e-8, lr=3e-3, k=1,
               raw_trace=False, g_bf16=False, kernel="auto", wd=0.0, replay=True, lag=False, g_scale=0.01,
               label=None, grads=None):
    api.set_table_kernel(kernel)
    try:
        _foam_run(api, shapes, steps, seed, refresh, pf, tol, eps, lr, k, raw_trace, g_bf16, wd, replay, lag,
                  g_scale, label or f"foam{shapes}s{seed}", grads)
    finally:
        api.set_table_kernel("auto")


def _foam_run(api, shapes, steps, seed, refresh, pf, tol, eps, lr, k, raw_trace, g_bf16, wd, replay, lag, g_scale,
              label, grads=None):
    rng = np.random.default_rng(seed)
    b1 = b2 = 0.95
    dev, ora, ora32, Ws, Ws32 = [], [], [], [], []
    for (m, n) in shapes:
        W = (rng.standard_normal((m, n)) * 0.02).astype(np.float32)
        st = O.FoamState.init(m, n)
        ora32.append(st.copy(np.float32))
        Ws32.append(W.copy())
        dev.append({"W": _t(W), "G": _gdev(np.zeros((m, n), np.float32), g_bf16), "M": _t(st.M), "r": _t(st.r),
                    "c": _t(st.c),
                    "R": _t(st.R), "QR": _t(st.QR), "perm_R": torch.zeros(n, dtype=torch.int32, device="cuda")})
        ora.append(st)
        Ws.append(W.astype(np.float64))
    batch = api.FoamBatch(dev, beta1=b1, beta2=b2, eps=eps, lr=lr, wd=wd, refresh=refresh, pf=pf, tol=tol, k=k,
                          lag=lag, tau_raw_trace=raw_trace, with_stats=True)
    seen_at = [None] * len(shapes)  # gradients R had taken in at its last refresh
    gpu_prev = [w.copy() for w in Ws]
    for t in range(1, steps + 1):
        Gs = grads(t) if grads is not None else [_grad(rng, s, g_scale, g_bf16) for s in shapes]
        for d, G in zip(dev, Gs):
            d["G"].copy_(_gdev(G, g_bf16))
        batch(t)
        assert batch.device_status() == 0
        torch.cuda.synchronize()
        stats = batch.stats_dict()
        for i, (m, n) in enumerate(shapes):
            d = dev[i]
            lab = f"{label} t={t} #{i} {m}x{n}"
            kw = dict(t=t, beta1=b1, beta2=b2, eps=eps, lr=lr, wd=wd, refresh_kind=KINDS[refresh], pf=pf, tol=tol,
                      k=k, raw_trace=raw_trace, lag=lag)
            res = O.foam_step(Ws[i], Gs[i].astype(np.float64), ora[i], **kw)
            pg = d["perm_R"].cpu().numpy()
            if res.refreshed and not np.array_equal(pg, res.perm_R):
                src = ora[i].R if lag else res.state.R
                keys = np.sort(O.rayleigh_keys(src, ora[i].QR))[::-1]
                _perm_check(pg, res.perm_R, keys)
                res = O.foam_step(Ws[i], Gs[i].astype(np.float64), ora[i], force_perm=pg, **kw)
            if res.rho >= 0 and abs(res.rho - tol) > 1e-5:
                assert bool(stats["refreshed"][i] & 1) == res.refreshed, (lab, res.rho)
                # the device forms rho^2 = 1 - sum diag(D)^2 / ||F Q||_F^2, exact for an
                # orthogonal Q: its absolute error is bounded by the fp32 basis's
                # ||Q^T Q - I||, about 1e-6 at these sizes
                assert abs(stats["offdiag_ratio"][i] ** 2 - res.rho ** 2) < 1e-5, (lab, res.rho)
            # the float32 evaluation of the same step (same ordering as the float64 one)
            src32 = (ora[i].copy(np.float32), Ws[i].astype(np.float32)) if replay else (ora32[i], Ws32[i])
            r32 = O.foam_step(src32[1], Gs[i], src32[0], dtype=np.float32,
                              force_perm=res.perm_R if res.refreshed else None, **kw)
            for name in ("M", "R", "r", "c"):
                _compare(lab, "foam " + name, _np(d[name]), getattr(res.state, name), STATE_TOL,
                         getattr(r32.state, name).astype(np.float64))
            if res.refreshed:
                seen_at[i] = t - 1 if lag else t
            full = seen_at[i] is None or seen_at[i] * m >= n
            q32 = r32.state.QR.astype(np.float64)
            gate = STATE_TOL if full else max(STATE_TOL, 2 * gates.rel(q32, res.state.QR))
            _compare(lab, "foam QR" + (" (full rank)" if full else " (rank-deficient)"), _np(d["QR"]),
                     res.state.QR, gate, q32)
            ref = res.W - Ws[i]
            ref32 = r32.W.astype(np.float64) - src32[1].astype(np.float64)
            gate = max(STATE_TOL, 2 * gates.rel(ref32, ref))
            _compare(lab, "foam dW", _np(d["W"]) - gpu_prev[i], ref, gate, ref32)
            gpu_prev[i] = _np(d["W"])
            rms_ref = float(np.linalg.norm(ref) / np.sqrt(m * n))
            gates.check(lab, "foam update_rms", abs(stats["update_rms"][i] - rms_ref) / rms_ref, gate)
            assert stats["nonfinite"][i] == 0
            if replay:
                ora[i] = O.FoamState(_np(d["M"]), _np(d["r"]), _np(d["c"]), _np(d["R"]), _np(d["QR"]))
                Ws[i] = _np(d["W"])
            else:
                ora[i], Ws[i] = res.state, res.W
                ora32[i], Ws32[i] = r32.state, r32.W


def test_foam_tall_adaptive_multistep(api):
    """Tall shapes (full-rank input factor), adaptive check every 2 steps."""
    _foam_case(api, [(256, 128), (320, 192), (192, 192)], steps=4, seed=11, pf=2)


def test_foam_free_running(api):
    """The same as above without replaying the device state: the oracle keeps its own
    float64 trajectory for five steps."""
    _foam_case(api, [(256, 128), (192, 192)], steps=5, seed=15, pf=2, replay=False)


def test_foam_every_step_and_raw_trace(api):
    _foam_case(api, [(200, 136)], steps=2, seed=12, refresh="every_k", raw_trace=True)
    _foam_case(api, [(128, 64)], steps=2, seed=13, refresh="never")


def test_foam_weight_decay_and_lag(api):
    _foam_case(api, [(192, 128), (128, 96)], steps=3, seed=16, refresh="every_k", wd=0.1, lr=1e-2)
    _foam_case(api, [(192, 128), (128, 96)], steps=4, seed=17, refresh="every_k", k=2, lag=True)


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
        _compare(f"kron t={t}", "foam kronecker W", _np(d["W"]), Wd, STATE_TOL)


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
