"""Muon / Muon+ through the C ABI against the float64 oracle on the same seeded
inputs.  Tolerance: 2e-2 relative Frobenius error on the orthogonalised
direction O and on the weight update dW (Newton-Schulz runs with bf16 operands,
whose unit roundoff is 2^-8); beside it the largest elementwise error of dW must
stay below ten times that, 0.2 of dW's RMS (the factor the SOAP / FOAM checks
use), so that a few wrong entries cannot hide inside the norm.  The momentum is fp32 arithmetic and must agree to fp32 rounding."""

import numpy as np
import pytest
import torch

from matrix_aware_optimizers_02_b200 import synth
from oracle import mao_oracle as O
from tests import gates

pytestmark = pytest.mark.gpu

NS_TOL = 2e-2
ELEM_TOL = 10 * NS_TOL


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


def _run(api, inputs, g_bf16, **kw):
    """Run one GPU step; return per matrix (W_new, M_new) as float64 numpy."""
    dev = []
    for (W, G, M) in inputs:
        Wt = torch.from_numpy(W).cuda()
        Gt = torch.from_numpy(G).cuda()
        if g_bf16:
            Gt = Gt.to(torch.bfloat16)
        Mt = torch.from_numpy(M).cuda()
        dev.append((Wt, Gt, Mt))
    step = api.MuonBatch(dev, **kw)
    step()
    assert step.device_status() == 0
    torch.cuda.synchronize()
    return [(w.double().cpu().numpy(), m.double().cpu().numpy()) for (w, _, m) in dev], step


def _check(inputs, outs, *, mu, lr, wd=0.0, norm=O.NORM_NONE, ns_steps=5, coefs=None, split=None,
           label="muon"):
    worst = 0.0
    for i, ((W, G, M), (Wg, Mg)) in enumerate(zip(inputs, outs)):
        m, n = W.shape
        sp = split[i] if split is not None else (1, 1)
        Wo, Mo, Oo = O.muon_step(W, G, M, mu=mu, lr=lr, wd=wd, norm=norm, ns_steps=ns_steps, ns_coefs=coefs,
                                 split=sp)
        lab = f"{label} #{i} {m}x{n}"
        # momentum: fp32 fused multiply-add vs float64
        assert np.allclose(Mg, Mo, rtol=1e-5, atol=1e-7 * max(np.abs(Mo).max(), 1e-30))
        dW_gpu = Wg - W
        dW_ref = Wo - W
        e = _rel(dW_gpu, dW_ref)
        gates.check(lab, "muon dW", e, NS_TOL)
        gates.check(lab, "muon dW max/rms", gates.max_over_rms(dW_gpu, dW_ref), ELEM_TOL)
        if wd == 0.0:
            # O = -dW / (lr sqrt(m_b/n_b)), the block shape of a split matrix
            s = lr * np.sqrt((m // sp[0]) / (n // sp[1]))
            eo = _rel(-dW_gpu / s, Oo)
            gates.check(lab, "muon O", eo, NS_TOL)
            e = max(e, eo)
        worst = max(worst, e)
    return worst


def test_muon_single_256x512(api):
    """The single-weight case: W, G, M ~ N(0, 0.02^2), seed 0, mu 0.95, lr 0.02, 5 NS steps."""
    W, G, M = synth.muon_single_inputs(0)
    inputs = [(W.astype(np.float64), G.astype(np.float64), M.astype(np.float64))]
    outs, _ = _run(api, [(W, G, M)], False, mu=0.95, lr=0.02)
    _check(inputs, outs, mu=0.95, lr=0.02)


RAGGED = [synth.MatSpec(200, 328, 0.02), synth.MatSpec(328, 200, 0.02), synth.MatSpec(64, 64, 0.02),
          synth.MatSpec(8, 1000, 0.02), synth.MatSpec(1000, 8, 0.02), synth.MatSpec(264, 264, 0.02),
          synth.MatSpec(520, 136, 0.02)]


@pytest.mark.parametrize("g_bf16", [False, True])
def test_muon_ragged_batch(api, g_bf16):
    """Mixed shapes (several tiles, ragged tails, both orientations) in one call."""
    inputs = synth.muon_inputs(RAGGED, seed=3, g_bf16=g_bf16, m_std=0.02)
    outs, _ = _run(api, inputs, g_bf16, mu=0.9, lr=0.05, wd=0.1)
    _check([tuple(a.astype(np.float64) for a in x) for x in inputs], outs, mu=0.9, lr=0.05, wd=0.1)


@pytest.mark.parametrize("norm", ["row", "col", "col_row", "row_col"])
def test_muon_plus_modes(api, norm):
    specs = [synth.MatSpec(192, 320, 0.02), synth.MatSpec(320, 192, 0.02), synth.MatSpec(128, 128, 0.02)]
    inputs = synth.muon_inputs(specs, seed=4, g_bf16=True)
    outs, _ = _run(api, inputs, True, mu=0.95, lr=0.02, norm=norm)
    mode = {"row": O.NORM_ROW, "col": O.NORM_COL, "col_row": O.NORM_COL_ROW, "row_col": O.NORM_ROW_COL}[norm]
    _check([tuple(a.astype(np.float64) for a in x) for x in inputs], outs, mu=0.95, lr=0.02, norm=mode)


def test_custom_coefficients_and_step_counts(api):
    specs = [synth.MatSpec(96, 160, 0.02)]
    inputs = synth.muon_inputs(specs, seed=5, m_std=0.02)
    f64 = [tuple(a.astype(np.float64) for a in x) for x in inputs]
    coefs = [(3.0, -3.2, 1.2), (2.0, -1.5, 0.5), (1.875, -1.25, 0.375)]
    outs, _ = _run(api, inputs, False, mu=0.95, lr=0.02, ns_steps=3, ns_coef=coefs)
    _check(f64, outs, mu=0.95, lr=0.02, ns_steps=3, coefs=coefs)
    for k in (0, 1, 2):
        outs, _ = _run(api, inputs, False, mu=0.95, lr=0.02, ns_steps=k)
        _check(f64, outs, mu=0.95, lr=0.02, ns_steps=k)


def test_gpt2_124m_batch(api):
    """The GPT-2-124M-shaped Muon+ set (48 matrices, bf16 G ~ N(0, 0.02^2), Col-Row) in one
    call; every matrix compared with the oracle."""
    specs = synth.specs_gpt2_124m()
    inputs = synth.muon_inputs(specs, seed=0, g_bf16=True)
    outs, _ = _run(api, inputs, True, mu=0.95, lr=0.02, norm="col_row")
    _check([tuple(a.astype(np.float64) for a in x) for x in inputs], outs, mu=0.95, lr=0.02, norm=O.NORM_COL_ROW,
           label="gpt2_124m")


def test_deterministic_and_stats(api):
    specs = [synth.MatSpec(256, 768, 0.02), synth.MatSpec(768, 256, 0.02)]
    inputs = synth.muon_inputs(specs, seed=6, g_bf16=True, m_std=0.01)
    o1, s1 = _run(api, inputs, True, mu=0.95, lr=0.02, with_stats=True)
    o2, _ = _run(api, inputs, True, mu=0.95, lr=0.02, with_stats=True)
    for (a, b), (c, d) in zip(o1, o2):
        assert np.array_equal(a, c) and np.array_equal(b, d)
    st = s1.stats_dict()
    for i, (W, G, M) in enumerate(inputs):
        dw = o1[i][0] - W.astype(np.float64)
        rms = np.linalg.norm(dw) / np.sqrt(dw.size)
        assert abs(st["update_rms"][i] - rms) <= 1e-3 * rms
        assert st["nonfinite"][i] == 0


@pytest.mark.parametrize("norm", ["none", "col_row"])
def test_fused_qkv_split(api, norm):
    """Fused projections stepped as their logical matrices ("SOAP, Muon and Beyond" review
    3-2 (2)): a GPT-2 [q | k | v] weight of 768 x 2304 split into three 768 x 768 blocks along
    its columns, a row-stacked 3072 x 768 split into four, and an unsplit matrix in the same
    call; each block has its own pre-normalisation, Newton-Schulz, Muon+ norms and scale."""
    specs = [synth.MatSpec(768, 2304, 0.02), synth.MatSpec(3072, 768, 0.02), synth.MatSpec(256, 384, 0.02)]
    split = [(1, 3), (4, 1), (1, 1)]
    inputs = synth.muon_inputs(specs, seed=9, g_bf16=True, m_std=0.01)
    outs, _ = _run(api, inputs, True, mu=0.95, lr=0.02, norm=norm, split=split)
    mode = {"none": O.NORM_NONE, "col_row": O.NORM_COL_ROW}[norm]
    f64 = [tuple(a.astype(np.float64) for a in x) for x in inputs]
    _check(f64, outs, mu=0.95, lr=0.02, norm=mode, split=split, label=f"qkv split {norm}")
    # the split changes the result: the whole-matrix step is far from the split one
    Wo, _, _ = O.muon_step(*f64[0], mu=0.95, lr=0.02, norm=mode)
    assert _rel(outs[0][0] - f64[0][0], Wo - f64[0][0]) > 10 * NS_TOL


MOP_TOL = 1e-4  # fp32 gate: the polar factor to fp32 accuracy


@pytest.mark.parametrize("norm", ["none", "col_row"])
def test_mop_exact_polar(api, norm):
    """MOP ("SOAP, Muon, and Beyond" summary, "Muon vs SOAP Comparison"): the direction is the
    exact polar factor U V^T of the momentum (oracle: SVD), reached here by the library's
    fixed fp32-faithful Newton-Schulz schedule; one split matrix included."""
    specs = [synth.MatSpec(256, 384, 0.02), synth.MatSpec(384, 256, 0.02), synth.MatSpec(192, 192, 0.02),
             synth.MatSpec(128, 96, 0.02), synth.MatSpec(96, 288, 0.02)]
    split = [(1, 1)] * 4 + [(1, 3)]
    inputs = synth.muon_inputs(specs, seed=10, g_bf16=False, m_std=0.01)
    outs, _ = _run(api, inputs, False, mu=0.95, lr=0.02, norm=norm, split=split, polar="exact")
    mode = {"none": O.NORM_NONE, "col_row": O.NORM_COL_ROW}[norm]
    for i, ((W, G, M), (Wg, Mg)) in enumerate(zip(inputs, outs)):
        W, G, M = (a.astype(np.float64) for a in (W, G, M))
        m, n = W.shape
        sp = split[i]
        Wo, Mo, Oo = O.muon_step(W, G, M, mu=0.95, lr=0.02, norm=mode, split=sp, polar="exact")
        lab = f"mop {norm} #{i} {m}x{n}"
        s = 0.02 * np.sqrt((m // sp[0]) / (n // sp[1]))
        Og = -(Wg - W) / s
        gates.check(lab, "mop O", _rel(Og, Oo), MOP_TOL)
        gates.check(lab, "mop O max/rms", gates.max_over_rms(Og, Oo), 10 * MOP_TOL)
        if norm == "none" and sp == (1, 1):
            k = min(m, n)
            Ow = Og if m <= n else Og.T
            gates.check(lab, "mop orthonormality", np.linalg.norm(Ow @ Ow.T - np.eye(k)) / np.sqrt(k), 1e-5)
