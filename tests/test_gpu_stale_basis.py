"""The stale eigenbasis ("SOAP, Muon, and Beyond" summary, "SOAP Instability
Diagnosis"; "SOAP, Muon and Beyond" review 2-1 (3)): refreshing the basis only
every 10 steps, from factors that have not yet taken in the current gradient,
leaves the preconditioner pointing at old directions.

Gradients are a seeded low-rank spike whose singular subspaces turn by a fixed
angle every step, plus noise (synth.drifting_spike_gradients).  Twenty steps of
SOAP and of FOAM run through the C ABI with the real-time order (refresh every
step, current gradient first) and with the standard implementation's order
(every 10 steps, lagged), each against the float64 oracle running freely on the
same gradients (gates as in test_gpu_soap_foam).  The device's bases then show
the mechanism: the real-time left basis keeps its leading columns on the current
spike, the lagged one falls behind between refreshes.
"""

import numpy as np
import pytest
import torch

from matrix_aware_optimizers_02_b200 import synth
from tests import test_gpu_soap_foam as P

pytestmark = pytest.mark.gpu

STEPS = 20
RANK = 4
SHAPES = [(64, 96), (96, 64)]


@pytest.fixture(scope="module")
def api():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from matrix_aware_optimizers_02_b200 import api as A
    return A


def _drifting(seed):
    per = [synth.drifting_spike_gradients(np.random.default_rng(seed + i), m, n, STEPS, rank=RANK, omega=0.08)
           for i, (m, n) in enumerate(SHAPES)]
    return (lambda t: [g[0][t - 1] for g in per]), [g[1] for g in per]


def _alignment(Q, U):
    """Mean squared cosine between the basis's leading RANK columns and the spike's span."""
    return float(np.sum((U.T @ Q[:, :RANK]) ** 2) / RANK)


def test_soap_drifting_free_running(api):
    align = {}
    for k, lag in ((1, False), (10, True)):
        grads, dirs = _drifting(40)
        trace = []

        def probe(t, dev):
            U, _ = dirs[0](t)
            trace.append(_alignment(dev[0]["QL"].double().cpu().numpy(), U))

        P._soap_case(api, SHAPES, steps=STEPS, seed=40, grads=grads, k=k, lag=lag, replay=False, probe=probe,
                     label=f"drift soap k={k} lag={int(lag)}")
        align[(k, lag)] = np.array(trace)
    fresh, stale = align[(1, False)], align[(10, True)]
    # the factors are EMAs (beta2 = 0.95) and one power step refreshes the basis, so even the
    # real-time basis trails a turning spike; the lagged one trails it further at every step
    assert np.all(fresh > stale), (fresh, stale)
    assert fresh.mean() - stale.mean() > 0.3, (fresh.mean(), stale.mean())
    # t = 1: the lagged refresh sees only the initial 1e-6 I (the basis stays I); t = 11: it
    # sees ten gradients and jumps back toward the spike, then decays while the spike turns
    assert stale[9] < 0.2 < 0.6 < stale[10], stale
    assert np.all(np.diff(stale[10:]) < 0), stale


@pytest.mark.parametrize("k,lag", [(1, False), (10, True)])
def test_foam_drifting_free_running(api, k, lag):
    grads, _ = _drifting(41)
    P._foam_case(api, SHAPES, steps=STEPS, seed=41, refresh="every_k", k=k, lag=lag, replay=False, grads=grads,
                 label=f"drift foam k={k} lag={int(lag)}")
