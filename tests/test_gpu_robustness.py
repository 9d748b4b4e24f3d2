"""Failure detection, determinism and resume, through the C ABI.

* Non-finite gradients: a NaN or an Inf placed in one matrix's G on the host.  The
  step propagates it (that matrix's weight becomes non-finite), reports the count
  in mao_stats.nonfinite, records MAO_ERR_NONFINITE in the workspace status word,
  and leaves every other matrix of the batch finite and equal, to fp32 rounding,
  to what a batch without the bad matrix computes (matrices never mix; the launch
  shapes, hence summation orders, may differ between the two batches).  No GPU
  fault is involved: the values are ordinary data.
* Determinism: two identical runs give bit-identical weights, states and stats.
* Resume: a step taken after copying the whole state to the host and back into
  fresh buffers (a checkpoint) is bit-identical to the uninterrupted run.
* Bounded waits: a wait on a barrier phase that nothing completes (a test entry of
  the library, through the same bounded wait every kernel uses) gives up after its
  limit, records MAO_ERR_TIMEOUT in the status word and returns; the context stays
  usable.  No GPU fault, trap or endless loop is involved.
"""

import ctypes

import numpy as np
import pytest
import torch

from matrix_aware_optimizers_02_b200 import _lib as L
from matrix_aware_optimizers_02_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def api():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from matrix_aware_optimizers_02_b200 import api as A
    return A


SHAPES = [(128, 192), (192, 96), (96, 96)]


def _soap_state(m, n, dev="cuda"):
    z = lambda *s: torch.zeros(s, device=dev)  # noqa: E731
    return {"M": z(m, n), "V": z(m, n), "L": torch.eye(m, device=dev) * 1e-6, "R": torch.eye(n, device=dev) * 1e-6,
            "QL": torch.eye(m, device=dev), "QR": torch.eye(n, device=dev),
            "perm_L": torch.zeros(m, dtype=torch.int32, device=dev),
            "perm_R": torch.zeros(n, dtype=torch.int32, device=dev)}


def _foam_state(m, n, dev="cuda"):
    z = lambda *s: torch.zeros(s, device=dev)  # noqa: E731
    return {"M": z(m, n), "r": z(m), "c": z(n), "R": torch.eye(n, device=dev) * 1e-6, "QR": torch.eye(n, device=dev),
            "perm_R": torch.zeros(n, dtype=torch.int32, device=dev)}


def _inputs(seed, shapes=SHAPES):
    rng = np.random.default_rng(seed)
    Ws = [(rng.standard_normal(s) * 0.02).astype(np.float32) for s in shapes]
    Gs = [[(rng.standard_normal(s) * 0.01).astype(np.float32) for s in shapes] for _ in range(3)]
    return Ws, Gs


def _make(api, kind, Ws, shapes, **kw):
    mats = []
    for W, (m, n) in zip(Ws, shapes):
        d = {"W": torch.from_numpy(W.copy()).cuda(), "G": torch.zeros((m, n), device="cuda")}
        d.update(_soap_state(m, n) if kind == "soap" else _foam_state(m, n))
        mats.append(d)
    if kind == "soap":
        return mats, api.SoapBatch(mats, beta1=0.95, beta2=0.95, eps=1e-8, lr=3e-3, with_stats=True, **kw)
    return mats, api.FoamBatch(mats, beta1=0.95, beta2=0.95, eps=1e-8, lr=3e-3, refresh="every_k", k=1,
                               with_stats=True, **kw)


def _run(api, kind, Ws, Gs, shapes=SHAPES, steps=2, **kw):
    mats, b = _make(api, kind, Ws, shapes, **kw)
    for t in range(1, steps + 1):
        for d, G in zip(mats, Gs[t - 1]):
            d["G"].copy_(torch.from_numpy(G))
        b(t)
    torch.cuda.synchronize()
    return mats, b


@pytest.mark.parametrize("kind", ["soap", "foam"])
@pytest.mark.parametrize("bad", [float("nan"), float("inf")])
def test_nonfinite_gradient_is_flagged_and_contained(api, kind, bad):
    Ws, Gs = _inputs(31)
    Gbad = [[g.copy() for g in step] for step in Gs]
    Gbad[0][1][5, 7] = bad  # matrix 1, first step
    mats, b = _run(api, kind, Ws, Gbad, steps=1)
    st = b.stats_dict()
    assert st["nonfinite"][1] > 0, st
    assert st["nonfinite"][0] == 0 and st["nonfinite"][2] == 0, st
    assert not torch.isfinite(mats[1]["W"]).all()
    assert b.device_status() == L.MAO_ERR_NONFINITE
    # the other matrices equal a batch that never held the bad one
    keep = [0, 2]
    ref, rb = _run(api, kind, [Ws[i] for i in keep], [[Gs[0][i] for i in keep]], shapes=[SHAPES[i] for i in keep],
                   steps=1)
    assert rb.device_status() == 0
    for j, i in enumerate(keep):
        assert torch.isfinite(mats[i]["W"]).all()
        assert torch.allclose(mats[i]["W"], ref[j]["W"], rtol=1e-5, atol=1e-8), i


@pytest.mark.parametrize("bad", [float("nan"), float("inf")])
def test_nonfinite_gradient_muon(api, bad):
    specs = [synth.MatSpec(128, 256, 0.02), synth.MatSpec(256, 128, 0.02)]
    inputs = synth.muon_inputs(specs, seed=32, m_std=0.01)
    G1 = inputs[1][1].copy()
    G1[3, 4] = bad
    dev = [(torch.from_numpy(W).cuda(), torch.from_numpy(G if i == 0 else G1).cuda(), torch.from_numpy(M).cuda())
           for i, (W, G, M) in enumerate(inputs)]
    ref = [(torch.from_numpy(inputs[0][0]).cuda(), torch.from_numpy(inputs[0][1]).cuda(),
            torch.from_numpy(inputs[0][2]).cuda())]
    b = api.MuonBatch(dev, mu=0.95, lr=0.02, with_stats=True)
    b()
    st = b.stats_dict()
    assert st["nonfinite"][0] == 0 and st["nonfinite"][1] > 0, st
    assert b.device_status() == L.MAO_ERR_NONFINITE
    rb = api.MuonBatch(ref, mu=0.95, lr=0.02)
    rb()
    torch.cuda.synchronize()
    assert torch.isfinite(dev[0][0]).all()
    assert torch.allclose(dev[0][0], ref[0][0], rtol=1e-5, atol=1e-8)
    # without stats nothing is counted, and the status word stays clear
    b2 = api.MuonBatch(dev, mu=0.95, lr=0.02)
    b2()
    assert b2.device_status() == 0


@pytest.mark.parametrize("kind", ["soap", "foam"])
def test_bitwise_repeat(api, kind):
    Ws, Gs = _inputs(33)
    a, ba = _run(api, kind, Ws, Gs, steps=3)
    b, bb = _run(api, kind, Ws, Gs, steps=3)
    for da, db in zip(a, b):
        for name in da:
            assert torch.equal(da[name], db[name]), name
    assert torch.equal(ba.stats, bb.stats)


@pytest.mark.parametrize("kind", ["soap", "foam"])
def test_resume_from_host_checkpoint(api, kind):
    """Three steps straight, against two steps, a checkpoint of every state tensor to host
    memory, a new batch over fresh device buffers restored from it, and the third step."""
    Ws, Gs = _inputs(34)
    full, _ = _run(api, kind, Ws, Gs, steps=3)
    part, _ = _run(api, kind, Ws, Gs, steps=2)
    ckpt = [{k: v.cpu().clone() for k, v in d.items()} for d in part]
    del part
    torch.cuda.empty_cache()
    mats, b = _make(api, kind, [c["W"].numpy() for c in ckpt], SHAPES)
    for d, c in zip(mats, ckpt):
        for k, v in c.items():
            d[k].copy_(v)
    for d, G in zip(mats, Gs[2]):
        d["G"].copy_(torch.from_numpy(G))
    b(3)
    torch.cuda.synchronize()
    for d, f in zip(mats, full):
        for name in ("W", "M", "R", "QR") + (("V", "L", "QL") if kind == "soap" else ("r", "c")):
            assert torch.equal(d[name], f[name]), name


def test_bounded_wait_gives_up_and_reports(api):
    lib = L.load()
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    addr = ws.data_ptr()
    assert addr % 256 == 0
    stream = torch.cuda.current_stream()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    L.check(lib.mao_test_wait_timeout(addr, ws.numel(), stream.cuda_stream), "wait timeout")
    ev1.record(stream)
    where = ctypes.c_int32(0)
    st = lib.mao_workspace_status(addr, stream.cuda_stream, ctypes.byref(where))
    assert st == L.MAO_ERR_TIMEOUT and where.value == 40, (st, where.value)
    waited_ms = ev0.elapsed_time(ev1)
    assert 900.0 <= waited_ms <= 5000.0, waited_ms  # the 1 s limit, then the kernel returned
    # the context is still usable: a product after the timeout is right
    A = torch.randn(2, 96, 64, device="cuda")
    B = torch.randn(2, 80, 64, device="cuda")
    D = api.gemm(A, B, kind="split3")
    ref = torch.bmm(A.double(), B.double().transpose(1, 2))
    assert (D.double() - ref).abs().max().item() < 1e-4
