"""The launch profiler's executed-work counters (mao_launch_info.exec_*).

The table-mode kernels count the work of every tile they compute in device
counters, so launches whose problems run or not on a device decision (the QR's
second projections and Cholesky-QR passes) report what actually ran; every other
launch reports its host-side count.
"""

import numpy as np
import pytest
import torch

from matrix_aware_optimizers_02_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def api():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from matrix_aware_optimizers_02_b200 import api as A
    return A


def _state(m, n, rng):
    f = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()
    G = synth.bf16_round((rng.standard_normal((m, n)) * 1e-2).astype(np.float32)).astype(np.float32)
    return {"W": f(rng.standard_normal((m, n)) * 0.02), "G": f(G).to(torch.bfloat16), "M": f(np.zeros((m, n))),
            "V": f(np.zeros((m, n))), "L": f(1e-6 * np.eye(m)), "R": f(1e-6 * np.eye(n)), "QL": f(np.eye(m)),
            "QR": f(np.eye(n))}


def test_profiler_counts_executed_work(api):
    from matrix_aware_optimizers_02_b200 import _lib as L
    lib = L.load()
    m, n = 1024, 768
    rng = np.random.default_rng(33)
    st = _state(m, n, rng)
    soap = api.SoapBatch([st], beta1=0.95, beta2=0.95, eps=1e-8, lr=3e-3, refresh="every_k", k=1)
    soap(1)
    st["G"].copy_(torch.from_numpy((rng.standard_normal((m, n)) * 1e-2).astype(np.float32)).to(torch.bfloat16))
    torch.cuda.synchronize()
    cap = 8192
    info = (L.LaunchInfo * cap)()
    L.check(lib.mao_profile_start(None, info, cap), "profile start")
    soap(2)
    cnt = lib.mao_profile_stop()
    torch.cuda.synchronize()
    assert 0 < cnt <= cap
    rows = [info[i] for i in range(cnt)]
    by = lambda name: [r for r in rows if L.KERNEL_NAMES.get(r.kernel) == name]
    # ungated products: the device's tile count equals the host's (bf16 x bf16: one product)
    fac = by("pc_factor")
    assert len(fac) == 2
    for r in fac:
        assert r.exec_flops == r.flops > 0 and r.exec_tc_flops == r.tc_flops == r.flops
    for r in by("pc_power") + by("pc_rotate") + by("pc_update"):
        assert r.exec_flops == r.flops and r.exec_tc_flops == r.tc_flops
    # QR projections: the passes decided on the device add to the host's count
    qr = by("pc_qr")
    assert qr and sum(r.exec_flops for r in qr) >= sum(r.flops for r in qr) > 0
    for r in qr:
        assert r.exec_tc_flops == 6.0 * r.exec_flops
        if r.flops > 0:
            assert r.exec_flops == r.flops
    # launches outside table mode report the host's count
    for r in by("pc_elementwise") + by("pc_sort") + by("pc_chol"):
        assert r.exec_flops == r.flops and r.exec_tc_flops == r.tc_flops
