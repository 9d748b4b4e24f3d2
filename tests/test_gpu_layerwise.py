"""The layer-wise distributed step on a GPU: a one-rank NCCL group drives the whole
path (gradient reduce to the owner, the owned batch, the side-stream all-gather-V
with its event wait) and must reproduce the plain batch bit for bit.  More ranks
than one need more GPUs than a test box has; the multi-rank logic is covered by
the two-rank gloo tests on CPU."""

import datetime
import os
import tempfile

import numpy as np
import pytest
import torch

from matrix_aware_optimizers_02_b200 import layerwise as LW
from matrix_aware_optimizers_02_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def api():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from matrix_aware_optimizers_02_b200 import api as A
    return A


@pytest.fixture(scope="module")
def nccl_group():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import torch.distributed as dist
    d = tempfile.mkdtemp()
    store = dist.FileStore(os.path.join(d, "store"), 1)
    dist.init_process_group("nccl", store=store, rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    yield dist
    dist.destroy_process_group()


SPECS = [synth.MatSpec(256, 512, 0.02), synth.MatSpec(512, 256, 0.02), synth.MatSpec(384, 384, 0.02)]


def _muon_mats(seed):
    inputs = synth.muon_inputs(SPECS, seed=seed, g_bf16=True, m_std=0.01)
    return [(torch.from_numpy(W).cuda(), torch.from_numpy(G).cuda().to(torch.bfloat16), torch.from_numpy(M).cuda())
            for (W, G, M) in inputs]


def test_layerwise_muon_one_rank_matches_batch(api, nccl_group):
    a, b = _muon_mats(60), _muon_mats(60)
    plain = api.MuonBatch(a, mu=0.95, lr=0.02, norm="col_row")
    lw = LW.LayerwiseStep(b, "muon", nccl_group, mu=0.95, lr=0.02, norm="col_row")
    assert lw.owners == [0, 0, 0]
    for _ in range(2):
        plain()
        lw()
    torch.cuda.synchronize()
    for (Wa, _, Ma), (Wb, _, Mb) in zip(a, b):
        assert torch.equal(Wa, Wb) and torch.equal(Ma, Mb)


def test_layerwise_soap_one_rank_matches_batch(api, nccl_group):
    rng = np.random.default_rng(61)
    shapes = [(128, 192), (192, 96)]

    def mats():
        out = []
        r = np.random.default_rng(62)
        for (m, n) in shapes:
            out.append({"W": torch.from_numpy((r.standard_normal((m, n)) * 0.02).astype(np.float32)).cuda(),
                        "G": torch.zeros((m, n), device="cuda"), "M": torch.zeros((m, n), device="cuda"),
                        "V": torch.zeros((m, n), device="cuda"), "L": torch.eye(m, device="cuda") * 1e-6,
                        "R": torch.eye(n, device="cuda") * 1e-6, "QL": torch.eye(m, device="cuda"),
                        "QR": torch.eye(n, device="cuda")})
        return out
    a, b = mats(), mats()
    plain = api.SoapBatch(a, beta1=0.95, beta2=0.95, eps=1e-8, lr=3e-3)
    lw = LW.LayerwiseStep(b, "soap", nccl_group, beta1=0.95, beta2=0.95, eps=1e-8, lr=3e-3)
    for t in (1, 2):
        for da, db, (m, n) in zip(a, b, shapes):
            g = torch.from_numpy((rng.standard_normal((m, n)) * 0.01).astype(np.float32)).cuda()
            da["G"].copy_(g)
            db["G"].copy_(g)
        plain(t)
        lw(t)
    torch.cuda.synchronize()
    for da, db in zip(a, b):
        for name in ("W", "M", "V", "L", "R", "QL", "QR"):
            assert torch.equal(da[name], db[name]), name
