"""The allocation-free Muon entry point (mao_muon_step_noalloc) against the
workspace entry point (mao_muon_step), through the C ABI.

mao_muon_step_noalloc serves callers that cannot allocate device memory for the
step's scratch (a fixed device-memory budget, or a framework allocator that owns
all device memory): it takes its scratch from a static device array inside the
library.  Its outputs must match the workspace entry point's within the Muon
step runs the same deterministic kernels on the same inputs, so its outputs
must be bit-identical to the workspace entry point's on two calls in a row (the
second call sees the state the first left, and the shared scratch still holds
the first call's contents); a scratch-overlap slip that moved values by a few
ulps would show.  Its status word, kept inside the static scratch, is read with
mao_muon_noalloc_status, and one of the calls asks for the per-matrix stats.  Collected last so that a failure here stops a -x run only after
every other test has run; it also passes alone in a fresh process.
"""

import ctypes

import numpy as np
import pytest
import torch

from matrix_aware_optimizers_02_b200 import _lib as L
from matrix_aware_optimizers_02_b200 import synth

pytestmark = pytest.mark.gpu



@pytest.fixture(scope="module")
def env():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from matrix_aware_optimizers_02_b200 import api
    return L.load(), api


def _device_copy(inputs, bf16_idx):
    out = []
    for i, (W, G, M) in enumerate(inputs):
        g = torch.from_numpy(G).cuda()
        if i in bf16_idx:
            g = g.to(torch.bfloat16)
        out.append((torch.from_numpy(W).cuda(), g, torch.from_numpy(M).cuda()))
    return out


def test_noalloc_matches_workspace_entry_point_twice(env):
    lib, api = env
    specs = [synth.MatSpec(256, 512, 0.02), synth.MatSpec(384, 128, 0.02), synth.MatSpec(200, 328, 0.02)]
    inputs = synth.muon_inputs(specs, seed=11, m_std=0.02)
    bf16_idx = {1}
    for i in bf16_idx:
        inputs[i] = (inputs[i][0], synth.bf16_round(inputs[i][1]), inputs[i][2])
    ref = _device_copy(inputs, bf16_idx)
    mine = _device_copy(inputs, bf16_idx)
    ref_step = api.MuonBatch(ref, mu=0.95, lr=0.02, norm="col_row", with_stats=True)
    n = len(mine)
    arr = (L.MuonMat * n)(*[L.MuonMat(W.shape[0], W.shape[1], W.data_ptr(), G.data_ptr(),
                                      L.MAO_BF16 if G.dtype == torch.bfloat16 else L.MAO_F32, M.data_ptr())
                            for (W, G, M) in mine])
    params = L.MuonParams(0.95, 0.02, 0.0, 1e-7, 5, None, L.NORM_MODES["col_row"])
    stats = torch.zeros((n, 4), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        ref_step()
        st = lib.mao_muon_step_noalloc(arr, n, ctypes.byref(params), stats.data_ptr() if call == 1 else None,
                                       stream)
        assert st == L.MAO_OK, L.status_string(st)
        where = ctypes.c_int32(-1)
        assert lib.mao_muon_noalloc_status(stream, ctypes.byref(where)) == L.MAO_OK, where.value
        torch.cuda.synchronize()
        for k, ((Wr, _, Mr), (Wm, _, Mm)) in enumerate(zip(ref, mine)):
            assert torch.equal(Wm, Wr), (call, k, (Wm - Wr).abs().max().item())
            assert torch.equal(Mm, Mr), (call, k)
    # the stats of the second call, computed in the static scratch, equal the workspace entry point's
    assert torch.equal(stats.cpu(), ref_step.stats[:n].cpu())
    assert ref_step.stats_dict()["nonfinite"] == [0] * n


def test_noalloc_rejects_batches_beyond_the_scratch(env):
    lib, _ = env
    big = L.MuonMat(4096, 4096, 0x10000, 0x10000, L.MAO_F32, 0x10000)
    arr = (L.MuonMat * 1)(big)
    params = L.MuonParams(0.95, 0.02, 0.0, 1e-7, 5, None, 0)
    need = ctypes.c_size_t(0)
    assert lib.mao_muon_workspace_size(arr, 1, ctypes.byref(params), ctypes.byref(need)) == L.MAO_OK
    assert need.value > (64 << 20)
    assert lib.mao_muon_step_noalloc(arr, 1, ctypes.byref(params), None, None) == L.MAO_ERR_WORKSPACE
