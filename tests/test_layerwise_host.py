"""Layer-wise distributed step, host side on CPU: the owner assignment, the cost
model, and the reduce-to-owner + all-gather-V exchange over two gloo ranks, with a
stand-in for the per-rank GPU step."""

import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

from matrix_aware_optimizers_02_b200 import layerwise as LW

SHAPES = ([(4096, 4096), (4096, 1024), (4096, 1024), (4096, 4096), (4096, 14336), (4096, 14336), (14336, 4096)]
          + [(2048, 768), (2048, 768), (768, 2048)] * 8)


@pytest.mark.parametrize("opt", ["muon", "soap", "foam"])
@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_assignment_covers_balances_and_repeats(opt, world):
    owners = LW.assign_owners(SHAPES, world, opt)
    assert len(owners) == len(SHAPES) and all(0 <= o < world for o in owners)
    assert owners == LW.assign_owners(SHAPES, world, opt)  # every rank computes the same owners
    c = [LW.step_cost(opt, m, n) for (m, n) in SHAPES]
    load = [sum(ci for ci, o in zip(c, owners) if o == r) for r in range(world)]
    # greedy longest-first: no rank exceeds the average by more than one matrix's cost
    assert max(load) <= sum(c) / world + max(c) + 1e-12
    if world <= len(SHAPES):
        assert min(load) > 0


def test_cost_model_follows_shape_not_size():
    # same element count, different cost: Newton-Schulz work depends on min(m, n)
    assert LW.step_flops("muon", 4096, 1024) == LW.step_flops("muon", 1024, 4096)
    assert LW.step_flops("muon", 2048, 2048) > LW.step_flops("muon", 4096, 1024)
    # SOAP carries both factors, FOAM only the input side
    assert LW.state_bytes("soap", 4096, 1024) > LW.state_bytes("foam", 4096, 1024)
    assert LW.state_bytes("foam", 4096, 1024) < LW.state_bytes("foam", 1024, 4096)


def test_cost_model_follows_the_batch_settings():
    # Newton-Schulz work is linear in the step count
    assert LW.step_flops("muon", 768, 2304, ns_steps=16) == pytest.approx(16 / 5 * LW.step_flops("muon", 768, 2304))
    # a refresh every k steps is paid once per k steps: the refresh part shrinks by k
    full = LW.step_flops("soap", 2048, 768, refresh_period=1)
    plain = LW.step_flops("soap", 2048, 768, refresh_period=1 << 40)
    assert LW.step_flops("soap", 2048, 768, refresh_period=10) == pytest.approx(plain + (full - plain) / 10)
    # the QR term is the built block Gram-Schmidt: 2 k^3 + 4 k^2 b with 128-column panels
    assert LW.qr_flops(4096) == 2 * 4096 ** 3 + 4 * 4096 ** 2 * 128
    c = LW.cost_for("soap", {"refresh": "every_k", "k": 10})
    assert c("soap", 4096, 1024) == LW.step_cost("soap", 4096, 1024, 5, 10)
    c = LW.cost_for("muon", {"ns_steps": 16})
    assert c("muon", 4096, 1024) == LW.step_cost("muon", 4096, 1024, 16, 1)
    assert LW.cost_for("foam", {})("foam", 1536, 4608) == LW.step_cost("foam", 1536, 4608, 5, 10)


def test_lpt_matches_brute_force_optimum_bound():
    # four jobs on two ranks: longest-first reaches the optimum here
    cost = {(4, 1): 7.0, (3, 1): 5.0, (2, 1): 4.0, (1, 1): 4.0}

    def c(opt, m, n):
        return cost[(m, n)]
    owners = LW.assign_owners([(4, 1), (3, 1), (2, 1), (1, 1)], 2, "muon", cost=c)
    loads = [sum(cost[s] for s, o in zip([(4, 1), (3, 1), (2, 1), (1, 1)], owners) if o == r) for r in range(2)]
    assert sorted(loads) == [9.0, 11.0]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        shapes = [(8, 16), (16, 8), (24, 16), (8, 8), (32, 16)]
        # every rank holds the same weights and its own local gradient: G_i = i + 10 rank
        mats = [{"W": torch.full(s, float(i), dtype=torch.float32),
                 "G": torch.full(s, float(i) + 10.0 * rank, dtype=torch.float32)} for i, s in enumerate(shapes)]
        stepped = []

        def make_batch(owned):
            def step(t):
                for d in owned:  # stand-in for the GPU step: W <- W - t * G (G reduced to its owner)
                    d["W"].sub_(t * d["G"])
                stepped.extend(id(d) for d in owned)
            return step

        lw = LW.LayerwiseStep(mats, "soap", dist, make_batch=make_batch)
        lw(2)
        q.put((rank, lw.owners, [d["W"].tolist() for d in mats], len(stepped)))
    finally:
        dist.destroy_process_group()


def test_two_ranks_step_owned_and_gather_all():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    owners0, owners1 = out[0][1], out[1][1]
    assert owners0 == owners1 and set(owners0) == {0, 1}
    shapes = [(8, 16), (16, 8), (24, 16), (8, 8), (32, 16)]
    for rank, owners, Ws, nstep in out:
        assert nstep == sum(1 for o in owners if o == rank)  # each rank stepped only what it owns
        for i, (W, o) in enumerate(zip(Ws, owners)):
            # the owner stepped with the mean gradient over the two ranks, i + 5, and every
            # rank received its update
            expect = float(i) - 2 * (float(i) + 5.0)
            t = torch.tensor(W)
            assert tuple(t.shape) == shapes[i]
            assert torch.all(t == expect), (rank, i, o)
