"""Layer-wise distributed optimizer step over data-parallel ranks.

"SOAP, Muon and Beyond" (the Korean review: §2-1 Main contribution, item 4, the
layer-wise distributed optimizer; §3-2 Module breakdown, item 7, layer-wise
optimizer ownership) keeps every weight matrix whole: each matrix is owned by one
data-parallel rank, which holds its full optimizer state and runs the matrix
optimizer on it, and the updated weights reach every rank through an all-gather
before the next forward pass.  The owners are balanced by optimizer cost (the
Newton-Schulz work and the factor sizes depend on the shape), memory and compute
together, not by parameter count.

Here: `assign_owners` is that assignment (longest-processing-time-first over a cost
model of the step's tensor-core and HBM time), `allgather_v` is the exchange (one
broadcast per owner of its packed updated weights, every rank issuing the same
collectives in the same order), and `LayerwiseStep` runs the owned matrices through
the single-GPU library (`api.MuonBatch`, `api.SoapBatch`, `api.FoamBatch`) and then
the exchange.  The collectives are torch.distributed's (NCCL over NVLink on GPUs).
"""

from __future__ import annotations

from typing import Callable, List, Optional, Sequence, Tuple

from . import _lib as L

# Roofline denominators of the cost model (measured on B200: sustained bf16 tensor
# rate and HBM copy bandwidth).  Only their ratio matters for the assignment.
_TC_FLOPS = 1.38e15
_HBM_BYTES = 6.5e12
# tensor-core products per fp32-faithful multiply-add (three bf16 planes each side)
_SPLIT3_PRODUCTS = 6


def step_flops(opt: str, m: int, n: int) -> float:
    """Multiply-add work of one step of an m x n matrix, in FLOP (2 per multiply-add).

    muon: 5 Newton-Schulz iterations on the wide orientation, 4 s^2 l + 2 s^3 each.
    soap: factors 2m^2n + 2mn^2, power step 2(m^3 + n^3), QR about 2(2 + 1/3)k^3 per
          factor, rotations in 4(m^2n + mn^2), rotation back 2(m^2n + mn^2).
    foam: factor 2mn^2, rotations in 4mn^2, rotation back 2mn^2 (plain step)."""
    if opt == "muon":
        s, l = min(m, n), max(m, n)
        return 5.0 * (4.0 * s * s * l + 2.0 * s ** 3)
    if opt == "soap":
        k3 = float(m) ** 3 + float(n) ** 3
        mn = float(m) * m * n + float(m) * n * n
        return 2.0 * mn + 2.0 * k3 + 2.0 * (2.0 + 1.0 / 3.0) * k3 + 6.0 * mn
    if opt == "foam":
        return 8.0 * m * float(n) * n
    raise ValueError(f"unknown optimizer {opt!r}")


def state_bytes(opt: str, m: int, n: int) -> float:
    """fp32 optimizer state of one matrix, from the library's own count."""
    lib = L.load()
    fn = {"muon": lib.mao_muon_state_elems, "soap": lib.mao_soap_state_elems,
          "foam": lib.mao_foam_state_elems}[opt]
    return 4.0 * fn(m, n)


def step_cost(opt: str, m: int, n: int) -> float:
    """Estimated seconds of one step: tensor-core time of its products plus one pass
    over the weights, gradient and state in HBM."""
    products = 1 if opt == "muon" else _SPLIT3_PRODUCTS
    flops = step_flops(opt, m, n) * products
    hbm = state_bytes(opt, m, n) * 2.0 + 10.0 * m * n  # state read + written; W, G, update
    return flops / _TC_FLOPS + hbm / _HBM_BYTES


def assign_owners(shapes: Sequence[Tuple[int, int]], world: int, opt: str,
                  cost: Optional[Callable[[str, int, int], float]] = None) -> List[int]:
    """Owner rank of every matrix: longest processing time first (matrices by cost,
    descending, ties by index; each to the least-loaded rank, ties to the lower rank).
    Deterministic, so every rank computes the same owners without communicating."""
    if world < 1:
        raise ValueError("world must be >= 1")
    cost = cost or step_cost
    c = [cost(opt, m, n) for (m, n) in shapes]
    order = sorted(range(len(shapes)), key=lambda i: (-c[i], i))
    load = [0.0] * world
    owners = [0] * len(shapes)
    for i in order:
        r = min(range(world), key=lambda q: (load[q], q))
        owners[i] = r
        load[r] += c[i]
    return owners


def allgather_v(tensors: Sequence, owners: Sequence[int], dist, group=None) -> None:
    """Every rank ends with every owner's values of `tensors` (owner-side values are
    the updated ones): per owner, its tensors are packed into one flat buffer and
    broadcast from it.  All ranks call this with the same tensors and owners, so the
    collectives match in number, order and size."""
    import torch
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    for r in range(world):
        idx = [i for i, o in enumerate(owners) if o == r]
        if not idx:
            continue
        parts = [tensors[i] for i in idx]
        dtype = parts[0].dtype
        if any(p.dtype != dtype for p in parts):
            raise TypeError("allgather_v packs one dtype per owner")
        flat = torch.empty(sum(p.numel() for p in parts), dtype=dtype, device=parts[0].device)
        if rank == r:
            torch.cat([p.reshape(-1) for p in parts], out=flat)
        dist.broadcast(flat, src=dist.get_global_rank(group, r) if group is not None else r, group=group)
        if rank != r:
            off = 0
            for p in parts:
                p.copy_(flat[off:off + p.numel()].view_as(p))
                off += p.numel()


class LayerwiseStep:
    """One optimizer step of a whole layer set over data-parallel ranks.

    mats: the full list, in the same order on every rank (Muon: (W, G, M) tuples;
    SOAP/FOAM: dicts as the batch classes take).  Each rank builds a batch object of
    the matrices it owns (`make_batch(owned_mats)`, by default the library's batch
    class for `opt` with `batch_kw`), steps them, then exchanges the updated W.  Every
    rank keeps full-size W (and, as in data parallelism, G); only the owner keeps a
    matrix's optimizer state up to date."""

    def __init__(self, mats: Sequence, opt: str, dist, group=None,
                 make_batch: Optional[Callable[[List], Callable]] = None, **batch_kw):
        self.mats = list(mats)
        self.opt = opt
        self.dist = dist
        self.group = group
        world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        shapes = [tuple(self._W(x).shape) for x in self.mats]
        self.owners = assign_owners(shapes, world, opt)
        owned = [x for x, o in zip(self.mats, self.owners) if o == self.rank]
        if make_batch is None:
            from . import api
            cls = {"muon": api.MuonBatch, "soap": api.SoapBatch, "foam": api.FoamBatch}[opt]

            def make_batch(ms):
                return cls(ms, **batch_kw)
        self.batch = make_batch(owned) if owned else None

    @staticmethod
    def _W(x):
        return x[0] if isinstance(x, (tuple, list)) else x["W"]

    def __call__(self, *args) -> None:
        if self.batch is not None:
            self.batch(*args)
        allgather_v([self._W(x) for x in self.mats], self.owners, self.dist, self.group)
