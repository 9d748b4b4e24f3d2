"""Layer-wise distributed optimizer step over data-parallel ranks.

"SOAP, Muon and Beyond" (the Korean review: §2-1 Main contribution, item 4, the
layer-wise distributed optimizer; §3-2 Module breakdown, item 7, layer-wise
optimizer ownership) keeps every weight matrix whole: each matrix is owned by one
data-parallel rank, which holds its full optimizer state and runs the matrix
optimizer on it, and the updated weights reach every rank through an all-gather
before the next forward pass.  The owners are balanced by optimizer cost (the
Newton-Schulz work and the factor sizes depend on the shape), memory and compute
together, not by parameter count.  The English summary ("Layer-Wise Distributed
Optimizer") adds that the variable-sized all-gather runs asynchronously, hidden
behind computation.

Here:
  * `assign_owners`: longest-processing-time-first over a cost model of the step's
    tensor-core and HBM time (`step_cost`);
  * `reduce_to_owners`: each gradient summed over the ranks into its owner (one
    packed reduce per owner, a reduce-scatter-V) and divided by the world size, for
    callers whose gradients are not yet averaged;
  * `AllGatherV`: the exchange of the updated weights, one packed broadcast per
    owner on a side stream.  Broadcasts from other owners write weights this rank
    does not step, so they start at once and overlap this rank's own step; this
    rank's broadcast waits for its step (an event);
  * `LayerwiseStep`: reduce (optional), the owned matrices through the single-GPU
    library (`api.MuonBatch`, `api.SoapBatch`, `api.FoamBatch`), the exchange.
Every rank issues the same collectives in the same order.  The collectives are
torch.distributed's (NCCL over NVLink on GPUs, gloo on CPU).
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
# columns of one QR panel in the library's block Gram-Schmidt
_PANEL = 128


def qr_flops(k: int) -> float:
    """The library's QR of a k x k matrix by panels of b columns (block Gram-Schmidt
    with Cholesky-QR inside each panel): the projections against the finished
    columns, C = Q^T P_j and P_j - Q C, total 2 k^3 over the panels; per panel a Gram
    (2 k b^2) and W R^-1 (2 k b^2), total 4 k^2 b.  Extra passes that the device
    decides only when cancellation shows are not counted."""
    return 2.0 * float(k) ** 3 + 4.0 * float(k) ** 2 * _PANEL


def step_flops(opt: str, m: int, n: int, ns_steps: int = 5, refresh_period: int = 1) -> float:
    """Multiply-add work of one step of an m x n matrix, in FLOP (2 per multiply-add),
    averaged over the refresh period.

    muon: `ns_steps` Newton-Schulz iterations on the wide orientation, 4 s^2 l + 2 s^3
          each.
    soap: factors 2m^2n + 2mn^2, rotations in 4(m^2n + mn^2), rotation back
          2(m^2n + mn^2); per refresh (every `refresh_period` steps) the power step
          2(m^3 + n^3) and the QR of both factors.
    foam: factor 2mn^2, rotations in 4mn^2, rotation back 2mn^2; per check or refresh
          (every `refresh_period` steps, counted as refreshing) the power step 2n^3
          and the QR of the input factor."""
    if opt == "muon":
        s, l = min(m, n), max(m, n)
        return ns_steps * (4.0 * s * s * l + 2.0 * s ** 3)
    per = max(int(refresh_period), 1)
    if opt == "soap":
        mn = float(m) * m * n + float(m) * n * n
        refresh = 2.0 * (float(m) ** 3 + float(n) ** 3) + qr_flops(m) + qr_flops(n)
        return 8.0 * mn + refresh / per
    if opt == "foam":
        refresh = 2.0 * float(n) ** 3 + qr_flops(n)
        return 8.0 * m * float(n) * n + refresh / per
    raise ValueError(f"unknown optimizer {opt!r}")


def state_bytes(opt: str, m: int, n: int) -> float:
    """fp32 optimizer state of one matrix, from the library's own count."""
    lib = L.load()
    fn = {"muon": lib.mao_muon_state_elems, "soap": lib.mao_soap_state_elems,
          "foam": lib.mao_foam_state_elems}[opt]
    return 4.0 * fn(m, n)


def step_cost(opt: str, m: int, n: int, ns_steps: int = 5, refresh_period: int = 1) -> float:
    """Estimated seconds of one step: tensor-core time of its products plus one pass
    over the weights, gradient and state in HBM."""
    products = 1 if opt == "muon" else _SPLIT3_PRODUCTS
    flops = step_flops(opt, m, n, ns_steps, refresh_period) * products
    hbm = state_bytes(opt, m, n) * 2.0 + 10.0 * m * n  # state read + written; W, G, update
    return flops / _TC_FLOPS + hbm / _HBM_BYTES


def cost_for(opt: str, batch_kw: dict) -> Callable[[str, int, int], float]:
    """The cost function that matches a batch's settings: Newton-Schulz steps (Muon),
    the refresh period (SOAP every k steps, FOAM's check period pf; none = 1 refresh in
    a very long run)."""
    ns = int(batch_kw.get("ns_steps", 5))
    if opt == "soap":
        kind = batch_kw.get("refresh", "every_k")
        per = {"every_k": int(batch_kw.get("k", 1)), "adaptive": int(batch_kw.get("pf", 10))}.get(kind, 1 << 20)
    elif opt == "foam":
        kind = batch_kw.get("refresh", "adaptive")
        per = {"every_k": int(batch_kw.get("k", 1)), "adaptive": int(batch_kw.get("pf", 10))}.get(kind, 1 << 20)
    else:
        per = 1

    def cost(o, m, n):
        return step_cost(o, m, n, ns, per)
    return cost


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


def _src(dist, group, r):
    return dist.get_global_rank(group, r) if group is not None else r


class _Packs:
    """Packing of a list of same-dtype tensors per owner rank into one persistent flat
    buffer, sized for the largest owner and reused owner after owner (the packs, the
    collectives and the unpacks of one exchange run in order on one stream)."""

    def __init__(self, tensors, owners, world):
        import torch
        self.idx = [[i for i, o in enumerate(owners) if o == r] for r in range(world)]
        self.size = [sum(tensors[i].numel() for i in ix) for ix in self.idx]
        dtypes = {tensors[i].dtype for ix in self.idx for i in ix}
        if len(dtypes) > 1:
            raise TypeError("one dtype for every packed tensor")
        self.buf = None
        if tensors:
            self.buf = torch.empty(max(max(self.size), 1), dtype=tensors[0].dtype, device=tensors[0].device)

    def flat(self, r):
        return self.buf[:self.size[r]] if self.size[r] else None

    def pack(self, tensors, r):
        import torch
        torch.cat([tensors[i].reshape(-1) for i in self.idx[r]], out=self.flat(r))

    def unpack(self, tensors, r):
        off = 0
        f = self.flat(r)
        for i in self.idx[r]:
            p = tensors[i]
            p.copy_(f[off:off + p.numel()].view_as(p))
            off += p.numel()


def reduce_to_owners(grads: Sequence, owners: Sequence[int], dist, group=None, packs: Optional[_Packs] = None):
    """Each owner ends with the mean over ranks of the gradients it owns; the other ranks'
    copies are left as they were.  One packed reduce per owner, in rank order."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    packs = packs or _Packs(grads, owners, world)
    for r in range(world):
        if not packs.size[r]:
            continue
        packs.pack(grads, r)
        dist.reduce(packs.flat(r), dst=_src(dist, group, r), op=dist.ReduceOp.SUM, group=group)
        if rank == r:
            packs.flat(r).div_(world)
            packs.unpack(grads, r)
    return packs


def allgather_v(tensors: Sequence, owners: Sequence[int], dist, group=None) -> None:
    """Every rank ends with every owner's values of `tensors` (owner-side values are
    the updated ones): per owner, its tensors are packed into one flat buffer and
    broadcast from it.  All ranks call this with the same tensors and owners, so the
    collectives match in number, order and size.  Synchronous, on the current stream."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    packs = _Packs(tensors, owners, world)
    for r in range(world):
        if not packs.size[r]:
            continue
        if rank == r:
            packs.pack(tensors, r)
        dist.broadcast(packs.flat(r), src=_src(dist, group, r), group=group)
        if rank != r:
            packs.unpack(tensors, r)


class AllGatherV:
    """The weight exchange of a layer-wise step, overlapped with this rank's own step.

    `start(done_event)` enqueues, on a side stream, every owner's broadcast in rank
    order: the broadcasts of other owners (into weights this rank does not step) right
    away, this rank's own after `done_event` (the end of its step on the compute
    stream) and a pack of its updated weights.  `wait()` makes the current stream wait
    for the exchange.  On CPU (gloo) it runs synchronously."""

    def __init__(self, tensors, owners, dist, group=None):
        self.tensors = list(tensors)
        self.owners = list(owners)
        self.dist = dist
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.packs = _Packs(self.tensors, self.owners, self.world)
        self.cuda = bool(self.tensors) and self.tensors[0].is_cuda
        self.stream = None
        self.done = None
        if self.cuda:
            import torch
            self.stream = torch.cuda.Stream(device=self.tensors[0].device)

    def _run(self, own_ready):
        for r in range(self.world):
            if not self.packs.size[r]:
                continue
            if r == self.rank:
                own_ready()
                self.packs.pack(self.tensors, r)
            self.dist.broadcast(self.packs.flat(r), src=_src(self.dist, self.group, r), group=self.group)
            if r != self.rank:
                self.packs.unpack(self.tensors, r)

    def start(self, done_event=None) -> None:
        if not self.cuda:
            self._run(lambda: None)
            return
        import torch
        with torch.cuda.stream(self.stream):
            self._run(lambda: self.stream.wait_event(done_event) if done_event is not None else None)
            self.done = torch.cuda.Event()
            self.done.record(self.stream)

    def wait(self) -> None:
        if self.cuda and self.done is not None:
            import torch
            torch.cuda.current_stream(self.tensors[0].device).wait_event(self.done)


class LayerwiseStep:
    """One optimizer step of a whole layer set over data-parallel ranks.

    mats: the full list, in the same order on every rank (Muon: (W, G, M) tuples;
    SOAP/FOAM: dicts as the batch classes take).  Each rank builds a batch object of
    the matrices it owns (`make_batch(owned_mats)`, by default the library's batch
    class for `opt` with `batch_kw`), steps them, then exchanges the updated W.  Every
    rank keeps full-size W and G; only the owner keeps a matrix's optimizer state.

    Gradients: with `grads_reduced=False` (default) each rank holds its own local
    gradient and the step first reduces every G to its owner as the mean over ranks
    (the owner's G buffer is overwritten with it).  Pass `grads_reduced=True` when the
    caller has already averaged the gradients on every rank (e.g. a DDP all-reduce).
    The owners balance `cost_for(opt, batch_kw)`.  `exchange` shares an AllGatherV built
    for the same weights and owners."""

    def __init__(self, mats: Sequence, opt: str, dist, group=None,
                 make_batch: Optional[Callable[[List], Callable]] = None, grads_reduced: bool = False,
                 exchange: Optional[AllGatherV] = None, **batch_kw):
        self.mats = list(mats)
        self.opt = opt
        self.dist = dist
        self.group = group
        self.grads_reduced = grads_reduced
        world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        shapes = [tuple(self._W(x).shape) for x in self.mats]
        self.owners = assign_owners(shapes, world, opt, cost_for(opt, batch_kw))
        owned = [x for x, o in zip(self.mats, self.owners) if o == self.rank]
        if make_batch is None:
            from . import api
            cls = {"muon": api.MuonBatch, "soap": api.SoapBatch, "foam": api.FoamBatch}[opt]

            def make_batch(ms):
                return cls(ms, **batch_kw)
        self.batch = make_batch(owned) if owned else None
        # several steps over the same weights (e.g. one per gradient buffer) may share one
        # exchange (and its pack buffer)
        self.exchange = exchange or AllGatherV([self._W(x) for x in self.mats], self.owners, dist, group)
        self.gpacks = None

    @staticmethod
    def _W(x):
        return x[0] if isinstance(x, (tuple, list)) else x["W"]

    @staticmethod
    def _G(x):
        return x[1] if isinstance(x, (tuple, list)) else x["G"]

    def __call__(self, *args) -> None:
        if not self.grads_reduced:
            self.gpacks = reduce_to_owners([self._G(x) for x in self.mats], self.owners, self.dist, self.group,
                                           self.gpacks)
        if self.batch is not None:
            self.batch(*args)
        done = None
        if self.exchange.cuda:
            import torch
            done = torch.cuda.Event()
            done.record()
        self.exchange.start(done)
        self.exchange.wait()
