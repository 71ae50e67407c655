"""Expert-parallel MoE layer ("Llama 3 Meets MoE", section "训练框架": the 5-D hybrid
parallelism places the experts of each MoE layer on different devices, and the
training configuration runs 8-way expert parallelism inside the NVLink domain).

N ranks, one process per GPU.  Rank r holds its own batch of tokens and the packed
weights of experts [r E/N, (r+1) E/N) only.  One layer step on rank r:

  1. route and dispatch its tokens with the library's kernels, without a capacity;
  2. gather every rank's per-expert counts (and its token count) and sum the
     router's token sums over the ranks (two small collectives);
  3. derive the exchange plan on the host (``moe_ep_plan``: the same on every rank)
     and mark the assignments the capacity drops in slot_row (``moe_ep_mask_slots``);
  4. send every kept run of rows to the rank that owns its expert; a run is the
     kept prefix of one expert's block of the dispatch output and lands at its
     place in the owner's expert-major buffer, so neither side packs or regroups;
  5. run the grouped SwiGLU GEMMs of the local experts on the received rows;
  6. send the output runs back along the same paths;
  7. combine with the gate weights, and compute the gate statistics over all ranks.

With capacity scope GLOBAL the result is the one-device layer on the ranks'
batches concatenated in rank order.  The collectives go through torch.distributed
(NCCL between GPUs); every arithmetic step runs in libmoe's kernels (``LibmoeOps``).

Host synchronisation: one per step.  The exchange sizes (step 4) are host-side
arguments of the point-to-point calls, so the gathered counts are copied into
pinned host memory and the host waits for that copy alone (an event), plans, and
issues the exchange; the device is idle meanwhile.  ``EpStep.host_plan_ms`` records
that wait plus the plan.
"""
import time

import torch
import torch.distributed as dist

from . import (EP_CAPACITY_GLOBAL, MIXTRAL, MOE_BF16, MoeError, MOE_ERR_SHAPE, Workspace,
               _dtype_code, h_ld, moe_combine, moe_dispatch_routed, moe_ep_gate_stats,
               moe_ep_mask_slots, moe_ep_plan, moe_expert_ffn, moe_route, moe_workspace_size,
               params)

__all__ = ["exchange_runs", "DistTransport", "ExpertParallelMoE", "EpStep", "LibmoeOps"]


def exchange_runs(src, src_runs, dst, dst_runs, rank, group=None):
    """Moves runs of rows between ranks.

    src_runs / dst_runs: (peer, first row, rows, expert) of every run this rank
    sends from ``src`` / receives into ``dst``.  Between two ranks, the run one
    sends for expert e must pair with the run the other receives for expert e.
    NCCL ignores point-to-point tags and pairs the messages between two ranks by
    their order alone, so each peer's non-empty runs must be listed in ascending
    expert order on both sides; that is checked here before any transfer (the
    expert is also passed as the tag, which gloo honours).  Empty runs move
    nothing; runs whose peer is this rank are copied locally.  Works on CUDA
    tensors (NCCL) and CPU tensors (gloo).
    """
    for runs, what in ((src_runs, "send"), (dst_runs, "receive")):
        last = {}
        for p, _, n, e in runs:
            if n > 0:
                if e <= last.get(p, -1):
                    raise ValueError("the %s runs to rank %d are not in ascending expert order "
                                     "(NCCL pairs messages by order)" % (what, p))
                last[p] = e
    own_src = [(r, n, e) for (p, r, n, e) in src_runs if p == rank and n > 0]
    own_dst = [(r, n, e) for (p, r, n, e) in dst_runs if p == rank and n > 0]
    if [(n, e) for (_, n, e) in own_src] != [(n, e) for (_, n, e) in own_dst]:
        raise ValueError("the local runs of the send and receive lists do not pair up")
    for (a, n, _), (b, _, _) in zip(own_src, own_dst):
        dst[b:b + n].copy_(src[a:a + n])
    ops = []
    for p, r, n, e in src_runs:
        if p != rank and n > 0:
            ops.append(dist.P2POp(dist.isend, src[r:r + n], p, group=group, tag=e))
    for p, r, n, e in dst_runs:
        if p != rank and n > 0:
            ops.append(dist.P2POp(dist.irecv, dst[r:r + n], p, group=group, tag=e))
    if ops:
        for w in dist.batch_isend_irecv(ops):
            w.wait()


class DistTransport:
    """The collectives of a layer step over a torch.distributed process group."""

    def __init__(self, group=None):
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)

    def all_gather(self, t):
        """[n] on every rank -> [world][n], rows in rank order."""
        parts = [torch.empty_like(t) for _ in range(self.world)]
        dist.all_gather(parts, t.contiguous(), group=self.group)
        return torch.stack(parts)

    def all_reduce_sum(self, t):
        dist.all_reduce(t, op=dist.ReduceOp.SUM, group=self.group)

    def exchange(self, src, src_runs, dst, dst_runs):
        exchange_runs(src, src_runs, dst, dst_runs, self.rank, self.group)


class EpStep:
    """Tensors of one layer step on one rank (outputs: y, loss, counts, importance, f, P)."""


class LibmoeOps:
    """The arithmetic of a layer step: libmoe's entry points (device tensors).  Every
    method takes the library's arguments and writes its outputs in place."""

    dtype_code = staticmethod(_dtype_code)

    @staticmethod
    def workspace(p, device):
        return Workspace(p, device=device)

    @staticmethod
    def workspace_size(p):
        return moe_workspace_size(p)

    # a1 then a2 on the same workspace: the dispatch reuses the router's chunk counts
    route = staticmethod(moe_route)
    dispatch = staticmethod(moe_dispatch_routed)
    mask_slots = staticmethod(moe_ep_mask_slots)
    expert_ffn = staticmethod(moe_expert_ffn)
    combine = staticmethod(moe_combine)
    gate_stats = staticmethod(moe_ep_gate_stats)


class ExpertParallelMoE:
    """The layer on one rank.  W13_local / W2_local: the packed weights (moe_partition_*
    layout) of this rank's E/N experts.  Wg, Wnoise, bias: the full router (every rank
    routes its own tokens over all E experts).  capacity: rows an expert keeps (< 0:
    none), counted over all ranks' tokens (EP_CAPACITY_GLOBAL) or per rank
    (EP_CAPACITY_LOCAL).

    ``forward`` runs the seven steps with ``transport`` (default: DistTransport over
    the default group).  The steps are also methods of their own, separated at the
    collectives, so a caller can drive several ranks' steps in lockstep.  ``ops``
    carries the arithmetic (default ``LibmoeOps``, the library's kernels)."""

    def __init__(self, d, E, k, m, W13_local, W2_local, Wg, Wnoise=None, bias=None,
                 dtype=torch.bfloat16, router_type=MIXTRAL, capacity=-1,
                 capacity_scope=EP_CAPACITY_GLOBAL, rescale=False, balance_lambda=0.0,
                 rank=None, world=None, transport=None, ops=None):
        self.ops = ops if ops is not None else LibmoeOps()
        if transport is None and (rank is None or world is None):
            transport = DistTransport()
        self.transport = transport
        self.rank = transport.rank if rank is None else rank
        self.world = transport.world if world is None else world
        if E % self.world != 0:
            raise MoeError(MOE_ERR_SHAPE, "the %d experts do not split over %d ranks"
                           % (E, self.world))
        self.d, self.E, self.k, self.m = d, E, k, m
        self.E_local = E // self.world
        self.W13, self.W2, self.Wg, self.Wnoise, self.bias = W13_local, W2_local, Wg, Wnoise, bias
        self.dtype = dtype
        self.router_type, self.capacity, self.scope = router_type, capacity, capacity_scope
        self.rescale, self.lam = rescale, balance_lambda
        self.device = Wg.device
        self._ws_route = None
        self._ws_ffn = None

    def _params(self, T, E, k):
        return params(T, self.d, E, k, self.m, self.ops.dtype_code(self.dtype), self.router_type,
                      -1, self.rescale, self.lam)

    def _workspace(self, attr, p):
        need = self.ops.workspace_size(p)
        ws = getattr(self, attr)
        if ws is None or ws.nbytes < need:
            ws = self.ops.workspace(p, self.device)
            setattr(self, attr, ws)
        return ws

    # -- step 1
    def begin(self, x, noise=None) -> EpStep:
        T, d, E, k = x.shape[0], self.d, self.E, self.k
        dev = self.device
        s = EpStep()
        s.T = T
        s.p = p = self._params(T, E, k)
        ws = self._workspace("_ws_route", p)
        rows = max(T * k, 1)
        E4 = (E + 3) // 4 * 4
        i32 = dict(dtype=torch.int32, device=dev)
        s.topk_idx = torch.empty((max(T, 1), k), **i32)
        s.topk_w = torch.empty((max(T, 1), k), dtype=torch.float32, device=dev)
        s.sums = torch.zeros(2 * E4, dtype=torch.float32, device=dev)
        s.probs_sum, s.importance = s.sums[:E], s.sums[E4:E4 + E]
        s.x_perm = torch.empty((rows, d), dtype=x.dtype, device=dev)
        s.row_token = torch.empty(rows, **i32)
        s.slot_row = torch.empty((max(T, 1), k), **i32)
        s.counts_T = torch.zeros(E4 + 4, **i32)
        s.counts = s.counts_T[:E]
        s.kept = torch.empty(E, **i32)
        s.offsets = torch.empty(E4 + 4, **i32)
        if T > 0:
            self.ops.route(p, x, self.Wg, self.Wnoise, noise, self.bias, ws, s.topk_idx,
                           s.topk_w, s.probs_sum, s.importance)
            self.ops.dispatch(p, x, s.topk_idx, ws, s.x_perm, s.row_token, s.slot_row, s.counts,
                              s.kept, s.offsets)
        s.counts_T[E] = T
        return s

    # -- step 2 (collectives)
    def gather_counts(self, s: EpStep, transport=None):
        tr = transport or self.transport
        s.counts_all_dev = tr.all_gather(s.counts_T)
        if s.counts_all_dev.is_cuda:  # into pinned memory; the host waits for this copy only
            s.counts_host = torch.empty(s.counts_all_dev.shape, dtype=torch.int32,
                                        pin_memory=True)
            s.counts_host.copy_(s.counts_all_dev, non_blocking=True)
            s.counts_ready = torch.cuda.Event()
            s.counts_ready.record()
        tr.all_reduce_sum(s.sums)

    # -- step 3 (host plan, slot mask, receive buffers)
    def plan(self, s: EpStep, counts_all_host=None):
        E = self.E
        t0 = time.perf_counter()
        if counts_all_host is None:
            ready = getattr(s, "counts_ready", None)
            if ready is not None:  # the pinned copy gather_counts started
                ready.synchronize()
                counts_all_host = s.counts_host
            else:
                counts_all_host = s.counts_all_dev.cpu()
        ca = counts_all_host[:, :E].contiguous()
        s.T_all = int(counts_all_host[:, E].sum())
        s.counts_all = s.counts_all_dev[:, :E].contiguous()
        s.ep = moe_ep_plan(ca, self.rank, self.capacity, self.scope)
        keep = s.ep.keep_all[self.rank]
        if s.T > 0 and bool((keep < ca[self.rank]).any()):
            self.ops.mask_slots(s.p, s.topk_idx, s.offsets, keep, s.slot_row)
        R_in = s.ep.rows_in
        s.R_in = R_in
        s.xin = torch.empty((max(R_in, 1), self.d), dtype=s.x_perm.dtype, device=self.device)
        s.in_offsets = s.ep.in_offsets.to(self.device)
        s.send_runs, s.recv_runs = s.ep.send_runs(), s.ep.recv_runs()
        s.host_plan_ms = 1000.0 * (time.perf_counter() - t0)

    # -- step 4 (collective)
    def send_rows(self, s: EpStep, transport=None):
        (transport or self.transport).exchange(s.x_perm, s.send_runs, s.xin, s.recv_runs)

    # -- step 5
    def experts(self, s: EpStep):
        dev, R_in = self.device, s.R_in
        s.out_local = torch.empty((max(R_in, 1), self.d), dtype=s.x_perm.dtype, device=dev)
        s.out = torch.zeros_like(s.x_perm)
        if R_in == 0:
            return
        pl = self._params(R_in, self.E_local, 1)
        ws = self._workspace("_ws_ffn", pl)
        s.h = torch.empty((R_in, h_ld(self.m)), dtype=s.x_perm.dtype, device=dev)
        self.ops.expert_ffn(pl, s.xin, s.in_offsets, self.W13, self.W2, s.h, s.out_local, ws)

    # -- step 6 (collective)
    def return_rows(self, s: EpStep, transport=None):
        (transport or self.transport).exchange(s.out_local, s.recv_runs, s.out, s.send_runs)

    # -- step 7
    def finish(self, s: EpStep) -> EpStep:
        dev, E = self.device, self.E
        s.y = torch.empty((s.T, self.d), dtype=s.x_perm.dtype, device=dev)
        if s.T > 0:
            self.ops.combine(s.p, s.out, s.slot_row, s.topk_w, s.y)
        s.counts_global = torch.empty(E, dtype=torch.int32, device=dev)
        s.f = torch.empty(E, dtype=torch.float32, device=dev)
        s.P = torch.empty(E, dtype=torch.float32, device=dev)
        s.loss = torch.empty(1, dtype=torch.float32, device=dev)
        pg = self._params(s.T_all, E, self.k)
        self.ops.gate_stats(pg, s.counts_all, self.world, s.probs_sum, s.counts_global, s.f, s.P,
                            s.loss)
        return s

    def forward(self, x, noise=None) -> EpStep:
        s = self.begin(x, noise)
        self.gather_counts(s)
        self.plan(s)
        self.send_rows(s)
        self.experts(s)
        self.return_rows(s)
        return self.finish(s)
