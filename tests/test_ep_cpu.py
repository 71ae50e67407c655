"""Expert-parallel layer on the CPU: the exchange plan of libmoe (host code, no GPU)
against a brute-force recount, and ``ExpertParallelMoE.forward`` itself in world
sizes 2 and 4 over gloo (its plan, slot mask, row exchange and gate statistics,
with the fp64 oracle standing in for the GPU kernels' arithmetic), against the
oracle's one-process layer on the ranks' batches concatenated in rank order
("Llama 3 Meets MoE", section "训练框架", Expert Parallelism; section 3 "容量因子"
for the capacity)."""
import json
import os
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import top_routing_grouped_noisy_b200 as moe  # noqa: E402

GLOBAL, LOCAL = moe.EP_CAPACITY_GLOBAL, moe.EP_CAPACITY_LOCAL


def _brute_keep(counts_all, capacity, scope):
    """Rank every (rank, expert) assignment in the order the layer sees them and keep
    those below the capacity (one list entry per assignment)."""
    N, E = counts_all.shape
    keep = np.zeros((N, E), np.int64)
    for e in range(E):
        seen = 0
        for p in range(N):
            local = 0
            for _ in range(int(counts_all[p, e])):
                pos = seen if scope == GLOBAL else local
                if capacity < 0 or pos < capacity:
                    keep[p, e] += 1
                seen += 1
                local += 1
    return keep


@pytest.mark.parametrize("N,E", [(1, 8), (2, 8), (4, 8), (8, 8), (4, 16), (8, 64), (3, 12)])
@pytest.mark.parametrize("capacity", [-1, 0, 3, 11, 1000])
@pytest.mark.parametrize("scope", [GLOBAL, LOCAL])
def test_plan_matches_recount_and_pairs_up(N, E, capacity, scope):
    rng = np.random.default_rng(N * 1000 + E * 10 + capacity + 7 * scope)
    counts = rng.integers(0, 9, size=(N, E)).astype(np.int32)
    counts[rng.random((N, E)) < 0.2] = 0
    plans = [moe.moe_ep_plan(torch.from_numpy(counts), r, capacity, scope) for r in range(N)]
    want = _brute_keep(counts, capacity, scope)
    El = E // N
    for r, pl in enumerate(plans):
        assert np.array_equal(pl.keep_all.numpy(), want)
        # sends: the kept prefix of each expert's block of the dropless dispatch output
        blocks = np.concatenate([[0], np.cumsum(counts[r])])
        assert np.array_equal(pl.send_row.numpy(), blocks[:E])
        assert np.array_equal(pl.send_cnt.numpy(), want[r])
        # receives tile [0, rows_in) expert-major, ranks ascending inside an expert
        runs = pl.recv_runs()
        pos = 0
        for l in range(El):
            assert int(pl.in_offsets[l]) == pos
            for p in range(N):
                peer, row, n, e = runs[p * El + l]
                assert (peer, e) == (p, r * El + l)
                assert row == pos and n == want[p, r * El + l]
                pos += n
        assert int(pl.in_offsets[El]) == pos == pl.rows_in
    # between every pair, the non-empty runs one sends pair with those the other receives
    for q in range(N):
        for p in range(N):
            sent = [(n, e) for (peer, _, n, e) in plans[q].send_runs() if peer == p and n > 0]
            got = [(n, e) for (peer, _, n, e) in plans[p].recv_runs() if peer == q and n > 0]
            assert sent == got


from hypothesis import given, settings, strategies as st  # noqa: E402


@settings(max_examples=200, deadline=None)
@given(st.data())
def test_plan_property_random_shapes(data):
    """Random rank counts, expert counts, capacities and scopes: the plan equals the
    brute-force recount, every receive buffer is tiled exactly, and the kept totals per
    expert are min(routed, C) under GLOBAL."""
    N = data.draw(st.sampled_from([1, 2, 4, 8]))
    E = N * data.draw(st.integers(1, 64 // N))
    counts = np.array(data.draw(st.lists(st.lists(st.integers(0, 20), min_size=E, max_size=E),
                                         min_size=N, max_size=N)), np.int32)
    C = data.draw(st.integers(-1, 50))
    scope = data.draw(st.sampled_from([GLOBAL, LOCAL]))
    want = _brute_keep(counts, C, scope)
    rows_in = 0
    for r in range(N):
        pl = moe.moe_ep_plan(torch.from_numpy(counts), r, C, scope)
        assert np.array_equal(pl.keep_all.numpy(), want)
        runs = sorted((row, n) for (_, row, n, _) in pl.recv_runs())
        pos = 0
        for row, n in runs:
            assert row == pos
            pos += n
        assert pos == pl.rows_in
        rows_in += pl.rows_in
    assert rows_in == want.sum()
    if scope == GLOBAL and C >= 0:
        assert np.array_equal(want.sum(0), np.minimum(counts.sum(0), C))


def test_plan_global_capacity_totals():
    counts = np.array([[5, 0, 2, 9], [4, 3, 0, 1], [6, 6, 6, 6], [0, 1, 2, 3]], np.int32)
    pl = moe.moe_ep_plan(torch.from_numpy(counts), 0, capacity=7, scope=GLOBAL)
    kept = pl.keep_all.numpy().sum(0)
    assert np.array_equal(kept, np.minimum(counts.sum(0), 7))
    pl = moe.moe_ep_plan(torch.from_numpy(counts), 0, capacity=7, scope=LOCAL)
    assert np.array_equal(pl.keep_all.numpy(), np.minimum(counts, 7))


@pytest.mark.parametrize("counts,rank,scope,code", [
    ([[1, 2, 3]], 0, GLOBAL, moe.MOE_OK),
    ([[1, 2, 3], [1, 1, 1]], 0, GLOBAL, moe.MOE_ERR_SHAPE),        # 2 ranks, 3 experts
    ([[1, 2], [1, 1]], 2, GLOBAL, moe.MOE_ERR_INVALID_ARG),        # rank outside [0, N)
    ([[1, -2], [1, 1]], 0, GLOBAL, moe.MOE_ERR_INVALID_ARG),       # negative count
    ([[1, 2], [1, 1]], 0, 5, moe.MOE_ERR_INVALID_ARG),             # scope
    ([[1] * 66, [1] * 66], 0, GLOBAL, moe.MOE_ERR_SHAPE),          # E > 64
    ([[2 ** 30, 2 ** 30]], 0, GLOBAL, moe.MOE_ERR_SHAPE),          # too many rows
])
def test_plan_errors(counts, rank, scope, code):
    c = torch.tensor(counts, dtype=torch.int32)
    if code == moe.MOE_OK:
        moe.moe_ep_plan(c, rank, -1, scope)
        return
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_ep_plan(c, rank, -1, scope)
    assert ei.value.code == code


# --------------------------------------------------------------------------- gloo layer

def _layer_inputs(Ts, d, E, m, seed):
    g = torch.Generator().manual_seed(seed)
    Tall = sum(Ts)
    x = torch.randn(Tall, d, generator=g)
    Wg = torch.randn(d, E, generator=g) * 0.3
    Wn = torch.randn(d, E, generator=g) * 0.3
    eps = torch.randn(Tall, E, generator=g)
    W1 = torch.randn(E, m, d, generator=g) * 0.2
    W3 = torch.randn(E, m, d, generator=g) * 0.2
    W2 = torch.randn(E, d, m, generator=g) * 0.2
    f = lambda t: t.numpy().astype(np.float32)
    return dict(x=f(x), Wg=f(Wg), Wn=f(Wn), eps=f(eps), W1=f(W1), W3=f(W3), W2=f(W2))


class OracleOps:
    """ExpertParallelMoE's arithmetic on the host in fp64 (the oracle), for CPU tensors
    of float64 that hold f32 values exactly: the same calls, arguments and in-place
    outputs as the library's entry points, which need a GPU.  Everything else of the
    layer -- the class's steps, the exchange plan (libmoe host code), the collectives
    and the row exchange over gloo -- is the code under test.  Outputs the library
    keeps in f32 (gate weights, token sums, statistics) are stored in the f32 tensors
    the class allocates for them."""

    def __init__(self, W1l, W3l, W2l, lam):
        self.W1l, self.W3l, self.W2l, self.lam = W1l, W3l, W2l, lam

    @staticmethod
    def dtype_code(dt):
        return moe.MOE_F32  # a tag of the call shapes; the tensors are float64

    class _Ws:
        nbytes = 1 << 62

    def workspace(self, p, device):
        return self._Ws()

    @staticmethod
    def workspace_size(p):
        return 0

    @staticmethod
    def _f32(t):
        return np.ascontiguousarray(t.numpy().astype(np.float32))

    def route(self, p, x, Wg, Wn, noise, bias, ws, topk_idx, topk_w, probs_sum, importance):
        import oracle
        r = oracle.router(self._f32(x), self._f32(Wg), None if Wn is None else self._f32(Wn),
                          None if noise is None else self._f32(noise),
                          None if bias is None else bias.numpy(), p.k, p.router_type)
        T = p.T
        topk_idx[:T] = torch.from_numpy(r["idx"])
        topk_w[:T] = torch.from_numpy(r["G"]).to(topk_w.dtype)
        probs_sum.copy_(torch.from_numpy(r["probs_sum"]))
        importance.copy_(torch.from_numpy(r["importance"]))

    def dispatch(self, p, x, topk_idx, ws, x_perm, row_token, slot_row, counts, kept, offsets):
        import oracle
        d = oracle.dispatch(topk_idx[:p.T].numpy(), p.E, p.capacity)
        R = d["R"]
        rt = torch.from_numpy(d["row_token"]).long()
        x_perm[:R] = x[rt]
        row_token[:R] = torch.from_numpy(d["row_token"])
        slot_row[:p.T] = torch.from_numpy(d["slot_row"])
        counts.copy_(torch.from_numpy(d["counts"]))
        kept.copy_(torch.from_numpy(d["kept"]))
        offsets[:p.E + 1] = torch.from_numpy(d["offsets"])

    @staticmethod
    def mask_slots(p, topk_idx, offsets, keep, slot_row):
        # an assignment whose position inside its expert's block is past keep[e] drops
        for t in range(p.T):
            for j in range(p.k):
                r = int(slot_row[t, j])
                if r >= 0:
                    e = int(topk_idx[t, j])
                    if r - int(offsets[e]) >= int(keep[e]):
                        slot_row[t, j] = -1

    def expert_ffn(self, p, xin, in_offsets, W13, W2, h, out, ws):
        import oracle
        R = p.T
        off = in_offsets.numpy()
        eor = (np.searchsorted(off, np.arange(R), side="right") - 1).astype(np.int32)
        out[:R] = torch.from_numpy(oracle.expert_ffn(self.W1l, self.W3l, self.W2l,
                                                     self._f32(xin[:R]), eor))

    @staticmethod
    def combine(p, out, slot_row, topk_w, y):
        import oracle
        scale = p.E / p.k if p.rescale else 1.0
        y.copy_(torch.from_numpy(oracle.combine(out.numpy(), slot_row[:p.T].numpy(),
                                                topk_w[:p.T].numpy().astype(np.float64),
                                                scale)))

    def gate_stats(self, pg, counts_all, N, probs_sum, counts, f, P, loss):
        import oracle
        c = counts_all.numpy().sum(0).astype(np.int32)
        fe, Pe, L = oracle.gate_stats(pg.T, pg.k, c, probs_sum.numpy().astype(np.float64),
                                      self.lam)
        counts.copy_(torch.from_numpy(c))
        f.copy_(torch.from_numpy(fe))
        P.copy_(torch.from_numpy(Pe))
        loss[0] = L


def _ep_worker(rank, world, port, out_dir, cfg):
    """One rank of the layer: ExpertParallelMoE.forward over gloo, oracle arithmetic."""
    sys.path.insert(0, ROOT)
    from top_routing_grouped_noisy_b200.expert_parallel import ExpertParallelMoE
    dist.init_process_group("gloo", init_method="tcp://127.0.0.1:%d" % port, rank=rank,
                            world_size=world)
    try:
        Ts, d, E, k, m = cfg["Ts"], cfg["d"], cfg["E"], cfg["k"], cfg["m"]
        inp = _layer_inputs(Ts, d, E, m, cfg["seed"])
        a = sum(Ts[:rank])
        T = Ts[rank]
        t64 = lambda v: torch.from_numpy(v.astype(np.float64))
        El = E // world
        lo = rank * El
        ops = OracleOps(inp["W1"][lo:lo + El], inp["W3"][lo:lo + El], inp["W2"][lo:lo + El], 0.01)
        layer = ExpertParallelMoE(d, E, k, m, None, None, t64(inp["Wg"]), t64(inp["Wn"]), None,
                                  torch.float64, cfg["router"], cfg["capacity"], cfg["scope"],
                                  cfg["rescale"], 0.01, ops=ops)
        s = layer.forward(t64(inp["x"][a:a + T]), t64(inp["eps"][a:a + T]))
        np.save(os.path.join(out_dir, "y%d.npy" % rank), s.y.numpy())
        with open(os.path.join(out_dir, "r%d.json" % rank), "w") as fh:
            json.dump({"counts_all": s.counts_all_dev.tolist(),
                       "sums": s.sums[:E].tolist() + s.sums[-(s.sums.numel() // 2):][:E].tolist(),
                       "keep_all": s.ep.keep_all.tolist(),
                       "slot_row": s.slot_row[:T].tolist(),
                       "counts": s.counts_global.tolist(), "f": s.f.tolist(), "P": s.P.tolist(),
                       "loss": float(s.loss[0]), "T_all": s.T_all}, fh)
    finally:
        dist.destroy_process_group()


def _one_process_layer(inp, Ts, E, k, capacity, scope, router, rescale):
    """The oracle's layer on the ranks' batches (concatenated under GLOBAL, each rank's
    batch alone under LOCAL), with the gate weights rounded to f32 as the layer stores
    them; y per rank."""
    import oracle
    scale = E / k if rescale else 1.0
    spans = [(sum(Ts[:i]), sum(Ts[:i + 1])) for i in range(len(Ts))]
    groups = [(0, sum(Ts))] if scope == GLOBAL else spans
    y = np.zeros((sum(Ts), inp["x"].shape[1]))
    for a, b in groups:
        if b == a:
            continue
        r = oracle.router(inp["x"][a:b], inp["Wg"], inp["Wn"], inp["eps"][a:b], None, k, router)
        dsp = oracle.dispatch(r["idx"], E, capacity)
        R = dsp["R"]
        eor = (np.searchsorted(dsp["offsets"], np.arange(R), side="right") - 1).astype(np.int32)
        out = oracle.expert_ffn(inp["W1"], inp["W3"], inp["W2"],
                                np.ascontiguousarray(inp["x"][a:b][dsp["row_token"]]), eor) \
            if R else np.zeros((1, inp["x"].shape[1]))
        G32 = r["G"].astype(np.float32).astype(np.float64)
        y[a:b] = oracle.combine(out, dsp["slot_row"], G32, scale)
    return [y[a:b] for a, b in spans]


@pytest.mark.parametrize("world,Ts,E,k,capacity,scope,router,rescale", [
    (2, [37, 20], 4, 2, -1, GLOBAL, 0, False),
    (2, [37, 20], 4, 2, 9, GLOBAL, 0, True),
    (2, [30, 41], 8, 3, 5, LOCAL, 1, True),
    (4, [13, 0, 21, 8], 8, 2, 4, GLOBAL, 0, False),
    (4, [16, 16, 16, 16], 4, 1, 6, GLOBAL, 1, False),
])
def test_ep_layer_over_gloo_equals_one_process_layer(tmp_path, world, Ts, E, k, capacity, scope,
                                                      router, rescale):
    """ExpertParallelMoE.forward on every rank (its plan, slot mask, row exchange over
    gloo and gate statistics; the oracle doing the arithmetic) gives each rank's rows of
    the one-process layer bit for bit, and the statistics of all ranks' tokens."""
    import oracle
    cfg = dict(Ts=Ts, d=16, E=E, k=k, m=8, capacity=capacity, scope=scope, router=router,
               rescale=rescale, seed=sum(Ts) + E)
    port = 29700 + (os.getpid() * 7 + world + E) % 900
    mp.spawn(_ep_worker, args=(world, port, str(tmp_path), cfg), nprocs=world, join=True)
    inp = _layer_inputs(Ts, 16, E, 8, cfg["seed"])
    res = [json.load(open(tmp_path / ("r%d.json" % i))) for i in range(world)]
    ys = [np.load(tmp_path / ("y%d.npy" % i)) for i in range(world)]
    counts_all = np.array(res[0]["counts_all"])[:, :E]
    want = _one_process_layer(inp, Ts, E, k, capacity, scope, router, rescale)
    for i in range(world):
        # the same per-row fp64 arithmetic; only the rows' places differ
        assert ys[i].shape == want[i].shape
        assert np.array_equal(ys[i], want[i]), i
    full = oracle.forward(inp["x"], inp["Wg"], inp["W1"], inp["W3"], inp["W2"], k, router,
                          inp["Wn"], inp["eps"], None, capacity, rescale, 0.01)
    # statistics over all ranks' tokens (pre-drop counts, f32 token sums)
    assert np.array_equal(counts_all.sum(0), full["dispatch"]["counts"])
    for rr in res:
        assert rr["counts"] == full["dispatch"]["counts"].tolist()
        assert rr["T_all"] == sum(Ts)
        s = np.array(rr["sums"])
        np.testing.assert_allclose(s[:E], full["router"]["probs_sum"], rtol=1e-6)
        np.testing.assert_allclose(s[E:], full["router"]["importance"], rtol=1e-6)
        assert rr["loss"] == pytest.approx(full["L"], rel=1e-5)
    if scope == GLOBAL:
        assert np.array_equal(np.array(res[0]["keep_all"]).sum(0), full["dispatch"]["kept"])
    # every rank got the same plan
    for i in range(1, world):
        assert res[i]["keep_all"] == res[0]["keep_all"]
    if capacity >= 0:
        assert any(v == -1 for rr in res for row in rr["slot_row"] for v in row)


@pytest.mark.parametrize("N,E,k,capacity", [(2, 8, 2, 5), (4, 8, 3, 7), (8, 16, 4, 2), (2, 4, 1, 0)])
def test_plan_global_drops_equal_oracle_dispatch_of_concatenated_batch(N, E, k, capacity):
    """The plan's kept prefix of each (rank, expert) block, applied to every rank's
    dropless dispatch, keeps exactly the assignments the oracle's dispatch keeps on the
    ranks' batches concatenated in rank order."""
    import oracle
    rng = np.random.default_rng(N * 97 + E + k)
    Ts = [int(t) for t in rng.integers(0, 40, size=N)]
    idx_all = np.stack([rng.permutation(E)[:k] for _ in range(sum(Ts))]).astype(np.int32) \
        if sum(Ts) else np.zeros((0, k), np.int32)
    full = oracle.dispatch(idx_all, E, capacity)
    counts = []
    dsp = []
    a = 0
    for T in Ts:
        d = oracle.dispatch(idx_all[a:a + T], E, -1)
        dsp.append(d)
        counts.append(d["counts"])
        a += T
    pl = moe.moe_ep_plan(torch.from_numpy(np.array(counts, np.int32)), 0, capacity, GLOBAL)
    keep = pl.keep_all.numpy()
    a = 0
    for r, T in enumerate(Ts):
        sr = dsp[r]["slot_row"]
        ix = idx_all[a:a + T]
        mine = (sr >= 0) & (sr - dsp[r]["offsets"][ix] < keep[r][ix])
        np.testing.assert_array_equal(mine, full["slot_row"][a:a + T] >= 0)
        a += T


def _dying_worker(rank, world, port, out_dir):
    """Rank 1 leaves between the count gather and the row exchange (with nothing in
    flight); rank 0 must get an error from its exchange, not wait for ever."""
    import datetime
    sys.path.insert(0, ROOT)
    from top_routing_grouped_noisy_b200 import moe_ep_plan
    from top_routing_grouped_noisy_b200.expert_parallel import DistTransport
    dist.init_process_group("gloo", init_method="tcp://127.0.0.1:%d" % port, rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=10))
    tr = DistTransport()
    counts_all = tr.all_gather(torch.tensor([3, 2, 1, 4, 0], dtype=torch.int32))
    if rank == 1:
        os._exit(0)
    plan = moe_ep_plan(counts_all[:, :4].contiguous(), rank)
    src = torch.zeros(10, 8)
    dst = torch.zeros(max(plan.rows_in, 1), 8)
    err = None
    try:
        tr.exchange(src, plan.send_runs(), dst, plan.recv_runs())
    except Exception as e:  # the peer is gone: gloo reports it or the group times out
        err = type(e).__name__
    with open(os.path.join(out_dir, "dying.json"), "w") as fh:
        json.dump({"error": err}, fh)
    os._exit(0)


@pytest.mark.timeout(180)
def test_exchange_reports_a_rank_that_left(tmp_path):
    port = 30700 + os.getpid() % 900
    mp.spawn(_dying_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True)
    res = json.load(open(tmp_path / "dying.json"))
    assert res["error"] is not None
