"""Expert-parallel layer on the GPU through the C ABI ("Llama 3 Meets MoE", section
"训练框架", Expert Parallelism).

The ranks are emulated on one GPU: the layer objects of N ranks run their steps
in lockstep in one process on one device, and a copy
transport (below) stands in for the collectives by matching each rank's send
runs with the receiving rank's runs of the same expert.  No kernel waits for
another rank.  The result is checked against the fp64 oracle on the ranks'
batches concatenated in rank order (capacity scope GLOBAL) or on each rank's batch
(LOCAL).  A one-rank NCCL process group (its own subprocess) runs the real
torch.distributed transport and must reproduce moe_forward bit for bit.
"""
import json
import os
import subprocess
import sys
from types import SimpleNamespace

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

import harness as H  # noqa: E402
import oracle  # noqa: E402
import top_routing_grouped_noisy_b200 as moe  # noqa: E402
import workloads as wl  # noqa: E402
from top_routing_grouped_noisy_b200.expert_parallel import ExpertParallelMoE  # noqa: E402

pytestmark = pytest.mark.gpu
W = wl.Workload
GLOBAL, LOCAL = moe.EP_CAPACITY_GLOBAL, moe.EP_CAPACITY_LOCAL


def _lockstep_gather(steps):
    counts_all = torch.stack([s.counts_T for s in steps])
    total = torch.stack([s.sums for s in steps]).sum(0)
    for s in steps:
        s.counts_all_dev = counts_all.clone()
        s.sums.copy_(total)


def _lockstep_exchange(steps, src, src_runs, dst, dst_runs):
    for q, sq in enumerate(steps):
        for p, row, n, e in getattr(sq, src_runs):
            if n == 0:
                continue
            m = [(r2, n2) for (pp, r2, n2, e2) in getattr(steps[p], dst_runs) if pp == q and e2 == e]
            assert len(m) == 1 and m[0][1] == n
            getattr(steps[p], dst)[m[0][0]:m[0][0] + n].copy_(getattr(sq, src)[row:row + n])


def _run_lockstep(w, inp, Ts, N, capacity, scope):
    dev = "cuda"
    W13_e, W2_e = H.gpu_weights(w, inp)
    E, El = w.E, w.E // N
    g = lambda n: None if inp.get(n) is None else inp[n].to(dev)
    x, eps = g("x"), g("eps")
    layers, steps = [], []
    for r in range(N):
        lo = r * El
        layers.append(ExpertParallelMoE(
            w.d, E, w.k, w.m, W13_e.view(E, -1)[lo:lo + El].reshape(-1),
            W2_e.view(E, -1)[lo:lo + El].reshape(-1), g("Wg"), g("Wnoise"), g("bias"),
            wl.torch_dtype(w), w.router, capacity, scope, w.rescale, w.lam, rank=r, world=N))
    for r in range(N):
        a, b = sum(Ts[:r]), sum(Ts[:r + 1])
        steps.append(layers[r].begin(x[a:b], None if eps is None else eps[a:b]))
    _lockstep_gather(steps)
    for r in range(N):
        layers[r].plan(steps[r])
    _lockstep_exchange(steps, "x_perm", "send_runs", "xin", "recv_runs")
    for r in range(N):
        layers[r].experts(steps[r])
    _lockstep_exchange(steps, "out_local", "recv_runs", "out", "send_runs")
    for r in range(N):
        layers[r].finish(steps[r])
    torch.cuda.synchronize()
    for L in layers:
        for ws in (L._ws_route, L._ws_ffn):
            if ws is not None:
                assert moe.moe_get_device_status(ws) == 0
    return steps


def _cat(steps, name, T):
    parts = [getattr(s, name)[:s.T] for s in steps if s.T > 0]
    return torch.cat(parts) if parts else None


CASES = {
    # name: (workload over all ranks, tokens per rank, ranks, capacity scope)
    "n2_e8_global_cap": (W("n2", T=1223, d=256, d_ff=1024, E=8, k=2, noisy=True, rescale=True,
                           cf=1.0, seed=61), [700, 523], 2, GLOBAL),
    "n4_e8_st_bias_empty_rank": (W("n4", T=827, d=200, d_ff=800, E=8, k=2, router=wl.ST,
                                   noisy=True, bias=True, cf=1.25, seed=62),
                                 [300, 0, 450, 77], 4, GLOBAL),
    "n2_e16_k4_local": (W("n2l", T=900, d=128, d_ff=16 * 48, E=16, k=4, noisy=True,
                          rescale=True, cf=1.0, seed=63), [450, 450], 2, LOCAL),
    "n8_e8_small_router": (W("n8", T=512, d=256, d_ff=8 * 96, E=8, k=2, noisy=True, seed=64),
                           [64] * 8, 8, GLOBAL),
    "n4_decode_rows": (W("n4d", T=14, d=264, d_ff=8 * 120, E=8, k=2, noisy=True, rescale=True,
                         seed=65), [5, 3, 4, 2], 4, GLOBAL),
    "n2_f32_cap": (W("n2f", T=300, d=64, d_ff=4 * 40, E=4, k=2, dtype="f32", noisy=True,
                     cf=0.75, seed=66), [120, 180], 2, GLOBAL),
    "n2_pair_rows": (W("n2p", T=4400, d=256, d_ff=8 * 256, E=8, k=2, noisy=True, rescale=True,
                       seed=67), [2200, 2200], 2, GLOBAL),
}


@pytest.mark.parametrize("name", list(CASES))
def test_ep_lockstep_matches_oracle(name):
    w, Ts, N, scope = CASES[name]
    assert sum(Ts) == w.T
    inp = wl.make_inputs(w)
    C = H.capacity_of(w) if scope == GLOBAL else (
        moe.moe_capacity(Ts[0], w.E, w.cf) if w.cf >= 0 else -1)
    if scope == LOCAL:
        assert len(set(Ts)) == 1
    steps = _run_lockstep(w, inp, Ts, N, C, scope)
    ns = SimpleNamespace(topk_idx=_cat(steps, "topk_idx", w.T), topk_w=_cat(steps, "topk_w", w.T),
                         probs_sum=steps[0].probs_sum, importance=steps[0].importance,
                         y=_cat(steps, "y", w.T), loss=steps[0].loss)
    r, ties = H.check_routing(w, inp, ns, 1e-5 if w.dtype == "f32" else 5e-5)
    gi = ns.topk_idx.cpu().numpy()
    OW = H.oracle_weights(w, inp)
    sr_gpu = _cat(steps, "slot_row", w.T).cpu().numpy()
    if scope == GLOBAL:
        dsp = oracle.dispatch(gi, w.E, C)
        # the kept set equals the one-device layer's on the concatenated batch
        np.testing.assert_array_equal(sr_gpu < 0, dsp["slot_row"] < 0)
        np.testing.assert_array_equal(steps[0].counts_global.cpu().numpy(), dsp["counts"])
        H.check_y(w, ns, r, dsp, OW, np.nonzero(~ties)[0], inp=inp)
    else:
        a = 0
        for s in steps:
            dsp_r = oracle.dispatch(gi[a:a + s.T], w.E, C)
            np.testing.assert_array_equal(sr_gpu[a:a + s.T] < 0, dsp_r["slot_row"] < 0)
            inp_r = dict(inp, x=inp["x"][a:a + s.T])
            tok = np.nonzero(~ties[a:a + s.T])[0]
            H.check_y(w.with_(T=s.T), SimpleNamespace(y=s.y), {"G": r["G"][a:a + s.T]}, dsp_r,
                      OW, tok, inp=inp_r)
            a += s.T
    H.check_loss(w, ns, r)
    for s in steps[1:]:
        assert torch.equal(s.loss, steps[0].loss)
        assert torch.equal(s.counts_global, steps[0].counts_global)
    if C >= 0 and name != "n2_pair_rows":
        assert (sr_gpu < 0).any()


def _one_rank_main(out_path):
    """Runs in its own process: a one-rank NCCL group, the layer with the
    torch.distributed transport, and moe_forward on the same batch."""
    import datetime
    import torch.distributed as dist
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", init_method="file://%s.store" % out_path, rank=0,
                            world_size=1, timeout=datetime.timedelta(seconds=60))
    res = {}
    try:
        for name, w in [("cap", W("one_cap", T=700, d=256, d_ff=1024, E=8, k=2, noisy=True,
                                  rescale=True, cf=1.0, seed=71)),
                        ("st_bias", W("one_st", T=333, d=200, d_ff=800, E=8, k=3, router=wl.ST,
                                      noisy=True, bias=True, seed=72))]:
            inp = wl.make_inputs(w)
            p, bufs, ws, status, (W13_e, W2_e) = H.run_forward(w, inp)
            g = lambda n: None if inp.get(n) is None else inp[n].to("cuda")
            L = ExpertParallelMoE(w.d, w.E, w.k, w.m, W13_e, W2_e, g("Wg"), g("Wnoise"),
                                  g("bias"), wl.torch_dtype(w), w.router, p.capacity, GLOBAL,
                                  w.rescale, w.lam)
            s = L.forward(g("x"), g("eps"))
            torch.cuda.synchronize()
            res[name] = {
                "status": status,
                "y": bool(torch.equal(s.y, bufs.y)),
                "drops": bool(torch.equal(s.slot_row < 0, bufs.slot_row < 0)),
                "counts": bool(torch.equal(s.counts_global, bufs.counts)),
                "loss": bool(torch.equal(s.loss, bufs.loss)),
                "f": bool(torch.equal(s.f, bufs.f)),
                "P": bool(torch.equal(s.P, bufs.P)),
                "importance": bool(torch.equal(s.importance, bufs.importance)),
                "rows_in": s.R_in,
                "R": int(bufs.offsets[w.E]),
            }
    finally:
        dist.destroy_process_group()
    with open(out_path, "w") as fh:
        json.dump(res, fh)


def test_ep_one_rank_nccl_reproduces_forward(tmp_path):
    out = tmp_path / "one_rank.json"
    env = dict(os.environ, MASTER_ADDR="127.0.0.1", NCCL_NVLS_ENABLE="0")
    rc = subprocess.run([sys.executable, os.path.abspath(__file__), "--one-rank", str(out)],
                        env=env, capture_output=True, text=True, timeout=300)
    assert rc.returncode == 0, rc.stderr[-3000:]
    res = json.load(open(out))
    for name, v in res.items():
        assert v["status"] == 0
        assert v["rows_in"] == v["R"]
        for key in ("y", "drops", "counts", "loss", "f", "P", "importance"):
            assert v[key], (name, key)


if __name__ == "__main__":
    if len(sys.argv) == 3 and sys.argv[1] == "--one-rank":
        _one_rank_main(sys.argv[2])
