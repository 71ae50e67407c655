"""Shared test plumbing: run a layer through the C ABI on the GPU and check every
step against the fp64 oracle on the same seeded inputs.

Parity rules (per the layer's statement of accuracy):
  * expert indices bit-exact, except tokens whose k-th and (k+1)-th routing logits,
    rounded to f32, lie within 1e-5 relative of each other (near ties, where the
    order of f32 accumulation may legitimately decide);
  * dispatch tables bit-exact when the oracle dispatches the GPU's own indices;
  * x_perm bit-exact (a copy);
  * y: max|y - y_ref| / max|y_ref| <= 1e-2 for bf16 layers, <= 1e-5 for f32 layers;
  * L_balance within 1e-4 relative.
"""
import numpy as np
import torch

import oracle
import top_routing_grouped_noisy_b200 as moe
import workloads as wl

TIE_REL = 1e-5
Y_TOL = {"bf16": 1e-2, "f32": 1e-5}
LOSS_REL = 1e-4


def raw(t):
    return wl.to_numpy_raw(t)


def f64(t):
    """Exact float64 values of a bf16/f32 tensor."""
    return t.detach().cpu().to(torch.float64).numpy()


def capacity_of(w: wl.Workload) -> int:
    return moe.moe_capacity(w.T, w.E, w.cf) if w.cf >= 0 else -1


def unpack_w13(W13_e, E, m, d):
    m16 = (m + 15) // 16 * 16
    A = W13_e.view(E, m16 // 16, 2, 16, d)
    return A[:, :, 0].reshape(E, m16, d)[:, :m], A[:, :, 1].reshape(E, m16, d)[:, :m]


def unpack_w2(W2_e, E, m, d):
    m8 = (m + 7) // 8 * 8
    return W2_e.view(E, d, m8)[:, :, :m]


def gpu_weights(w: wl.Workload, inp: dict, ws=None):
    """a0 on the GPU: packed expert weights for workload w."""
    dev = "cuda"
    if w.partition == wl.COPY and "W1s" in inp:
        return moe.moe_partition_experts(inp["W1s"].to(dev), inp["W3s"].to(dev),
                                         inp["W2s"].to(dev), w.E, moe.STACKED, ws=ws)
    if w.partition == wl.COPY:
        return moe.moe_partition_experts(inp["W1"].to(dev), inp["W3"].to(dev),
                                         inp["W2"].to(dev), w.E, moe.COPY, ws=ws)
    return moe.moe_partition_experts(inp["W1"].to(dev), inp["W3"].to(dev), inp["W2"].to(dev),
                                     w.E, moe.DISJOINT, perm=inp["perm"].to(dev), ws=ws)


def oracle_weights(w: wl.Workload, inp: dict):
    """Per-expert standard-layout weights for the oracle (same element values)."""
    if w.partition == wl.COPY and "W1s" in inp:
        return raw(inp["W1s"]), raw(inp["W3s"]), raw(inp["W2s"])
    mode = oracle.COPY if w.partition == wl.COPY else oracle.DISJOINT
    perm = None if inp["perm"] is None else raw(inp["perm"])
    return oracle.partition(raw(inp["W1"]), raw(inp["W3"]), raw(inp["W2"]), w.E, mode, perm)


def layer_params(w: wl.Workload, capacity=None):
    C = capacity_of(w) if capacity is None else capacity
    return moe.params(w.T, w.d, w.E, w.k, w.m, wl.torch_dtype(w), w.router, C, w.rescale, w.lam)


def run_forward(w: wl.Workload, inp: dict, capacity=None, weights=None):
    """Whole layer through moe_forward; returns (params, buffers, workspace, status)."""
    dev = "cuda"
    p = layer_params(w, capacity)
    ws = moe.Workspace(p)
    W13_e, W2_e = weights if weights is not None else gpu_weights(w, inp, ws)
    bufs = moe.ForwardBuffers(p)
    g = lambda n: None if inp.get(n) is None else inp[n].to(dev)
    moe.moe_forward(p, g("x"), g("Wg"), W13_e, W2_e, ws, bufs, Wnoise=g("Wnoise"),
                    noise=g("eps"), bias=g("bias"))
    torch.cuda.synchronize()
    status = moe.moe_get_device_status(ws)
    return p, bufs, ws, status, (W13_e, W2_e)


def near_tie_tokens(H: np.ndarray, k: int) -> np.ndarray:
    """Tokens whose k-th and (k+1)-th f32-rounded routing logits are within TIE_REL."""
    T, E = H.shape
    if k >= E or T == 0:
        return np.zeros(T, bool)
    h32 = H.astype(np.float32).astype(np.float64)
    s = -np.sort(-h32, axis=1)
    a, b = s[:, k - 1], s[:, k]
    return np.abs(a - b) <= TIE_REL * np.maximum(np.abs(a), np.abs(b))


def check_routing(w, inp, bufs, G_atol):
    """a1 parity; returns (oracle router result, near-tie mask)."""
    r = oracle.router(raw(inp["x"]), raw(inp["Wg"]),
                      None if inp.get("Wnoise") is None else raw(inp["Wnoise"]),
                      None if inp.get("eps") is None else raw(inp["eps"]),
                      None if inp.get("bias") is None else raw(inp["bias"]), w.k, w.router)
    ties = near_tie_tokens(r["H"], w.k)
    gi = bufs.topk_idx.cpu().numpy()
    gw = bufs.topk_w.cpu().numpy().astype(np.float64)
    ok = ~ties
    np.testing.assert_array_equal(gi[ok], r["idx"][ok])
    np.testing.assert_allclose(gw[ok], r["G"][ok], rtol=0, atol=G_atol)
    if ties.any():  # a near tie may swap order; the chosen set is still a valid top-k
        for t in np.nonzero(ties)[0]:
            h32 = r["H"][t].astype(np.float32).astype(np.float64)
            kth = -np.sort(-h32)[w.k - 1]
            assert (h32[gi[t]] >= kth - 2 * TIE_REL * abs(kth)).all()
    T = w.T
    ps = bufs.probs_sum.cpu().numpy().astype(np.float64)
    imp = bufs.importance.cpu().numpy().astype(np.float64)
    scale = max(T, 1)
    np.testing.assert_allclose(ps, r["probs_sum"], rtol=0, atol=1e-4 * scale / w.E + 1e-6)
    np.testing.assert_allclose(imp, r["importance"], rtol=0,
                               atol=1e-4 * scale / w.E + 1e-6 + 2.0 * ties.sum())
    return r, ties


def check_dispatch(w, inp, p, bufs):
    """a2 parity: the oracle dispatches the GPU's indices; everything bit-exact."""
    gi = bufs.topk_idx.cpu().numpy()
    d = oracle.dispatch(gi, w.E, p.capacity)
    assert bufs.counts.cpu().numpy().tolist() == d["counts"].tolist()
    assert bufs.kept.cpu().numpy().tolist() == d["kept"].tolist()
    assert bufs.offsets.cpu().numpy().tolist() == d["offsets"].tolist()
    R = d["R"]
    np.testing.assert_array_equal(bufs.row_token[:R].cpu().numpy(), d["row_token"])
    np.testing.assert_array_equal(bufs.slot_row.cpu().numpy(), d["slot_row"])
    if R:
        xp = bufs.x_perm[:R].cpu()
        xr = inp["x"].cpu()[torch.from_numpy(d["row_token"]).long()]
        assert torch.equal(xp.view(torch.int16) if xp.dtype == torch.bfloat16 else xp,
                           xr.view(torch.int16) if xr.dtype == torch.bfloat16 else xr)
    return d


def x_rows_of(inp, dsp, rows):
    """The activations of kept rows, taken from x through the oracle's row tables."""
    x = raw(inp["x"])
    return np.ascontiguousarray(x[dsp["row_token"][rows]])


def rel_err(a, b):
    den = np.abs(b).max() if b.size else 0.0
    return float(np.abs(a - b).max() / den) if den > 0 else float(np.abs(a - b).max())


def check_expert_rows(w, bufs, dsp, OW, rows=None, inp=None):
    """a3/a4 parity on kept rows (the GPU's x_perm through the oracle's experts)."""
    R = dsp["R"]
    if R == 0:
        return 0.0
    if rows is None:
        rows = np.arange(R)
    expert_of_row = np.searchsorted(dsp["offsets"], rows, side="right") - 1
    x_rows = x_rows_of(inp, dsp, rows)
    out_ref, h_ref = oracle.expert_ffn(*OW, x_rows, expert_of_row, want_h=True)
    out_g = f64(bufs.out[torch.from_numpy(rows).long().cuda()])
    h_g = f64(bufs.h[torch.from_numpy(rows).long().cuda()][:, :w.m])
    tol = Y_TOL[w.dtype]
    eh, eo = rel_err(h_g, h_ref), rel_err(out_g, out_ref)
    assert eh <= tol, "h rel err %g" % eh
    assert eo <= tol, "out rel err %g" % eo
    return eo


def check_y(w, bufs, r, dsp, OW, tokens, inp=None):
    """End-to-end y for `tokens` (non-tie tokens): y_ref from the oracle's experts and
    gate weights over the dispatch of the GPU's indices."""
    tokens = np.asarray(tokens, np.int64)
    if len(tokens) == 0:
        return 0.0
    sr = dsp["slot_row"][tokens]
    rows = np.unique(sr[sr >= 0])
    y_g = f64(bufs.y[torch.from_numpy(tokens).cuda()])
    if len(rows):
        expert_of_row = np.searchsorted(dsp["offsets"], rows, side="right") - 1
        x_rows = x_rows_of(inp, dsp, rows)
        out_u = oracle.expert_ffn(*OW, x_rows, expert_of_row)
        remap = {int(v): i for i, v in enumerate(rows)}
        sr_local = np.vectorize(lambda v: remap.get(int(v), -1))(sr).astype(np.int32)
    else:
        out_u = np.zeros((1, w.d))
        sr_local = np.full_like(sr, -1)
    scale = w.E / w.k if w.rescale else 1.0
    y_ref = oracle.combine(out_u, sr_local, r["G"][tokens], scale)
    e = rel_err(y_g, y_ref)
    assert e <= Y_TOL[w.dtype], "y rel err %g (tol %g)" % (e, Y_TOL[w.dtype])
    return e


def check_loss(w, bufs, r):
    """L_balance from the oracle's own routing (pre-drop counts, probs of H)."""
    od = oracle.dispatch(r["idx"], w.E, -1)
    _, _, L = oracle.gate_stats(w.T, w.k, od["counts"], r["probs_sum"], w.lam)
    Lg = float(bufs.loss.cpu()[0])
    assert abs(Lg - L) <= LOSS_REL * abs(L) + 1e-12, (Lg, L)
    return Lg, L
