"""Backward of the MoE layer on the GPU against the fp64 oracle's backward (itself
pinned by finite differences): the gradient of l(y) + c L_balance given dy, for the
combine, the two expert GEMMs with the SwiGLU backward, the router (Mixtral / ST,
softplus noise, balance term) and the input.  bf16 gradients: max|err| / max|ref|
<= 2e-2 (bf16 rounding of out, h, d_out, dh, dGU on the GPU against f64)."""
import numpy as np
import pytest
import torch

import harness as H
import oracle
import top_routing_grouped_noisy_b200 as moe
import workloads as wl

pytestmark = pytest.mark.gpu

TOL = 2e-2
W = wl.Workload
CASES = {
    "bwd_mid": W("bwd_mid", T=1000, d=512, d_ff=2752, E=8, k=2, noisy=True, rescale=True,
                 lam=0.01, seed=80),
    "bwd_st_bias_cap": W("bwd_st_bias_cap", T=700, d=256, d_ff=1024, E=8, k=2, router=wl.ST,
                         noisy=True, bias=True, cf=1.0, rescale=True, lam=0.05, seed=81),
    "bwd_ragged": W("bwd_ragged", T=333, d=200, d_ff=400, E=4, k=2, noisy=True, seed=82),
    "bwd_decode": W("bwd_decode", T=8, d=256, d_ff=1088, E=8, k=2, rescale=True, seed=83),
    "bwd_e16k4": W("bwd_e16k4", T=512, d=256, d_ff=1024, E=16, k=4, router=wl.ST, noisy=True,
                   bias=True, lam=0.01, seed=84),
    "bwd_copy": W("bwd_copy", T=256, d=128, d_ff=256, E=4, k=2, partition=wl.COPY, seed=85),
    "bwd_e64": W("bwd_e64", T=300, d=128, d_ff=1024, E=64, k=2, noisy=True, bias=True, lam=0.05,
                 seed=87),
    "bwd_e12_ragged_d": W("bwd_e12_ragged_d", T=150, d=72, d_ff=480, E=12, k=3, router=wl.ST,
                          noisy=True, seed=88),
    # T*k >= 4096: the 2-SM (cta_group::2) backward GEMMs
    "bwd_pair_st_cap": W("bwd_pair_st_cap", T=2100, d=256, d_ff=1024, E=8, k=2, router=wl.ST,
                         noisy=True, bias=True, cf=1.0, rescale=True, lam=0.05, seed=92),
    "bwd_pair_e16k4": W("bwd_pair_e16k4", T=2048, d=136, d_ff=576, E=16, k=4, noisy=True,
                        seed=93),
}


def rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.abs(a - b).max() / max(np.abs(b).max(), 1e-30))


def _run(w, inp, dLb=1.0):
    dev = "cuda"
    p, bufs, ws, st, (W13_e, W2_e) = H.run_forward(w, inp)
    assert st == 0
    g = lambda n: None if inp.get(n) is None else inp[n].to(dev)
    dy = wl.make_grad_output(w, w.seed + 1).to(dev)
    gb = moe.BackwardBuffers(p, w.noisy, w.bias)
    wsb = moe.Workspace(p, nbytes=moe.moe_backward_workspace_size(p))
    moe.moe_backward(p, g("x"), g("Wg"), W13_e, W2_e, bufs, gb, dy, wsb, Wnoise=g("Wnoise"),
                     noise=g("eps"), bias=g("bias"), dLb=dLb)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(wsb) == 0
    return p, bufs, gb, dy


def _oracle(w, inp, dy, dLb=1.0):
    W1e, W3e, W2e = H.oracle_weights(w, inp)
    r = lambda n: None if inp.get(n) is None else H.raw(inp[n])
    eps = None if inp.get("eps") is None else inp["eps"].numpy()
    bias = None if inp.get("bias") is None else inp["bias"].numpy()
    rt = oracle.MIXTRAL if w.router == wl.MIXTRAL else oracle.ST
    return oracle.backward(H.raw(inp["x"]), H.raw(inp["Wg"]), W1e, W3e, W2e, w.k, H.f64(dy), rt,
                           r("Wnoise"), eps, bias, H.capacity_of(w), w.rescale, w.lam, dLb)


def _check(w, inp, p, bufs, gb, dy, dLb=1.0):
    ref = _oracle(w, inp, dy.cpu(), dLb)
    fwd = ref["fwd"]
    idx = bufs.topk_idx.cpu().numpy()
    assert (idx == fwd["router"]["idx"]).all(), "routing differs: pick a seed without near ties"
    R = int(fwd["dispatch"]["R"])
    assert int(bufs.offsets[-1]) == R
    m, d, E = w.m, w.d, w.E
    errs = {
        "dG": rel(gb.dG.cpu().numpy(), ref["dG"]),
        "d_out": rel(H.f64(gb.d_out[:R]), ref["d_out"]),
        "dh": rel(H.f64(gb.dh[:R, :m]), ref["dh"]),
        "dx_perm": rel(H.f64(gb.dx_perm[:R]), ref["dx_rows"]),
        "dx": rel(H.f64(gb.dx), ref["dx"]),
        "dWg": rel(gb.dWg.cpu().numpy(), ref["dWg"]),
    }
    dW1, dW3 = H.unpack_w13(gb.dW13_e, E, m, d)
    errs["dW1e"] = rel(H.f64(dW1), ref["dW1e"])
    errs["dW3e"] = rel(H.f64(dW3), ref["dW3e"])
    errs["dW2e"] = rel(H.f64(H.unpack_w2(gb.dW2_e, E, m, d)), ref["dW2e"])
    if gb.dWnoise is not None:
        errs["dWnoise"] = rel(gb.dWnoise.cpu().numpy(), ref["dWnoise"])
    if gb.dbias is not None:
        errs["dbias"] = rel(gb.dbias.cpu().numpy(), ref["dbias"])
    bad = {k: v for k, v in errs.items() if not v <= TOL}
    assert not bad, (w.name, errs)
    # the padding of the packed gradients is zero, like the packed weights
    m16, m8 = (m + 15) // 16 * 16, (m + 7) // 8 * 8
    A = gb.dW13_e.view(E, m16 // 16, 2, 16, d).permute(0, 2, 1, 3, 4).reshape(E, 2, m16, d)
    assert (A[:, :, m:] == 0).all()
    assert (gb.dW2_e.view(E, d, m8)[:, :, m:] == 0).all()
    return errs


@pytest.mark.parametrize("name", list(CASES))
def test_backward_parity(name):
    w = CASES[name]
    inp = wl.make_inputs(w)
    p, bufs, gb, dy = _run(w, inp)
    _check(w, inp, p, bufs, gb, dy)


def test_expert_without_rows_gets_zero_gradient():
    """A large negative bias keeps the last expert unselected: its weight gradient
    (the K-grouped GEMM with no K blocks) is zero, the others match the oracle."""
    w = W("bwd_idle", T=300, d=256, d_ff=1024, E=8, k=2, noisy=True, bias=True, lam=0.02,
          seed=86)
    inp = wl.make_inputs(w)
    inp["bias"][w.E - 1] = -1.0e4
    p, bufs, gb, dy = _run(w, inp)
    assert int(bufs.counts[w.E - 1]) == 0
    dW1, dW3 = H.unpack_w13(gb.dW13_e, w.E, w.m, w.d)
    assert (dW1[w.E - 1] == 0).all() and (dW3[w.E - 1] == 0).all()
    assert (H.unpack_w2(gb.dW2_e, w.E, w.m, w.d)[w.E - 1] == 0).all()
    _check(w, inp, p, bufs, gb, dy)


def test_steps_equal_the_whole_backward():
    """The step calls in order give bit-identical results to moe_backward."""
    w = CASES["bwd_st_bias_cap"]
    inp = wl.make_inputs(w)
    p, bufs, gb, dy = _run(w, inp)
    dev = "cuda"
    g = lambda n: None if inp.get(n) is None else inp[n].to(dev)
    W13_e, W2_e = H.gpu_weights(w, inp)
    s = moe.BackwardBuffers(p, w.noisy, w.bias)
    ws = moe.Workspace(p, nbytes=moe.moe_backward_workspace_size(p))
    moe.moe_combine_backward(p, dy, bufs.out, bufs.slot_row, bufs.topk_w, s.d_out, s.dG)
    moe.moe_expert_down_backward(p, s.d_out, bufs.h, bufs.offsets, W2_e, s.dh, s.dW2_e, ws)
    moe.moe_expert_up_backward(p, bufs.x_perm, s.dh, bufs.offsets, W13_e, s.dx_perm, s.dW13_e,
                               ws)
    moe.moe_route_backward(p, g("x"), g("Wg"), bufs.topk_idx, bufs.topk_w, s.dG, bufs.counts,
                           s.dx_perm, bufs.slot_row, s.dx, s.dWg, ws, Wnoise=g("Wnoise"),
                           noise=g("eps"), bias=g("bias"), dWnoise=s.dWnoise, dbias=s.dbias)
    torch.cuda.synchronize()
    for n in ("dx", "dWg", "dWnoise", "dbias", "dW13_e", "dW2_e", "dG"):
        assert torch.equal(getattr(s, n), getattr(gb, n)), n
    R = int(bufs.offsets[-1])  # row buffers: rows past R are unused
    for n in ("d_out", "dh", "dx_perm"):
        assert torch.equal(getattr(s, n)[:R], getattr(gb, n)[:R]), n


# --------------------------------------------------------------------------- residual layer

RES_CASES = {
    "res_bwd_mid": W("res_bwd_mid", T=600, d=256, d_ff=1152, E=8, k=2, noisy=True, rescale=True,
                     shared=128, lam=0.02, seed=90),
    "res_bwd_st_cap": W("res_bwd_st_cap", T=400, d=200, d_ff=840, E=4, k=2, router=wl.ST,
                        noisy=True, bias=True, cf=1.0, shared=40, seed=91),
}


@pytest.mark.parametrize("name", list(RES_CASES))
def test_residual_backward_parity(name):
    """y = FFN_S(x) + s sum G E(x): the routed gradients, the shared block's weight
    gradients and the total dx against the oracle."""
    w = RES_CASES[name]
    inp = wl.make_inputs(w)
    dev = "cuda"
    p = H.layer_params(w)
    ws = moe.Workspace(p)
    g = lambda n: None if inp.get(n) is None else inp[n].to(dev)
    W13_e, W2_e, W13_s, W2_s = moe.moe_partition_residual(
        g("W1"), g("W3"), g("W2"), w.E, g("shared_idx"), g("perm_rest"), ws=ws)
    b = moe.ForwardBuffers(p)
    h_s = torch.empty(w.T, moe.h_ld(w.shared), dtype=torch.bfloat16, device=dev)
    out_s = torch.empty(w.T, w.d, dtype=torch.bfloat16, device=dev)
    moe.moe_forward_residual(p, g("x"), g("Wg"), W13_e, W2_e, W13_s, W2_s, w.shared, ws, b, h_s,
                             out_s, Wnoise=g("Wnoise"), noise=g("eps"), bias=g("bias"))
    dy = wl.make_grad_output(w, w.seed + 1).to(dev)
    gb = moe.BackwardBuffers(p, w.noisy, w.bias)
    dh_s = torch.empty(w.T, moe.h_ld(w.shared), dtype=torch.bfloat16, device=dev)
    dx_s = torch.empty(w.T, w.d, dtype=torch.bfloat16, device=dev)
    dW13_s = torch.empty(moe.packed_w13_elems(1, w.shared, w.d), dtype=torch.bfloat16,
                         device=dev)
    dW2_s = torch.empty(moe.packed_w2_elems(1, w.shared, w.d), dtype=torch.bfloat16, device=dev)
    wsb = moe.Workspace(p, nbytes=moe.moe_backward_residual_workspace_size(p, w.shared))
    moe.moe_backward_residual(p, g("x"), g("Wg"), W13_e, W2_e, W13_s, W2_s, w.shared, h_s, b, gb,
                              dy, dh_s, dx_s, dW13_s, dW2_s, wsb, Wnoise=g("Wnoise"),
                              noise=g("eps"), bias=g("bias"))
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(wsb) == 0
    raw = H.raw
    experts, blk = oracle.partition_residual(raw(inp["W1"]), raw(inp["W3"]), raw(inp["W2"]),
                                             w.E, raw(inp["shared_idx"]), raw(inp["perm_rest"]))
    opt = lambda n: None if inp.get(n) is None else raw(inp[n])
    ref = oracle.backward_residual(raw(inp["x"]), raw(inp["Wg"]), experts, blk, w.k,
                                   H.f64(dy), w.router, opt("Wnoise"),
                                   None if inp.get("eps") is None else inp["eps"].numpy(),
                                   None if inp.get("bias") is None else inp["bias"].numpy(),
                                   p.capacity, w.rescale, w.lam, 1.0)
    assert (b.topk_idx.cpu().numpy() == ref["fwd"]["router"]["idx"]).all()
    m_s, m, d, E = w.shared, w.m, w.d, w.E
    dW1s, dW3s = H.unpack_w13(dW13_s, 1, m_s, d)
    dW1, dW3 = H.unpack_w13(gb.dW13_e, E, m, d)
    errs = {
        "dx": rel(H.f64(gb.dx), ref["dx"]),
        "dx_s": rel(H.f64(dx_s), ref["dx_s"]),
        "dh_s": rel(H.f64(dh_s[:, :m_s]), ref["dh_s"]),
        "dW1s": rel(H.f64(dW1s[0]), ref["dW1s"]),
        "dW3s": rel(H.f64(dW3s[0]), ref["dW3s"]),
        "dW2s": rel(H.f64(H.unpack_w2(dW2_s, 1, m_s, d)[0]), ref["dW2s"]),
        "dW1e": rel(H.f64(dW1), ref["dW1e"]),
        "dW3e": rel(H.f64(dW3), ref["dW3e"]),
        "dW2e": rel(H.f64(H.unpack_w2(gb.dW2_e, E, m, d)), ref["dW2e"]),
        "dWg": rel(gb.dWg.cpu().numpy(), ref["dWg"]),
    }
    bad = {k2: v for k2, v in errs.items() if not v <= TOL}
    assert not bad, (name, errs)


# --------------------------------------------------------------------------- full size

def test_full_size_sampled_backward():
    """moe_2of8 (T=16384, d=4096, 8 x 1376, top-2 noisy Mixtral, rescale, lambda=0.01) in the
    bench's launch configuration; the oracle routes the whole batch and then computes
    one by one: dx of 16 sampled tokens (their expert rows and the router term,
    normalised by the whole batch), and for 6 sampled (expert, neuron) pairs the rows of
    dW1 / dW3 and the column of dW2 summed over all of that expert's rows."""
    w = wl.WORKLOADS["moe_2of8"]
    inp = wl.make_inputs(w)
    p, bufs, gb, dy = _run(w, inp)
    raw = H.raw
    x, Wg, Wn = raw(inp["x"]), raw(inp["Wg"]), raw(inp["Wnoise"])
    eps = inp["eps"].numpy()
    r = oracle.router(x, Wg, Wn, eps, None, w.k, oracle.MIXTRAL)
    ties = H.near_tie_tokens(r["H"], w.k)
    gidx = bufs.topk_idx.cpu().numpy()
    assert ((gidx == r["idx"]).all(axis=1) | ties).all()
    assert ties.sum() < 32
    dsp = oracle.dispatch(r["idx"], w.E, -1)
    W1e, W3e, W2e = H.oracle_weights(w, inp)
    s = w.E / w.k
    dy64 = H.f64(dy)
    rng = np.random.default_rng(3)
    m, d, E, k = w.m, w.d, w.E, w.k
    # -- dx of sampled tokens
    toks = np.sort(rng.choice(np.nonzero(~ties)[0], 16, replace=False))
    sr = dsp["slot_row"][toks]
    rows = sr[sr >= 0]
    eor = np.searchsorted(dsp["offsets"], rows, side="right") - 1
    xr = x[dsp["row_token"][rows]]
    out_rows = oracle.expert_ffn(W1e, W3e, W2e, xr, eor)
    local = np.full(sr.shape, -1, np.int32)
    local[sr >= 0] = np.arange(len(rows))
    d_out, dG = oracle.combine_backward(out_rows, local, r["G"][toks], s, dy64[toks])
    eb = oracle.expert_ffn_backward(W1e, W3e, W2e, xr, eor, d_out)
    rb = oracle.router_backward_tokens(x[toks], Wg, r["idx"][toks], r["G"][toks], dG,
                                       dsp["counts"], k, w.T, oracle.MIXTRAL, Wn, eps[toks], None,
                                       w.lam, 1.0)
    dx_ref = rb["dx"].copy()
    for a, (t_i, j) in enumerate(zip(*np.nonzero(sr >= 0))):
        dx_ref[t_i] += eb["dx_rows"][local[t_i, j]]
    e_dx = rel(H.f64(gb.dx[torch.from_numpy(toks).cuda()]), dx_ref)
    assert e_dx <= TOL, e_dx
    # -- sampled neurons of three experts
    dW1, dW3 = H.unpack_w13(gb.dW13_e, E, m, d)
    dW2 = H.unpack_w2(gb.dW2_e, E, m, d)
    worst = 0.0
    for e in rng.choice(E, 3, replace=False):
        rows_e = np.arange(dsp["offsets"][e], dsp["offsets"][e + 1])
        loc = np.full(dsp["slot_row"].shape, -1, np.int32)
        hit = (dsp["slot_row"] >= dsp["offsets"][e]) & (dsp["slot_row"] < dsp["offsets"][e + 1])
        loc[hit] = dsp["slot_row"][hit] - dsp["offsets"][e]
        d_out_e, _ = oracle.combine_backward(np.zeros((len(rows_e), d)), loc, r["G"], s, dy64)
        xr_e = x[dsp["row_token"][rows_e]]
        for i in rng.choice(m, 2, replace=False):
            d1, d3, d2 = oracle.neuron_wgrad(W1e, W3e, W2e, int(e), int(i), xr_e, d_out_e)
            worst = max(worst, rel(H.f64(dW1[e, i]), d1), rel(H.f64(dW3[e, i]), d3),
                        rel(H.f64(dW2[e, :, i]), d2))
    assert worst <= TOL, worst
