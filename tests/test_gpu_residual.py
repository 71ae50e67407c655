"""Residual MoE (shared neurons plus disjoint experts) on the GPU against the fp64
oracle: y = FFN_S(x) + s sum_j G_j E_j(x), with the shared block run as a
one-expert grouped GEMM over all tokens ("LLaMA-MoE v2", section 共享神经元划分)."""
import numpy as np
import pytest
import torch

import harness as H
import oracle
import top_routing_grouped_noisy_b200 as moe
import workloads as wl

pytestmark = pytest.mark.gpu

W = wl.Workload
CASES = {
    "res_mid": W("res_mid", T=1000, d=512, d_ff=2752, E=8, k=2, noisy=True, rescale=True,
                 shared=352, seed=50),
    "res_pair_st_cap": W("res_pair_st_cap", T=2100, d=256, d_ff=2048, E=8, k=2, router=wl.ST,
                         noisy=True, bias=True, cf=1.0, rescale=True, shared=256, seed=51),
    "res_decode": W("res_decode", T=8, d=256, d_ff=1088, E=8, k=2, rescale=True, shared=128,
                    seed=52),
    "res_ragged": W("res_ragged", T=333, d=200, d_ff=840, E=4, k=2, noisy=True, shared=40,
                    seed=53),
    "res_f32": W("res_f32", T=190, d=96, d_ff=400, E=8, k=2, dtype="f32", noisy=True,
                 rescale=True, shared=80, seed=54),
}


def _weights(w, inp, ws):
    dev = "cuda"
    W13_e, W2_e, W13_s, W2_s = moe.moe_partition_residual(
        inp["W1"].to(dev), inp["W3"].to(dev), inp["W2"].to(dev), w.E,
        inp["shared_idx"].to(dev), inp["perm_rest"].to(dev), ws=ws)
    return W13_e, W2_e, W13_s, W2_s


def _run(w, inp, capacity=None):
    dev = "cuda"
    p = H.layer_params(w, capacity)
    ws = moe.Workspace(p)
    W13_e, W2_e, W13_s, W2_s = _weights(w, inp, ws)
    b = moe.ForwardBuffers(p)
    dt = wl.torch_dtype(w)
    h_s = torch.empty(max(w.T, 1), moe.h_ld(w.shared), dtype=dt, device=dev)
    out_s = torch.empty(max(w.T, 1), w.d, dtype=dt, device=dev)
    g = lambda n: None if inp.get(n) is None else inp[n].to(dev)
    moe.moe_forward_residual(p, g("x"), g("Wg"), W13_e, W2_e, W13_s, W2_s, w.shared, ws, b, h_s,
                             out_s, Wnoise=g("Wnoise"), noise=g("eps"), bias=g("bias"))
    torch.cuda.synchronize()
    return p, ws, b, h_s, out_s, (W13_e, W2_e, W13_s, W2_s)


def _oracle(w, inp, p, tokens):
    raw = H.raw
    experts, blk = oracle.partition_residual(raw(inp["W1"]), raw(inp["W3"]), raw(inp["W2"]),
                                             w.E, raw(inp["shared_idx"]), raw(inp["perm_rest"]))
    opt = lambda n: None if inp.get(n) is None else raw(inp[n])
    return oracle.forward_residual(raw(inp["x"]), raw(inp["Wg"]), experts, blk, w.k, w.router,
                                   opt("Wnoise"), opt("eps"), opt("bias"), p.capacity,
                                   w.rescale, w.lam, tokens=tokens)


def _check(w, inp, p, ws, b, out_s, tok_sample=None):
    assert moe.moe_get_device_status(ws) == 0
    r, ties = H.check_routing(w, inp, b, 1e-5 if w.dtype == "f32" else 5e-5)
    H.check_dispatch(w, inp, p, b)
    good = np.nonzero(~ties)[0]
    if tok_sample is not None and len(good) > tok_sample:
        good = np.sort(np.random.default_rng(w.seed).choice(good, tok_sample, replace=False))
    ref = _oracle(w, inp, p, good)
    tol = H.Y_TOL[w.dtype]
    e_s = H.rel_err(H.f64(out_s[torch.from_numpy(good).cuda()]), ref["y_shared"])
    assert e_s <= tol, "shared block rel err %g" % e_s
    e_y = H.rel_err(H.f64(b.y[torch.from_numpy(good).cuda()]), ref["y"])
    assert e_y <= tol, "y rel err %g" % e_y
    H.check_loss(w, b, r)
    return e_y


@pytest.mark.parametrize("name", list(CASES))
def test_residual_layer_parity(name):
    w = CASES[name]
    inp = wl.make_inputs(w)
    p, ws, b, h_s, out_s, _ = _run(w, inp)
    _check(w, inp, p, ws, b, out_s)


def test_residual_capacity_zero_is_the_shared_block():
    w = CASES["res_mid"]
    inp = wl.make_inputs(w)
    p, ws, b, h_s, out_s, _ = _run(w, inp, capacity=0)
    assert moe.moe_get_device_status(ws) == 0
    assert (b.slot_row == -1).all()
    assert torch.equal(b.y.view(torch.int16), out_s.view(torch.int16))
    ref = _oracle(w, inp, p, np.arange(w.T))
    assert H.rel_err(H.f64(b.y), ref["y"]) <= H.Y_TOL[w.dtype]


def test_residual_steps_reproduce_forward_bit_exactly():
    """moe_forward_residual equals the step calls: the routed layer, the shared
    block as a one-expert moe_expert_ffn over x, moe_combine_residual."""
    w = CASES["res_pair_st_cap"]
    inp = wl.make_inputs(w)
    p, ws, b, h_s, out_s, (W13_e, W2_e, W13_s, W2_s) = _run(w, inp)
    dev = "cuda"
    x, Wg, Wn, eps, bias = (None if inp.get(n) is None else inp[n].to(dev)
                            for n in ("x", "Wg", "Wnoise", "eps", "bias"))
    b2 = moe.ForwardBuffers(p)
    moe.moe_route(p, x, Wg, Wn, eps, bias, ws, b2.topk_idx, b2.topk_w, b2.probs_sum,
                  b2.importance)
    moe.moe_dispatch(p, x, b2.topk_idx, ws, b2.x_perm, b2.row_token, b2.slot_row, b2.counts,
                     b2.kept, b2.offsets)
    moe.moe_expert_ffn(p, b2.x_perm, b2.offsets, W13_e, W2_e, b2.h, b2.out, ws)
    ps = moe.params(w.T, w.d, 1, 1, w.shared, wl.torch_dtype(w), w.router, -1, w.rescale, w.lam)
    rng = torch.tensor([0, w.T], dtype=torch.int32, device=dev)
    h2 = torch.empty_like(h_s)
    o2 = torch.empty_like(out_s)
    moe.moe_expert_ffn(ps, x, rng, W13_s, W2_s, h2, o2, ws)
    moe.moe_combine_residual(p, b2.out, b2.slot_row, b2.topk_w, o2, b2.y)
    torch.cuda.synchronize()
    assert torch.equal(o2.view(torch.int16), out_s.view(torch.int16))
    assert torch.equal(b2.y.view(torch.int16), b.y.view(torch.int16))


def test_residual_full_size_sampled():
    w = wl.WORKLOADS["moe_res_2of8"]
    inp = wl.make_inputs(w)
    p, ws, b, h_s, out_s, _ = _run(w, inp)
    _check(w, inp, p, ws, b, out_s, tok_sample=48)
