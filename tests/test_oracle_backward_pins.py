"""Pins of the oracle's backward (the gradient of l(y) + c L_balance) to facts that
do not come from the backward code: central finite differences of the oracle's own
f64 forward pass (itself pinned in test_oracle_pins.py), closed forms, and a plain
torch autograd restatement of the dense SwiGLU FFN."""
import numpy as np
import pytest
import torch

GATES = ["mixtral", "st"]


def _rng(seed):
    return np.random.default_rng(seed)


def _problem(seed, T=6, d=8, m=4, E=4, k=2, noisy=True, bias=True):
    r = _rng(seed)
    f32 = np.float32
    x = r.standard_normal((T, d)).astype(f32)
    Wg = (0.6 * r.standard_normal((d, E))).astype(f32)
    Wn = (0.4 * r.standard_normal((d, E))).astype(f32) if noisy else None
    eps = r.standard_normal((T, E)).astype(f32) if noisy else None
    b = (0.3 * r.standard_normal(E)).astype(f32) if bias else None
    W1e = (0.5 * r.standard_normal((E, m, d))).astype(f32)
    W3e = (0.5 * r.standard_normal((E, m, d))).astype(f32)
    W2e = (0.5 * r.standard_normal((E, d, m))).astype(f32)
    dy = r.standard_normal((T, d))
    return dict(x=x, Wg=Wg, Wnoise=Wn, eps=eps, bias=b, W1e=W1e, W3e=W3e, W2e=W2e, dy=dy)


def _loss(orc, P, k, rt, C, rescale, lam, c):
    f = orc.forward(P["x"], P["Wg"], P["W1e"], P["W3e"], P["W2e"], k, rt, P["Wnoise"],
                    P["eps"], P["bias"], C, rescale, lam)
    return float((f["y"] * P["dy"]).sum() + c * f["L"]), f


def _margin(f, k):
    """Smallest gap between the k-th and (k+1)-th routing logit over tokens."""
    H = np.sort(f["router"]["H"], axis=1)[:, ::-1]
    return float((H[:, k - 1] - H[:, k]).min()) if H.shape[1] > k else np.inf


@pytest.mark.parametrize("gate", GATES)
@pytest.mark.parametrize("variant", ["plain", "capacity_rescale_balance"])
def test_backward_matches_central_differences(orc, gate, variant):
    rt = orc.MIXTRAL if gate == "mixtral" else orc.ST
    k = 2
    C, rescale, lam, c = (-1, False, 0.0, 0.0) if variant == "plain" else (2, True, 0.3, 0.7)
    P = _problem(11 if gate == "mixtral" else 12)
    base, f0 = _loss(orc, P, k, rt, C, rescale, lam, c)
    assert _margin(f0, k) > 1e-2  # no top-k decision sits near a tie
    if C >= 0:
        assert (f0["dispatch"]["slot_row"] < 0).any()  # the case really drops
    g = orc.backward(P["x"], P["Wg"], P["W1e"], P["W3e"], P["W2e"], k, P["dy"], rt, P["Wnoise"],
                     P["eps"], P["bias"], C, rescale, lam, c)
    grads = dict(x=g["dx"], Wg=g["dWg"], Wnoise=g["dWnoise"], bias=g["dbias"], W1e=g["dW1e"],
                 W3e=g["dW3e"], W2e=g["dW2e"])
    r = _rng(5)
    for name, G in grads.items():
        arr = P[name]
        for _ in range(6):
            i = tuple(int(r.integers(0, s)) for s in arr.shape)
            v = float(arr[i])
            h = 2.0 ** -12 * max(1.0, abs(v))
            vp, vm = np.float32(v + h), np.float32(v - h)
            Pp = dict(P)
            Pp[name] = arr.copy()
            Pp[name][i] = vp
            lp, fp = _loss(orc, Pp, k, rt, C, rescale, lam, c)
            Pp[name][i] = vm
            lm, fm = _loss(orc, Pp, k, rt, C, rescale, lam, c)
            for ff in (fp, fm):  # the piecewise-constant choices did not move
                assert (ff["router"]["idx"] == f0["router"]["idx"]).all()
            fd = (lp - lm) / (float(vp) - float(vm))
            assert abs(fd - G[i]) <= 1e-6 * max(1.0, abs(fd)), (name, i, fd, G[i])


def test_expert_backward_matches_torch_autograd(orc):
    """One expert row by row: the oracle's dx, dW1, dW3, dW2 against torch autograd
    of silu(W1 x) * (W3 x) -> W2 (f64)."""
    r = _rng(21)
    E, m, d, n = 3, 5, 7, 9
    W1e = r.standard_normal((E, m, d)).astype(np.float32)
    W3e = r.standard_normal((E, m, d)).astype(np.float32)
    W2e = r.standard_normal((E, d, m)).astype(np.float32)
    x = r.standard_normal((n, d)).astype(np.float32)
    eor = r.integers(0, E, n).astype(np.int32)
    d_out = r.standard_normal((n, d))
    got = orc.expert_ffn_backward(W1e, W3e, W2e, x, eor, d_out)
    t = lambda a: torch.tensor(np.asarray(a, np.float64), requires_grad=True)
    W1, W3, W2, X = t(W1e), t(W3e), t(W2e), t(x)
    out = torch.stack([W2[e] @ (torch.nn.functional.silu(W1[e] @ X[i]) * (W3[e] @ X[i]))
                       for i, e in enumerate(eor)])
    (out * torch.tensor(d_out)).sum().backward()
    np.testing.assert_allclose(got["dx_rows"], X.grad.numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(got["dW1e"], W1.grad.numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(got["dW3e"], W3.grad.numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(got["dW2e"], W2.grad.numpy(), rtol=1e-12, atol=1e-12)


def test_mixtral_top1_router_gets_only_the_balance_gradient(orc):
    """k = 1 Mixtral: G = softmax over one logit is identically 1, so y carries no
    gradient into the router; with lambda = 0 the router gradients vanish."""
    P = _problem(31, noisy=False, bias=True)
    g = orc.backward(P["x"], P["Wg"], P["W1e"], P["W3e"], P["W2e"], 1, P["dy"], orc.MIXTRAL,
                     None, None, P["bias"], -1, False, 0.0, 1.0)
    assert np.abs(g["dH"]).max() < 1e-13
    assert np.abs(g["dWg"]).max() < 1e-12 and np.abs(g["dbias"]).max() < 1e-13


def test_balance_gradient_closed_form(orc):
    """With dy = 0 only L_balance = lambda sum_e f_e P_e contributes: dH_te =
    p_te (b_e - sum_l p_tl b_l), b_e = c lambda f_e / T (softmax Jacobian)."""
    P = _problem(33, noisy=False, bias=False)
    P["dy"] = np.zeros_like(P["dy"])
    lam, c, k = 0.5, 2.0, 2
    g = orc.backward(P["x"], P["Wg"], P["W1e"], P["W3e"], P["W2e"], k, P["dy"], orc.ST, None,
                     None, None, -1, False, lam, c)
    f = g["fwd"]
    H = f["router"]["H"]
    p = np.exp(H - H.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    T = H.shape[0]
    b = c * lam * f["f"] / T
    ref = p * (b[None, :] - (p * b[None, :]).sum(1, keepdims=True))
    np.testing.assert_allclose(g["dH"], ref, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(g["dWg"], P["x"].astype(np.float64).T @ ref, rtol=1e-11,
                               atol=1e-14)


def test_residual_backward_matches_central_differences(orc):
    """Residual layer y = FFN_S(x) + s sum G E(x): finite differences of the oracle's
    forward_residual for x, the router and both the shared and the routed weights."""
    r = _rng(61)
    f32 = np.float32
    T, d, d_ff, E, k, m_s = 5, 8, 24, 4, 2, 8
    x = r.standard_normal((T, d)).astype(f32)
    Wg = (0.6 * r.standard_normal((d, E))).astype(f32)
    W1 = (0.5 * r.standard_normal((d_ff, d))).astype(f32)
    W3 = (0.5 * r.standard_normal((d_ff, d))).astype(f32)
    W2 = (0.5 * r.standard_normal((d, d_ff))).astype(f32)
    perm = r.permutation(d_ff).astype(np.int32)
    shared, rest = perm[:m_s], perm[m_s:]
    experts, blk = orc.partition_residual(W1, W3, W2, E, shared, rest)
    experts = [e.astype(f32) for e in experts]
    blk = [np.ascontiguousarray(b, f32) for b in blk]
    dy = r.standard_normal((T, d))
    lam, c = 0.2, 0.5

    def loss(x_, Wg_, ex, bl):
        f = orc.forward_residual(x_, Wg_, ex, bl, k, rescale=True, lam=lam)
        return float((f["y"] * dy).sum() + c * f["L"])

    g = orc.backward_residual(x, Wg, experts, blk, k, dy, rescale=True, lam=lam, dLb=c)
    checks = [("x", x, g["dx"]), ("Wg", Wg, g["dWg"]), ("W1e", experts[0], g["dW1e"]),
              ("W2e", experts[2], g["dW2e"]), ("W1s", blk[0], g["dW1s"]),
              ("W3s", blk[1], g["dW3s"]), ("W2s", blk[2], g["dW2s"])]
    for name, arr, G in checks:
        for _ in range(5):
            i = tuple(int(r.integers(0, s)) for s in arr.shape)
            v = float(arr[i])
            h = 2.0 ** -12 * max(1.0, abs(v))
            vals = []
            for vv in (np.float32(v + h), np.float32(v - h)):
                a2 = arr.copy()
                a2[i] = vv
                args = {"x": x, "Wg": Wg, "ex": list(experts), "bl": list(blk)}
                if name == "x":
                    args["x"] = a2
                elif name == "Wg":
                    args["Wg"] = a2
                elif name.endswith("e"):
                    args["ex"][{"W1e": 0, "W2e": 2}[name]] = a2
                else:
                    args["bl"][{"W1s": 0, "W3s": 1, "W2s": 2}[name]] = a2
                vals.append(loss(args["x"], args["Wg"], args["ex"], args["bl"]))
            fd = (vals[0] - vals[1]) / (float(np.float32(v + h)) - float(np.float32(v - h)))
            assert abs(fd - G[i]) <= 1e-6 * max(1.0, abs(fd)), (name, i, fd, G[i])


def test_sampled_backward_pieces_equal_the_full_backward(orc):
    """The sampling helpers the full-size parity test uses reproduce the full
    backward: the per-neuron weight gradient, and the router backward of a token
    subset normalised by the whole batch."""
    P = _problem(71, T=9, d=8, m=5, E=3, k=2, noisy=True, bias=True)
    lam, c = 0.3, 0.7
    g = orc.backward(P["x"], P["Wg"], P["W1e"], P["W3e"], P["W2e"], 2, P["dy"], orc.MIXTRAL,
                     P["Wnoise"], P["eps"], P["bias"], -1, True, lam, c)
    f = g["fwd"]
    dsp = f["dispatch"]
    for e in range(3):
        rows = np.arange(dsp["offsets"][e], dsp["offsets"][e + 1])
        xr = P["x"][dsp["row_token"][rows]]
        for i in range(5):
            d1, d3, d2 = orc.neuron_wgrad(P["W1e"], P["W3e"], P["W2e"], e, i, xr,
                                          g["d_out"][rows])
            np.testing.assert_allclose(d1, g["dW1e"][e, i], rtol=1e-12, atol=1e-14)
            np.testing.assert_allclose(d3, g["dW3e"][e, i], rtol=1e-12, atol=1e-14)
            np.testing.assert_allclose(d2, g["dW2e"][e][:, i], rtol=1e-12, atol=1e-14)
    toks = np.array([1, 4, 7])
    rb = orc.router_backward_tokens(P["x"][toks], P["Wg"], f["router"]["idx"][toks],
                                    f["router"]["G"][toks], g["dG"][toks], dsp["counts"], 2, 9,
                                    orc.MIXTRAL, P["Wnoise"], P["eps"][toks], P["bias"], lam, c)
    np.testing.assert_allclose(rb["dH"], g["dH"][toks], rtol=1e-12, atol=1e-15)
