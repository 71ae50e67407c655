"""Failure detection on the GPU without a GPU fault: every bounded wait inside the
tensor-core GEMM kernels is made to run out at once (wait limit 0), the kernel
must report MOE_ERR_DEVICE_TIMEOUT through the workspace status word and return,
and the context must stay usable (a normal layer afterwards passes parity)."""
import numpy as np
import pytest
import torch

import harness as H
import top_routing_grouped_noisy_b200 as moe
import workloads as wl

pytestmark = pytest.mark.gpu

DEFAULT_LIMIT_NS = 2_000_000_000


@pytest.mark.parametrize("T", [300, 2500], ids=["one_sm_kernel", "two_sm_kernel"])
def test_wait_timeout_is_reported_and_context_survives(T):
    w = wl.Workload("to", T=T, d=256, d_ff=1024, E=8, k=2, noisy=True, seed=81)
    inp = wl.make_inputs(w)
    p = H.layer_params(w)
    ws = moe.Workspace(p)
    W13_e, W2_e = H.gpu_weights(w, inp, ws)
    b = moe.ForwardBuffers(p)
    dev = "cuda"
    x, Wg, Wn, eps = (inp[n].to(dev) for n in ("x", "Wg", "Wnoise", "eps"))
    moe.moe_route(p, x, Wg, Wn, eps, None, ws, b.topk_idx, b.topk_w, b.probs_sum, b.importance)
    moe.moe_dispatch(p, x, b.topk_idx, ws, b.x_perm, b.row_token, b.slot_row, b.counts, b.kept,
                     b.offsets)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    moe.moe_set_wait_limit_ns(0)
    try:
        moe.moe_expert_up(p, b.x_perm, b.offsets, W13_e, b.h, ws)
        torch.cuda.synchronize()
    finally:
        moe.moe_set_wait_limit_ns(DEFAULT_LIMIT_NS)
    assert moe.moe_get_device_status(ws) == moe.MOE_ERR_DEVICE_TIMEOUT
    assert moe.moe_get_device_status(ws) == 0  # cleared by the read
    # the same context still computes the layer correctly
    p2, bufs, ws2, status, _ = H.run_forward(w, inp, weights=(W13_e, W2_e))
    assert status == 0
    r, ties = H.check_routing(w, inp, bufs, 5e-5)
    dsp = H.check_dispatch(w, inp, p2, bufs)
    H.check_y(w, bufs, r, dsp, H.oracle_weights(w, inp), np.nonzero(~ties)[0], inp=inp)



@pytest.mark.parametrize("T", [300, 2500], ids=["one_sm_kernels", "two_sm_kernels"])
def test_backward_wait_timeout_is_reported_and_context_survives(T):
    """The backward GEMMs (row-grouped with the SwiGLU-backward epilogue, dgrad and the
    K-grouped wgrad, 1-SM and 2-SM forms) give up at a wait limit of 0, report
    MOE_ERR_DEVICE_TIMEOUT and return; a normal backward afterwards is correct."""
    import oracle
    w = wl.Workload("to_bwd", T=T, d=256, d_ff=1024, E=8, k=2, noisy=True, seed=82)
    inp = wl.make_inputs(w)
    p, bufs, ws, status, (W13_e, W2_e) = H.run_forward(w, inp)
    assert status == 0
    dev = "cuda"
    dy = wl.make_grad_output(w, 5).to(dev)
    g = moe.BackwardBuffers(p, True, False)
    wsb = moe.Workspace(p, nbytes=moe.moe_backward_workspace_size(p))
    moe.moe_combine_backward(p, dy, bufs.out, bufs.slot_row, bufs.topk_w, g.d_out, g.dG)
    torch.cuda.synchronize()
    moe.moe_set_wait_limit_ns(0)
    try:
        moe.moe_expert_down_backward(p, g.d_out, bufs.h, bufs.offsets, W2_e, g.dh, g.dW2_e, wsb)
        moe.moe_expert_up_backward(p, bufs.x_perm, g.dh, bufs.offsets, W13_e, g.dx_perm,
                                   g.dW13_e, wsb)
        torch.cuda.synchronize()
    finally:
        moe.moe_set_wait_limit_ns(DEFAULT_LIMIT_NS)
    assert moe.moe_get_device_status(wsb) == moe.MOE_ERR_DEVICE_TIMEOUT
    assert moe.moe_get_device_status(wsb) == 0
    # the same context then runs the whole backward correctly
    x, Wg, Wn, eps = (inp[n].to(dev) for n in ("x", "Wg", "Wnoise", "eps"))
    moe.moe_backward(p, x, Wg, W13_e, W2_e, bufs, g, dy, wsb, Wnoise=Wn, noise=eps)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(wsb) == 0
    W1e, W3e, W2e = H.oracle_weights(w, inp)
    ref = oracle.backward(H.raw(inp["x"]), H.raw(inp["Wg"]), W1e, W3e, W2e, w.k, H.f64(dy.cpu()),
                          oracle.MIXTRAL, H.raw(inp["Wnoise"]), inp["eps"].numpy(), None, -1,
                          False, w.lam, 1.0)
    assert (bufs.topk_idx.cpu().numpy() == ref["fwd"]["router"]["idx"]).all()
    dx = H.f64(g.dx)
    assert np.abs(dx - ref["dx"]).max() <= 2e-2 * np.abs(ref["dx"]).max()


def test_decode_forward_wait_timeout_is_reported_and_context_survives():
    """The one-launch decode layer (bulk-copy ring, grid barrier) gives up at a wait
    limit of 0, reports MOE_ERR_DEVICE_TIMEOUT and returns; its grid barrier words are
    back at zero, so the next forward on the same workspace is correct."""
    w = wl.Workload("to_dec", T=4, d=512, d_ff=8 * 96, E=8, k=2, noisy=True, rescale=True,
                    seed=83)
    inp = wl.make_inputs(w)
    p, bufs, ws, status, weights = H.run_forward(w, inp)
    assert status == 0
    dev = "cuda"
    W13_e, W2_e = weights
    x, Wg, Wn, eps = (inp[n].to(dev) for n in ("x", "Wg", "Wnoise", "eps"))
    moe.moe_set_wait_limit_ns(0)
    try:
        moe.moe_forward(p, x, Wg, W13_e, W2_e, ws, bufs, Wnoise=Wn, noise=eps)
        torch.cuda.synchronize()
    finally:
        moe.moe_set_wait_limit_ns(DEFAULT_LIMIT_NS)
    assert moe.moe_get_device_status(ws) == moe.MOE_ERR_DEVICE_TIMEOUT
    assert moe.moe_get_device_status(ws) == 0
    moe.moe_forward(p, x, Wg, W13_e, W2_e, ws, bufs, Wnoise=Wn, noise=eps)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    r, ties = H.check_routing(w, inp, bufs, 5e-5)
    dsp = H.check_dispatch(w, inp, p, bufs)
    H.check_y(w, bufs, r, dsp, H.oracle_weights(w, inp), np.nonzero(~ties)[0], inp=inp)


def test_front_small_wait_timeout_is_reported_and_context_survives():
    """The small-batch front of moe_forward (routing, dispatch and gate statistics in
    one cooperative launch with two grid barriers) gives up at a wait limit of 0,
    reports MOE_ERR_DEVICE_TIMEOUT and returns with its barrier words back at zero, so
    the next forward on the same workspace is correct without a status clear."""
    w = wl.Workload("to_front", T=40, d=256, d_ff=8 * 64, E=8, k=2, noisy=True, seed=84)
    inp = wl.make_inputs(w)
    p, bufs, ws, status, weights = H.run_forward(w, inp)
    assert status == 0
    dev = "cuda"
    W13_e, W2_e = weights
    x, Wg, Wn, eps = (inp[n].to(dev) for n in ("x", "Wg", "Wnoise", "eps"))
    moe.moe_set_wait_limit_ns(0)
    try:
        moe.moe_forward(p, x, Wg, W13_e, W2_e, ws, bufs, Wnoise=Wn, noise=eps)
        torch.cuda.synchronize()
    finally:
        moe.moe_set_wait_limit_ns(DEFAULT_LIMIT_NS)
    assert moe.moe_get_device_status(ws, clear=False) == moe.MOE_ERR_DEVICE_TIMEOUT
    hdr = ws.buf[:32].view(torch.int32).cpu()
    assert int(hdr[6]) == 0 and int(hdr[7]) == 0  # the front barrier words
    assert moe.moe_get_device_status(ws) == moe.MOE_ERR_DEVICE_TIMEOUT  # read and clear
    moe.moe_forward(p, x, Wg, W13_e, W2_e, ws, bufs, Wnoise=Wn, noise=eps)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    r, ties = H.check_routing(w, inp, bufs, 5e-5)
    dsp = H.check_dispatch(w, inp, p, bufs)
    H.check_y(w, bufs, r, dsp, H.oracle_weights(w, inp), np.nonzero(~ties)[0], inp=inp)


def test_small_batch_gemm_reports_an_expert_with_more_rows_than_tokens():
    """At most 64 tokens give each expert at most 64 rows, which the small-batch GEMM
    ring is sized for; offsets that give an expert more (no dispatch can) are reported
    as MOE_ERR_DEVICE_BADINDEX, every access stays inside the buffers (the rows past 64
    are computed from whatever the stage held), and the next call is unaffected."""
    T, d, E, k, m = 64, 256, 4, 2, 64
    p = moe.params(T, d, E, k, m)
    ws = moe.Workspace(p)
    gen = torch.Generator().manual_seed(85)
    rows = T * k
    x_perm = (torch.randn(rows, d, generator=gen) * 0.5).to(torch.bfloat16).cuda()
    W13 = (torch.randn(E, 2 * m, d, generator=gen) * 0.05).to(torch.bfloat16).cuda()
    h = torch.zeros(rows, m, dtype=torch.bfloat16, device="cuda")
    bad = torch.tensor([0, 100, 110, 120, rows], dtype=torch.int32, device="cuda")
    moe.moe_expert_up(p, x_perm, bad, W13, h, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == moe.MOE_ERR_DEVICE_BADINDEX
    good = torch.tensor([0, 40, 70, 100, rows], dtype=torch.int32, device="cuda")
    moe.moe_expert_up(p, x_perm, good, W13, h, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    # expert 1's rows against a plain f32 product: h = silu(g) * u over 32-row groups
    xe = x_perm[40:70].float()
    W = W13[1].float()  # rows: per 32-row group 16 W1 rows, then the 16 W3 rows
    g = torch.cat([W[32 * i:32 * i + 16] for i in range(m // 16)]) @ xe.T
    u = torch.cat([W[32 * i + 16:32 * i + 32] for i in range(m // 16)]) @ xe.T
    ref = (torch.nn.functional.silu(g) * u).T
    assert torch.allclose(h[40:70].float(), ref, atol=2e-2, rtol=2e-2)
