"""The host-buffer pipeline (include/moe_pipeline.h): batches submitted from host
memory with several in flight give, batch by batch, exactly what moe_forward gives
on the same inputs, and one batch is checked against the fp64 oracle."""
import numpy as np
import pytest
import torch

import harness as H
import top_routing_grouped_noisy_b200 as moe
import workloads as wl

pytestmark = pytest.mark.gpu

W = wl.Workload
CASES = {
    "mid_noisy_d2": (W("pipe_mid_noisy", T=1000, d=512, d_ff=2752, E=8, k=2, noisy=True,
                       rescale=True, lam=0.01, seed=40), 2),
    "pair_st_cap_d3": (W("pipe_pair_st", T=2100, d=256, d_ff=2048, E=16, k=4, router=wl.ST,
                         noisy=True, bias=True, cf=1.1, lam=0.01, seed=41), 3),
    "decode_t8_d4": (W("pipe_decode", T=8, d=256, d_ff=1024, E=8, k=2, lam=0.01, seed=42), 4),
    "f32_d2": (W("pipe_f32", T=190, d=96, d_ff=384, E=16, k=4, dtype="f32", noisy=True,
                 seed=43), 2),
}


def _batch(w, i):
    """Activations and noise of batch i (everything else is shared)."""
    b = wl.make_inputs(w.with_(seed=w.seed * 100 + i))
    return b["x"], b["eps"]


@pytest.mark.parametrize("name", list(CASES))
def test_pipeline_matches_forward(name):
    w, depth = CASES[name]
    inp = wl.make_inputs(w)
    p = H.layer_params(w)
    ws = moe.Workspace(p)
    W13_e, W2_e = H.gpu_weights(w, inp, ws)
    dev = lambda t: None if t is None else t.cuda()
    Wg, Wn, bias = dev(inp["Wg"]), dev(inp["Wnoise"]), dev(inp["bias"])
    nb = 2 * depth + 1
    batches = [_batch(w, i) for i in range(nb)]
    pin = lambda t: None if t is None else t.contiguous().pin_memory()
    xs = [pin(x) for x, _ in batches]
    ns = [pin(n) for _, n in batches]
    dt = wl.torch_dtype(w)
    ys = [torch.empty(w.T, w.d, dtype=dt).pin_memory() for _ in range(nb)]
    ls = [torch.empty(1, dtype=torch.float32).pin_memory() for _ in range(nb)]
    with moe.Pipeline(p, Wg, W13_e, W2_e, Wnoise=Wn, bias=bias, depth=depth) as pl:
        tickets = [pl.submit(xs[i], ys[i], ls[i], noise_host=ns[i]) for i in range(nb)]
        assert tickets == list(range(nb))
        pl.wait(tickets[1])  # an earlier ticket after later ones were queued
        pl.wait(tickets[-1])
    bufs = moe.ForwardBuffers(p)
    for i in range(nb):
        moe.moe_forward(p, xs[i].cuda(), Wg, W13_e, W2_e, ws, bufs, Wnoise=Wn,
                        noise=dev(ns[i]), bias=bias)
        torch.cuda.synchronize()
        assert moe.moe_get_device_status(ws) == 0
        y_ref = bufs.y.cpu()
        assert torch.equal(ys[i].view(torch.int16) if dt == torch.bfloat16 else ys[i],
                           y_ref.view(torch.int16) if dt == torch.bfloat16 else y_ref), i
        assert ls[i].item() == bufs.loss.cpu().item(), i
    # the last batch against the oracle (routing, dispatch, y, L_balance)
    last = dict(inp, x=batches[-1][0], eps=batches[-1][1])
    r, ties = H.check_routing(w, last, bufs, 1e-5 if w.dtype == "f32" else 5e-5)
    dsp = H.check_dispatch(w, last, p, bufs)
    OW = H.oracle_weights(w, last)
    H.check_y(w, bufs, r, dsp, OW, np.nonzero(~ties)[0], inp=last)
    H.check_loss(w, bufs, r)


def test_pipeline_reports_bad_index_status():
    """A NaN routing logit in batch 1 is reported by wait() for that batch only:
    batches 0 and 2, queued around it before any wait, report MOE_OK, and batch 0's
    status stays its own although batch 1's kernels ran before it was read."""
    w = W("pipe_nan", T=300, d=128, d_ff=512, E=8, k=2, seed=44)
    inp = wl.make_inputs(w)
    p = H.layer_params(w)
    ws = moe.Workspace(p)
    W13_e, W2_e = H.gpu_weights(w, inp, ws)
    x_ok = inp["x"].contiguous().pin_memory()
    x_bad = inp["x"].clone()
    x_bad[17, :] = float("nan")
    x_bad = x_bad.pin_memory()
    y = [torch.empty(w.T, w.d, dtype=torch.bfloat16).pin_memory() for _ in range(4)]
    loss = [torch.empty(1).pin_memory() for _ in range(4)]
    with moe.Pipeline(p, inp["Wg"].cuda(), W13_e, W2_e, depth=2) as pl:
        t0 = pl.submit(x_ok, y[0], loss[0])
        t1 = pl.submit(x_bad, y[1], loss[1])
        t2 = pl.submit(x_ok, y[2], loss[2])
        pl.wait(t2)  # every batch is done; each status was snapshotted on its own
        pl.wait(t0)
        with pytest.raises(moe.MoeError) as ei:
            pl.wait(t1)
        assert ei.value.code == moe.MOE_ERR_DEVICE_BADINDEX
        pl.wait(t2)
        t3 = pl.submit(x_ok, y[3], loss[3])
        pl.wait(t3)
    assert torch.equal(y[0].view(torch.int16), y[2].view(torch.int16))
