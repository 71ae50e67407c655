"""GPU parity of every step of the layer against the fp64 oracle, through the C ABI.

Small cases span several 128x256 tensor-core tiles with ragged row, column and K
tails; the full-size cases run the workloads the benchmark times, in the same
launch configuration, and compare routing and dispatch on every token and the
layer output on a seeded sample of tokens.
"""
import numpy as np
import pytest
import torch

import harness as H
import oracle
import top_routing_grouped_noisy_b200 as moe
import workloads as wl

pytestmark = pytest.mark.gpu

W = wl.Workload
SMALL = {
    "mid_mixtral_noisy": W("mid_mixtral_noisy", T=1000, d=512, d_ff=2752, E=8, k=2, noisy=True,
                           rescale=True, seed=11),
    "mid_st_bias_cap": W("mid_st_bias_cap", T=700, d=256, d_ff=1024, E=16, k=4, router=wl.ST,
                         noisy=True, bias=True, rescale=True, cf=1.0, seed=12),
    "e64_k8": W("e64_k8", T=300, d=128, d_ff=1024, E=64, k=8, noisy=True, seed=13),
    "e32_st": W("e32_st", T=500, d=256, d_ff=768, E=32, k=3, router=wl.ST, noisy=True, seed=14),
    "odd_m_d": W("odd_m_d", T=333, d=200, d_ff=800, E=8, k=2, seed=15),
    "copy_perturbed_cf1": W("copy_perturbed_cf1", T=600, d=256, d_ff=384, E=4, k=2, cf=1.0,
                            partition=wl.COPY, perturb=1e-3, seed=16),
    "copy_exact": W("copy_exact", T=256, d=128, d_ff=256, E=4, k=2, partition=wl.COPY,
                    seed=17),
    "single_expert": W("single_expert", T=100, d=64, d_ff=64, E=1, k=1, rescale=True, seed=18),
    "k_eq_E": W("k_eq_E", T=128, d=64, d_ff=128, E=4, k=4, seed=19),
    "one_token": W("one_token", T=1, d=256, d_ff=512, E=8, k=2, noisy=True, seed=20),
    "tiny_cap": W("tiny_cap", T=200, d=64, d_ff=256, E=8, k=2, cf=0.25, seed=21),
    # T*k >= 4096 rows: the 2-SM (cta_group::2) GEMM kernel
    "pair_mid": W("pair_mid", T=2100, d=256, d_ff=2048, E=8, k=2, noisy=True, rescale=True,
                  seed=24),
    "pair_e16_odd": W("pair_e16_odd", T=1200, d=200, d_ff=1600, E=16, k=4, router=wl.ST,
                      noisy=True, bias=True, cf=1.1, seed=25),
    "pair_e64": W("pair_e64", T=600, d=128, d_ff=1024, E=64, k=8, noisy=True, seed=26),
    # T <= 16: the weight-streaming decode kernels (larger small batches: tcgen05)
    "decode_t64_m344": W("decode_t64_m344", T=64, d=512, d_ff=8 * 344, E=8, k=2, rescale=True,
                         seed=27),
    "decode_skewed_rows": W("decode_skewed_rows", T=40, d=256, d_ff=4 * 96, E=4, k=2, bias=True,
                            seed=28),
    "decode_ragged_d": W("decode_ragged_d", T=8, d=200, d_ff=8 * 100, E=8, k=2, noisy=True,
                         seed=29),
    "decode_t16_st_cap": W("decode_t16_st_cap", T=16, d=264, d_ff=8 * 120, E=8, k=3,
                           router=wl.ST, noisy=True, bias=True, cf=1.0, rescale=True, seed=31),
    # wide rows and 12 tokens: the decode kernel's 1024-column GEMM 1 stages
    "decode_t12_wide": W("decode_t12_wide", T=12, d=4096, d_ff=8 * 64, E=8, k=2, noisy=True,
                         rescale=True, seed=32),
    # 17..64 tokens: one cooperative launch routes, dispatches and takes the gate
    # statistics in moe_forward (f32 here, capacity drops, ST, noise and bias)
    "front_f32_st_cap": W("front_f32_st_cap", T=33, d=72, d_ff=8 * 40, E=8, k=3, dtype="f32",
                          router=wl.ST, noisy=True, bias=True, cf=0.5, seed=35),
    "f32_noisy_st_cap": W("f32_noisy_st_cap", T=257, d=64, d_ff=160, E=8, k=2, dtype="f32",
                          router=wl.ST, noisy=True, bias=True, cf=1.5, seed=22),
    "f32_e16_k4": W("f32_e16_k4", T=190, d=96, d_ff=16 * 24, E=16, k=4, dtype="f32",
                    noisy=True, rescale=True, seed=23),
}


def _G_atol(w):
    return 1e-5 if w.dtype == "f32" else 5e-5


def _full_check(w, inp, rows_sample=None, tok_sample=None, capacity=None):
    p, bufs, ws, status, weights = H.run_forward(w, inp, capacity=capacity)
    assert status == 0, "device status %d" % status
    r, ties = H.check_routing(w, inp, bufs, _G_atol(w))
    dsp = H.check_dispatch(w, inp, p, bufs)
    OW = H.oracle_weights(w, inp)
    rows = None
    if rows_sample is not None and dsp["R"] > rows_sample:
        rows = np.sort(np.random.default_rng(w.seed).choice(dsp["R"], rows_sample, replace=False))
    H.check_expert_rows(w, bufs, dsp, OW, rows, inp=inp)
    good = np.nonzero(~ties)[0]
    if tok_sample is not None and len(good) > tok_sample:
        good = np.sort(np.random.default_rng(w.seed + 1).choice(good, tok_sample, replace=False))
    e = H.check_y(w, bufs, r, dsp, OW, good, inp=inp)
    H.check_loss(w, bufs, r)
    return dict(p=p, bufs=bufs, ws=ws, r=r, ties=ties, dsp=dsp, y_err=e, weights=weights)


@pytest.mark.parametrize("name", list(SMALL))
def test_layer_parity_small(name):
    w = SMALL[name]
    inp = wl.make_inputs(w)
    if name == "decode_skewed_rows":  # two experts take (nearly) every token: > 32 rows each
        inp["bias"] = torch.tensor([6.0, 6.0, -6.0, -6.0])
    res = _full_check(w, inp)
    if name == "decode_skewed_rows":
        assert int(res["bufs"].kept.max()) > 32


def test_tiny_fp32_workload_full():
    w = wl.WORKLOADS["tiny_fp32"]
    inp = wl.make_inputs(w)
    res = _full_check(w, inp)
    assert res["y_err"] <= 1e-5


@pytest.mark.parametrize("mode", ["disjoint_bf16", "copy_f32", "stacked_bf16", "odd_m"])
def test_partition_parity(mode):
    if mode == "disjoint_bf16":
        w = W("p", T=1, d=128, d_ff=1024, E=8, k=2, seed=31)
    elif mode == "copy_f32":
        w = W("p", T=1, d=64, d_ff=96, E=4, k=2, dtype="f32", partition=wl.COPY, seed=32)
    elif mode == "stacked_bf16":
        w = W("p", T=1, d=64, d_ff=80, E=3, k=2, partition=wl.COPY, perturb=1e-2, seed=33)
    else:
        w = W("p", T=1, d=40, d_ff=8 * 13, E=8, k=2, seed=34)  # m = 13
    inp = wl.make_inputs(w)
    W13_e, W2_e = H.gpu_weights(w, inp)
    torch.cuda.synchronize()
    W1e, W3e, W2e = H.oracle_weights(w, inp)
    g1, g3 = H.unpack_w13(W13_e, w.E, w.m, w.d)
    g2 = H.unpack_w2(W2_e, w.E, w.m, w.d)
    np.testing.assert_array_equal(H.raw(g1.contiguous()), W1e)
    np.testing.assert_array_equal(H.raw(g3.contiguous()), W3e)
    np.testing.assert_array_equal(H.raw(g2.contiguous()), W2e)
    # padding rows/columns are zero
    m16, m8 = (w.m + 15) // 16 * 16, (w.m + 7) // 8 * 8
    full = W13_e.view(w.E, m16 // 16, 2, 16, w.d)
    gate_all = full[:, :, 0].reshape(w.E, m16, w.d)
    assert not gate_all[:, w.m:].float().abs().sum()
    assert not W2_e.view(w.E, w.d, m8)[:, :, w.m:].float().abs().sum()


STEP_CASES = {
    "mid_st_bias_cap": SMALL["mid_st_bias_cap"],
    # small batches (weight-streaming kernels up to 16 tokens, tcgen05 above)
    "decode_t64_m344": SMALL["decode_t64_m344"],
    "decode_ragged_d": SMALL["decode_ragged_d"],
    "decode_t16_st_cap": SMALL["decode_t16_st_cap"],
    "one_token": SMALL["one_token"],
    "decode_t12_wide": SMALL["decode_t12_wide"],
    "decode_st_bias_cap": W("decode_st_bias_cap", T=48, d=192, d_ff=16 * 40, E=16, k=4,
                            router=wl.ST, noisy=True, bias=True, cf=1.0, rescale=True,
                            lam=0.01, seed=30),
    "front_f32_st_cap": SMALL["front_f32_st_cap"],
    "front_e32_k8": W("front_e32_k8", T=64, d=128, d_ff=32 * 16, E=32, k=8, noisy=True,
                      cf=0.8, seed=36),
    # E = 64 without noise: the front's gate runs one thread per token (E > 32)
    "front_e64_plain": W("front_e64_plain", T=64, d=128, d_ff=64 * 16, E=64, k=8, cf=1.0,
                         seed=38),
    # E = 64 with noise: too many logits for the split-K router, so both sides route
    # on the tensor cores
    "e64_k8_t64": W("e64_k8_t64", T=64, d=128, d_ff=64 * 16, E=64, k=8, noisy=True,
                    cf=0.8, seed=37),
}


@pytest.mark.parametrize("name", list(STEP_CASES))
def test_steps_reproduce_forward_bit_exactly(name):
    """The six step calls give the same bytes as moe_forward, and reruns are identical."""
    w = STEP_CASES[name]
    inp = wl.make_inputs(w)
    p, bufs, ws, status, (W13_e, W2_e) = H.run_forward(w, inp)
    assert status == 0
    b2 = moe.ForwardBuffers(p)
    x, Wg, Wn, eps, bias = (None if inp.get(n) is None else inp[n].to("cuda")
                            for n in ("x", "Wg", "Wnoise", "eps", "bias"))
    moe.moe_route(p, x, Wg, Wn, eps, bias, ws, b2.topk_idx, b2.topk_w, b2.probs_sum,
                  b2.importance)
    moe.moe_dispatch(p, x, b2.topk_idx, ws, b2.x_perm, b2.row_token, b2.slot_row, b2.counts,
                     b2.kept, b2.offsets)
    moe.moe_expert_up(p, b2.x_perm, b2.offsets, W13_e, b2.h, ws)
    moe.moe_expert_down(p, b2.h, b2.offsets, W2_e, b2.out, ws)
    moe.moe_combine(p, b2.out, b2.slot_row, b2.topk_w, b2.y)
    moe.moe_gate_stats(p, b2.counts, b2.probs_sum, b2.f, b2.P, b2.loss)
    torch.cuda.synchronize()
    R = int(bufs.offsets[-1])
    for n in ("y", "topk_idx", "topk_w", "probs_sum", "importance", "counts", "kept",
              "offsets", "slot_row", "loss", "f", "P"):
        assert torch.equal(getattr(bufs, n), getattr(b2, n)), n
    assert torch.equal(bufs.out[:R], b2.out[:R])
    assert torch.equal(bufs.row_token[:R], b2.row_token[:R])
    assert torch.equal(bufs.x_perm[:R], b2.x_perm[:R])
    assert torch.equal(bufs.h[:R, :w.m], b2.h[:R, :w.m])


ROUTED_CASES = {
    # the tensor-core router counts the chunks in its epilogue (vector and scalar B
    # writer: E % 8 == 0 and E = 5; NOUT 16, 32 and 128; ragged last chunk)
    "tc_noisy_cap": W("r_tc_noisy_cap", T=1000, d=256, d_ff=8 * 64, E=8, k=2, noisy=True,
                      cf=1.1, seed=50),
    "tc_e16_st_bias": W("r_tc_e16_st", T=2100, d=192, d_ff=16 * 48, E=16, k=4, router=wl.ST,
                        noisy=True, bias=True, cf=0.9, seed=51),
    "tc_e64_k8": W("r_tc_e64_k8", T=777, d=128, d_ff=64 * 16, E=64, k=8, noisy=True, seed=52),
    "tc_e5_plain": W("r_tc_e5", T=301, d=136, d_ff=5 * 32, E=5, k=2, cf=0.7, seed=53),
    # the other router paths end with the count kernel
    "small_t40": W("r_small_t40", T=40, d=256, d_ff=8 * 32, E=8, k=2, noisy=True, cf=1.0,
                   seed=54),
    "f32": W("r_f32", T=300, d=64, d_ff=8 * 24, E=8, k=3, dtype="f32", cf=1.2, seed=55),
}


@pytest.mark.parametrize("name", list(ROUTED_CASES))
def test_routed_dispatch_equals_dispatch(name):
    """moe_dispatch_routed (the router's own chunk counts) gives the bytes moe_dispatch
    gives on the same indices, with the routing call's capacity and with another one,
    twice in a row; the tables are those of the oracle's dispatch of those indices."""
    w = ROUTED_CASES[name]
    inp = wl.make_inputs(w)
    p = H.layer_params(w)
    ws = moe.Workspace(p)
    x, Wg, Wn, eps, bias = (None if inp.get(n) is None else inp[n].to("cuda")
                            for n in ("x", "Wg", "Wnoise", "eps", "bias"))
    for rep, cap in enumerate((p.capacity, max(1, w.T * w.k // (2 * w.E)), p.capacity)):
        q = H.layer_params(w, capacity=cap)
        a, b = moe.ForwardBuffers(q), moe.ForwardBuffers(q)
        moe.moe_route(p, x, Wg, Wn, eps, bias, ws, a.topk_idx, a.topk_w, a.probs_sum,
                      a.importance)
        moe.moe_dispatch_routed(q, x, a.topk_idx, ws, a.x_perm, a.row_token, a.slot_row,
                                a.counts, a.kept, a.offsets)
        moe.moe_dispatch(q, x, a.topk_idx, ws, b.x_perm, b.row_token, b.slot_row, b.counts,
                         b.kept, b.offsets)
        torch.cuda.synchronize()
        assert moe.moe_get_device_status(ws) == 0
        R = int(b.offsets[-1])
        for n in ("counts", "kept", "offsets", "slot_row"):
            assert torch.equal(getattr(a, n), getattr(b, n)), (rep, n)
        assert torch.equal(a.row_token[:R], b.row_token[:R]), rep
        assert torch.equal(a.x_perm[:R], b.x_perm[:R]), rep
        H.check_dispatch(w, inp, q, a)


@pytest.mark.parametrize("T,d,E,k", [(600, 320, 8, 2), (2500, 320, 8, 2), (2500, 200, 8, 2),
                                     (1100, 136, 16, 4)],
                         ids=["one_sm_kernel", "two_sm_kernel", "two_sm_k_tail",
                              "two_sm_e16_k_tail"])
def test_gather_gemm_equals_permuted_copy_gemm(T, d, E, k):
    """moe_expert_up_gather (rows of x gathered through row_token: TMA gather4 in the
    1-SM kernel, cp.async in the 2-SM kernel) gives the same bytes as moe_expert_up
    on the permuted copy x_perm, and moe_dispatch_rows the same tables as
    moe_dispatch."""
    w = W("gather", T=T, d=d, d_ff=E * 176, E=E, k=k, noisy=True, cf=1.2, seed=45)
    inp = wl.make_inputs(w)
    p = H.layer_params(w)
    ws = moe.Workspace(p)
    W13_e, W2_e = H.gpu_weights(w, inp, ws)
    a, b = moe.ForwardBuffers(p), moe.ForwardBuffers(p)
    x, Wg, Wn, eps = (inp[n].cuda() for n in ("x", "Wg", "Wnoise", "eps"))
    moe.moe_route(p, x, Wg, Wn, eps, None, ws, a.topk_idx, a.topk_w, a.probs_sum, a.importance)
    moe.moe_dispatch(p, x, a.topk_idx, ws, a.x_perm, a.row_token, a.slot_row, a.counts, a.kept,
                     a.offsets)
    moe.moe_dispatch_rows(p, a.topk_idx, ws, b.row_token, b.slot_row, b.counts, b.kept,
                          b.offsets)
    moe.moe_expert_up(p, a.x_perm, a.offsets, W13_e, a.h, ws)
    moe.moe_expert_up_gather(p, x, b.row_token, b.offsets, W13_e, b.h, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    R = int(a.offsets[-1])
    for n in ("counts", "kept", "offsets", "slot_row"):
        assert torch.equal(getattr(a, n), getattr(b, n)), n
    assert torch.equal(a.row_token[:R], b.row_token[:R])
    m = w.m
    assert torch.equal(a.h[:R, :m], b.h[:R, :m])
    # and the permuted copy itself is x's rows in dispatch order
    assert torch.equal(a.x_perm[:R], x[a.row_token[:R].long()])


def test_empty_batch():
    w = W("empty", T=0, d=64, d_ff=128, E=4, k=2, noisy=True, seed=40)
    inp = wl.make_inputs(w)
    p, bufs, ws, status, _ = H.run_forward(w, inp)
    assert status == 0
    assert bufs.counts.tolist() == [0] * 4 and bufs.offsets.tolist() == [0] * 5
    assert bufs.probs_sum.abs().sum().item() == 0 and float(bufs.loss[0]) == 0.0


def test_capacity_zero_drops_everything():
    w = W("cap0", T=77, d=64, d_ff=128, E=4, k=2, seed=41)
    inp = wl.make_inputs(w)
    p, bufs, ws, status, _ = H.run_forward(w, inp, capacity=0)
    assert status == 0
    assert bufs.kept.tolist() == [0] * 4 and int(bufs.offsets[-1]) == 0
    assert (bufs.slot_row == -1).all()
    assert bufs.y.float().abs().sum().item() == 0.0
    assert bufs.counts.sum().item() == 77 * 2


def test_nan_input_sets_badindex_status():
    w = W("nan", T=64, d=64, d_ff=128, E=4, k=2, seed=42)
    inp = wl.make_inputs(w)
    inp["x"][5, 3] = float("nan")
    p, bufs, ws, status, _ = H.run_forward(w, inp)
    assert status == moe.MOE_ERR_DEVICE_BADINDEX
    assert (bufs.topk_idx[5] == -1).all() and (bufs.slot_row[5] == -1).all()
    assert moe.moe_get_device_status(ws) == 0  # cleared by the previous read


def test_out_of_range_index_is_dropped_and_reported():
    w = W("badidx", T=40, d=64, d_ff=128, E=4, k=2, seed=43)
    inp = wl.make_inputs(w)
    p = H.layer_params(w)
    ws = moe.Workspace(p)
    b = moe.ForwardBuffers(p)
    idx = torch.tensor([[0, 1]] * 40, dtype=torch.int32, device="cuda")
    idx[3, 1] = 7
    idx[9, 0] = -2
    x = inp["x"].cuda()
    moe.moe_dispatch(p, x, idx, ws, b.x_perm, b.row_token, b.slot_row, b.counts, b.kept,
                     b.offsets)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == moe.MOE_ERR_DEVICE_BADINDEX
    d = oracle.dispatch(idx.cpu().numpy(), 4, -1)
    np.testing.assert_array_equal(b.slot_row.cpu().numpy(), d["slot_row"])
    assert b.counts.tolist() == d["counts"].tolist()


def test_dense_equivalence_on_gpu():
    """All E disjoint experts at gate weight 1 (k = E fed through dispatch and the
    expert GEMMs, combine weights 1, no rescale) reproduce the dense FFN."""
    w = W("dense", T=200, d=256, d_ff=1024, E=8, k=8, seed=44)
    inp = wl.make_inputs(w)
    p = H.layer_params(w)
    ws = moe.Workspace(p)
    W13_e, W2_e = H.gpu_weights(w, inp, ws)
    b = moe.ForwardBuffers(p)
    x = inp["x"].cuda()
    idx = torch.arange(8, dtype=torch.int32, device="cuda").repeat(w.T, 1).contiguous()
    ones = torch.ones(w.T, 8, dtype=torch.float32, device="cuda")
    moe.moe_dispatch(p, x, idx, ws, b.x_perm, b.row_token, b.slot_row, b.counts, b.kept,
                     b.offsets)
    moe.moe_expert_ffn(p, b.x_perm, b.offsets, W13_e, W2_e, b.h, b.out, ws)
    moe.moe_combine(p, b.out, b.slot_row, ones, b.y)
    torch.cuda.synchronize()
    dense = oracle.dense_ffn(H.raw(inp["W1"]), H.raw(inp["W3"]), H.raw(inp["W2"]),
                             H.raw(inp["x"]))
    assert H.rel_err(H.f64(b.y), dense) <= 1e-2


# ------------------------------------------------------------------ full-size workloads

FULL = ["tiny_fp32", "moe_2of8", "moe_4of16", "e8t2_cf1", "e8t2_cf4", "decode_t1", "decode_t8",
        "decode_t64"]


@pytest.mark.slow
@pytest.mark.parametrize("name", FULL)
def test_full_size_workload(name):
    w = wl.WORKLOADS[name]
    inp = wl.make_inputs(w, device="cuda")
    big = w.name.startswith("e8t2")
    res = _full_check(w, inp, rows_sample=64 if big else 256, tok_sample=32 if big else 128)
    if w.cf >= 0:
        C = moe.moe_capacity(w.T, w.E, w.cf)
        assert C == oracle.capacity(w.T, w.E, w.cf)
        assert (res["bufs"].kept.cpu() <= C).all()


def test_gemm_band_order_changes_no_result():
    """The 2-SM expert GEMMs give the same bytes whatever band of rows the concurrent
    clusters sweep N over (whole experts, and bands of one, three and eight m-tiles)."""
    w = W("band", T=5000, d=256, d_ff=8 * 176, E=8, k=2, noisy=True, cf=1.3, seed=56)
    inp = wl.make_inputs(w)
    p = H.layer_params(w)
    ws = moe.Workspace(p)
    W13_e, W2_e = H.gpu_weights(w, inp, ws)
    b = moe.ForwardBuffers(p)
    x, Wg, Wn, eps = (inp[n].cuda() for n in ("x", "Wg", "Wnoise", "eps"))
    moe.moe_route(p, x, Wg, Wn, eps, None, ws, b.topk_idx, b.topk_w, b.probs_sum, b.importance)
    moe.moe_dispatch_routed(p, x, b.topk_idx, ws, b.x_perm, b.row_token, b.slot_row, b.counts,
                            b.kept, b.offsets)
    R = int(b.offsets[-1].item())
    res = []
    try:
        for band in (0, 256, 700, 2048):
            moe.moe_set_gemm_band_rows(band)
            h = torch.zeros_like(b.h)
            out = torch.zeros_like(b.out)
            moe.moe_expert_ffn(p, b.x_perm, b.offsets, W13_e, W2_e, h, out, ws)
            torch.cuda.synchronize()
            res.append((h[:R, :w.m].clone(), out[:R].clone()))
    finally:
        moe.moe_set_gemm_band_rows(2048)
    assert moe.moe_get_device_status(ws) == 0
    for h, out in res[1:]:
        assert torch.equal(h, res[0][0]) and torch.equal(out, res[0][1])


@pytest.mark.parametrize("name", ["mid_mixtral_noisy", "mid_st_bias_cap", "e64_k8", "odd_m_d",
                                  "pair_e16_odd", "copy_exact"])
def test_packed_router_weights_give_the_same_layer(name):
    """moe_route_packed with the weights packed once by moe_router_pack, and moe_forward
    given them, produce the bytes of moe_route / moe_forward packing per call."""
    w = SMALL[name]
    inp = wl.make_inputs(w)
    p, bufs, ws, status, (W13_e, W2_e) = H.run_forward(w, inp)
    assert status == 0
    x, Wg, Wn, eps, bias = (None if inp.get(n) is None else inp[n].to("cuda")
                            for n in ("x", "Wg", "Wnoise", "eps", "bias"))
    Wt = moe.moe_router_pack(p, Wg, Wn)
    assert Wt.numel() == moe.moe_router_packed_bytes(p, Wn is not None)
    a = moe.ForwardBuffers(p)
    moe.moe_route_packed(p, x, Wg, Wn, Wt, eps, bias, ws, a.topk_idx, a.topk_w, a.probs_sum,
                         a.importance)
    c = moe.ForwardBuffers(p)
    moe.moe_forward(p, x, Wg, W13_e, W2_e, ws, c, Wnoise=Wn, noise=eps, bias=bias,
                    router_packed=Wt)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    for n in ("topk_idx", "topk_w", "probs_sum", "importance"):
        assert torch.equal(getattr(a, n), getattr(bufs, n)), n
    for n in ("y", "topk_idx", "topk_w", "probs_sum", "importance", "counts", "kept", "offsets",
              "slot_row", "loss"):
        assert torch.equal(getattr(c, n), getattr(bufs, n)), n
