"""Pins of the fp64 CPU oracle to facts that do not come from the oracle itself:
hand-worked fixtures (tests/golden), closed forms, special cases that reduce to
library routines (numpy/scipy), brute force on tiny inputs, and invariants of
the layer stated on the pages (dense equivalence of a disjoint partition, the
copy invariant of upcycling, softmax normalisation, the capacity formula).
"""
import itertools
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16_bits(a: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16) \
        .view(torch.int16).numpy().view(np.uint16)


def _rng(seed):
    return np.random.default_rng(seed)


def _layer(seed, T, d, d_ff, E, dtype="f32"):
    r = _rng(seed)
    x = r.standard_normal((T, d)).astype(np.float32)
    W1 = (0.1 * r.standard_normal((d_ff, d))).astype(np.float32)
    W3 = (0.1 * r.standard_normal((d_ff, d))).astype(np.float32)
    W2 = (0.1 * r.standard_normal((d, d_ff))).astype(np.float32)
    Wg = (0.1 * r.standard_normal((d, E))).astype(np.float32)
    perm = r.permutation(d_ff).astype(np.int32)
    if dtype == "bf16":
        x, W1, W3, W2, Wg = map(_bf16_bits, (x, W1, W3, W2, Wg))
    return x, W1, W3, W2, Wg, perm


def _numpy_dense_ffn(W1, W3, W2, x):
    """Dense SwiGLU FFN with library matmul and scipy's logistic function."""
    import oracle
    W1, W3, W2, x = map(oracle.to_f64, (W1, W3, W2, x))
    g = x @ W1.T
    u = x @ W3.T
    return (g * scipy.special.expit(g) * u) @ W2.T


# --------------------------------------------------------------------------- scalars

def test_softplus_matches_logaddexp(orc):
    for z in np.concatenate([np.linspace(-40, 40, 161), [-700.0, -1e-9, 0.0, 1e-9, 700.0]]):
        assert orc.softplus(z) == pytest.approx(np.logaddexp(0.0, z), rel=1e-14, abs=1e-300)
    assert orc.softplus(0.0) == pytest.approx(math.log(2.0), rel=1e-15)


def test_silu_matches_scipy_expit(orc):
    for z in np.linspace(-30, 30, 121):
        assert orc.silu(z) == pytest.approx(z * scipy.special.expit(z), rel=1e-14, abs=1e-300)


# --------------------------------------------------------------------------- a0 partition

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_partition_is_disjoint_equal_gather(orc, dtype):
    T, d, d_ff, E = 3, 24, 40, 4
    x, W1, W3, W2, Wg, perm = _layer(1, T, d, d_ff, E, dtype)
    W1e, W3e, W2e = orc.partition(W1, W3, W2, E, orc.DISJOINT, perm)
    m = d_ff // E
    assert W1e.shape == (E, m, d) and W2e.shape == (E, d, m)
    sets = [set(perm[e * m:(e + 1) * m].tolist()) for e in range(E)]
    assert all(len(s) == m for s in sets)
    assert set().union(*sets) == set(range(d_ff))
    for a, b in itertools.combinations(sets, 2):
        assert not (a & b)
    for e in range(E):
        ids = perm[e * m:(e + 1) * m]
        np.testing.assert_array_equal(W1e[e], W1[ids])
        np.testing.assert_array_equal(W3e[e], W3[ids])
        np.testing.assert_array_equal(W2e[e], W2[:, ids])
    C1, C3, C2 = orc.partition(W1, W3, W2, E, orc.COPY)
    for e in range(E):
        np.testing.assert_array_equal(C1[e], W1)
        np.testing.assert_array_equal(C2[e], W2)


def test_partition_rejects_indivisible(orc):
    x, W1, W3, W2, Wg, perm = _layer(2, 2, 8, 10, 3)
    with pytest.raises(ValueError):
        orc.partition(W1, W3, W2, 3, orc.DISJOINT, perm)


def test_generated_perm_is_a_permutation():
    w = wl.WORKLOADS["moe_2of8"]
    inp = wl.make_inputs(w.with_(T=4))
    p = inp["perm"].numpy()
    assert np.array_equal(np.sort(p), np.arange(w.d_ff))


# --------------------------------------------------------------------------- dense equivalence

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_dense_ffn_matches_library(orc, dtype):
    x, W1, W3, W2, Wg, perm = _layer(3, 9, 32, 48, 4, dtype)
    y = orc.dense_ffn(W1, W3, W2, x)
    ref = _numpy_dense_ffn(W1, W3, W2, x)
    np.testing.assert_allclose(y, ref, rtol=1e-11, atol=1e-12 * np.abs(ref).max())


@pytest.mark.parametrize("dtype,E", [("f32", 4), ("bf16", 8), ("f32", 1)])
def test_disjoint_experts_all_selected_equal_dense(orc, dtype, E):
    """With every disjoint expert selected at gate weight 1 and no rescale, the MoE
    layer is the dense FFN (the partition only regroups the intermediate neurons)."""
    T, d, d_ff = 11, 32, 64
    x, W1, W3, W2, Wg, perm = _layer(4, T, d, d_ff, E, dtype)
    W1e, W3e, W2e = orc.partition(W1, W3, W2, E, orc.DISJOINT, perm)
    idx = np.tile(np.arange(E, dtype=np.int32), (T, 1))
    dsp = orc.dispatch(idx, E, -1)
    assert dsp["R"] == T * E
    eor = np.searchsorted(dsp["offsets"], np.arange(dsp["R"]), side="right") - 1
    out = orc.expert_ffn(W1e, W3e, W2e, x[dsp["row_token"]], eor)
    y = orc.combine(out, dsp["slot_row"], np.ones((T, E)), 1.0)
    dense = orc.dense_ffn(W1, W3, W2, x)
    np.testing.assert_allclose(y, dense, rtol=1e-11, atol=1e-12 * np.abs(dense).max())


def test_copy_invariant_mixtral_and_st(orc):
    """Upcycled copies: Mixtral weights sum to one, so y = FFN(x); ST weights give
    y = (sum_j G_j) FFN(x)."""
    T, d, d_ff, E, k = 13, 16, 24, 4, 2
    x, W1, W3, W2, Wg, perm = _layer(5, T, d, d_ff, E)
    W1e, W3e, W2e = orc.partition(W1, W3, W2, E, orc.COPY)
    dense = orc.dense_ffn(W1, W3, W2, x)
    res = orc.forward(x, Wg, W1e, W3e, W2e, k, orc.MIXTRAL)
    np.testing.assert_allclose(res["y"], dense, rtol=1e-11, atol=1e-12 * np.abs(dense).max())
    res = orc.forward(x, Wg, W1e, W3e, W2e, k, orc.ST)
    gs = res["router"]["G"].sum(1, keepdims=True)
    np.testing.assert_allclose(res["y"], gs * dense, rtol=1e-11,
                               atol=1e-12 * np.abs(dense).max())


def test_single_expert_rescale(orc):
    T, d, d_ff = 7, 16, 24
    x, W1, W3, W2, Wg, perm = _layer(6, T, d, d_ff, 1)
    W1e, W3e, W2e = orc.partition(W1, W3, W2, 1, orc.DISJOINT, perm)
    res = orc.forward(x, Wg, W1e, W3e, W2e, 1, orc.MIXTRAL, rescale=True)
    dense = orc.dense_ffn(W1, W3, W2, x)
    np.testing.assert_allclose(res["y"], dense, rtol=1e-11, atol=1e-12 * np.abs(dense).max())


# --------------------------------------------------------------------------- a1 router

def _load_router_cases():
    cases = []
    with open(os.path.join(GOLDEN, "router_closed_form.txt")) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            f = [s.strip() for s in line.split("|")]
            vec = (lambda s: None if s == "-" else [float(v) for v in s.split()])
            env = {"exp": math.exp, "e": math.e, "ln": math.log, "__builtins__": {}}
            cases.append(dict(name=f[0], router=f[1], k=int(f[2]), L=vec(f[3]), Ln=vec(f[4]),
                              eps=vec(f[5]), bias=vec(f[6]), idx=[int(v) for v in f[7].split()],
                              G=[eval(s, env) for s in f[8].split(";")]))
    return cases


@pytest.mark.parametrize("case", _load_router_cases(), ids=lambda c: c["name"])
def test_router_closed_forms(orc, case):
    E, d = len(case["L"]), 8
    x = np.zeros((1, d), np.float32)
    x[0, 0] = 1.0
    Wg = np.zeros((d, E), np.float32)
    Wg[0] = case["L"]
    Wn = eps = None
    if case["Ln"] is not None:
        Wn = np.zeros((d, E), np.float32)
        Wn[0] = case["Ln"]
        eps = np.array([case["eps"]], np.float32)
    bias = None if case["bias"] is None else np.array(case["bias"], np.float32)
    rt = orc.MIXTRAL if case["router"] == "mixtral" else orc.ST
    r = orc.router(x, Wg, Wn, eps, bias, case["k"], rt)
    assert r["idx"][0].tolist() == case["idx"]
    np.testing.assert_allclose(r["G"][0], case["G"], rtol=1e-14)


def _random_router(orc, seed, T, d, E, k, rt, noisy, bias, dtype="f32"):
    r = _rng(seed)
    x = r.standard_normal((T, d)).astype(np.float32)
    Wg = (0.3 * r.standard_normal((d, E))).astype(np.float32)
    Wn = (0.3 * r.standard_normal((d, E))).astype(np.float32) if noisy else None
    eps = r.standard_normal((T, E)).astype(np.float32) if noisy else None
    b = r.standard_normal(E).astype(np.float32) if bias else None
    if dtype == "bf16":
        x, Wg = _bf16_bits(x), _bf16_bits(Wg)
        Wn = _bf16_bits(Wn) if noisy else None
    return orc.router(x, Wg, Wn, eps, b, k, rt), (x, Wg, Wn, eps, b)


@pytest.mark.parametrize("rt", [0, 1])
def test_router_weight_sums_and_full_softmax(orc, rt):
    T, d, E, k = 40, 16, 8, 3
    res, _ = _random_router(orc, 7, T, d, E, k, rt, True, True)
    G, H = res["G"], res["H"]
    full = scipy.special.softmax(H, axis=1)
    if rt == orc.MIXTRAL:
        np.testing.assert_allclose(G.sum(1), 1.0, rtol=1e-13)
    else:
        assert np.all(G.sum(1) <= 1.0 + 1e-13)
        np.testing.assert_allclose(G, np.take_along_axis(full, res["idx"], 1), rtol=1e-13)
    # P uses the full softmax of the routing logits H (noise and bias included)
    np.testing.assert_allclose(res["probs_sum"], full.sum(0), rtol=1e-12)
    # importance = per-expert sum of the gate weights
    imp = np.zeros(E)
    np.add.at(imp, res["idx"].ravel(), G.ravel())
    np.testing.assert_allclose(res["importance"], imp, rtol=1e-12)
    # k = E: Mixtral and ST both give the full softmax in descending order
    resE, _ = _random_router(orc, 7, T, d, E, E, rt, True, True)
    np.testing.assert_allclose(resE["G"], np.take_along_axis(full, resE["idx"], 1), rtol=1e-12)
    np.testing.assert_allclose(resE["G"].sum(1), 1.0, rtol=1e-13)


def test_router_noise_is_eps_times_softplus(orc):
    """H - L = eps * softplus(x.W_noise), checked against numpy's logaddexp."""
    T, d, E = 20, 12, 6
    res, (x, Wg, Wn, eps, b) = _random_router(orc, 8, T, d, E, 2, 0, True, False)
    L = x.astype(np.float64) @ Wg.astype(np.float64)
    Ln = x.astype(np.float64) @ Wn.astype(np.float64)
    np.testing.assert_allclose(res["H"], L + eps * np.logaddexp(0.0, Ln), rtol=1e-12, atol=1e-13)


def test_k1_mixtral_weight_is_one(orc):
    res, _ = _random_router(orc, 9, 30, 8, 8, 1, 0, True, False)
    np.testing.assert_array_equal(res["G"], 1.0)


def test_topk_brute_force_with_ties(orc):
    """Sort-based KeepTopK against enumeration of all k-subsets: the chosen set has the
    largest sum and, among equal sums, the lexicographically smallest index set."""
    r = _rng(10)
    n = 0
    for E in range(1, 9):
        for k in range(1, E + 1):
            for _ in range(12):
                h = r.integers(-2, 3, size=E).astype(np.float64)  # many ties
                if r.random() < 0.3:
                    h = r.standard_normal(E)
                got = orc.topk(h, k)
                best = max(itertools.combinations(range(E), k),
                           key=lambda s: (sum(h[list(s)]), [-i for i in s]))
                assert sorted(got.tolist()) == list(best)
                # slot order: descending value, ties by lower index
                keys = [(-h[i], i) for i in got]
                assert keys == sorted(keys)
                n += 1
    assert n > 400


def test_topk_rejects_nan(orc):
    with pytest.raises(ValueError):
        orc.topk(np.array([0.0, np.nan, 1.0]), 2)


# --------------------------------------------------------------------------- a2 dispatch

def test_capacity_formula(orc):
    # tokens per batch / N x CF for the upcycling workload
    assert orc.capacity(32768, 8, 1.0) == 32768 // 8 * 1 == 4096
    assert orc.capacity(32768, 8, 4.0) == 16384
    assert orc.capacity(10, 3, 1.0) == 4          # rounded up to a whole token
    assert orc.capacity(16384, 16, 1.25) == 1280
    assert orc.capacity(100, 8, -1.0) == -1


def _load_dispatch_golden():
    spec, cases, cur = {}, [], None
    with open(os.path.join(GOLDEN, "dispatch_capacity.txt")) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, _, rest = line.partition(" ")
            vals = [int(v) for v in rest.split()] if key != "case" else rest
            if key == "case":
                cur = {"C": int(rest.split("=")[1])}
                cases.append(cur)
            elif cur is None:
                spec[key] = vals
            else:
                cur[key] = vals
    return spec, cases


def test_dispatch_golden(orc):
    spec, cases = _load_dispatch_golden()
    T, E, k = spec["T"][0], spec["E"][0], spec["k"][0]
    idx = np.array(spec["idx"], np.int32).reshape(T, k)
    assert len(cases) == 3
    for c in cases:
        got = orc.dispatch(idx, E, c["C"])
        for key in ("counts", "kept", "offsets", "row_token"):
            assert got[key].tolist() == c[key], (c["C"], key)
        assert got["slot_row"].ravel().tolist() == c["slot_row"], c["C"]


@pytest.mark.parametrize("C", [-1, 0, 1, 5, 37, 1000])
def test_dispatch_matches_stable_sort_recount(orc, C):
    r = _rng(11)
    T, E, k = 333, 7, 3
    idx = np.stack([r.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    got = orc.dispatch(idx, E, C)
    counts = np.bincount(idx.ravel(), minlength=E)
    kept = counts if C < 0 else np.minimum(counts, C)
    assert got["counts"].tolist() == counts.tolist()
    assert got["kept"].tolist() == kept.tolist()
    assert got["R"] == kept.sum() == got["offsets"][-1]
    flat_e = idx.ravel()
    order = np.argsort(flat_e, kind="stable")          # assignments grouped by expert
    tok = order // k
    slot = np.full(T * k, -1)
    row = 0
    for e in range(E):
        sel = order[flat_e[order] == e]
        keep = sel[:kept[e]]
        np.testing.assert_array_equal(got["row_token"][row:row + kept[e]], keep // k)
        slot[keep] = np.arange(row, row + kept[e])
        row += kept[e]
    np.testing.assert_array_equal(got["slot_row"].ravel(), slot)
    assert len(tok) == T * k


def test_dispatch_treats_bad_index_as_dropped(orc):
    idx = np.array([[0, 5], [-1, 1]], np.int32)
    got = orc.dispatch(idx, 2, -1)
    assert got["counts"].tolist() == [1, 1]
    assert got["slot_row"].tolist() == [[0, -1], [-1, 1]]


# --------------------------------------------------------------------------- a5 / a6

def test_all_dropped_token_is_zero(orc):
    out = np.arange(6, dtype=np.float64).reshape(2, 3)
    y = orc.combine(out, np.array([[0, -1], [-1, -1]], np.int32), np.ones((2, 2)), 2.0)
    np.testing.assert_array_equal(y, [[0.0, 2.0, 4.0], [0.0, 0.0, 0.0]])


def test_balance_closed_form_all_ties(orc):
    """W_g = 0, no noise, no bias: every logit ties, the first k experts take every
    token, so f = 1/k on them, P = 1/E everywhere and L = lambda / E."""
    T, d, E, k, lam = 50, 8, 8, 2, 0.01
    x = _rng(12).standard_normal((T, d)).astype(np.float32)
    Wg = np.zeros((d, E), np.float32)
    r = orc.router(x, Wg, k=k)
    assert (r["idx"] == np.arange(k)).all()
    dsp = orc.dispatch(r["idx"], E, -1)
    f, P, L = orc.gate_stats(T, k, dsp["counts"], r["probs_sum"], lam)
    np.testing.assert_allclose(f, [1 / k] * k + [0.0] * (E - k), rtol=1e-15)
    np.testing.assert_allclose(P, 1.0 / E, rtol=1e-14)
    assert L == pytest.approx(lam / E, rel=1e-14)


def test_gate_stats_empty_batch(orc):
    f, P, L = orc.gate_stats(0, 2, np.zeros(4, np.int32), np.zeros(4), 0.01)
    assert L == 0.0 and not f.any() and not P.any()


# --------------------------------------------------------------------------- T = 0

def test_empty_batch(orc):
    x, W1, W3, W2, Wg, perm = _layer(13, 0, 16, 32, 4)
    W1e, W3e, W2e = orc.partition(W1, W3, W2, 4, orc.DISJOINT, perm)
    res = orc.forward(x, Wg, W1e, W3e, W2e, 2)
    assert res["y"].shape == (0, 16)
    assert res["dispatch"]["R"] == 0
    assert res["dispatch"]["counts"].tolist() == [0, 0, 0, 0]


# --------------------------------------------------------------------------- page-2 code sample

def test_cross_read_of_v2_code_sample(orc):
    """An independent torch fp64 restatement of the LLaMA-MoE v2 code sample's layer
    (loop over experts with boolean masks; ST gate = topk of the softmax; output
    times N/k; inference mode, so no noise) agrees with the oracle's forward."""
    T, d, d_ff, E, k = 37, 24, 64, 8, 2
    x, W1, W3, W2, Wg, perm = _layer(14, T, d, d_ff, E)
    W1e, W3e, W2e = orc.partition(W1, W3, W2, E, orc.DISJOINT, perm)
    res = orc.forward(x, Wg, W1e, W3e, W2e, k, orc.ST, rescale=True)

    X = torch.from_numpy(x).double()
    logits = X @ torch.from_numpy(Wg).double()
    probs = torch.softmax(logits, dim=-1)
    w, ix = torch.topk(probs, k, dim=-1)
    gate = torch.zeros(T, E, dtype=torch.float64).scatter(1, ix, w)
    y = torch.zeros_like(X)
    for e in range(E):
        mask = gate[:, e] > 0
        if not mask.any():
            continue
        xe = X[mask]
        a = xe @ torch.from_numpy(W1e[e]).double().T
        b = xe @ torch.from_numpy(W3e[e]).double().T
        oe = (torch.nn.functional.silu(a) * b) @ torch.from_numpy(W2e[e]).double().T
        y[mask] += oe * gate[mask, e].unsqueeze(-1)
    y = y * (E / k)
    np.testing.assert_allclose(res["y"], y.numpy(), rtol=1e-11, atol=1e-12 * y.abs().max().item())

    # its load-balancing term: normalised weight sums x mean clean softmax x N
    freq = gate.sum(0) / (gate.sum() + 1e-6)
    Lb = float((freq * probs.mean(0)).sum() * E)
    r = res["router"]
    assert orc.balance_sketch(r["idx"], r["G"], r["clean_probs_sum"]) == pytest.approx(Lb, rel=1e-12)


def test_forward_sample_equals_full(orc):
    T, d, d_ff, E, k = 29, 16, 32, 4, 2
    x, W1, W3, W2, Wg, perm = _layer(15, T, d, d_ff, E, "bf16")
    W1e, W3e, W2e = orc.partition(W1, W3, W2, E, orc.DISJOINT, perm)
    full = orc.forward(x, Wg, W1e, W3e, W2e, k, capacity_rows=10)
    toks = [0, 3, 17, 28]
    part = orc.forward(x, Wg, W1e, W3e, W2e, k, capacity_rows=10, tokens=toks)
    np.testing.assert_array_equal(part["y"], full["y"][toks])
    assert full["dispatch"]["R"] < T * k  # some assignments dropped


# --------------------------------------------------------------------------- residual MoE

def _residual_split(seed, d_ff, m_s):
    perm = _rng(seed).permutation(d_ff).astype(np.int32)
    return perm[:m_s], perm[m_s:]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_residual_all_experts_selected_equal_dense(orc, dtype):
    """Shared block plus every disjoint expert at gate weight 1 (no rescale) is the
    dense FFN: S and the experts together regroup all intermediate neurons."""
    T, d, d_ff, E, m_s = 9, 32, 72, 4, 8
    x, W1, W3, W2, Wg, _ = _layer(21, T, d, d_ff, E, dtype)
    shared, rest = _residual_split(22, d_ff, m_s)
    (W1e, W3e, W2e), blk = orc.partition_residual(W1, W3, W2, E, shared, rest)
    idx = np.tile(np.arange(E, dtype=np.int32), (T, 1))
    dsp = orc.dispatch(idx, E, -1)
    eor = np.searchsorted(dsp["offsets"], np.arange(dsp["R"]), side="right") - 1
    out = orc.expert_ffn(W1e, W3e, W2e, x[dsp["row_token"]], eor)
    y = orc.combine(out, dsp["slot_row"], np.ones((T, E)), 1.0) + orc.dense_ffn(*blk, x)
    ref = _numpy_dense_ffn(W1, W3, W2, x)
    np.testing.assert_allclose(y, ref, rtol=1e-10, atol=1e-11 * np.abs(ref).max())


def test_residual_capacity_zero_leaves_the_shared_block(orc):
    """With capacity 0 every routed assignment is dropped: y is exactly the shared
    block, the SwiGLU FFN restricted to the neurons of S (numpy)."""
    T, d, d_ff, E, k, m_s = 10, 24, 40, 4, 2, 8
    x, W1, W3, W2, Wg, _ = _layer(23, T, d, d_ff, E)
    shared, rest = _residual_split(24, d_ff, m_s)
    experts, blk = orc.partition_residual(W1, W3, W2, E, shared, rest)
    r = orc.forward_residual(x, Wg, experts, blk, k, capacity_rows=0, rescale=True)
    ref = _numpy_dense_ffn(W1[shared], W3[shared], W2[:, shared], x)
    assert (r["dispatch"]["slot_row"] == -1).all()
    np.testing.assert_allclose(r["y"], ref, rtol=1e-11, atol=1e-12 * np.abs(ref).max())


def test_residual_is_shared_block_plus_routed_layer(orc):
    """The routed part of the residual layer is the plain MoE layer over the
    non-shared neurons; E/k rescale applies to it and not to the shared block."""
    T, d, d_ff, E, k, m_s = 12, 16, 56, 4, 2, 16
    x, W1, W3, W2, Wg, _ = _layer(25, T, d, d_ff, E)
    shared, rest = _residual_split(26, d_ff, m_s)
    experts, blk = orc.partition_residual(W1, W3, W2, E, shared, rest)
    r = orc.forward_residual(x, Wg, experts, blk, k, rescale=True)
    # the routed experts rebuilt independently from the numpy weights
    m = (d_ff - m_s) // E
    y_moe = np.zeros((T, d))
    G = r["router"]["G"]
    for t in range(T):
        for j in range(k):
            e = int(r["router"]["idx"][t, j])
            cols = rest[e * m:(e + 1) * m]
            y_moe[t] += G[t, j] * _numpy_dense_ffn(W1[cols], W3[cols], W2[:, cols], x[t:t + 1])[0]
    ref = _numpy_dense_ffn(W1[shared], W3[shared], W2[:, shared], x) + (E / k) * y_moe
    np.testing.assert_allclose(r["y"], ref, rtol=1e-10, atol=1e-11 * np.abs(ref).max())


# --------------------------------------------------------------------------- clustering

def _load_cluster_golden():
    cases, cur = [], None
    with open(os.path.join(GOLDEN, "cluster_hand.txt")) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, _, rest = line.partition(" ")
            if key == "case":
                cur = {"name": rest}
                cases.append(cur)
            elif key == "centers":
                cur[key] = [int(n) / int(q) for n, q in (v.split("/") for v in rest.split())]
            else:
                cur[key] = [int(v) for v in rest.split()]
    return cases


def test_cluster_golden(orc):
    cases = _load_cluster_golden()
    assert len(cases) == 7
    for c in cases:
        d, E = c["d"][0], c["E"][0]
        F = np.array(c["F"], np.float32).reshape(-1, d)
        assign, centers, perm = orc.cluster(F, E, c["iters"][0], c["init"])
        assert assign.tolist() == c["assign"], c["name"]
        assert perm.tolist() == c["perm"], c["name"]
        assert centers.ravel().tolist() == c["centers"], c["name"]


def _separated_groups(seed, E, m, d):
    """E groups of m neurons around far-apart anchors, rows shuffled."""
    r = _rng(seed)
    anchors = 10.0 * r.standard_normal((E, d))
    label = np.repeat(np.arange(E), m)
    F = anchors[label] + 0.05 * r.standard_normal((E * m, d))
    order = r.permutation(E * m)
    return F[order].astype(np.float32), label[order]


@pytest.mark.parametrize("E,m,d", [(4, 6, 16), (8, 5, 24)])
def test_cluster_separated_groups_match_lloyd(orc, E, m, d):
    """When the nearest-center assignment is already balanced, the balanced
    k-means is Lloyd's k-means: compare with scikit-learn's, started from the
    same centers."""
    from sklearn.cluster import KMeans
    F, label = _separated_groups(31 + E, E, m, d)
    r = _rng(7)
    init = np.array([r.choice(np.flatnonzero(label == g)) for g in r.permutation(E)], np.int32)
    assign, centers, perm = orc.cluster(F, E, 3, init)
    km = KMeans(n_clusters=E, init=F[init].astype(np.float64), n_init=1, max_iter=3,
                algorithm="lloyd", tol=0.0).fit(F.astype(np.float64))
    assert assign.tolist() == km.labels_.tolist()
    np.testing.assert_allclose(centers, km.cluster_centers_, rtol=1e-12, atol=1e-12)
    # the groups come back whole: cluster e is the group of its initial neuron
    for e in range(E):
        assert set(np.flatnonzero(assign == e)) == set(np.flatnonzero(label == label[init[e]]))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_cluster_invariants_and_first_round(orc, dtype):
    """Balance, permutation layout, centers = numpy mean of the members; and for
    one iteration, the first round of the assignment against scipy distances:
    a cluster whose nearest-neuron set fits keeps all of it, one that overflows
    keeps its m nearest."""
    from scipy.spatial.distance import cdist
    E, m, d = 6, 7, 20
    r = _rng(41)
    F = r.standard_normal((E * m, d)).astype(np.float32)
    if dtype == "bf16":
        F = _bf16_bits(F)
    F64 = orc.to_f64(F)
    init = r.choice(E * m, E, replace=False).astype(np.int32)
    for iters in (1, 4):
        assign, centers, perm = orc.cluster(F, E, iters, init)
        assert np.bincount(assign, minlength=E).tolist() == [m] * E
        assert sorted(perm.tolist()) == list(range(E * m))
        for e in range(E):
            seg = perm[e * m:(e + 1) * m]
            assert (np.diff(seg) > 0).all() and (assign[seg] == e).all()
            np.testing.assert_allclose(centers[e], F64[seg].mean(axis=0), rtol=1e-13, atol=1e-15)
    assign, _, _ = orc.cluster(F, E, 1, init)
    D = cdist(F64, F64[init], "sqeuclidean")
    near = D.argmin(axis=1)
    for e in range(E):
        P = np.flatnonzero(near == e)
        kept = P if len(P) <= m else P[np.argsort(D[P, e], kind="stable")[:m]]
        assert (assign[kept] == e).all(), e
        if len(P) > m:
            assert (assign[np.setdiff1d(P, kept)] != e).all(), e


def test_cluster_special_cases(orc):
    r = _rng(43)
    F = r.standard_normal((12, 5)).astype(np.float32)
    # E = 1: one cluster, its center the mean of all rows
    assign, centers, perm = orc.cluster(F, 1, 2, [4])
    assert (assign == 0).all() and perm.tolist() == list(range(12))
    np.testing.assert_allclose(centers[0], F.astype(np.float64).mean(axis=0), rtol=1e-13)
    # m = 1: every neuron is the center of its own cluster
    init = r.permutation(12).astype(np.int32)
    assign, centers, perm = orc.cluster(F, 12, 1, init)
    assert perm.tolist() == init.tolist()
    assert assign[init].tolist() == list(range(12))
    np.testing.assert_array_equal(centers, F[init].astype(np.float64))


def test_cluster_rejects_bad_arguments(orc):
    F = np.zeros((8, 4), np.float32)
    for E, it, init in ((3, 1, [0, 1, 2]), (2, 0, [0, 1]), (2, 1, [1, 1]), (2, 1, [0, 8])):
        with pytest.raises(ValueError):
            orc.cluster(F, E, it, init)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_sqdist_matches_scipy(orc, dtype):
    from scipy.spatial.distance import cdist
    r = _rng(47)
    F = r.standard_normal((37, 29)).astype(np.float32)
    if dtype == "bf16":
        F = _bf16_bits(F)
    Cc = r.standard_normal((5, 29))
    D = orc.sqdist(F, Cc)
    np.testing.assert_allclose(D, cdist(orc.to_f64(F), Cc, "sqeuclidean"), rtol=1e-13)
