"""Python face of the fp64 CPU oracle (``oracle/moe_oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package; the product library never
does.  It shares no code with the CUDA path.

Arrays are numpy.  Floating-point inputs are either ``float32`` (fp32 data) or
``uint16`` holding raw bfloat16 bit patterns (bf16 data); the C code widens them
exactly to double.  All floating-point results are ``float64``.
"""
import ctypes as C
import os

import numpy as np

from . import build as _build

MIXTRAL = 0
ST = 1
DISJOINT = 0
COPY = 1

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        _lib = C.CDLL(path)
        d = C.c_double
        p = C.c_void_p
        i = C.c_int
        _lib.oracle_softplus.restype = d
        _lib.oracle_softplus.argtypes = [d]
        _lib.oracle_silu.restype = d
        _lib.oracle_silu.argtypes = [d]
        _lib.oracle_capacity.argtypes = [i, i, d]
        _lib.oracle_set_num_threads.argtypes = [i]
        _lib.oracle_set_num_threads.restype = None
        _lib.oracle_partition.argtypes = [p, p, p, i, i, i, i, i, p, p, p, p]
        _lib.oracle_topk.argtypes = [i, i, p, p]
        _lib.oracle_router.argtypes = [i, i, i, i, i, p, i, p, p, p, p, p, p, p, p, p, p]
        _lib.oracle_dispatch.argtypes = [i, i, i, p, i, p, p, p, p, p]
        _lib.oracle_expert_ffn.argtypes = [i, i, i, p, p, p, i, p, i, p, i, p, p]
        _lib.oracle_dense_ffn.argtypes = [i, i, p, p, p, i, p, i, i, p]
        _lib.oracle_combine.argtypes = [i, i, i, p, p, p, d, p]
        _lib.oracle_gate_stats.argtypes = [i, i, i, p, p, d, p, p, p]
        _lib.oracle_balance_sketch.argtypes = [i, i, i, p, p, p, p]
        _lib.oracle_cluster.argtypes = [p, i, i, i, i, i, p, p, p, p]
        _lib.oracle_sqdist.argtypes = [p, i, i, i, i, p, p]
        _lib.oracle_combine_backward.argtypes = [i, i, i, p, p, p, d, p, p, p]
        _lib.oracle_expert_ffn_backward.argtypes = [i, i, i, p, p, p, i, p, i, p, i, p, p, p, p,
                                                    p, p, p, p]
        _lib.oracle_router_backward.argtypes = [i, i, i, i, i, p, i, p, p, p, p, p, p, p, p, d,
                                                d, p, p, p, p, p, p]
        _lib.oracle_router_backward_norm.argtypes = [i, i, i, i, i, i, p, i, p, p, p, p, p, p, p,
                                                     p, d, d, p, p, p, p, p, p]
        _lib.oracle_neuron_wgrad.argtypes = [i, i, i, p, p, p, i, p, i, i, p, p, p, p]
    return _lib


def num_threads() -> int:
    return int(lib().oracle_num_threads())


def set_num_threads(n: int) -> None:
    """Host threads of the oracle's parallel loops from now on (results do not change)."""
    lib().oracle_set_num_threads(int(n))


def _dt(a: np.ndarray) -> int:
    if a.dtype == np.float32:
        return 0
    if a.dtype == np.uint16:
        return 1
    raise TypeError("oracle inputs are float32 or uint16 (raw bf16 bits), got %s" % a.dtype)


def _c(a, dtype=None):
    a = np.ascontiguousarray(a if dtype is None else a.astype(dtype, copy=False))
    return a


def _ptr(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _check(rc, what):
    if rc < 0:
        raise ValueError("oracle %s rejected its arguments (rc=%d)" % (what, rc))
    return rc


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of raw bf16 bit patterns (uint16) as float64."""
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def to_f64(a: np.ndarray) -> np.ndarray:
    return bf16_to_f64(a) if a.dtype == np.uint16 else a.astype(np.float64)


def softplus(z: float) -> float:
    return lib().oracle_softplus(float(z))


def silu(z: float) -> float:
    return lib().oracle_silu(float(z))


def capacity(T: int, E: int, cf: float) -> int:
    return int(lib().oracle_capacity(int(T), int(E), float(cf)))


def partition(W1, W3, W2, E: int, mode: int = DISJOINT, perm=None):
    """a0: per-expert W1e, W3e [E][m][d] and W2e [E][d][m] (same element type)."""
    W1, W3, W2 = _c(W1), _c(W3), _c(W2)
    dt = _dt(W1)
    d_ff, d = W1.shape
    m = d_ff // E if mode == DISJOINT else d_ff
    W1e = np.empty((E, m, d), W1.dtype)
    W3e = np.empty((E, m, d), W1.dtype)
    W2e = np.empty((E, d, m), W1.dtype)
    pp = None if perm is None else _c(perm, np.int32)
    _check(lib().oracle_partition(_ptr(W1), _ptr(W3), _ptr(W2), dt, d, d_ff, E, mode,
                                  _ptr(pp), _ptr(W1e), _ptr(W3e), _ptr(W2e)), "partition")
    return W1e, W3e, W2e


def topk(h, k: int):
    h = _c(h, np.float64)
    idx = np.empty(k, np.int32)
    _check(lib().oracle_topk(h.shape[0], k, _ptr(h), _ptr(idx)), "topk")
    return idx


def router(x, Wg, Wnoise=None, eps=None, bias=None, k=2, router_type=MIXTRAL):
    """a1: routing logits, Top-k indices and gate weights, plus the token sums."""
    x, Wg = _c(x), _c(Wg)
    dt = _dt(x)
    assert _dt(Wg) == dt
    T, d = x.shape
    E = Wg.shape[1]
    Wn = None if Wnoise is None else _c(Wnoise)
    ep = None if eps is None else _c(eps, np.float32)
    b = None if bias is None else _c(bias, np.float32)
    H = np.empty((T, E), np.float64)
    idx = np.empty((T, k), np.int32)
    G = np.empty((T, k), np.float64)
    ps = np.empty(E, np.float64)
    cps = np.empty(E, np.float64)
    imp = np.empty(E, np.float64)
    _check(lib().oracle_router(T, d, E, k, router_type, _ptr(x), dt, _ptr(Wg), _ptr(Wn),
                               _ptr(ep), _ptr(b), _ptr(H), _ptr(idx), _ptr(G), _ptr(ps),
                               _ptr(cps), _ptr(imp)), "router")
    return dict(H=H, idx=idx, G=G, probs_sum=ps, clean_probs_sum=cps, importance=imp)


def dispatch(idx, E: int, C_cap: int):
    """a2: counting-sort dispatch with capacity; returns the integer tables."""
    idx = _c(idx, np.int32)
    T, k = idx.shape
    counts = np.empty(E, np.int32)
    kept = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    row_token = np.full(max(T * k, 1), -1, np.int32)
    slot_row = np.empty((T, k), np.int32)
    R = _check(lib().oracle_dispatch(T, E, k, _ptr(idx), int(C_cap), _ptr(counts), _ptr(kept),
                                     _ptr(offsets), _ptr(row_token), _ptr(slot_row)), "dispatch")
    return dict(counts=counts, kept=kept, offsets=offsets, row_token=row_token[:R],
                slot_row=slot_row, R=R)


def expert_ffn(W1e, W3e, W2e, x_rows, expert_of_row, want_h=False):
    """a3+a4: SwiGLU expert outputs for each given row (float64 [n][d])."""
    W1e, W3e, W2e = _c(W1e), _c(W3e), _c(W2e)
    E, m, d = W1e.shape
    x_rows = _c(x_rows)
    eor = _c(expert_of_row, np.int32)
    n = x_rows.shape[0]
    out = np.empty((n, d), np.float64)
    h = np.empty((n, m), np.float64) if want_h else None
    _check(lib().oracle_expert_ffn(d, m, E, _ptr(W1e), _ptr(W3e), _ptr(W2e), _dt(W1e),
                                   _ptr(x_rows), _dt(x_rows), _ptr(eor), n, _ptr(out),
                                   _ptr(h)), "expert_ffn")
    return (out, h) if want_h else out


def dense_ffn(W1, W3, W2, x):
    """The dense SwiGLU FFN the experts were cut from (float64 [n][d])."""
    W1, W3, W2, x = _c(W1), _c(W3), _c(W2), _c(x)
    d_ff, d = W1.shape
    n = x.shape[0]
    y = np.empty((n, d), np.float64)
    _check(lib().oracle_dense_ffn(d, d_ff, _ptr(W1), _ptr(W3), _ptr(W2), _dt(W1), _ptr(x),
                                  _dt(x), n, _ptr(y)), "dense_ffn")
    return y


def combine(out_rows, slot_row, G, scale: float):
    """a5: gate-weighted combine (float64 [T][d])."""
    out_rows = _c(out_rows, np.float64)
    slot_row = _c(slot_row, np.int32)
    G = _c(G, np.float64)
    T, k = slot_row.shape
    d = out_rows.shape[1] if out_rows.ndim == 2 and out_rows.shape[0] > 0 else out_rows.shape[-1]
    y = np.empty((T, d), np.float64)
    if out_rows.shape[0] == 0:
        out_rows = np.zeros((1, d), np.float64)
    _check(lib().oracle_combine(T, d, k, _ptr(out_rows), _ptr(slot_row), _ptr(G), float(scale),
                                _ptr(y)), "combine")
    return y


def gate_stats(T: int, k: int, counts, probs_sum, lam: float):
    """a6: f, P and L_balance."""
    counts = _c(counts, np.int32)
    ps = _c(probs_sum, np.float64)
    E = counts.shape[0]
    f = np.empty(E, np.float64)
    P = np.empty(E, np.float64)
    L = np.empty(1, np.float64)
    _check(lib().oracle_gate_stats(T, E, k, _ptr(counts), _ptr(ps), float(lam), _ptr(f),
                                   _ptr(P), _ptr(L)), "gate_stats")
    return f, P, float(L[0])


def balance_sketch(idx, G, clean_probs_sum):
    """Load-balance loss as the LLaMA-MoE v2 code sample computes it (information only)."""
    idx = _c(idx, np.int32)
    G = _c(G, np.float64)
    cps = _c(clean_probs_sum, np.float64)
    T, k = idx.shape
    L = np.empty(1, np.float64)
    _check(lib().oracle_balance_sketch(T, cps.shape[0], k, _ptr(idx), _ptr(G), _ptr(cps),
                                       _ptr(L)), "balance_sketch")
    return float(L[0])


def forward(x, Wg, W1e, W3e, W2e, k, router_type=MIXTRAL, Wnoise=None, eps=None, bias=None,
            capacity_rows=-1, rescale=False, lam=0.0, tokens=None):
    """The whole layer: a1 -> a2 -> a3/a4 -> a5 -> a6.

    Routing, dispatch and statistics always cover every token.  The expert FFN and
    the combine are evaluated for ``tokens`` (all tokens when None), so large
    layers can be checked on a sample.  Returns a dict with every intermediate.
    """
    E = Wg.shape[1]
    T = x.shape[0]
    r = router(x, Wg, Wnoise, eps, bias, k, router_type)
    dsp = dispatch(r["idx"], E, capacity_rows)
    f, P, L = gate_stats(T, k, dsp["counts"], r["probs_sum"], lam)
    toks = np.arange(T) if tokens is None else np.asarray(tokens, np.int64)
    sr = dsp["slot_row"][toks]
    rows = sr[sr >= 0]
    uniq = np.unique(rows)
    remap = {int(v): i for i, v in enumerate(uniq)}
    expert_of_row = np.searchsorted(dsp["offsets"], uniq, side="right") - 1
    x_rows = np.ascontiguousarray(x[dsp["row_token"][uniq]]) if len(uniq) else x[:0]
    out_u = expert_ffn(W1e, W3e, W2e, x_rows, expert_of_row) if len(uniq) else \
        np.zeros((0, x.shape[1]))
    sr_local = np.where(sr >= 0, np.vectorize(lambda v: remap.get(int(v), -1))(sr) if sr.size
                        else sr, -1).astype(np.int32)
    scale = (E / k) if rescale else 1.0
    y = combine(out_u, sr_local, r["G"][toks], scale)
    return dict(router=r, dispatch=dsp, f=f, P=P, L=L, tokens=toks, y=y, out_rows=out_u,
                rows=uniq)


# --------------------------------------------------------------------------- residual MoE
# "LLaMA-MoE v2", section "共享神经元划分" (Shared Neuron Partitioning): the neurons of a
# set S are shared by all experts, the rest are split into E equal disjoint experts.
# The pages give no output formula; the layer is read as a residual block every token
# passes through next to the routed experts:
#     y = FFN_S(x) + s * sum_j G_j E_j(x)
# (FFN_S the SwiGLU FFN on the neurons of S, unscaled, applied to dropped tokens too).

def partition_residual(W1, W3, W2, E: int, shared_idx, perm_rest):
    """a0 of the residual MoE: the shared block (W1, W3 rows and W2 columns of S) and
    E disjoint experts over perm_rest (expert e gets perm_rest[e m, (e+1) m))."""
    shared = np.asarray(shared_idx, np.int64)
    rest = np.asarray(perm_rest, np.int64)
    W1, W3, W2 = np.asarray(W1), np.asarray(W3), np.asarray(W2)
    blk = (np.ascontiguousarray(W1[shared]), np.ascontiguousarray(W3[shared]),
           np.ascontiguousarray(W2[:, shared]))
    experts = partition(np.ascontiguousarray(W1[rest]), np.ascontiguousarray(W3[rest]),
                        np.ascontiguousarray(W2[:, rest]), E, DISJOINT,
                        np.arange(len(rest), dtype=np.int32))
    return experts, blk


def forward_residual(x, Wg, experts, shared_block, k, router_type=MIXTRAL, Wnoise=None,
                     eps=None, bias=None, capacity_rows=-1, rescale=False, lam=0.0,
                     tokens=None):
    """The residual MoE layer: forward() over the routed experts plus FFN_S(x) for
    every token evaluated.  Adds ``y_shared`` to the returned dict."""
    r = forward(x, Wg, *experts, k, router_type, Wnoise, eps, bias, capacity_rows, rescale,
                lam, tokens)
    xs = np.ascontiguousarray(np.asarray(x)[r["tokens"]])
    ys = dense_ffn(*shared_block, xs)
    r["y_moe"] = r["y"]
    r["y_shared"] = ys
    r["y"] = r["y"] + ys
    return r


def cluster(F, E: int, n_iter: int, init):
    """f4: balanced k-means partition of the rows of F [d_ff][d] into E clusters
    of d_ff/E neurons.  Returns (assign [d_ff] int32, centers [E][d] float64,
    perm [d_ff] int32)."""
    F = _c(F)
    dt = _dt(F)
    d_ff, d = F.shape
    ini = _c(np.asarray(init), np.int32)
    assign = np.empty(d_ff, np.int32)
    centers = np.empty((E, d), np.float64)
    perm = np.empty(d_ff, np.int32)
    _check(lib().oracle_cluster(_ptr(F), dt, d, d_ff, E, n_iter, _ptr(ini), _ptr(assign),
                                _ptr(centers), _ptr(perm)), "cluster")
    return assign, centers, perm


def sqdist(F, C):
    """D [d_ff][E] float64: squared Euclidean distances of the rows of F to the rows of C."""
    F = _c(F)
    Cc = _c(C, np.float64)
    d_ff, d = F.shape
    E = Cc.shape[0]
    D = np.empty((d_ff, E), np.float64)
    _check(lib().oracle_sqdist(_ptr(F), _dt(F), d, d_ff, E, _ptr(Cc), _ptr(D)), "sqdist")
    return D


# --------------------------------------------------------------------------- backward (f1)

def combine_backward(out_rows, slot_row, G, scale: float, dy):
    """d_out [R][d] and dG [T][k] of y = s sum_j G_j out_{r(t,j)}."""
    out_rows = _c(out_rows, np.float64)
    slot_row = _c(slot_row, np.int32)
    G = _c(G, np.float64)
    dy = _c(dy, np.float64)
    T, k = slot_row.shape
    d = dy.shape[1]
    R = out_rows.shape[0]
    d_out = np.zeros((max(R, 1), d), np.float64)
    dG = np.empty((T, k), np.float64)
    src = out_rows if R > 0 else np.zeros((1, d))
    _check(lib().oracle_combine_backward(T, d, k, _ptr(src), _ptr(slot_row), _ptr(G),
                                         float(scale), _ptr(dy), _ptr(d_out), _ptr(dG)),
           "combine_backward")
    return d_out[:R], dG


def expert_ffn_backward(W1e, W3e, W2e, x_rows, expert_of_row, d_out):
    """Expert backward for the given rows: dx_rows [n][d], dW1e / dW3e [E][m][d],
    dW2e [E][d][m], and the per-row dh, dg, du [n][m] (all float64)."""
    W1e, W3e, W2e = _c(W1e), _c(W3e), _c(W2e)
    E, m, d = W1e.shape
    x_rows = _c(x_rows)
    eor = _c(expert_of_row, np.int32)
    d_out = _c(d_out, np.float64)
    n = x_rows.shape[0]
    dx = np.zeros((max(n, 1), d), np.float64)
    dW1 = np.empty((E, m, d), np.float64)
    dW3 = np.empty((E, m, d), np.float64)
    dW2 = np.empty((E, d, m), np.float64)
    dh = np.empty((max(n, 1), m), np.float64)
    dg = np.empty((max(n, 1), m), np.float64)
    du = np.empty((max(n, 1), m), np.float64)
    xr = x_rows if n > 0 else np.zeros((1, d), x_rows.dtype)
    dor = d_out if n > 0 else np.zeros((1, d))
    _check(lib().oracle_expert_ffn_backward(d, m, E, _ptr(W1e), _ptr(W3e), _ptr(W2e), _dt(W1e),
                                            _ptr(xr), _dt(xr), _ptr(eor), n, _ptr(dor), _ptr(dx),
                                            _ptr(dW1), _ptr(dW3), _ptr(dW2), _ptr(dh), _ptr(dg),
                                            _ptr(du)), "expert_ffn_backward")
    return dict(dx_rows=dx[:n], dW1e=dW1, dW3e=dW3, dW2e=dW2, dh=dh[:n], dg=dg[:n], du=du[:n])


def router_backward(x, Wg, idx, G, dG, counts, k, router_type=MIXTRAL, Wnoise=None, eps=None,
                    bias=None, lam=0.0, dLb=1.0, dx=None):
    """Router backward; adds W_g dL + W_noise dN to dx (a new zero array when None)."""
    x, Wg = _c(x), _c(Wg)
    dt = _dt(x)
    T, d = x.shape
    E = Wg.shape[1]
    Wn = None if Wnoise is None else _c(Wnoise)
    ep = None if eps is None else _c(eps, np.float32)
    b = None if bias is None else _c(bias, np.float32)
    idx = _c(idx, np.int32)
    G = _c(G, np.float64)
    dG = _c(dG, np.float64)
    counts = _c(counts, np.int32)
    dx = np.zeros((T, d), np.float64) if dx is None else dx
    assert dx.dtype == np.float64 and dx.flags.c_contiguous
    dWg = np.empty((d, E), np.float64)
    dWn = np.empty((d, E), np.float64) if Wnoise is not None else None
    db = np.empty(E, np.float64) if bias is not None else None
    dH = np.empty((T, E), np.float64)
    dN = np.empty((T, E), np.float64)
    _check(lib().oracle_router_backward(T, d, E, k, router_type, _ptr(x), dt, _ptr(Wg), _ptr(Wn),
                                        _ptr(ep), _ptr(b), _ptr(idx), _ptr(G), _ptr(dG),
                                        _ptr(counts), float(lam), float(dLb), _ptr(dx),
                                        _ptr(dWg), _ptr(dWn), _ptr(db), _ptr(dH), _ptr(dN)),
           "router_backward")
    return dict(dx=dx, dWg=dWg, dWnoise=dWn, dbias=db, dH=dH, dN=dN)


def backward(x, Wg, W1e, W3e, W2e, k, dy, router_type=MIXTRAL, Wnoise=None, eps=None,
             bias=None, capacity_rows=-1, rescale=False, lam=0.0, dLb=1.0):
    """Gradients of l(y) + dLb * L_balance for the whole layer, given dy = dl/dy:
    dx, dWg, dWnoise, dbias, dW1e, dW3e, dW2e, plus every intermediate (d_out,
    dG, dh, dg, du, dx_rows, dH, dN) and the forward pass (key 'fwd')."""
    E = Wg.shape[1]
    T = x.shape[0]
    f = forward(x, Wg, W1e, W3e, W2e, k, router_type, Wnoise, eps, bias, capacity_rows,
                rescale, lam)
    r, dsp = f["router"], f["dispatch"]
    scale = (E / k) if rescale else 1.0
    d_out, dG = combine_backward(f["out_rows"], dsp["slot_row"], r["G"], scale, dy)
    R = dsp["R"]
    expert_of_row = np.searchsorted(dsp["offsets"], np.arange(R), side="right") - 1
    x_rows = np.ascontiguousarray(np.asarray(x)[dsp["row_token"]])
    eb = expert_ffn_backward(W1e, W3e, W2e, x_rows, expert_of_row, d_out)
    dx = np.zeros((T, x.shape[1]), np.float64)
    for t in range(T):
        for j in range(k):
            row = dsp["slot_row"][t, j]
            if row >= 0:
                dx[t] += eb["dx_rows"][row]
    rb = router_backward(x, Wg, r["idx"], r["G"], dG, dsp["counts"], k, router_type, Wnoise,
                         eps, bias, lam, dLb, dx)
    return dict(dx=dx, dWg=rb["dWg"], dWnoise=rb["dWnoise"], dbias=rb["dbias"],
                dW1e=eb["dW1e"], dW3e=eb["dW3e"], dW2e=eb["dW2e"], d_out=d_out, dG=dG,
                dh=eb["dh"], dg=eb["dg"], du=eb["du"], dx_rows=eb["dx_rows"], dH=rb["dH"],
                dN=rb["dN"], fwd=f)


def backward_residual(x, Wg, experts, shared_block, k, dy, router_type=MIXTRAL, Wnoise=None,
                      eps=None, bias=None, capacity_rows=-1, rescale=False, lam=0.0, dLb=1.0):
    """Gradients of the residual MoE layer y = FFN_S(x) + s sum_j G_j E_j(x): the routed
    layer's backward() plus the shared block's (an expert over every token whose output
    gradient is dy).  Adds dx_s, dW1s, dW3s, dW2s, dh_s to backward()'s dict; dx is the
    total."""
    g = backward(x, Wg, *experts, k, dy, router_type, Wnoise, eps, bias, capacity_rows,
                 rescale, lam, dLb)
    W1s, W3s, W2s = shared_block
    T = x.shape[0]
    sb = expert_ffn_backward(np.ascontiguousarray(W1s)[None], np.ascontiguousarray(W3s)[None],
                             np.ascontiguousarray(W2s)[None], x, np.zeros(T, np.int32), dy)
    g["dx_s"] = sb["dx_rows"]
    g["dx"] = g["dx"] + sb["dx_rows"]
    g["dW1s"], g["dW3s"], g["dW2s"] = sb["dW1e"][0], sb["dW3e"][0], sb["dW2e"][0]
    g["dh_s"] = sb["dh"]
    return g


def router_backward_tokens(x, Wg, idx, G, dG, counts, k, T_norm, router_type=MIXTRAL,
                           Wnoise=None, eps=None, bias=None, lam=0.0, dLb=1.0):
    """Router backward for some of a batch's tokens (rows of x etc. are those tokens;
    counts and T_norm are the whole batch's).  Returns the router term of dx and dL/dN."""
    x, Wg = _c(x), _c(Wg)
    T, d = x.shape
    E = Wg.shape[1]
    Wn = None if Wnoise is None else _c(Wnoise)
    ep = None if eps is None else _c(eps, np.float32)
    b = None if bias is None else _c(bias, np.float32)
    dx = np.zeros((T, d), np.float64)
    dWg = np.empty((d, E), np.float64)
    dWn = np.empty((d, E), np.float64)
    db = np.empty(E, np.float64)
    dH = np.empty((T, E), np.float64)
    dN = np.empty((T, E), np.float64)
    _check(lib().oracle_router_backward_norm(
        T, int(T_norm), d, E, k, router_type, _ptr(x), _dt(x), _ptr(Wg), _ptr(Wn), _ptr(ep),
        _ptr(b), _ptr(_c(idx, np.int32)), _ptr(_c(G, np.float64)), _ptr(_c(dG, np.float64)),
        _ptr(_c(counts, np.int32)), float(lam), float(dLb), _ptr(dx), _ptr(dWg),
        _ptr(dWn if Wnoise is not None else None), _ptr(db if bias is not None else None),
        _ptr(dH), _ptr(dN)), "router_backward_norm")
    return dict(dx=dx, dH=dH, dN=dN)


def neuron_wgrad(W1e, W3e, W2e, e: int, i: int, x_rows, d_out):
    """Gradients of neuron i of expert e over the given rows of that expert:
    (dW1 row [d], dW3 row [d], dW2 column [d]), float64."""
    W1e, W3e, W2e = _c(W1e), _c(W3e), _c(W2e)
    E, m, d = W1e.shape
    x_rows = _c(x_rows)
    d_out = _c(d_out, np.float64)
    out = [np.empty(d, np.float64) for _ in range(3)]
    w1 = np.ascontiguousarray(W1e[e, i])
    w3 = np.ascontiguousarray(W3e[e, i])
    w2 = np.ascontiguousarray(W2e[e])
    _check(lib().oracle_neuron_wgrad(d, m, i, _ptr(w1), _ptr(w3), _ptr(w2), _dt(W1e),
                                     _ptr(x_rows), _dt(x_rows), x_rows.shape[0], _ptr(d_out),
                                     _ptr(out[0]), _ptr(out[1]), _ptr(out[2])), "neuron_wgrad")
    return out
