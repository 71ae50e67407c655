"""Python binding of libmoe.so, the B200 (sm_100a) sparse Mixture-of-Experts SwiGLU
FFN layer: the forward pass (noisy Top-K routing, capacity dispatch, grouped expert
GEMMs on tcgen05 tensor cores, gate-weighted combine, gate statistics), its backward
(moe_backward and its steps), the residual layer with shared neurons, the expert
construction (moe_partition_*), the clustering partition (moe_cluster_partition) and
the non-collective steps of the expert-parallel layer (moe_ep_*; the layer itself is
``expert_parallel.ExpertParallelMoE``).

The functions mirror the C ABI in ``include/moe.h`` one to one and only marshal
arguments: torch tensors are passed as device pointers together with torch's
current CUDA stream; every step of the layer runs in the library's kernels.
PyTorch provides device memory and streams only.  There is no fallback: if the
library is missing or a call fails, an exception is raised.
"""
import ctypes as C
import os

import torch

__all__ = [
    "MoeError", "Params", "lib", "params", "moe_capacity", "moe_version", "moe_launch_count",
    "moe_partition_experts", "moe_workspace_size", "Workspace", "moe_route", "moe_route_packed",
    "moe_router_pack", "moe_router_packed_bytes", "moe_dispatch", "moe_dispatch_routed", "moe_dispatch_noalloc", "moe_dispatch_rows", "moe_expert_up_gather",
    "moe_expert_up", "moe_expert_down", "moe_expert_ffn", "moe_combine", "moe_gate_stats",
    "moe_forward", "ForwardBuffers", "moe_get_device_status", "moe_set_wait_limit_ns",
    "moe_set_gemm_band_rows",
    "packed_w13_elems", "packed_w2_elems", "h_ld", "Pipeline", "moe_partition_residual",
    "moe_combine_residual", "moe_forward_residual", "moe_cluster_workspace_size",
    "moe_cluster_partition", "moe_cluster_distances", "moe_backward_workspace_size",
    "moe_combine_backward", "moe_expert_down_backward", "moe_expert_up_backward",
    "moe_route_backward", "moe_backward", "BackwardBuffers",
    "moe_backward_residual_workspace_size", "moe_backward_residual", "EpPlan", "moe_ep_plan",
    "moe_ep_mask_slots", "moe_ep_gate_stats", "EP_CAPACITY_GLOBAL", "EP_CAPACITY_LOCAL",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = -1
MOE_ERR_SHAPE = -2
MOE_ERR_ALIGN = -3
MOE_ERR_DTYPE = -4
MOE_ERR_CUDA = -5
MOE_ERR_DEVICE_TIMEOUT = -6
MOE_ERR_DEVICE_BADINDEX = -7
MOE_ERR_WORKSPACE = -8
MOE_ERR_UNSUPPORTED = -9

MOE_F32 = 0
MOE_BF16 = 1
MIXTRAL = 0
ST = 1
DISJOINT = 0
COPY = 1
STACKED = 2
EP_CAPACITY_GLOBAL = 0
EP_CAPACITY_LOCAL = 1


class MoeError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__("libmoe error %d: %s" % (code, msg))
        self.code = code


class Params(C.Structure):
    _fields_ = [("T", C.c_int32), ("d", C.c_int32), ("E", C.c_int32), ("k", C.c_int32),
                ("m", C.c_int32), ("dtype", C.c_int32), ("router_type", C.c_int32),
                ("capacity", C.c_int32), ("rescale", C.c_int32), ("balance_lambda", C.c_float)]


_BUF_FIELDS = ["x", "Wg", "Wnoise", "noise", "bias", "W13_e", "W2_e", "y", "loss", "counts",
               "importance", "f", "P", "topk_idx", "topk_w", "probs_sum", "x_perm", "row_token",
               "slot_row", "kept", "offsets", "h", "out", "router_packed"]


class _Buffers(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in _BUF_FIELDS]


_BWD_FIELDS = ["dy", "dx", "dWg", "dWnoise", "dbias", "dW13_e", "dW2_e", "d_out", "dG", "dh",
               "dx_perm"]


class _BwdBuffers(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in _BWD_FIELDS]


_lib = None


def lib():
    """The loaded libmoe.so (raises ImportError when it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError("libmoe.so not found at %s; build it with "
                              "`python -m top_routing_grouped_noisy_b200.build`" % LIB_PATH)
        L = C.CDLL(LIB_PATH)
        v, i32, i64, sz, f64 = C.c_void_p, C.c_int32, C.c_int64, C.c_size_t, C.c_double
        P = C.POINTER(Params)
        sig = {
            "moe_version": (C.c_char_p, []),
            "moe_last_error_string": (C.c_char_p, []),
            "moe_launch_count": (C.c_uint64, []),
            "moe_set_wait_limit_ns": (None, [C.c_uint64]),
            "moe_set_gemm_band_rows": (None, [C.c_int32]),
            "moe_capacity": (i32, [i32, i32, f64]),
            "moe_packed_w13_elems": (i64, [i32, i32, i32]),
            "moe_packed_w2_elems": (i64, [i32, i32, i32]),
            "moe_h_ld": (i32, [i32]),
            "moe_partition_experts": (C.c_int, [v, v, v, i32, i32, i32, i32, v, i32, v, v, v, v]),
            "moe_workspace_size": (sz, [P]),
            "moe_workspace_init": (C.c_int, [v, sz, v]),
            "moe_route": (C.c_int, [P, v, v, v, v, v, v, v, v, v, v, sz, v]),
            "moe_route_packed": (C.c_int, [P, v, v, v, v, v, v, v, v, v, v, v, sz, v]),
            "moe_router_pack": (C.c_int, [P, v, v, v, v]),
            "moe_router_packed_bytes": (sz, [P, i32]),
            "moe_dispatch": (C.c_int, [P, v, v, v, v, v, v, v, v, v, sz, v]),
            "moe_dispatch_routed": (C.c_int, [P, v, v, v, v, v, v, v, v, v, sz, v]),
            "moe_dispatch_noalloc": (C.c_int, [P, v, v, v, v, v, v, v, v, v, v]),
            "moe_dispatch_rows": (C.c_int, [P, v, v, v, v, v, v, v, sz, v]),
            "moe_expert_up_gather": (C.c_int, [P, v, v, v, v, v, v, sz, v]),
            "moe_expert_up": (C.c_int, [P, v, v, v, v, v, sz, v]),
            "moe_expert_down": (C.c_int, [P, v, v, v, v, v, sz, v]),
            "moe_expert_ffn": (C.c_int, [P, v, v, v, v, v, v, v, sz, v]),
            "moe_combine": (C.c_int, [P, v, v, v, v, v]),
            "moe_gate_stats": (C.c_int, [P, v, v, v, v, v, v]),
            "moe_forward": (C.c_int, [P, C.POINTER(_Buffers), v, sz, v]),
            "moe_get_device_status": (C.c_int, [v, C.POINTER(i32), i32, v]),
            "moe_partition_residual": (C.c_int, [v, v, v, i32, i32, i32, v, i32, v, i32, v, v,
                                                 v, v, v, v]),
            "moe_combine_residual": (C.c_int, [P, v, v, v, v, v, v]),
            "moe_forward_residual": (C.c_int, [P, C.POINTER(_Buffers), v, v, i32, v, v, v, sz,
                                               v]),
            "moe_cluster_workspace_size": (sz, [i32, i32, i32]),
            "moe_cluster_partition": (C.c_int, [v, i32, i32, i32, i32, i32, v, v, v, v, v, sz,
                                                v]),
            "moe_cluster_distances": (C.c_int, [v, i32, i32, i32, i32, v, v, v]),
            "moe_backward_workspace_size": (sz, [P]),
            "moe_combine_backward": (C.c_int, [P, v, v, v, v, v, v, v]),
            "moe_expert_down_backward": (C.c_int, [P, v, v, v, v, v, v, v, sz, v]),
            "moe_expert_up_backward": (C.c_int, [P, v, v, v, v, v, v, v, sz, v]),
            "moe_route_backward": (C.c_int, [P, v, v, v, v, v, v, v, v, v, C.c_float, v, v, v,
                                             v, v, v, v, sz, v]),
            "moe_backward": (C.c_int, [P, C.POINTER(_Buffers), C.POINTER(_BwdBuffers),
                                       C.c_float, v, sz, v]),
            "moe_backward_residual_workspace_size": (sz, [P, i32]),
            "moe_backward_residual": (C.c_int, [P, C.POINTER(_Buffers), C.POINTER(_BwdBuffers), v,
                                                v, i32, v, v, v, v, v, C.c_float, v, sz, v]),
            "moe_ep_plan": (C.c_int, [v, i32, i32, i32, i32, i32, v, v, v, v, v, v]),
            "moe_ep_mask_slots": (C.c_int, [P, v, v, v, v, v]),
            "moe_ep_gate_stats": (C.c_int, [P, v, i32, v, v, v, v, v, v]),
            "moe_pipeline_create": (C.c_int, [P, v, v, v, v, v, i32, C.POINTER(v)]),
            "moe_pipeline_submit": (C.c_int, [v, v, v, v, v, C.POINTER(i64)]),
            "moe_pipeline_wait": (C.c_int, [v, i64]),
            "moe_pipeline_destroy": (C.c_int, [v]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(rc):
    if rc != MOE_OK:
        raise MoeError(rc, lib().moe_last_error_string().decode())


def _p(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor, got %r" % type(t))
    if not t.is_cuda:
        raise ValueError("libmoe takes CUDA tensors (got a %s tensor)" % t.device)
    if not t.is_contiguous():
        raise ValueError("libmoe takes contiguous tensors")
    return t.data_ptr() or None


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _dtype_code(dt):
    if dt == torch.bfloat16:
        return MOE_BF16
    if dt == torch.float32:
        return MOE_F32
    raise TypeError("libmoe computes in bf16 or f32, not %s" % dt)


def moe_version() -> str:
    return lib().moe_version().decode()


def moe_launch_count() -> int:
    return int(lib().moe_launch_count())


def moe_set_wait_limit_ns(ns: int) -> None:
    lib().moe_set_wait_limit_ns(int(ns))


def moe_set_gemm_band_rows(rows: int) -> None:
    """Tuning knob of the 2-SM expert GEMMs' tile order (results do not change)."""
    lib().moe_set_gemm_band_rows(int(rows))


def moe_capacity(T: int, E: int, cf: float) -> int:
    return int(lib().moe_capacity(T, E, float(cf)))


def packed_w13_elems(E, m, d):
    return int(lib().moe_packed_w13_elems(E, m, d))


def packed_w2_elems(E, m, d):
    return int(lib().moe_packed_w2_elems(E, m, d))


def h_ld(m):
    return int(lib().moe_h_ld(m))


def params(T, d, E, k, m, dtype=torch.bfloat16, router_type=MIXTRAL, capacity=-1,
           rescale=False, balance_lambda=0.0) -> Params:
    return Params(T, d, E, k, m, _dtype_code(dtype) if isinstance(dtype, torch.dtype) else dtype,
                  router_type, capacity, 1 if rescale else 0, balance_lambda)


def moe_workspace_size(p: Params) -> int:
    return int(lib().moe_workspace_size(C.byref(p)))


class Workspace:
    """Caller-owned scratch for the library (a zeroed torch uint8 buffer)."""

    def __init__(self, p: Params, device=None, nbytes=None):
        n = nbytes if nbytes is not None else moe_workspace_size(p)
        if n <= 0:
            raise MoeError(MOE_ERR_INVALID_ARG, "invalid parameters for the workspace")
        self.buf = torch.empty(n, dtype=torch.uint8, device=device or "cuda")
        self.nbytes = n
        _check(lib().moe_workspace_init(_p(self.buf), n, _stream()))

    @property
    def ptr(self):
        return self.buf.data_ptr()


def moe_get_device_status(ws: Workspace, clear=True, stream=None) -> int:
    st = C.c_int32(0)
    _check(lib().moe_get_device_status(ws.ptr, C.byref(st), 1 if clear else 0, _stream(stream)))
    return st.value


def moe_partition_experts(W1, W3, W2, E, mode=DISJOINT, perm=None, ws=None, out=None,
                          stream=None):
    """a0: packed expert weights (W13_e, W2_e) from a dense FFN (or stacked experts)."""
    dt = _dtype_code(W1.dtype)
    if mode == STACKED:
        d_ff, d = W1.shape[1], W1.shape[2]
    else:
        d_ff, d = W1.shape
    m = d_ff // E if mode == DISJOINT else d_ff
    if out is None:
        W13_e = torch.empty(packed_w13_elems(E, m, d), dtype=W1.dtype, device=W1.device)
        W2_e = torch.empty(packed_w2_elems(E, m, d), dtype=W1.dtype, device=W1.device)
    else:
        W13_e, W2_e = out
    _check(lib().moe_partition_experts(_p(W1), _p(W3), _p(W2), d, d_ff, E, mode, _p(perm), dt,
                                       _p(W13_e), _p(W2_e), ws.ptr if ws is not None else None,
                                       _stream(stream)))
    return W13_e, W2_e


def moe_route(p, x, Wg, Wnoise, noise, bias, ws, topk_idx, topk_w, probs_sum, importance,
              stream=None):
    _check(lib().moe_route(C.byref(p), _p(x), _p(Wg), _p(Wnoise), _p(noise), _p(bias),
                           _p(topk_idx), _p(topk_w), _p(probs_sum), _p(importance), ws.ptr,
                           ws.nbytes, _stream(stream)))


def moe_router_packed_bytes(p, noisy) -> int:
    return int(lib().moe_router_packed_bytes(C.byref(p), 1 if noisy else 0))


def moe_router_pack(p, Wg, Wnoise=None, out=None, stream=None):
    """The router weights packed once for the tensor-core router (include/moe.h);
    returns the packed device buffer (uint8)."""
    n = moe_router_packed_bytes(p, Wnoise is not None)
    if out is None:
        out = torch.empty(n, dtype=torch.uint8, device=Wg.device)
    _check(lib().moe_router_pack(C.byref(p), _p(Wg), _p(Wnoise), _p(out), _stream(stream)))
    return out


def moe_route_packed(p, x, Wg, Wnoise, Wt, noise, bias, ws, topk_idx, topk_w, probs_sum,
                     importance, stream=None):
    _check(lib().moe_route_packed(C.byref(p), _p(x), _p(Wg), _p(Wnoise), _p(Wt), _p(noise),
                                  _p(bias), _p(topk_idx), _p(topk_w), _p(probs_sum),
                                  _p(importance), ws.ptr, ws.nbytes, _stream(stream)))


def moe_dispatch(p, x, topk_idx, ws, x_perm, row_token, slot_row, counts, kept, offsets,
                 stream=None):
    _check(lib().moe_dispatch(C.byref(p), _p(x), _p(topk_idx), _p(x_perm), _p(row_token),
                              _p(slot_row), _p(counts), _p(kept), _p(offsets), ws.ptr,
                              ws.nbytes, _stream(stream)))


def moe_dispatch_routed(p, x, topk_idx, ws, x_perm, row_token, slot_row, counts, kept, offsets,
                        stream=None):
    """a2 right after moe_route on the same workspace: reuses the chunk counts the
    router left there (topk_idx must be that call's output, unchanged)."""
    _check(lib().moe_dispatch_routed(C.byref(p), _p(x), _p(topk_idx), _p(x_perm),
                                     _p(row_token), _p(slot_row), _p(counts), _p(kept),
                                     _p(offsets), ws.ptr, ws.nbytes, _stream(stream)))


def moe_dispatch_rows(p, topk_idx, ws, row_token, slot_row, counts, kept, offsets, stream=None):
    """a2 tables only (no permuted copy of x)."""
    _check(lib().moe_dispatch_rows(C.byref(p), _p(topk_idx), _p(row_token), _p(slot_row),
                                   _p(counts), _p(kept), _p(offsets), ws.ptr, ws.nbytes,
                                   _stream(stream)))


def moe_expert_up_gather(p, x, row_token, offsets, W13_e, h, ws, stream=None):
    """a3 gathering rows of x through row_token (bf16)."""
    _check(lib().moe_expert_up_gather(C.byref(p), _p(x), _p(row_token), _p(offsets), _p(W13_e),
                                      _p(h), ws.ptr, ws.nbytes, _stream(stream)))


def moe_dispatch_noalloc(p, x, topk_idx, x_perm, row_token, slot_row, counts, kept, offsets,
                         status, stream=None):
    """a2 without a workspace (fixed scratch inside the library; see include/moe.h).
    ``status`` is a device int32 tensor the caller zeroes; it is required for T > 0,
    being the only place a bad expert index is reported."""
    _check(lib().moe_dispatch_noalloc(C.byref(p), _p(x), _p(topk_idx), _p(x_perm),
                                      _p(row_token), _p(slot_row), _p(counts), _p(kept),
                                      _p(offsets), _p(status), _stream(stream)))


def moe_expert_up(p, x_perm, offsets, W13_e, h, ws, stream=None):
    _check(lib().moe_expert_up(C.byref(p), _p(x_perm), _p(offsets), _p(W13_e), _p(h), ws.ptr,
                               ws.nbytes, _stream(stream)))


def moe_expert_down(p, h, offsets, W2_e, out, ws, stream=None):
    _check(lib().moe_expert_down(C.byref(p), _p(h), _p(offsets), _p(W2_e), _p(out), ws.ptr,
                                 ws.nbytes, _stream(stream)))


def moe_expert_ffn(p, x_perm, offsets, W13_e, W2_e, h, out, ws, stream=None):
    _check(lib().moe_expert_ffn(C.byref(p), _p(x_perm), _p(offsets), _p(W13_e), _p(W2_e), _p(h),
                                _p(out), ws.ptr, ws.nbytes, _stream(stream)))


def moe_combine(p, out, slot_row, topk_w, y, stream=None):
    _check(lib().moe_combine(C.byref(p), _p(out), _p(slot_row), _p(topk_w), _p(y),
                             _stream(stream)))


def moe_gate_stats(p, counts, probs_sum, f, P, loss, stream=None):
    _check(lib().moe_gate_stats(C.byref(p), _p(counts), _p(probs_sum), _p(f), _p(P), _p(loss),
                                _stream(stream)))


class EpPlan:
    """Exchange plan of one rank of the expert-parallel layer (host int32 tensors):
    keep_all [N][E], send_row/send_cnt [E] (indexed by expert), recv_row/recv_cnt [E]
    (entry p*(E/N)+l: rank p's run for local expert l), in_offsets [E/N+1]."""

    def __init__(self, N, E, rank, keep_all, send_row, send_cnt, recv_row, recv_cnt, in_offsets):
        self.N, self.E, self.rank = N, E, rank
        self.E_local = E // N
        self.keep_all, self.send_row, self.send_cnt = keep_all, send_row, send_cnt
        self.recv_row, self.recv_cnt, self.in_offsets = recv_row, recv_cnt, in_offsets

    @property
    def rows_in(self) -> int:
        return int(self.in_offsets[-1])

    def send_runs(self):
        """(peer, first row, rows, expert) of the run this rank sends for each expert."""
        El = self.E_local
        return [(e // El, int(self.send_row[e]), int(self.send_cnt[e]), e)
                for e in range(self.E)]

    def recv_runs(self):
        """(peer, first row, rows, expert) of every run this rank receives, grouped by
        peer and in expert order inside a peer (the order the peer sends them in)."""
        El = self.E_local
        return [(i // El, int(self.recv_row[i]), int(self.recv_cnt[i]), self.rank * El + i % El)
                for i in range(self.E)]


def _host_i32(t, name):
    if not isinstance(t, torch.Tensor) or t.is_cuda or t.dtype != torch.int32 or \
            not t.is_contiguous():
        raise ValueError("%s must be a contiguous host int32 tensor" % name)
    return t.data_ptr()


def moe_ep_plan(counts_all, rank, capacity=-1, scope=EP_CAPACITY_GLOBAL) -> EpPlan:
    """counts_all: host int32 [N][E] (every rank's routed counts).  Runs on the host."""
    c = torch.as_tensor(counts_all, dtype=torch.int32).contiguous()
    if c.dim() != 2:
        raise ValueError("counts_all must be [N][E]")
    N, E = c.shape
    El = E // N if N > 0 and E >= N else 0
    z = lambda *s: torch.zeros(*s, dtype=torch.int32)
    keep, srow, scnt, rrow, rcnt, ioff = z(N, E), z(E), z(E), z(E), z(E), z(El + 1)
    _check(lib().moe_ep_plan(_host_i32(c, "counts_all"), N, E, int(rank), int(capacity),
                             int(scope), keep.data_ptr(), srow.data_ptr(), scnt.data_ptr(),
                             rrow.data_ptr(), rcnt.data_ptr(), ioff.data_ptr()))
    return EpPlan(N, E, int(rank), keep, srow, scnt, rrow, rcnt, ioff)


def moe_ep_mask_slots(p, topk_idx, offsets, keep, slot_row, stream=None):
    """keep: host int32 [E] (this rank's row of EpPlan.keep_all)."""
    keep = torch.as_tensor(keep, dtype=torch.int32).contiguous()
    if keep.numel() < p.E:
        raise ValueError("keep needs E entries")
    _check(lib().moe_ep_mask_slots(C.byref(p), _p(topk_idx), _p(offsets),
                                   _host_i32(keep, "keep"), _p(slot_row), _stream(stream)))


def moe_ep_gate_stats(p, counts_all, N, probs_sum, counts, f, P, loss, stream=None):
    _check(lib().moe_ep_gate_stats(C.byref(p), _p(counts_all), int(N), _p(probs_sum),
                                   _p(counts), _p(f), _p(P), _p(loss), _stream(stream)))


class ForwardBuffers:
    """Every intermediate and output tensor of one layer forward, allocated with torch."""

    def __init__(self, p: Params, device="cuda"):
        dt = torch.bfloat16 if p.dtype == MOE_BF16 else torch.float32
        T, d, E, k = p.T, p.d, p.E, p.k
        rows = max(T * k, 1)
        i32 = dict(dtype=torch.int32, device=device)
        f32 = dict(dtype=torch.float32, device=device)
        self.y = torch.empty(max(T, 1), d, dtype=dt, device=device)[:T]
        self.loss = torch.empty(1, **f32)
        self.counts = torch.empty(E, **i32)
        self.importance = torch.empty(E, **f32)
        self.f = torch.empty(E, **f32)
        self.P = torch.empty(E, **f32)
        self.topk_idx = torch.empty(max(T, 1), k, **i32)[:T]
        self.topk_w = torch.empty(max(T, 1), k, **f32)[:T]
        self.probs_sum = torch.empty(E, **f32)
        self.x_perm = torch.empty(rows, d, dtype=dt, device=device)
        self.row_token = torch.empty(rows, **i32)
        self.slot_row = torch.empty(max(T, 1), k, **i32)[:T]
        self.kept = torch.empty(E, **i32)
        self.offsets = torch.empty(E + 1, **i32)
        self.h = torch.empty(rows, h_ld(p.m), dtype=dt, device=device)
        self.out = torch.empty(rows, d, dtype=dt, device=device)
        self.router_packed = None  # optional: moe_router_pack output for moe_forward


def moe_forward(p, x, Wg, W13_e, W2_e, ws, bufs: ForwardBuffers, Wnoise=None, noise=None,
                bias=None, stream=None, router_packed=None):
    b = _Buffers()
    vals = dict(x=x, Wg=Wg, Wnoise=Wnoise, noise=noise, bias=bias, W13_e=W13_e, W2_e=W2_e)
    if router_packed is not None:  # else bufs.router_packed (None: packed per call)
        vals["router_packed"] = router_packed
    for n in _BUF_FIELDS:
        t = vals[n] if n in vals else getattr(bufs, n)
        setattr(b, n, _p(t))
    _check(lib().moe_forward(C.byref(p), C.byref(b), ws.ptr, ws.nbytes, _stream(stream)))
    return bufs


def moe_partition_residual(W1, W3, W2, E, shared_idx, perm_rest, ws=None, stream=None):
    """a0 of the residual MoE: E disjoint experts over perm_rest and the shared block
    over shared_idx; returns (W13_e, W2_e, W13_s, W2_s) (include/moe.h)."""
    dt = _dtype_code(W1.dtype)
    d_ff, d = W1.shape
    m_s = shared_idx.numel()
    m = (d_ff - m_s) // E
    mk = lambda n: torch.empty(n, dtype=W1.dtype, device=W1.device)
    W13_e, W2_e = mk(packed_w13_elems(E, m, d)), mk(packed_w2_elems(E, m, d))
    W13_s, W2_s = mk(packed_w13_elems(1, m_s, d)), mk(packed_w2_elems(1, m_s, d))
    _check(lib().moe_partition_residual(_p(W1), _p(W3), _p(W2), d, d_ff, E, _p(shared_idx), m_s,
                                        _p(perm_rest), dt, _p(W13_e), _p(W2_e), _p(W13_s),
                                        _p(W2_s), ws.ptr if ws is not None else None,
                                        _stream(stream)))
    return W13_e, W2_e, W13_s, W2_s


def moe_combine_residual(p, out, slot_row, topk_w, resid, y, stream=None):
    _check(lib().moe_combine_residual(C.byref(p), _p(out), _p(slot_row), _p(topk_w), _p(resid),
                                      _p(y), _stream(stream)))


def moe_forward_residual(p, x, Wg, W13_e, W2_e, W13_s, W2_s, m_s, ws, bufs: ForwardBuffers, h_s,
                         out_s, Wnoise=None, noise=None, bias=None, stream=None):
    """The residual MoE layer: routed experts plus the shared block (include/moe.h)."""
    b = _Buffers()
    vals = dict(x=x, Wg=Wg, Wnoise=Wnoise, noise=noise, bias=bias, W13_e=W13_e, W2_e=W2_e)
    for n in _BUF_FIELDS:
        t = vals[n] if n in vals else getattr(bufs, n)
        setattr(b, n, _p(t))
    _check(lib().moe_forward_residual(C.byref(p), C.byref(b), _p(W13_s), _p(W2_s), int(m_s),
                                      _p(h_s), _p(out_s), ws.ptr, ws.nbytes, _stream(stream)))
    return bufs


def _host_ptr(t, name):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s: expected a torch.Tensor, got %r" % (name, type(t)))
    if t.is_cuda:
        raise ValueError("%s: the pipeline takes host tensors (pinned for overlap)" % name)
    if not t.is_contiguous():
        raise ValueError("%s: the pipeline takes contiguous tensors" % name)
    return t.data_ptr() or None


class Pipeline:
    """Host-buffer pipeline (include/moe_pipeline.h): batches in host memory go
    through the layer with up to ``depth`` of them in flight, copies overlapping
    the compute.  The weights are device tensors that must outlive the pipeline."""

    def __init__(self, p: Params, Wg, W13_e, W2_e, Wnoise=None, bias=None, depth=2):
        self._p = p
        self._keep = (Wg, W13_e, W2_e, Wnoise, bias)
        h = C.c_void_p(None)
        _check(lib().moe_pipeline_create(C.byref(p), _p(Wg), _p(Wnoise), _p(bias), _p(W13_e),
                                         _p(W2_e), int(depth), C.byref(h)))
        self._h = h
        self._held = {}

    def submit(self, x_host, y_host, loss_host, noise_host=None) -> int:
        """Enqueue one batch; returns its ticket.  The host tensors are held until
        wait() has returned for that ticket."""
        t = C.c_int64(-1)
        _check(lib().moe_pipeline_submit(self._h, _host_ptr(x_host, "x_host"),
                                         _host_ptr(noise_host, "noise_host"),
                                         _host_ptr(y_host, "y_host"),
                                         _host_ptr(loss_host, "loss_host"), C.byref(t)))
        self._held[t.value] = (x_host, noise_host, y_host, loss_host)
        return t.value

    def wait(self, ticket: int) -> None:
        _check(lib().moe_pipeline_wait(self._h, int(ticket)))
        for k in [k for k in self._held if k <= ticket]:
            del self._held[k]

    def close(self) -> None:
        if self._h is not None and self._h.value is not None:
            h, self._h = self._h, None
            self._held.clear()
            _check(lib().moe_pipeline_destroy(h))

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def moe_cluster_workspace_size(d, d_ff, E) -> int:
    return int(lib().moe_cluster_workspace_size(d, d_ff, E))


def moe_cluster_partition(F, E, n_iter, init_idx, ws=None, stream=None):
    """Balanced k-means partition of the rows of F [d_ff][d] into E clusters of
    d_ff/E neurons (include/moe.h).  Returns (assign, centers, perm, ws); ws is a
    Workspace-like object whose status word records a bad init index."""
    dt = _dtype_code(F.dtype)
    d_ff, d = F.shape
    dev = F.device
    if ws is None:
        n = moe_cluster_workspace_size(d, d_ff, E)
        if n <= 0:
            raise MoeError(MOE_ERR_SHAPE, "invalid shape for the clustering workspace")
        ws = Workspace(None, device=dev, nbytes=n)
    assign = torch.empty(d_ff, dtype=torch.int32, device=dev)
    perm = torch.empty(d_ff, dtype=torch.int32, device=dev)
    centers = torch.empty(E, d, dtype=torch.float64, device=dev)
    _check(lib().moe_cluster_partition(_p(F), d, d_ff, E, dt, n_iter, _p(init_idx), _p(assign),
                                       _p(centers), _p(perm), ws.ptr, ws.nbytes,
                                       _stream(stream)))
    return assign, centers, perm, ws


def moe_cluster_distances(F, centers, out=None, stream=None):
    """D [d_ff][E] f64: squared distances of the rows of F to the centers (f64)."""
    d_ff, d = F.shape
    E = centers.shape[0]
    D = out if out is not None else torch.empty(d_ff, E, dtype=torch.float64, device=F.device)
    _check(lib().moe_cluster_distances(_p(F), d, d_ff, E, _dtype_code(F.dtype), _p(centers),
                                       _p(D), _stream(stream)))
    return D


# --------------------------------------------------------------------------- backward

def moe_backward_workspace_size(p) -> int:
    return int(lib().moe_backward_workspace_size(C.byref(p)))


class BackwardBuffers:
    """Outputs and intermediates of moe_backward for layer p (include/moe.h)."""

    def __init__(self, p: Params, noisy: bool, biased: bool, device="cuda"):
        T, d, E, k = p.T, p.d, p.E, p.k
        dt = torch.bfloat16
        f32 = dict(dtype=torch.float32, device=device)
        rows = max(T * k, 1)
        self.dx = torch.empty(T, d, dtype=dt, device=device)
        self.dWg = torch.empty(d, E, **f32)
        self.dWnoise = torch.empty(d, E, **f32) if noisy else None
        self.dbias = torch.empty(E, **f32) if biased else None
        self.dW13_e = torch.empty(packed_w13_elems(E, p.m, d), dtype=dt, device=device)
        self.dW2_e = torch.empty(packed_w2_elems(E, p.m, d), dtype=dt, device=device)
        self.d_out = torch.empty(rows, d, dtype=dt, device=device)
        self.dG = torch.empty(T, k, **f32)
        self.dh = torch.empty(rows, h_ld(p.m), dtype=dt, device=device)
        self.dx_perm = torch.empty(rows, d, dtype=dt, device=device)


def moe_combine_backward(p, dy, out, slot_row, topk_w, d_out, dG, stream=None):
    _check(lib().moe_combine_backward(C.byref(p), _p(dy), _p(out), _p(slot_row), _p(topk_w),
                                      _p(d_out), _p(dG), _stream(stream)))


def moe_expert_down_backward(p, d_out, h, offsets, W2_e, dh, dW2_e, ws, stream=None):
    _check(lib().moe_expert_down_backward(C.byref(p), _p(d_out), _p(h), _p(offsets), _p(W2_e),
                                          _p(dh), _p(dW2_e), ws.ptr, ws.nbytes, _stream(stream)))


def moe_expert_up_backward(p, x_perm, dh, offsets, W13_e, dx_perm, dW13_e, ws, stream=None):
    _check(lib().moe_expert_up_backward(C.byref(p), _p(x_perm), _p(dh), _p(offsets), _p(W13_e),
                                        _p(dx_perm), _p(dW13_e), ws.ptr, ws.nbytes,
                                        _stream(stream)))


def moe_route_backward(p, x, Wg, topk_idx, topk_w, dG, counts, dx_perm, slot_row, dx, dWg, ws,
                       Wnoise=None, noise=None, bias=None, dWnoise=None, dbias=None, dLb=1.0,
                       stream=None):
    _check(lib().moe_route_backward(C.byref(p), _p(x), _p(Wg), _p(Wnoise), _p(noise), _p(bias),
                                    _p(topk_idx), _p(topk_w), _p(dG), _p(counts), float(dLb),
                                    _p(dx_perm), _p(slot_row), _p(dx), _p(dWg), _p(dWnoise),
                                    _p(dbias), ws.ptr, ws.nbytes, _stream(stream)))


def moe_backward(p, x, Wg, W13_e, W2_e, fwd: "ForwardBuffers", g: BackwardBuffers, dy, ws,
                 Wnoise=None, noise=None, bias=None, dLb=1.0, stream=None):
    """The whole backward of the batch whose forward filled `fwd` (include/moe.h)."""
    b = _Buffers()
    vals = dict(x=x, Wg=Wg, Wnoise=Wnoise, noise=noise, bias=bias, W13_e=W13_e, W2_e=W2_e)
    for n in _BUF_FIELDS:
        t = vals[n] if n in vals else getattr(fwd, n)
        setattr(b, n, _p(t))
    gb = _BwdBuffers()
    for n in _BWD_FIELDS:
        setattr(gb, n, _p(dy if n == "dy" else getattr(g, n)))
    _check(lib().moe_backward(C.byref(p), C.byref(b), C.byref(gb), float(dLb), ws.ptr, ws.nbytes,
                              _stream(stream)))
    return g


def moe_backward_residual_workspace_size(p, m_s) -> int:
    return int(lib().moe_backward_residual_workspace_size(C.byref(p), int(m_s)))


def moe_backward_residual(p, x, Wg, W13_e, W2_e, W13_s, W2_s, m_s, h_s, fwd: "ForwardBuffers",
                          g: BackwardBuffers, dy, dh_s, dx_s, dW13_s, dW2_s, ws, Wnoise=None,
                          noise=None, bias=None, dLb=1.0, stream=None):
    """Backward of the residual MoE layer (include/moe.h)."""
    b = _Buffers()
    vals = dict(x=x, Wg=Wg, Wnoise=Wnoise, noise=noise, bias=bias, W13_e=W13_e, W2_e=W2_e)
    for n in _BUF_FIELDS:
        t = vals[n] if n in vals else getattr(fwd, n)
        setattr(b, n, _p(t))
    gb = _BwdBuffers()
    for n in _BWD_FIELDS:
        setattr(gb, n, _p(dy if n == "dy" else getattr(g, n)))
    _check(lib().moe_backward_residual(C.byref(p), C.byref(b), C.byref(gb), _p(W13_s), _p(W2_s),
                                       int(m_s), _p(h_s), _p(dh_s), _p(dx_s), _p(dW13_s),
                                       _p(dW2_s), float(dLb), ws.ptr, ws.nbytes, _stream(stream)))
    return g
