"""moe_dispatch_noalloc: the dispatch step for callers that cannot allocate device
memory or hand the library a workspace (e.g. a host engine whose plugin interface
passes a layer only its inputs and outputs and forbids allocation while it
enqueues work).  It must give exactly the bytes moe_dispatch gives.

Collected last on purpose (file name), so a run that stops at the first failure
has already run every other test; it depends on no other test.
"""
import ctypes as C

import pytest
import torch

import top_routing_grouped_noisy_b200 as moe
import workloads as wl

pytestmark = pytest.mark.gpu


def _dispatch_both(w, idx, x, p, ws):
    L = moe.lib()
    a = moe.ForwardBuffers(p)
    b = moe.ForwardBuffers(p)
    moe.moe_dispatch(p, x, idx, ws, a.x_perm, a.row_token, a.slot_row, a.counts, a.kept,
                     a.offsets)
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    rc = L.moe_dispatch_noalloc(C.byref(p), x.data_ptr(), idx.data_ptr(), b.x_perm.data_ptr(),
                                b.row_token.data_ptr(), b.slot_row.data_ptr(),
                                b.counts.data_ptr(), b.kept.data_ptr(), b.offsets.data_ptr(),
                                status.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == moe.MOE_OK, L.moe_last_error_string()
    torch.cuda.synchronize()
    return a, b, int(status[0])


def test_noalloc_dispatch_matches_workspace_dispatch_twice():
    w = wl.Workload("na", T=3000, d=512, d_ff=1024, E=16, k=4, seed=91)
    inp = wl.make_inputs(w)
    x = inp["x"].cuda()
    p = moe.params(w.T, w.d, w.E, w.k, w.m, torch.bfloat16, capacity=700)
    ws = moe.Workspace(p)
    g = torch.Generator().manual_seed(5)
    for call in range(2):  # two calls in a row: the shared scratch must not leak
        idx = torch.stack([torch.randperm(w.E, generator=g)[:w.k] for _ in range(w.T)])
        if call == 1:
            idx[:, 0] = 3  # a skewed second call, so stale counts would show
        idx = idx.to(torch.int32).cuda().contiguous()
        a, b, st = _dispatch_both(w, idx, x, p, ws)
        assert st == 0
        R = int(a.offsets[-1])
        assert R > 0
        for n in ("counts", "kept", "offsets", "slot_row"):
            assert torch.equal(getattr(a, n), getattr(b, n)), (call, n)
        assert torch.equal(a.row_token[:R], b.row_token[:R]), call
        assert torch.equal(a.x_perm[:R], b.x_perm[:R]), call


def test_noalloc_dispatch_rejects_oversize_and_reports_bad_index():
    L = moe.lib()
    big = moe.params(40000, 64, 64, 2, 16)
    f = [C.c_void_p(0x100000 + 256 * i) for i in range(10)]
    assert L.moe_dispatch_noalloc(C.byref(big), *f[:8], None, None) == moe.MOE_ERR_SHAPE
    assert b"fixed scratch" in L.moe_last_error_string()
    small = moe.params(64, 64, 4, 2, 16)
    # no status word for a non-empty batch: a bad index would go unreported
    assert L.moe_dispatch_noalloc(C.byref(small), *f[:8], None, None) == moe.MOE_ERR_INVALID_ARG
    assert b"status is NULL" in L.moe_last_error_string()
    w = wl.Workload("nb", T=64, d=64, d_ff=128, E=4, k=2, seed=92)
    x = wl.make_inputs(w)["x"].cuda()
    p = moe.params(w.T, w.d, w.E, w.k, w.m, torch.bfloat16)
    ws = moe.Workspace(p)
    idx = torch.tensor([[0, 1]] * w.T, dtype=torch.int32, device="cuda")
    idx[7, 1] = 9
    a, b, st = _dispatch_both(w, idx, x, p, ws)
    assert st == moe.MOE_ERR_DEVICE_BADINDEX
    assert torch.equal(a.slot_row, b.slot_row) and int(b.slot_row[7, 1]) == -1
