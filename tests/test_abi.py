"""The C ABI without a GPU: libmoe.so loads, exports every function include/moe.h
declares, its host-only helpers agree with the oracle, and argument validation
rejects bad calls before anything reaches the device."""
import ctypes as C
import os
import re

import pytest

import oracle
import top_routing_grouped_noisy_b200 as moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src))
    return sorted(names)


@pytest.fixture(scope="module")
def L():
    return moe.lib()


def test_library_exports_every_declared_function(L):
    names = _declared_functions()
    assert len(names) >= 20
    for n in names:
        assert hasattr(L, n), "libmoe.so does not export %s" % n
    assert len(L.moe_version()) > 0


def test_binding_wraps_every_declared_function():
    src = open(os.path.join(ROOT, "top_routing_grouped_noisy_b200", "__init__.py")).read()
    for n in _declared_functions():
        assert '"%s"' % n in src, "binding has no signature for %s" % n


@pytest.mark.parametrize("T,E,cf", [(32768, 8, 1.0), (32768, 8, 4.0), (10, 3, 1.0),
                                    (16384, 16, 1.25), (7, 8, 0.5), (100, 8, -1.0), (0, 4, 2.0)])
def test_capacity_matches_oracle(T, E, cf):
    assert moe.moe_capacity(T, E, cf) == oracle.capacity(T, E, cf)


def test_layout_helpers():
    assert moe.packed_w13_elems(8, 1376, 4096) == 8 * 2 * 1376 * 4096
    assert moe.packed_w13_elems(8, 100, 64) == 8 * 2 * 112 * 64
    assert moe.packed_w2_elems(8, 100, 64) == 8 * 64 * 104
    assert moe.h_ld(1376) == 1376 and moe.h_ld(172) == 176
    assert moe.packed_w13_elems(0, 1, 1) == 0


def test_workspace_size_and_invalid_params():
    p = moe.params(16384, 4096, 8, 2, 1376)
    assert moe.moe_workspace_size(p) > 0
    bigger = moe.params(32768, 4096, 8, 2, 1376)
    assert moe.moe_workspace_size(bigger) >= moe.moe_workspace_size(p)
    # non-decreasing in T across the small-batch sizes, so a workspace sized for a
    # batch serves every smaller one
    sizes = [moe.moe_workspace_size(moe.params(T, 4096, 8, 2, 1376))
             for T in (1, 2, 8, 9, 63, 64, 65, 300, 16384)]
    assert sizes == sorted(sizes), sizes
    for bad in (moe.params(16, 4096, 8, 9, 1376), moe.params(16, 4096, 65, 2, 1376),
                moe.params(16, 100, 8, 2, 1376), moe.params(-1, 64, 8, 2, 16),
                moe.params(16, 64, 8, 0, 16), moe.params(16, 64, 8, 2, 0)):
        assert moe.moe_workspace_size(bad) == 0


def _fake(addr=1 << 20):
    return C.c_void_p(addr)


def test_validation_codes_without_touching_the_device(L):
    """Every one of these returns before any CUDA call is made."""
    P = moe.params(64, 64, 8, 2, 16)
    f = [_fake(0x100000 + 256 * i) for i in range(12)]
    ws_bytes = moe.moe_workspace_size(P)
    # NULL params
    assert L.moe_route(None, *f[:10], ws_bytes, None) == moe.MOE_ERR_INVALID_ARG
    # k > E
    bad = moe.params(64, 64, 4, 5, 16)
    assert L.moe_route(C.byref(bad), *f[:10], ws_bytes, None) == moe.MOE_ERR_INVALID_ARG
    assert b"k=5" in L.moe_last_error_string()
    # d not a multiple of 8
    bad = moe.params(64, 60, 8, 2, 16)
    assert L.moe_dispatch(C.byref(bad), *f[:9], ws_bytes, None) == moe.MOE_ERR_SHAPE
    # bad dtype
    bad = moe.params(64, 64, 8, 2, 16, dtype=7)
    assert L.moe_combine(C.byref(bad), *f[:4], None) == moe.MOE_ERR_DTYPE
    # misaligned pointer
    mis = list(f[:10])
    mis[0] = _fake(0x100008)
    assert L.moe_route(C.byref(P), *mis, ws_bytes, None) == moe.MOE_ERR_ALIGN
    assert b"'x'" in L.moe_last_error_string()
    # NULL required output
    nul = list(f[:10])
    nul[8] = None
    assert L.moe_route(C.byref(P), *nul, ws_bytes, None) == moe.MOE_ERR_INVALID_ARG
    # noise projection without the noise draws
    nn = list(f[:10])
    nn[3] = None
    assert L.moe_route(C.byref(P), *nn, ws_bytes, None) == moe.MOE_ERR_INVALID_ARG
    # workspace too small
    assert L.moe_route(C.byref(P), *f[:10], ws_bytes - 1, None) == moe.MOE_ERR_WORKSPACE
    # partition: d_ff not divisible by E, missing perm, bad mode
    assert L.moe_partition_experts(*f[:3], 64, 100, 8, moe.DISJOINT, f[3], moe.MOE_BF16,
                                   f[4], f[5], None, None) == moe.MOE_ERR_SHAPE
    assert L.moe_partition_experts(*f[:3], 64, 128, 8, moe.DISJOINT, None, moe.MOE_BF16,
                                   f[4], f[5], None, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_partition_experts(*f[:3], 64, 128, 8, 9, None, moe.MOE_BF16,
                                   f[4], f[5], None, None) == moe.MOE_ERR_INVALID_ARG
    # status readback with NULL output
    assert L.moe_get_device_status(f[0], None, 0, None) == moe.MOE_ERR_INVALID_ARG


def test_empty_batch_needs_no_token_buffers(L):
    """T = 0: token-sized buffers may be NULL; the expert GEMMs and the combine return
    at once without launching anything."""
    P = moe.params(0, 64, 8, 2, 16)
    ws_bytes = moe.moe_workspace_size(P)
    off, w, ws = _fake(0x200000), _fake(0x300000), _fake(0x400000)
    before = moe.moe_launch_count()
    assert L.moe_expert_up(C.byref(P), None, off, w, None, ws, ws_bytes, None) == moe.MOE_OK
    assert L.moe_expert_down(C.byref(P), None, off, w, None, ws, ws_bytes, None) == moe.MOE_OK
    assert L.moe_combine(C.byref(P), None, None, None, None, None) == moe.MOE_OK
    assert moe.moe_launch_count() == before


def test_wait_limit_setter_is_host_only(L):
    moe.moe_set_wait_limit_ns(123)
    moe.moe_set_wait_limit_ns(2_000_000_000)


def test_pipeline_rejects_bad_arguments_before_the_device(L):
    p = moe.params(1000, 512, 8, 2, 344)
    out = C.c_void_p(123)
    dummy = C.c_void_p(16)
    assert L.moe_pipeline_create(C.byref(p), dummy, None, None, dummy, dummy, 2, None) == \
        moe.MOE_ERR_INVALID_ARG
    assert L.moe_pipeline_create(C.byref(p), dummy, None, None, dummy, dummy, 1,
                                 C.byref(out)) == moe.MOE_ERR_INVALID_ARG
    assert out.value is None
    assert L.moe_pipeline_create(C.byref(p), dummy, None, None, dummy, dummy, 5,
                                 C.byref(out)) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_pipeline_create(C.byref(p), None, None, None, dummy, dummy, 2,
                                 C.byref(out)) == moe.MOE_ERR_INVALID_ARG
    p0 = moe.params(0, 512, 8, 2, 344)
    assert L.moe_pipeline_create(C.byref(p0), dummy, None, None, dummy, dummy, 2,
                                 C.byref(out)) == moe.MOE_ERR_INVALID_ARG
    assert b"T must be" in L.moe_last_error_string()
    t = C.c_int64(0)
    assert L.moe_pipeline_submit(None, dummy, None, dummy, dummy, C.byref(t)) == \
        moe.MOE_ERR_INVALID_ARG
    assert L.moe_pipeline_wait(None, 0) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_pipeline_destroy(None) == moe.MOE_OK


def test_cluster_rejects_bad_arguments_before_the_device(L):
    a = C.c_void_p(256)
    n = L.moe_cluster_workspace_size(4096, 11008, 8)
    assert n > 11008 * 8 * 8 and L.moe_cluster_workspace_size(4096, 11008, 7) == 0
    assert L.moe_cluster_workspace_size(4096, 11008, 65) == 0
    assert L.moe_cluster_workspace_size(4096, 11008, 4) < n  # monotone in E
    call = lambda F=a, d=64, d_ff=32, E=4, dt=moe.MOE_BF16, it=1, init=a, asg=a, cen=a, perm=a, \
        ws=a, nb=1 << 20: L.moe_cluster_partition(F, d, d_ff, E, dt, it, init, asg, cen, perm, ws,
                                                  nb, None)
    assert call(F=None) == moe.MOE_ERR_INVALID_ARG
    assert call(perm=None) == moe.MOE_ERR_INVALID_ARG
    assert call(F=C.c_void_p(258)) == moe.MOE_ERR_ALIGN
    assert call(cen=C.c_void_p(264)) == moe.MOE_ERR_ALIGN
    assert call(dt=7) == moe.MOE_ERR_DTYPE
    assert call(E=0) == moe.MOE_ERR_INVALID_ARG
    assert call(E=65, d_ff=65 * 2) == moe.MOE_ERR_INVALID_ARG
    assert call(it=0) == moe.MOE_ERR_INVALID_ARG
    assert call(d=60) == moe.MOE_ERR_SHAPE
    assert call(d_ff=30) == moe.MOE_ERR_SHAPE
    assert call(nb=100) == moe.MOE_ERR_WORKSPACE
    assert b"workspace" in L.moe_last_error_string()


def test_backward_rejects_bad_arguments_before_the_device(L):
    p = moe.params(64, 256, 8, 2, 128)
    a = C.c_void_p(256)
    n = L.moe_backward_workspace_size(C.byref(p))
    assert n > 0
    assert L.moe_backward_workspace_size(C.byref(moe.params(128, 256, 8, 2, 128))) > n
    assert L.moe_backward_workspace_size(C.byref(moe.params(0, 256, 8, 2, 128))) == 0
    pf = moe.params(64, 256, 8, 2, 128, dtype=moe.MOE_F32)
    assert L.moe_combine_backward(C.byref(pf), a, a, a, a, a, a, None) == moe.MOE_ERR_DTYPE
    assert L.moe_combine_backward(C.byref(p), None, a, a, a, a, a, None) == \
        moe.MOE_ERR_INVALID_ARG
    assert L.moe_combine_backward(C.byref(p), C.c_void_p(258), a, a, a, a, a, None) == \
        moe.MOE_ERR_ALIGN
    assert L.moe_expert_down_backward(C.byref(p), a, a, a, a, a, a, a, n - 1, None) == \
        moe.MOE_ERR_WORKSPACE
    assert L.moe_expert_up_backward(C.byref(p), a, a, a, a, a, None, a, n, None) == \
        moe.MOE_ERR_INVALID_ARG
    # noise inputs and their gradient go together
    assert L.moe_route_backward(C.byref(p), a, a, a, None, None, a, a, a, a, C.c_float(1.0), a,
                                a, a, a, None, None, a, n, None) == moe.MOE_ERR_INVALID_ARG
    assert b"together" in L.moe_last_error_string()


def test_expert_parallel_calls_reject_bad_arguments_before_the_device(L):
    a = C.c_void_p(256)
    p = moe.params(64, 256, 8, 2, 128)
    keep = (C.c_int32 * 8)(*([3] * 8))
    mask = lambda pp=p, idx=a, off=a, kp=keep, sr=a: L.moe_ep_mask_slots(
        C.byref(pp), idx, off, kp, sr, None)
    assert mask(idx=None) == moe.MOE_ERR_INVALID_ARG
    assert mask(kp=None) == moe.MOE_ERR_INVALID_ARG
    assert mask(pp=moe.params(64, 256, 8, 9, 128)) == moe.MOE_ERR_INVALID_ARG
    neg = (C.c_int32 * 8)(*([3] * 7 + [-1]))
    assert mask(kp=neg) == moe.MOE_ERR_INVALID_ARG
    assert mask(pp=moe.params(0, 256, 8, 2, 128)) == moe.MOE_OK  # nothing to mark
    stats = lambda pp=p, ca=a, N=2, ps=a, out=a: L.moe_ep_gate_stats(
        C.byref(pp), ca, N, ps, out, a, a, a, None)
    assert stats(ca=None) == moe.MOE_ERR_INVALID_ARG
    assert stats(out=None) == moe.MOE_ERR_INVALID_ARG
    assert stats(N=3) == moe.MOE_ERR_SHAPE
    assert stats(N=0) == moe.MOE_ERR_SHAPE
    assert stats(N=16) == moe.MOE_ERR_SHAPE
    assert b"N must divide E" in L.moe_last_error_string()


def test_plain_c_program_links_and_plans(tmp_path):
    """The boundary is plain C: a C99 program compiled against include/moe.h and linked
    with libmoe.so calls the host-only exchange plan (no GPU needed)."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    src = tmp_path / "plan.c"
    src.write_text(r'''
#include <stdio.h>
#include "moe.h"
int main(void)
{
    const int32_t counts[2][4] = {{3, 1, 0, 2}, {1, 2, 2, 2}};
    int32_t keep[2][4], srow[4], scnt[4], rrow[4], rcnt[4], off[3];
    int rc = moe_ep_plan(&counts[0][0], 2, 4, 1, 3, MOE_EP_CAPACITY_GLOBAL, &keep[0][0], srow,
                         scnt, rrow, rcnt, off);
    if (rc != MOE_OK)
        return 1;
    for (int p = 0; p < 2; ++p)
        for (int e = 0; e < 4; ++e)
            printf("%d ", keep[p][e]);
    printf("| %d %d %d\n", off[0], off[1], off[2]);
    return moe_ep_plan(&counts[0][0], 2, 3, 0, -1, 0, &keep[0][0], srow, scnt, rrow, rcnt,
                       off) == MOE_ERR_SHAPE ? 0 : 2;
}
''')
    exe = tmp_path / "plan"
    libdir = os.path.dirname(moe.LIB_PATH)
    inc = os.path.join(os.path.dirname(libdir), "include")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", inc, str(src), "-o", str(exe),
                    moe.LIB_PATH, "-Wl,-rpath," + libdir], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stderr
    # expert 0: rank 0 fills the capacity of 3; expert 3: rank 0 holds 2, rank 1 keeps 1
    assert out.stdout.split() == "3 1 0 2 0 2 2 1 | 0 2 5".split()
