"""Clustering partition (balanced k-means over the neurons' W1 rows, "LLaMA-MoE
v2", section 专家构建方法, IndependentClustering) on the GPU against the fp64
oracle.  Both sides compute every distance, decision and mean in f64 with one
rounding per operation and the same summation order, so assignments,
permutations and centers are compared bit for bit."""
import os

import numpy as np
import pytest
import torch

import oracle
import top_routing_grouped_noisy_b200 as moe
import workloads as wl

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _raw(t):
    return wl.to_numpy_raw(t)


def _gpu(F, E, n_iter, init):
    assign, centers, perm, ws = moe.moe_cluster_partition(F.cuda(), E, n_iter, init.cuda())
    st = moe.moe_get_device_status(ws)
    torch.cuda.synchronize()
    return assign.cpu().numpy(), centers.cpu().numpy(), perm.cpu().numpy(), st


def _compare(F, E, n_iter, init):
    a, c, p, st = _gpu(F, E, n_iter, init)
    assert st == 0
    ra, rc, rp = oracle.cluster(_raw(F), E, n_iter, init.numpy())
    np.testing.assert_array_equal(a, ra)
    np.testing.assert_array_equal(p, rp)
    np.testing.assert_array_equal(c, rc)  # bit for bit
    return ra


def _features(seed, d_ff, d, dtype):
    g = torch.Generator()
    g.manual_seed(seed)
    F = 0.02 * torch.randn(d_ff, d, generator=g)
    return F.to(torch.bfloat16 if dtype == "bf16" else torch.float32)


def _load_golden():
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


def test_hand_worked_cases():
    """The hand-worked fixtures, features zero-padded to 8 columns (zero columns
    add exact zeros to every distance and keep zero centers)."""
    for c in _load_golden():
        d, E = c["d"][0], c["E"][0]
        F = torch.tensor(c["F"], dtype=torch.float32).reshape(-1, d)
        Fp = torch.zeros(F.shape[0], 8)
        Fp[:, :d] = F
        a, cen, p, st = _gpu(Fp, E, c["iters"][0], torch.tensor(c["init"], dtype=torch.int32))
        assert st == 0
        assert a.tolist() == c["assign"], c["name"]
        assert p.tolist() == c["perm"], c["name"]
        assert cen[:, :d].ravel().tolist() == c["centers"], c["name"]
        assert (cen[:, d:] == 0).all()


CASES = [
    # name, d_ff, d, E, n_iter, dtype, seed
    ("bf16_small_ragged_d", 96, 40, 4, 3, "bf16", 60),
    ("f32_two_chunks_tail", 200, 136, 8, 4, "f32", 61),
    ("bf16_e12", 360, 64, 12, 3, "bf16", 62),
    ("bf16_e64", 320, 72, 64, 2, "bf16", 63),
    ("bf16_one_per_cluster", 16, 24, 16, 2, "bf16", 64),
    ("bf16_one_cluster", 48, 16, 1, 2, "bf16", 65),
    ("bf16_mid", 2752, 512, 8, 5, "bf16", 66),
]


@pytest.mark.parametrize("name,d_ff,d,E,n_iter,dtype,seed", CASES, ids=[c[0] for c in CASES])
def test_parity(name, d_ff, d, E, n_iter, dtype, seed):
    F = _features(seed, d_ff, d, dtype)
    init = wl.make_cluster_init(d_ff, E, 7)
    ra = _compare(F, E, n_iter, init)
    assert np.bincount(ra, minlength=E).tolist() == [d_ff // E] * E


def test_crowded_cluster_ranks_across_tiles_and_ctas():
    """Most neurons propose to one center first (a central neuron against an
    outlier), so the acceptance ranks > 512 proposals over several CTAs."""
    d_ff, d, E = 2048, 16, 2
    F = _features(5, d_ff, d, "f32")
    F[7] = 0.0          # the mean of the cloud
    F[11] = 0.5         # far away
    init = torch.tensor([7, 11], dtype=torch.int32)
    D0 = ((F.double() - F[7].double()) ** 2).sum(1) < ((F.double() - F[11].double()) ** 2).sum(1)
    assert int(D0.sum()) > 1500
    _compare(F, E, 3, init)


def test_bad_init_sets_the_status_word():
    F = _features(9, 64, 16, "bf16")
    for init in ([3, 3], [0, 64], [-1, 2]):
        _, _, _, st = _gpu(F, 2, 1, torch.tensor(init, dtype=torch.int32))
        assert st == moe.MOE_ERR_DEVICE_BADINDEX, init


def test_full_size_w1_of_the_llama_ffn():
    """Llama-2-7B FFN width (d = 4096, d_ff = 11008), E = 8 clusters of 1376 neurons,
    on W1 of the moe_2of8 workload; two iterations, compared in full."""
    w = wl.WORKLOADS["moe_2of8"]
    F = wl.make_inputs(w, device="cuda")["W1"].cpu()
    init = wl.make_cluster_init(w.d_ff, w.E, w.seed)
    _compare(F, w.E, 2, init)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_distance_step_alone(dtype):
    """moe_cluster_distances against the oracle's distance step, bit for bit, with
    arbitrary f64 centers (not features), a ragged column tail and E = 5."""
    F = _features(70, 77, 200, dtype)
    g = torch.Generator()
    g.manual_seed(71)
    Cc = torch.randn(5, 200, generator=g, dtype=torch.float64) * 0.02
    D = moe.moe_cluster_distances(F.cuda(), Cc.cuda()).cpu().numpy()
    np.testing.assert_array_equal(D, oracle.sqdist(_raw(F), Cc.numpy()))
