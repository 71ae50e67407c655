"""Multi-rank host logic of bench.py on CPU (gloo, world size 2): the timing is
the max over ranks, throughput aggregates every rank's tokens over that time
(independent replicas, weak scaling), and the reference arm prints on rank 0 only."""
import json
import os
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method="tcp://127.0.0.1:%d" % port, rank=rank,
                            world_size=world)
    try:
        ms = [12.5, 20.0][rank]
        mx = bench.max_over_ranks(ms, world, device="cpu")
        v = bench.tokens_per_s(1000, 10, world, mx)
        with open(os.path.join(out_dir, "r%d.json" % rank), "w") as fh:
            json.dump({"max": mx, "value": v}, fh)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_aggregate(tmp_path):
    port = 29500 + os.getpid() % 1000
    mp.spawn(_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True)
    r = [json.load(open(tmp_path / ("r%d.json" % i))) for i in range(2)]
    assert r[0]["max"] == r[1]["max"] == 20.0
    assert r[0]["value"] == pytest.approx(1000 * 10 * 2 / 0.020)


@pytest.mark.parametrize("rank", [0, 1])
def test_reference_arm_prints_on_rank_zero_only(rank):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank))
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "tiny_fp32", "--steps", "2", "--warmup", "1",
                          "--gpus", "2"], env=env, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    if rank == 0:
        assert len(lines) == 1
        d = json.loads(lines[0])
        assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
        assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
        assert d["e2e"]["h2d_bytes_per_step"] == 0
    else:
        assert lines == []
