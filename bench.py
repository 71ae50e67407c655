"""Throughput of the MoE-layer forward on B200 (one JSON line on stdout).

A step is one pass of the whole layer (route -> dispatch -> expert GEMM 1 with
SwiGLU -> expert GEMM 2 -> combine -> gate statistics) over one batch of seeded
synthetic input already resident in HBM; the working set per step (x, the packed
expert weights and the intermediates) is several times the 126 MB L2, so no flush
is needed between steps.  Every step is issued as the six C-ABI step calls with
CUDA events between them on the launching stream, which gives the per-kernel
times used for the roofline line.  The end-to-end leg times ``moe_forward`` with
the inputs copied from pinned host memory and the result read back every step.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

N > 1 runs under torchrun: every rank runs an independent replica of the layer on
its own batch (weak scaling, no data-path collective); times are the max over ranks.
``--impl reference`` times the fp64 CPU oracle on a bounded sample of the same
workload (host cores; rank 0 only).
"""
import argparse
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads as wl  # noqa: E402

METRIC = "MoE-layer tokens/sec and TFLOP/s at 1 B200; % of bf16 tensor peak / % HBM BW"
# the largest single-GPU configuration: Llama-3-E8T2 upcycled layer at capacity factor 4
HEADLINE = "e8t2_cf4"
# the other forward workloads, measured in the same run with fewer steps
EXTRA = ["moe_2of8", "moe_4of16", "e8t2_cf1", "tiny_fp32", "decode_t1", "decode_t8",
         "decode_t64"]
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM bytes of one a3 launch (expert GEMM 1 + SwiGLU) from an ncu capture, keyed by
# the source it was taken on; reported as null once the kernel source changes.
# (default tile band of 2048 rows)
NCU_TRAFFIC = {
    "moe_2of8": {"src": "ed7e29b9fa5e804b", "T": 16384, "bytes_per_launch": 471.48e6 + 82.46e6},
    "e8t2_cf4": {"src": "ed7e29b9fa5e804b", "T": 32768,
                 "bytes_per_launch": 23875.10e6 + 1875.45e6},
}


def _src_hash(rel):
    with open(os.path.join(ROOT, rel), "rb") as fh:
        return hashlib.sha256(fh.read()).hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            pk = json.load(fh)
        return pk, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def tensor_roof(achieved, peaks, peak_src):
    """Fraction of the bf16 tensor peak.  The headline fraction divides by the burst
    figure (a cuBLAS GEMM timed alone, the larger of the two measured figures), so it
    stays at or below about 1; the fraction of the seconds-long, power-capped
    sustained figure is reported beside it."""
    burst = peaks["bf16_tflops"]
    sus = peaks.get("bf16_tflops_sustained", burst)
    return {"peak": burst, "frac": achieved / burst, "frac_of_sustained": achieved / sus,
            "peak_source": "%s bf16_tflops (burst) %.1f; frac_of_sustained against "
                           "bf16_tflops_sustained %.1f" % (peak_src, burst, sus)}


def config_of(w: wl.Workload, C: int):
    return {
        "workload": w.name, "T": w.T, "d": w.d, "d_ff": w.d_ff, "E": w.E, "k": w.k, "m": w.m,
        "router": "mixtral" if w.router == wl.MIXTRAL else "st", "noisy": w.noisy,
        "bias": w.bias, "rescale": w.rescale, "capacity": C, "cf": w.cf,
        "partition": "disjoint" if w.partition == wl.DISJOINT else "copy",
        "shared_neurons": w.shared,
        "global_batch": w.T, "seq_len": 4096,
        "l2": "no flush: per-step working set (x, packed weights, intermediates) >> 126 MB L2",
    }


# --------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while it runs."""

    Q = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, dev_index):
        self.samples = []
        self.proc = None
        try:
            uuid = str(torch.cuda.get_device_properties(dev_index).uuid)
            target = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            target = str(dev_index)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=" + self.Q, "--format=csv,noheader,nounits",
                 "-lms", "50", "-i", target], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0, t1):
        rows = []
        for ts, line in self.samples:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append((ts, float(f[1]), float(f[2]), f[5:9]))
            except ValueError:
                continue
        inwin = [r for r in rows if t0 <= r[0] <= t1]
        note = "samples inside the timed region"
        if not inwin and rows:
            mid = 0.5 * (t0 + t1)
            inwin = sorted(rows, key=lambda r: abs(r[0] - mid))[:3]
            note = "timed region shorter than the sampling period: nearest samples"
        if not inwin:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "note": "nvidia-smi unavailable"}
        reasons = sorted({self.NAMES[i] for r in inwin for i, v in enumerate(r[3])
                          if v.lower() == "active"})
        return {"sm_mhz": float(np.median([r[1] for r in inwin])),
                "sm_max_mhz": max(r[2] for r in inwin), "reasons": reasons,
                "samples": len(inwin), "note": note}


# --------------------------------------------------------------------------- oracle timing

def oracle_sample_forward(w, x_s, eps_s, Wg, Wn, bias, OW, C, rescale):
    """The oracle's layer forward on a sample of tokens (router, dispatch, experts,
    combine, statistics); returns y."""
    import oracle
    r = oracle.router(x_s, Wg, Wn, eps_s, bias, w.k, w.router)
    d = oracle.dispatch(r["idx"], w.E, C)
    oracle.gate_stats(x_s.shape[0], w.k, d["counts"], r["probs_sum"], w.lam)
    R = d["R"]
    if R:
        eor = np.searchsorted(d["offsets"], np.arange(R), side="right") - 1
        out = oracle.expert_ffn(*OW, np.ascontiguousarray(x_s[d["row_token"]]), eor)
    else:
        out = np.zeros((1, w.d))
    return oracle.combine(out, d["slot_row"], r["G"], (w.E / w.k) if rescale else 1.0)


def oracle_inputs(w, inp):
    import oracle
    raw = wl.to_numpy_raw
    if w.partition == wl.COPY and "W1s" in inp:
        OW = (raw(inp["W1s"]), raw(inp["W3s"]), raw(inp["W2s"]))
    else:
        OW = oracle.partition(raw(inp["W1"]), raw(inp["W3"]), raw(inp["W2"]), w.E,
                              oracle.COPY if w.partition == wl.COPY else oracle.DISJOINT,
                              None if inp["perm"] is None else raw(inp["perm"]))
    x = raw(inp["x"])
    eps = None if inp["eps"] is None else raw(inp["eps"])
    Wn = None if inp["Wnoise"] is None else raw(inp["Wnoise"])
    bias = None if inp["bias"] is None else raw(inp["bias"])
    return x, eps, raw(inp["Wg"]), Wn, bias, OW


def cpu_model():
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def time_oracle_single_thread():
    """The oracle on the whole tiny_fp32 layer (512 tokens, fp32 inputs) on one host
    thread: the single-core figure of the CPU baseline."""
    import oracle
    w = wl.WORKLOADS["tiny_fp32"]
    inp = wl.make_inputs(w)
    x, eps, Wg, Wn, bias, OW = oracle_inputs(w, inp)
    n0 = oracle.num_threads()
    oracle.set_num_threads(1)
    try:
        oracle_sample_forward(w, x[:8], None, Wg, Wn, bias, OW, -1, w.rescale)
        t0 = time.perf_counter()
        reps = 0
        while True:
            oracle_sample_forward(w, x, None, Wg, Wn, bias, OW, -1, w.rescale)
            reps += 1
            if time.perf_counter() - t0 > 2.0:
                break
        t = time.perf_counter() - t0
    finally:
        oracle.set_num_threads(n0)
    return {"value": reps * w.T / t, "unit": "tokens/s", "cores": 1,
            "sample": "tiny_fp32, all %d tokens, %d passes, %.1f s" % (w.T, reps, t)}


def time_oracle(w, inp, C, target_s=12.0, max_tokens=8192):
    """Oracle tokens/s on a bounded, seeded sample of the workload's tokens."""
    import oracle
    x, eps, Wg, Wn, bias, OW = oracle_inputs(w, inp)
    rng = np.random.default_rng(w.seed)

    def run(n):
        toks = np.sort(rng.choice(w.T, size=min(n, w.T), replace=False))
        xs = np.ascontiguousarray(x[toks])
        es = None if eps is None else np.ascontiguousarray(eps[toks])
        t0 = time.perf_counter()
        oracle_sample_forward(w, xs, es, Wg, Wn, bias, OW, C, w.rescale)
        return len(toks), time.perf_counter() - t0

    n0, t_probe = run(4)
    per_tok = t_probe / max(n0, 1)
    n = int(max(4, min(max_tokens, target_s / max(per_tok, 1e-9))))
    n_done, t = run(n)
    return {"value": n_done / t, "unit": "tokens/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": "%d of %d tokens of %s (seeded), full layer: router, dispatch (capacity "
                      "%d), SwiGLU experts, combine, statistics; fp64, %.1f s" %
                      (n_done, w.T, w.name, C, t)}


# --------------------------------------------------------------------------- main

def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=HEADLINE, choices=sorted(wl.WORKLOADS))
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the other forward workloads (reported under 'workloads')")
    ap.add_argument("--impl", default="libmoe", choices=["libmoe", "reference"])
    ap.add_argument("--tokens", type=int, default=None,
                    help="override the workload's T (small cases for profiling)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--cluster", action="store_true",
                    help="time the clustering partition (balanced k-means of the W1 rows) "
                         "of the workload's FFN instead of the layer")
    ap.add_argument("--cluster-iters", type=int, default=10)
    ap.add_argument("--expert-parallel", action="store_true",
                    help="time the expert-parallel layer: each of the N ranks holds the "
                         "workload's T tokens and E/N experts, rows move over NCCL")
    ap.add_argument("--backward", action="store_true",
                    help="time a training step (forward + backward) of the layer")
    return ap.parse_args()


def dist_setup(n):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n:
        raise SystemExit("--gpus %d but WORLD_SIZE=%d (launch N>1 with torchrun)" % (n, world))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                              device_id=torch.device("cuda", local))
    return rank, world, local


def max_over_ranks(v, world, device="cuda"):
    """The slowest rank's time (every rank calls it, in the same order)."""
    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def tokens_per_s(tokens_per_rank, steps, world, ms_max):
    """Whole-job throughput of independent replicas (weak scaling): every rank's
    tokens over the slowest rank's time."""
    return tokens_per_rank * steps * world / (ms_max / 1000.0)


def barrier(world):
    if world > 1:
        torch.distributed.barrier()

def e2e_pipeline(args, w, p, moe, x, Wg, Wn, eps, bias, W13_e, W2_e, world, depth=2):
    """End to end through the host-buffer pipeline (moe_pipeline_*): every step copies
    its x (and noise) in from pinned host memory and its y, L_balance and status word
    back out; with `depth` batches in flight the copies overlap the layer.  Host wall
    clock around the whole run, device idle on both sides, max over ranks."""
    x_h = x.cpu().pin_memory()
    eps_h = eps.cpu().pin_memory() if eps is not None else None
    y_h = [torch.empty(x.shape, dtype=x.dtype).pin_memory() for _ in range(depth)]
    loss_h = [torch.empty(1, dtype=torch.float32).pin_memory() for _ in range(depth)]
    pl = moe.Pipeline(p, Wg, W13_e, W2_e, Wnoise=Wn, bias=bias, depth=depth)

    def run(n):
        t = None
        for i in range(n):
            t = pl.submit(x_h, y_h[i % depth], loss_h[i % depth], noise_host=eps_h)
        pl.wait(t)

    run(args.warmup)
    torch.cuda.synchronize()
    barrier(world)
    t0 = time.perf_counter()
    run(args.steps)
    t1 = time.perf_counter()
    barrier(world)
    pl.close()
    ms = max_over_ranks((t1 - t0) * 1000.0, world)
    h2d = x.numel() * x.element_size() + (eps.numel() * 4 if eps is not None else 0)
    d2h = x.numel() * x.element_size() + 4 + 4
    return {"value": w.T * args.steps * world / (ms / 1000.0), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": ms / args.steps,
            "api": "moe_pipeline_submit/moe_pipeline_wait, %d batches in flight, host wall "
                   "clock" % depth}


def run_decode(args, w, p, moe, ws, b, x, Wg, Wn, eps, bias, W13_e, W2_e, C, rank, world,
               local):
    """Decode-shaped batches (T <= 64): the layer is launch- and weight-streaming-bound,
    so one moe_forward is captured in a CUDA graph and the graph is replayed; the
    figure of merit is the HBM rate of streaming the selected experts' weights.  The
    selected experts' weights (67.6 MB at T = 1) fit in the 126 MB L2, so a 512 MB
    buffer is read (not written: no dirty lines left to write back) between timed
    replays, and each replay is bracketed by its own events."""
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            moe.moe_forward(p, x, Wg, W13_e, W2_e, ws, b, Wnoise=Wn, noise=eps, bias=bias)
    stream.synchronize()
    status = moe.moe_get_device_status(ws)
    if status != 0:
        raise SystemExit("device status %d after warm-up" % status)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        moe.moe_forward(p, x, Wg, W13_e, W2_e, ws, b, Wnoise=Wn, noise=eps, bias=bias)
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()
    kept = b.kept.cpu()
    experts_used = int((kept > 0).sum())
    es = 2
    w_bytes = experts_used * (2 * w.m * w.d + w.d * w.m) * es
    io_bytes = 2 * w.T * w.d * es + w.d * w.E * es
    cur = torch.cuda.current_stream()
    flush = torch.ones(128 << 20, dtype=torch.float32, device="cuda")
    acc = torch.zeros((), dtype=torch.float32, device="cuda")
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    sampler = ClockSampler(local)
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    t_wall0 = time.time()
    for a, c in evs:
        torch.sum(flush, dim=0, out=acc)
        a.record(cur)
        graph.replay()
        c.record(cur)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    barrier(world)
    time.sleep(0.15)
    sampler.stop()
    ms = max_over_ranks(sum(a.elapsed_time(c) for a, c in evs), world)
    us = 1000.0 * ms / args.steps
    del flush
    peaks, peak_src = load_peaks()
    gbs = (w_bytes + io_bytes) / (us * 1e-6) / 1e9
    launches_per_forward = None
    l1 = moe.moe_launch_count()
    moe.moe_forward(p, x, Wg, W13_e, W2_e, ws, b, Wnoise=Wn, noise=eps, bias=bias)
    launches_per_forward = moe.moe_launch_count() - l1
    torch.cuda.synchronize()
    e2e = None if args.no_e2e else e2e_pipeline(args, w, p, moe, x, Wg, Wn, eps, bias, W13_e,
                                                W2_e, world)
    line = {
        "metric": METRIC, "value": w.T * args.steps * world / (ms / 1000.0), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms / args.steps, "us_per_layer": us, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(config_of(w, C), parallelism="dp%d replicas" % world,
                       experts_streamed=experts_used,
                       timing="CUDA graph of one moe_forward, events around each replay",
                       l2="512 MB buffer read between timed replays"),
        "roofline": {"kernel": "whole layer (selected experts' weights streamed once)",
                     "bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": gbs / peaks["hbm_gbs"], "traffic": None,
                     "peak_source": "%s hbm_gbs" % peak_src,
                     "algorithmic": "%d experts x 3*d*m*2 B + x, y, W_g = %.4g B per layer"
                                    % (experts_used, w_bytes + io_bytes)},
        "cpu_baseline": None, "e2e": e2e,
        "gpu_launches": launches_per_forward * args.steps,
        "clocks": sampler.summary(t_wall0, t_wall1),
    }
    return line


# FP64 lanes per SM on B200: NVIDIA's published 37-40 TFLOP/s FP64 over
# (2 FLOP per FMA x 148 SMs x 1.965 GHz) gives 64-69; 64 is the power of two.
FP64_LANES_PER_SM = 64
SM_COUNT = 148
SM_MAX_MHZ = 1965.0


def run_cluster(args, rank, world, local):
    """The clustering partition (balanced k-means over the W1 rows, E clusters of
    d_ff/E neurons, --cluster-iters iterations) on the workload's FFN.  One step =
    one whole moe_cluster_partition call.  F (W1) is below the 126 MB L2, so a
    256 MB buffer is written between timed calls.  The roofline kernel is the
    distance step (f64 ALU bound), timed alone with the same L2 flush."""
    import top_routing_grouped_noisy_b200 as moe
    w = wl.WORKLOADS[args.workload]
    inp = wl.make_inputs(w, device="cuda", seed=w.seed + 7919 * rank)
    F = inp["W1"]
    del inp
    n_iter = args.cluster_iters
    init = wl.make_cluster_init(w.d_ff, w.E, w.seed + rank).cuda()
    nbytes = moe.moe_cluster_workspace_size(w.d, w.d_ff, w.E)
    ws = moe.Workspace(None, device="cuda", nbytes=nbytes)
    assign = torch.empty(w.d_ff, dtype=torch.int32, device="cuda")
    perm = torch.empty(w.d_ff, dtype=torch.int32, device="cuda")
    centers = torch.empty(w.E, w.d, dtype=torch.float64, device="cuda")
    D = torch.empty(w.d_ff, w.E, dtype=torch.float64, device="cuda")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    lib = moe.lib()
    dt = moe.MOE_BF16 if F.dtype == torch.bfloat16 else moe.MOE_F32

    def call():
        rc = lib.moe_cluster_partition(F.data_ptr(), w.d, w.d_ff, w.E, dt, n_iter,
                                       init.data_ptr(), assign.data_ptr(), centers.data_ptr(),
                                       perm.data_ptr(), ws.ptr, ws.nbytes, stream.cuda_stream)
        if rc != 0:
            raise SystemExit("moe_cluster_partition: %s" % lib.moe_last_error_string().decode())

    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    if moe.moe_get_device_status(ws) != 0:
        raise SystemExit("device status set by the clustering")
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    sampler = ClockSampler(local)
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    l0 = moe.moe_launch_count()
    t_wall0 = time.time()
    for a, b in evs:
        flush.fill_(1)
        a.record(stream)
        call()
        b.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    launches = moe.moe_launch_count() - l0
    # the distance step alone, same flush
    devs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(args.steps)]
    for a, b in devs:
        flush.fill_(1)
        a.record(stream)
        moe.moe_cluster_distances(F, centers, out=D)
        b.record(stream)
    torch.cuda.synchronize()
    time.sleep(0.15)
    sampler.stop()
    clocks = sampler.summary(t_wall0, t_wall1)
    ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs) / args.steps, world)
    dist_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in devs) / args.steps, world)
    counts = torch.bincount(assign.long(), minlength=w.E).tolist()
    if counts != [w.d_ff // w.E] * w.E:
        raise SystemExit("unbalanced clusters %s" % counts)

    ops = 3.0 * w.d_ff * w.E * w.d  # subtract, multiply, add per (neuron, center, column)
    achieved = ops / (dist_ms / 1000.0) / 1e12
    peak = SM_COUNT * FP64_LANES_PER_SM * SM_MAX_MHZ * 1e6 / 1e12
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        Fh = wl.to_numpy_raw(F)
        it_s = 2
        t0 = time.time()
        oracle.cluster(Fh, w.E, it_s, init.cpu().numpy())
        t1 = time.time()
        cpu = {"value": (t1 - t0) * 1000.0 * n_iter / it_s, "unit": "ms", "cores":
               oracle.num_threads(), "kind": "oracle",
               "sample": "%d of the %d iterations on the same W1, scaled to %d" %
                         (it_s, n_iter, n_iter)}
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank != 0:
        return 0
    line = {
        "metric": "clustering partition time (balanced k-means over the W1 rows)",
        "value": ms, "unit": "ms", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "cluster_%s_w1" % w.name, "d": w.d, "d_ff": w.d_ff, "E": w.E,
                   "n_iter": n_iter, "features": "W1 [d_ff][d] %s" % wl.torch_dtype(w),
                   "parallelism": "dp%d replicas" % world,
                   "l2": "256 MB buffer written between timed calls"},
        "roofline": {"kernel": "cluster_dist_kernel (distance step, moe_cluster_distances)",
                     "bound": "alu", "achieved": achieved, "peak": peak,
                     "unit": "TFLOP/s (f64 add/sub/mul)", "frac": achieved / peak,
                     "traffic": None,
                     "peak_source": "derived: %d SMs x %d FP64 lanes x %.0f MHz" %
                                    (SM_COUNT, FP64_LANES_PER_SM, SM_MAX_MHZ),
                     "algorithmic": "3 f64 ops per (neuron, center, column) = %.4g per launch"
                                    % ops},
        "kernels": {"distance_step_ms": dist_ms, "per_iteration_ms": ms / n_iter},
        "cpu_baseline": cpu, "e2e": None, "gpu_launches": launches, "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_expert_parallel(args, rank, world, local):
    """The expert-parallel layer (expert_parallel.ExpertParallelMoE over NCCL): rank r
    routes its own T tokens over all E experts and runs the grouped GEMMs of experts
    [r E/N, (r+1) E/N) on the rows every rank sends it.  Capacity (if the workload has
    one) over all ranks' tokens.  One step = one whole layer forward, host plan and
    row exchanges included; weak scaling (T tokens per rank).  With N = 1 the group
    has one rank and the exchanges are local copies."""
    import datetime

    import top_routing_grouped_noisy_b200 as moe
    from top_routing_grouped_noisy_b200.expert_parallel import ExpertParallelMoE
    if world == 1:
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        os.environ.setdefault("MASTER_PORT", str(29300 + os.getpid() % 600))
        torch.distributed.init_process_group("nccl", rank=0, world_size=1,
                                              timeout=datetime.timedelta(seconds=120),
                                              device_id=torch.device("cuda", local))
    w = wl.WORKLOADS[args.workload]
    if args.tokens is not None:
        w = w.with_(T=args.tokens)
    if w.E % world != 0 or w.shared > 0 or w.partition != wl.DISJOINT:
        raise SystemExit("--expert-parallel needs a disjoint workload whose E divides N")
    dt = wl.torch_dtype(w)
    # the model (weights, router) is the same on every rank; the tokens differ
    inp = wl.make_inputs(w, device="cuda", seed=w.seed)
    tok = wl.make_inputs(w, device="cuda", seed=w.seed + 7919 * rank)
    x, eps = tok["x"], tok["eps"]
    del tok
    C = moe.moe_capacity(w.T * world, w.E, w.cf) if w.cf >= 0 else -1
    p = moe.params(w.T, w.d, w.E, w.k, w.m, dt, w.router, C, w.rescale, w.lam)
    ws = moe.Workspace(p)
    W13_e, W2_e = moe.moe_partition_experts(inp["W1"], inp["W3"], inp["W2"], w.E, moe.DISJOINT,
                                            perm=inp["perm"], ws=ws)
    El = w.E // world
    lo = rank * El
    W13_l = W13_e.view(w.E, -1)[lo:lo + El].clone().reshape(-1)
    W2_l = W2_e.view(w.E, -1)[lo:lo + El].clone().reshape(-1)
    del W13_e, W2_e
    L = ExpertParallelMoE(w.d, w.E, w.k, w.m, W13_l, W2_l, inp["Wg"], inp["Wnoise"], inp["bias"],
                          dt, w.router, C, moe.EP_CAPACITY_GLOBAL, w.rescale, w.lam)
    for n in ("W1", "W3", "W2", "x", "eps"):
        inp.pop(n, None)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        s = L.begin(x, eps)
        L.gather_counts(s)
        L.plan(s)
        L.send_rows(s)
        if ev is not None:
            ev[0].record(stream)
        L.experts(s)
        if ev is not None:
            ev[1].record(stream)
        L.return_rows(s)
        return L.finish(s)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    exp = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    sampler = ClockSampler(local)
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    l0 = moe.moe_launch_count()
    t_wall0 = time.time()
    rows = 0
    plan_ms = 0.0
    for (a, b), e in zip(evs, exp):
        a.record(stream)
        s = step(e)
        b.record(stream)
        rows += s.R_in
        plan_ms += s.host_plan_ms
    torch.cuda.synchronize()
    barrier(world)
    t_wall1 = time.time()
    launches = moe.moe_launch_count() - l0
    time.sleep(0.15)
    sampler.stop()
    clocks = sampler.summary(t_wall0, t_wall1)
    for wsx in (L._ws_route, L._ws_ffn):
        if wsx is not None and moe.moe_get_device_status(wsx) != 0:
            raise SystemExit("device status set by the expert-parallel layer")
    # every step waits on the host for the counts (the plan), so the device time of a
    # step is bracketed by its own events; the sum over the steps is the timed region
    ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs), world)
    exp_ms = sum(a.elapsed_time(b) for a, b in exp) / args.steps
    flop = 6.0 * w.d * w.m * rows / args.steps
    tf = flop / (exp_ms / 1000.0) / 1e12
    tf_slow = -max_over_ranks(-tf, world)  # the slowest rank's expert GEMMs
    peaks, peak_src = load_peaks()
    torch.distributed.destroy_process_group()
    if rank != 0:
        return 0
    line = {
        "metric": "MoE-layer tokens/s (expert parallel)",
        "value": tokens_per_s(w.T, args.steps, world, ms), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(config_of(w, C), workload="ep%d_%s" % (world, w.name),
                       parallelism="ep%d" % world, tokens_per_rank=w.T,
                       experts_per_rank=El, capacity_scope="global",
                       global_batch=w.T * world),
        "roofline": dict({"kernel": "moe_expert_ffn on the received rows (grouped GEMM 1 + "
                                    "SwiGLU, GEMM 2) of the slowest rank",
                          "bound": "tensor", "achieved": tf_slow, "unit": "TFLOP/s",
                          "traffic": None, "algorithmic": "6*d*m FLOP per received row"},
                         **tensor_roof(tf_slow, peaks, peak_src)),
        "kernels": {"expert_ffn_ms": exp_ms, "rows_in_per_step": rows / args.steps,
                    "host_plan_ms": plan_ms / args.steps,
                    "host_plan": "per step, the host waits for the gathered counts (pinned "
                                 "copy) and plans the exchange while the device idles; "
                                 "included in ms_per_step"},
        "cpu_baseline": None, "e2e": None, "gpu_launches": launches, "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_train(args, w, p, moe, fwd_step, b, x, Wg, Wn, eps, bias, W13_e, W2_e, C, inp, shared,
              rank, world, local):
    """A training step of the layer: the forward (the six step calls) and the backward
    (combine, expert GEMM 2, expert GEMM 1 + SwiGLU, router + input) for l(y) + L_balance
    with a seeded dl/dy.  The roofline figure is moe_expert_up_backward, timed inside the
    step loop: three tcgen05 GEMMs (g/u recompute with the SwiGLU backward, dgrad,
    wgrad) plus the transposes that feed the weight-gradient GEMM.  For a residual layer
    (shared neurons) the backward is the one call moe_backward_residual, which is then
    the roofline figure (its 16 d m R + 16 d m_s T FLOP)."""
    if w.dtype != "bf16":
        raise SystemExit("--backward runs bf16 layers")
    stream = torch.cuda.current_stream()
    dy = wl.make_grad_output(w, w.seed + 1 + 7919 * rank, device="cuda")
    g = moe.BackwardBuffers(p, Wn is not None, bias is not None)
    res = shared is not None
    if res:
        W13_s, W2_s, h_s = shared
        dh_s = torch.empty_like(h_s)
        dx_s = torch.empty(w.T, w.d, dtype=torch.bfloat16, device="cuda")
        dW13_s = torch.empty_like(W13_s)
        dW2_s = torch.empty_like(W2_s)
        wsb = moe.Workspace(p, nbytes=moe.moe_backward_residual_workspace_size(p, w.shared))
    else:
        wsb = moe.Workspace(p, nbytes=moe.moe_backward_workspace_size(p))
    SEG = ["forward", "backward"] if res else ["forward", "combine_bwd", "down_bwd", "up_bwd",
                                              "route_bwd"]

    def step(ev=None, up=None):
        def mark(i):
            if ev is not None:
                ev[i].record(stream)
        mark(0)
        fwd_step()
        mark(1)
        if res:
            if up is not None:
                up[0].record(stream)
            moe.moe_backward_residual(p, x, Wg, W13_e, W2_e, W13_s, W2_s, w.shared, h_s, b, g,
                                      dy, dh_s, dx_s, dW13_s, dW2_s, wsb, Wnoise=Wn, noise=eps,
                                      bias=bias, dLb=1.0)
            if up is not None:
                up[1].record(stream)
            mark(2)
            return
        moe.moe_combine_backward(p, dy, b.out, b.slot_row, b.topk_w, g.d_out, g.dG)
        mark(2)
        moe.moe_expert_down_backward(p, g.d_out, b.h, b.offsets, W2_e, g.dh, g.dW2_e, wsb)
        mark(3)
        if up is not None:
            up[0].record(stream)
        moe.moe_expert_up_backward(p, b.x_perm, g.dh, b.offsets, W13_e, g.dx_perm, g.dW13_e, wsb)
        if up is not None:
            up[1].record(stream)
        mark(4)
        moe.moe_route_backward(p, x, Wg, b.topk_idx, b.topk_w, g.dG, b.counts, g.dx_perm,
                               b.slot_row, g.dx, g.dWg, wsb, Wnoise=Wn, noise=eps, bias=bias,
                               dWnoise=g.dWnoise, dbias=g.dbias, dLb=1.0)
        mark(5)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = moe.moe_get_device_status(wsb)
    if st != 0:
        raise SystemExit("device status %d after warm-up" % st)
    R = int(b.offsets[-1])
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # events around the roofline call on every 8th step only (an event between two
    # kernels keeps the second from starting early under programmatic dependent launch)
    up_evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              if i % 8 == 0 else None for i in range(args.steps)]
    sampler = ClockSampler(local)
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    l0 = moe.moe_launch_count()
    t_wall0 = time.time()
    start.record(stream)
    for i in range(args.steps):
        step(up=up_evs[i])
    end.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    barrier(world)
    launches = moe.moe_launch_count() - l0
    time.sleep(0.15)
    sampler.stop()
    clocks = sampler.summary(t_wall0, t_wall1)
    if moe.moe_get_device_status(wsb) != 0:
        raise SystemExit("device status set in the timed region")
    ms = max_over_ranks(start.elapsed_time(end), world)
    up_pairs = [ev for ev in up_evs if ev is not None]
    up_ms = max_over_ranks(sum(a.elapsed_time(c) for a, c in up_pairs) / len(up_pairs), world)
    nseg = min(args.steps, 50)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(SEG) + 1)]
           for _ in range(nseg)]
    for i in range(nseg):
        step(evs[i])
    torch.cuda.synchronize()
    seg = np.zeros(len(SEG))
    for e in evs:
        for k2 in range(len(SEG)):
            seg[k2] += e[k2].elapsed_time(e[k2 + 1])
    seg = [max_over_ranks(v / nseg, world) for v in seg]
    value = tokens_per_s(w.T, args.steps, world, ms)
    dmr = float(w.d) * w.m * R
    dms = float(w.d) * w.shared * w.T  # shared block (residual layer), every token
    # forward 6, GEMM 2 backward 4, GEMM 1 backward 12 (with recompute); same for the block
    flop_step = 22.0 * (dmr + dms)
    peaks, peak_src = load_peaks()
    up_flop = 16.0 * (dmr + dms) if res else 12.0 * dmr
    up_tf = up_flop / (up_ms / 1000.0) / 1e12
    kernels = {n: {"ms": v} for n, v in zip(SEG, seg)}
    kernels["forward"]["TFLOP/s"] = 6.0 * (dmr + dms) / (seg[0] / 1000.0) / 1e12
    if res:
        kernels["backward"]["TFLOP/s"] = up_tf
    else:
        kernels["down_bwd"]["TFLOP/s"] = 4.0 * dmr / (seg[2] / 1000.0) / 1e12
        kernels["up_bwd"]["TFLOP/s"] = 12.0 * dmr / (seg[3] / 1000.0) / 1e12
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not res:
        import oracle
        n_s = 128
        sub = {k2: (v[:n_s].cpu() if k2 in ("x", "eps") and v is not None else
                    (v.cpu() if isinstance(v, torch.Tensor) else v)) for k2, v in inp.items()}
        if w.partition == wl.COPY:
            W1e, W3e, W2e = oracle.partition(wl.to_numpy_raw(sub["W1"]), wl.to_numpy_raw(
                sub["W3"]), wl.to_numpy_raw(sub["W2"]), w.E, oracle.COPY)
        else:
            W1e, W3e, W2e = oracle.partition(wl.to_numpy_raw(sub["W1"]), wl.to_numpy_raw(
                sub["W3"]), wl.to_numpy_raw(sub["W2"]), w.E, oracle.DISJOINT,
                wl.to_numpy_raw(sub["perm"]))
        dy_s = dy[:n_s].cpu().to(torch.float64).numpy()
        C_s = moe.moe_capacity(n_s, w.E, w.cf) if w.cf >= 0 else -1
        t0 = time.time()
        oracle.backward(wl.to_numpy_raw(sub["x"]), wl.to_numpy_raw(sub["Wg"]), W1e, W3e, W2e,
                        w.k, dy_s, w.router, None if sub["Wnoise"] is None else
                        wl.to_numpy_raw(sub["Wnoise"]), None if sub["eps"] is None else
                        sub["eps"].numpy(), None if sub["bias"] is None else sub["bias"].numpy(),
                        C_s, w.rescale, w.lam, 1.0)
        el = time.time() - t0
        cpu = {"value": n_s / el, "unit": "tokens/s", "cores": oracle.num_threads(),
               "kind": "oracle", "sample": "forward + backward of the first %d tokens (same "
               "weights, capacity for %d tokens), %.1f s" % (n_s, n_s, el)}
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank != 0:
        return 0
    line = {
        "metric": "MoE-layer training step (forward + backward) tokens/s at 1 B200",
        "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(config_of(w, C), parallelism="dp%d replicas" % world, kept_rows=R,
                       loss="sum(y * dy) + L_balance, dy ~ N(0,1) seeded"),
        "tflops": flop_step * args.steps * world / (ms / 1000.0) / 1e12,
        "roofline": dict({"kernel": ("moe_backward_residual: the routed and the shared "
                                     "block's backward GEMMs + transposes + router" if res else
                                     "moe_expert_up_backward: bwd_gemm_kernel x3 (recompute + "
                                     "SwiGLU backward, dgrad, wgrad) + 3 transposes"),
                          "bound": "tensor", "achieved": up_tf, "unit": "TFLOP/s",
                          "traffic": None,
                          "algorithmic": ("16*d*(m*R + m_s*T) = %.4g FLOP per call" % up_flop
                                          if res else "12*d*m FLOP per kept row x R=%d = %.4g "
                                          "FLOP per call" % (R, up_flop))},
                         **tensor_roof(up_tf, peaks, peak_src)),
        "kernels": kernels, "cpu_baseline": cpu, "e2e": None, "gpu_launches": launches,
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = wl.WORKLOADS[args.workload]
    if args.tokens is not None:
        w = w.with_(T=args.tokens)
    inp = wl.make_inputs(w, device="cpu")
    C = -1 if w.cf < 0 else int(np.ceil(w.T * w.cf / w.E - 1e-12))
    import oracle
    x, eps, Wg, Wn, bias, OW = oracle_inputs(w, inp)
    rng = np.random.default_rng(w.seed)
    # size each step's sample so that warm-up + timed steps take about two minutes
    t0 = time.perf_counter()
    oracle_sample_forward(w, x[:2], None if eps is None else eps[:2], Wg, Wn, bias, OW, C,
                          w.rescale)
    per_tok = (time.perf_counter() - t0) / 2
    n = int(max(1, min(64, 120.0 / max((args.steps + args.warmup) * per_tok, 1e-9))))
    total_tok, total_t = 0, 0.0
    for i in range(args.warmup + args.steps):
        toks = np.sort(rng.choice(w.T, size=n, replace=False))
        xs = np.ascontiguousarray(x[toks])
        es = None if eps is None else np.ascontiguousarray(eps[toks])
        t0 = time.perf_counter()
        oracle_sample_forward(w, xs, es, Wg, Wn, bias, OW, C, w.rescale)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            total_tok += n
            total_t += dt
    v = total_tok / total_t
    sample = ("%d seeded tokens of %s per step (full layer in fp64 on the host, "
              "oracle as is)" % (n, w.name))
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * total_t / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, C),
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    rank, world, local = dist_setup(args.gpus)
    torch.cuda.set_device(local)
    if args.cluster:
        return run_cluster(args, rank, world, local)
    if args.expert_parallel:
        return run_expert_parallel(args, rank, world, local)
    w = wl.WORKLOADS[args.workload]
    if args.tokens is not None:
        w = w.with_(T=args.tokens)
    line = forward_line(args, w, rank, world, local)
    if line is None:  # the training step printed its own line
        return 0
    if not args.no_extra and args.tokens is None and not args.backward:
        extra = {}
        for name in EXTRA:
            if name == w.name:
                continue
            torch.cuda.empty_cache()
            w2 = wl.WORKLOADS[name]
            decode = w2.T <= 64
            a2 = argparse.Namespace(**vars(args))
            # fewer steps for the extra workloads; decode steps are microseconds long
            a2.steps = 500 if decode else max(10, min(args.steps, 30))
            a2.warmup = 20 if decode else 3
            a2.no_e2e, a2.no_cpu_baseline, a2.backward = True, True, False
            try:
                l2 = forward_line(a2, w2, rank, world, local)
            except Exception as exc:  # never lose the headline to an extra workload
                extra[name] = {"error": "%s: %s" % (type(exc).__name__, exc)}
                continue
            for key in ("metric", "n_gpus", "higher_is_better", "scaling", "vs_baseline",
                        "data", "cpu_baseline", "e2e"):
                l2.pop(key, None)
            extra[name] = l2
        line["workloads"] = extra
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def forward_line(args, w, rank, world, local):
    """Measures the layer forward of workload ``w`` and returns its JSON line (rank 0's
    view; every rank takes the same collective steps)."""
    import top_routing_grouped_noisy_b200 as moe

    inp = wl.make_inputs(w, device="cuda", seed=w.seed + 7919 * rank)
    C = moe.moe_capacity(w.T, w.E, w.cf) if w.cf >= 0 else -1
    dt = wl.torch_dtype(w)
    p = moe.params(w.T, w.d, w.E, w.k, w.m, dt, w.router, C, w.rescale, w.lam)
    ws = moe.Workspace(p)
    if w.partition == wl.COPY and "W1s" in inp:
        W13_e, W2_e = moe.moe_partition_experts(inp["W1s"], inp["W3s"], inp["W2s"], w.E,
                                                moe.STACKED, ws=ws)
    elif w.partition == wl.COPY:
        W13_e, W2_e = moe.moe_partition_experts(inp["W1"], inp["W3"], inp["W2"], w.E, moe.COPY,
                                                ws=ws)
    elif w.shared > 0:  # residual MoE: shared block plus disjoint experts
        W13_e, W2_e, W13_s, W2_s = moe.moe_partition_residual(
            inp["W1"], inp["W3"], inp["W2"], w.E, inp["shared_idx"], inp["perm_rest"], ws=ws)
    else:
        W13_e, W2_e = moe.moe_partition_experts(inp["W1"], inp["W3"], inp["W2"], w.E,
                                                moe.DISJOINT, perm=inp["perm"], ws=ws)
    res = w.shared > 0
    if res:
        ps = moe.params(w.T, w.d, 1, 1, w.shared, dt, w.router, -1, w.rescale, w.lam)
        tok_range = torch.tensor([0, w.T], dtype=torch.int32, device="cuda")
        h_s = torch.empty(w.T, moe.h_ld(w.shared), dtype=dt, device="cuda")
        out_s = torch.empty(w.T, w.d, dtype=dt, device="cuda")
    b = moe.ForwardBuffers(p)
    x, Wg, Wn, eps, bias = inp["x"], inp["Wg"], inp["Wnoise"], inp["eps"], inp["bias"]
    # the router weights in the tensor-core router's layout, packed once like W13_e / W2_e
    Wt = moe.moe_router_pack(p, Wg, Wn) if dt == torch.bfloat16 else None
    b.router_packed = Wt
    stream = torch.cuda.current_stream()
    # moe_forward's path: the dispatch materialises x_perm (the row-gathering GEMM 1
    # variant, moe_expert_up_gather, is slower on B200)
    gather = False
    SEG = ["route", "dispatch", "expert_up", "expert_down"] + (["shared"] if res else []) + \
        ["combine", "gate_stats"]
    NSEG = len(SEG)

    def step(ev=None, up_only=None):
        # ev: events between all steps; up_only: a (start, end) pair around expert
        # GEMM 1 alone (the roofline kernel), for the timed loop
        seg = iter(range(NSEG + 1))

        def mark():
            i = next(seg)
            if ev is not None:
                ev[i].record(stream)

        mark()
        if Wt is not None:  # router weights packed once per weight set
            moe.moe_route_packed(p, x, Wg, Wn, Wt, eps, bias, ws, b.topk_idx, b.topk_w,
                                 b.probs_sum, b.importance)
        else:
            moe.moe_route(p, x, Wg, Wn, eps, bias, ws, b.topk_idx, b.topk_w, b.probs_sum,
                          b.importance)
        mark()
        if gather:
            moe.moe_dispatch_rows(p, b.topk_idx, ws, b.row_token, b.slot_row, b.counts, b.kept,
                                  b.offsets)
        else:
            # moe_forward's dispatch: the router already counted the chunks
            moe.moe_dispatch_routed(p, x, b.topk_idx, ws, b.x_perm, b.row_token, b.slot_row,
                                    b.counts, b.kept, b.offsets)
        mark()
        if up_only is not None:
            up_only[0].record(stream)
        if gather:
            moe.moe_expert_up_gather(p, x, b.row_token, b.offsets, W13_e, b.h, ws)
        else:
            moe.moe_expert_up(p, b.x_perm, b.offsets, W13_e, b.h, ws)
        if up_only is not None:
            up_only[1].record(stream)
        mark()
        moe.moe_expert_down(p, b.h, b.offsets, W2_e, b.out, ws)
        mark()
        if res:  # the shared block: one expert over every token
            moe.moe_expert_ffn(ps, x, tok_range, W13_s, W2_s, h_s, out_s, ws)
            mark()
            moe.moe_combine_residual(p, b.out, b.slot_row, b.topk_w, out_s, b.y)
        else:
            moe.moe_combine(p, b.out, b.slot_row, b.topk_w, b.y)
        mark()
        moe.moe_gate_stats(p, b.counts, b.probs_sum, b.f, b.P, b.loss)
        mark()

    if args.backward:
        run_train(args, w, p, moe, step, b, x, Wg, Wn, eps, bias, W13_e, W2_e, C, inp,
                  (W13_s, W2_s, h_s) if res else None, rank, world, local)
        return None
    if w.T <= 64:
        return run_decode(args, w, p, moe, ws, b, x, Wg, Wn, eps, bias, W13_e, W2_e, C, rank,
                          world, local)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    status = moe.moe_get_device_status(ws)
    if status != 0:
        raise SystemExit("device status %d after warm-up" % status)
    R = int(b.offsets[-1])

    # the timed loop: K whole steps back to back; the only events inside it bracket
    # expert GEMM 1 (its time is the roofline figure) on every UP_EVERY-th step -- an
    # event recorded between two kernels keeps the second from starting early under
    # programmatic dependent launch, so bracketing every step would slow the loop
    UP_EVERY = 8
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    up_evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              if i % UP_EVERY == 0 else None for i in range(args.steps)]
    sampler = ClockSampler(local)
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    l0 = moe.moe_launch_count()
    t_wall0 = time.time()
    start.record(stream)
    for i in range(args.steps):
        step(up_only=up_evs[i])
    end.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    barrier(world)
    launches = moe.moe_launch_count() - l0
    time.sleep(0.15)
    sampler.stop()
    clocks = sampler.summary(t_wall0, t_wall1)
    status = moe.moe_get_device_status(ws)
    if status != 0:
        raise SystemExit("device status %d after the timed region" % status)
    ms_local = start.elapsed_time(end)
    # per-step breakdown: a second pass of the same steps with events between them
    # (the events keep each kernel from overlapping its neighbours' launch)
    nseg_steps = min(args.steps, 100)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(NSEG + 1)]
           for _ in range(nseg_steps)]
    torch.cuda.synchronize()
    for i in range(nseg_steps):
        step(evs[i])
    torch.cuda.synchronize()
    seg_ms = np.zeros(NSEG)
    for e in evs:
        for s in range(NSEG):
            seg_ms[s] += e[s].elapsed_time(e[s + 1])
    seg_ms /= nseg_steps
    up_pairs = [ev for ev in up_evs if ev is not None]
    up_ms_timed = sum(a.elapsed_time(b) for a, b in up_pairs) / len(up_pairs)
    ms = max_over_ranks(ms_local, world)
    seg_ms = np.array([max_over_ranks(v, world) for v in seg_ms])
    value = tokens_per_s(w.T, args.steps, world, ms)
    flop_step = 6.0 * w.d * w.m * R + (6.0 * w.d * w.shared * w.T if res else 0.0)
    tflops = flop_step * args.steps * world / (ms / 1000.0) / 1e12

    # roofline of the dominant kernel (expert GEMM 1 + SwiGLU), timed inside the step loop
    peaks, peak_src = load_peaks()
    es = 2 if dt == torch.bfloat16 else 4
    up_flop = 4.0 * w.d * w.m * R
    down_flop = 2.0 * w.d * w.m * R
    peak_t = peaks["bf16_tflops"]
    peak_s = peaks.get("bf16_tflops_sustained", peak_t)
    up_ms_timed = max_over_ranks(up_ms_timed, world)
    up_tf = up_flop / (up_ms_timed / 1000.0) / 1e12
    traffic = None
    key = _src_hash("top_routing_grouped_noisy_b200/csrc/ffn_tc.cu")
    tr = NCU_TRAFFIC.get(w.name)
    if tr is not None and tr["src"] == key and tr["T"] == w.T:
        traffic = tr["bytes_per_launch"]
    kname = ("grouped_gemm_2sm_kernel" if w.T * w.k >= 4096 else "grouped_gemm_kernel")
    kname += "<SwiGLU, gather> (expert GEMM 1, moe_expert_up_gather)" if gather else \
        "<SwiGLU> (expert GEMM 1, moe_expert_up)"
    roofline = dict({"kernel": kname, "bound": "tensor", "achieved": up_tf, "unit": "TFLOP/s",
                     "traffic": traffic,
                     "algorithmic": "4*d*m FLOP per kept row x R=%d rows = %.4g FLOP per "
                                    "launch; %.4g B per launch (x_perm, W13, h)"
                                    % (R, up_flop, R * w.d * es + 2 * w.m * w.d * es *
                                       int((b.kept > 0).sum()) + R * w.m * es)},
                    **tensor_roof(up_tf, peaks, peak_src))
    hbm = peaks["hbm_gbs"]
    route_bytes = w.T * w.d * es + (w.T * w.E * 4 if eps is not None else 0) + w.T * w.k * 8
    disp_bytes = (w.T * w.k * 12 if gather else w.T * w.d * es + R * w.d * es + w.T * w.k * 12)
    comb_bytes = R * w.d * es + w.T * w.d * es + w.T * w.k * 8
    sm = dict(zip(SEG, seg_ms))
    kernels = {
        "route": {"ms": seg_ms[0], "bound": "hbm", "GB/s": route_bytes / seg_ms[0] / 1e6,
                  "frac": route_bytes / seg_ms[0] / 1e6 / hbm},
        "dispatch": {"ms": seg_ms[1], "bound": "hbm", "GB/s": disp_bytes / seg_ms[1] / 1e6,
                     "frac": disp_bytes / seg_ms[1] / 1e6 / hbm,
                     "x_perm": "not materialised (GEMM 1 gathers rows of x)" if gather
                     else "materialised"},
        "expert_up": {"ms": seg_ms[2], "bound": "tensor",
                      "TFLOP/s": up_flop / (seg_ms[2] / 1000.0) / 1e12,
                      "frac": up_flop / (seg_ms[2] / 1000.0) / 1e12 / peak_t,
                      "ms_in_timed_loop": up_ms_timed},
        "expert_down": {"ms": seg_ms[3], "bound": "tensor",
                        "TFLOP/s": down_flop / (seg_ms[3] / 1000.0) / 1e12,
                        "frac": down_flop / (seg_ms[3] / 1000.0) / 1e12 / peak_t},
        "combine": {"ms": sm["combine"], "bound": "hbm",
                    "GB/s": comb_bytes / sm["combine"] / 1e6,
                    "frac": comb_bytes / sm["combine"] / 1e6 / hbm},
        "gate_stats": {"ms": sm["gate_stats"]},
    }
    if res:
        sh_flop = 6.0 * w.d * w.shared * w.T
        kernels["shared"] = {"ms": sm["shared"], "bound": "tensor",
                             "TFLOP/s": sh_flop / (sm["shared"] / 1000.0) / 1e12,
                             "frac": sh_flop / (sm["shared"] / 1000.0) / 1e12 / peak_t,
                             "what": "shared block FFN_S: GEMM 1 + SwiGLU and GEMM 2 over all "
                                     "%d tokens, %d shared neurons" % (w.T, w.shared)}

    # the host pipeline runs moe_forward (no shared block): no end-to-end figure for
    # a residual layer
    e2e = None if (args.no_e2e or res) else e2e_pipeline(args, w, p, moe, x, Wg, Wn, eps, bias,
                                                          W13_e, W2_e, world)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not res:
        inp_cpu = {k2: (v.cpu() if isinstance(v, torch.Tensor) else v) for k2, v in inp.items()}
        cpu = time_oracle(w, inp_cpu, C)
        del inp_cpu
        cpu["cpu_model"] = cpu_model()
        cpu["single_thread"] = time_oracle_single_thread()

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if dt == torch.bfloat16 else "f32", "data": "synthetic",
        "config": dict(config_of(w, C), parallelism="dp%d replicas" % world, kept_rows=R),
        "tflops": tflops, "tflops_frac_of_peak": tflops / peak_t,
        "tflops_frac_of_sustained": tflops / peak_s,
        "roofline": roofline, "kernels": kernels, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": launches, "clocks": clocks,
    }
    return line


if __name__ == "__main__":
    sys.exit(main())
