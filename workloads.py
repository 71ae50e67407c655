"""Seeded synthetic inputs for the MoE-layer forward, shared by the CUDA-path
tests, the benchmark and the oracle checks.

This module only draws random numbers and holds the workload shapes; it
contains none of the layer's arithmetic.  Floating-point tensors are drawn in
fp32 from a seeded ``torch.Generator`` and, for bf16 workloads, rounded to bf16
(round-to-nearest-even, torch's conversion).  Draw order is fixed:
x, W1, W3, W2, W_g, W_noise, eps, bias, perm, perturbation.

Workloads (shapes of the models on the pages; data is synthetic):
  tiny_fp32       T=512,  d=512,  d_ff=1376  -> 8 disjoint experts of 172, top-2 Mixtral, fp32
  moe_2of8        T=16384, d=4096, d_ff=11008 -> 8 x 1376, noisy top-2 Mixtral, rescale E/k, bf16
  moe_4of16       T=16384, d=4096, d_ff=11008 -> 16 x 688, noisy top-4 ST, bias N(0,1), lambda 0.01
  e8t2_cf1/_cf4   T=32768, d=4096, 8 copies of d_ff=14336 (+ N(0,1e-3) per expert), top-2
                  Mixtral, capacity factor 1 or 4 with overflow dropping
  decode_t{1,8,64} T in {1,8,64}, d=4096, 8 x 1376, top-2, no noise, rescale E/k
  moe_res_2of8    residual MoE: T=16384, d=4096, d_ff=11008 -> 1376 shared neurons +
                  8 x 1204 experts, noisy top-2 Mixtral, rescale E/k
With ``shared`` > 0 (residual MoE) the seeded permutation also chooses the shared
neurons: perm[:shared] is the shared set, perm[shared:] the experts' neurons in order.
"""
from dataclasses import dataclass, replace
from typing import Optional

import torch

MIXTRAL = 0
ST = 1
DISJOINT = 0
COPY = 1
STACKED = 2


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    d_ff: int
    E: int
    k: int
    dtype: str = "bf16"          # "bf16" or "f32"
    router: int = MIXTRAL
    noisy: bool = False
    bias: bool = False
    rescale: bool = False
    cf: float = -1.0             # < 0: no capacity limit
    lam: float = 0.01
    partition: int = DISJOINT    # DISJOINT, or COPY (upcycling)
    perturb: float = 0.0         # std of the per-expert perturbation of copies
    seed: int = 1000
    shared: int = 0              # > 0: residual MoE with this many shared neurons

    @property
    def m(self) -> int:
        if self.partition != DISJOINT:
            return self.d_ff
        return (self.d_ff - self.shared) // self.E

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", T=512, d=512, d_ff=1376, E=8, k=2, dtype="f32",
                          seed=1000),
    "moe_2of8": Workload("moe_2of8", T=16384, d=4096, d_ff=11008, E=8, k=2, noisy=True,
                         rescale=True, seed=1001),
    "moe_4of16": Workload("moe_4of16", T=16384, d=4096, d_ff=11008, E=16, k=4, router=ST,
                          noisy=True, bias=True, rescale=True, lam=0.01, seed=1002),
    "e8t2_cf1": Workload("e8t2_cf1", T=32768, d=4096, d_ff=14336, E=8, k=2, cf=1.0,
                         partition=COPY, perturb=1e-3, seed=1003),
    "e8t2_cf4": Workload("e8t2_cf4", T=32768, d=4096, d_ff=14336, E=8, k=2, cf=4.0,
                         partition=COPY, perturb=1e-3, seed=1003),
    "decode_t1": Workload("decode_t1", T=1, d=4096, d_ff=11008, E=8, k=2, rescale=True,
                          seed=1004),
    "decode_t8": Workload("decode_t8", T=8, d=4096, d_ff=11008, E=8, k=2, rescale=True,
                          seed=1004),
    "decode_t64": Workload("decode_t64", T=64, d=4096, d_ff=11008, E=8, k=2, rescale=True,
                           seed=1004),
    "moe_res_2of8": Workload("moe_res_2of8", T=16384, d=4096, d_ff=11008, E=8, k=2, noisy=True,
                             rescale=True, shared=1376, seed=1005),
}


def torch_dtype(w: Workload):
    return torch.bfloat16 if w.dtype == "bf16" else torch.float32


def make_inputs(w: Workload, device: str = "cpu", seed: Optional[int] = None):
    """Draws every input of workload ``w``.

    Returns a dict of tensors on ``device``:
      x [T,d]; W1, W3 [d_ff,d]; W2 [d,d_ff]; Wg, Wnoise [d,E] (Wnoise None unless noisy);
      eps [T,E] f32 (None unless noisy); bias [E] f32 (None unless biased);
      perm [d_ff] int32 (disjoint partition only);
      W1s, W3s [E,d_ff,d], W2s [E,d,d_ff] (perturbed copies only).
    """
    g = torch.Generator(device=device)
    g.manual_seed(w.seed if seed is None else seed)
    dt = torch_dtype(w)

    def randn(*shape, std=1.0):
        t = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
        if std != 1.0:
            t.mul_(std)
        return t

    out = {}
    out["x"] = randn(w.T, w.d).to(dt)
    W1 = randn(w.d_ff, w.d, std=0.02)
    W3 = randn(w.d_ff, w.d, std=0.02)
    W2 = randn(w.d, w.d_ff, std=0.02)
    out["Wg"] = randn(w.d, w.E, std=0.02).to(dt)
    out["Wnoise"] = randn(w.d, w.E, std=0.02).to(dt) if w.noisy else None
    out["eps"] = randn(w.T, w.E) if w.noisy else None
    out["bias"] = randn(w.E) if w.bias else None
    if w.partition == DISJOINT:
        out["perm"] = torch.randperm(w.d_ff, generator=g, device=device).to(torch.int32)
        if w.shared > 0:  # residual MoE: the permutation's head is the shared set
            out["shared_idx"] = out["perm"][:w.shared].contiguous()
            out["perm_rest"] = out["perm"][w.shared:].contiguous()
    else:
        out["perm"] = None
    if w.partition == COPY and w.perturb > 0:
        W1s = torch.empty(w.E, w.d_ff, w.d, dtype=dt, device=device)
        W3s = torch.empty(w.E, w.d_ff, w.d, dtype=dt, device=device)
        W2s = torch.empty(w.E, w.d, w.d_ff, dtype=dt, device=device)
        for e in range(w.E):
            W1s[e] = (W1 + randn(w.d_ff, w.d, std=w.perturb)).to(dt)
            W3s[e] = (W3 + randn(w.d_ff, w.d, std=w.perturb)).to(dt)
            W2s[e] = (W2 + randn(w.d, w.d_ff, std=w.perturb)).to(dt)
        out["W1s"], out["W3s"], out["W2s"] = W1s, W3s, W2s
    out["W1"], out["W3"], out["W2"] = W1.to(dt), W3.to(dt), W2.to(dt)
    return out


def to_numpy_raw(t: torch.Tensor):
    """CPU numpy view of a tensor for the oracle: float32 as is, bf16 as raw uint16 bits."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view("uint16")
    if t.dtype == torch.float32:
        return t.numpy()
    if t.dtype in (torch.int32, torch.int64):
        return t.numpy()
    raise TypeError(t.dtype)


def make_cluster_init(d_ff: int, E: int, seed: int) -> torch.Tensor:
    """E distinct neuron indices drawn uniformly (the initial k-means centers of the
    clustering partition), int32 on the CPU."""
    g = torch.Generator()
    g.manual_seed(seed)
    return torch.randperm(d_ff, generator=g)[:E].to(torch.int32).contiguous()


def make_grad_output(w: Workload, seed: int, device: str = "cpu") -> torch.Tensor:
    """dl/dy for the backward pass: N(0, 1) entries [T][d] in the workload's dtype."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return torch.randn(w.T, w.d, generator=g, device=device).to(torch_dtype(w))
