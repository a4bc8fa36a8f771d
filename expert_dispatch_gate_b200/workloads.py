"""Seeded synthetic inputs for the MoE layer workloads.

This module only draws random numbers and names shapes; it holds none of the layer's
arithmetic. The same tensors feed the CUDA library and the CPU oracle.

Recipe (per tensor): a ``torch.Generator`` on the target device seeded with
``20261202 + 100 * workload_index + tensor_id``; ``torch.randn`` in float32 scaled by the
standard deviation, then rounded to bfloat16 (round-to-nearest-even) for the bf16 workloads.

* x ~ N(0, 1)                         [T, H]       tensor_id 0
* w_router ~ N(0, 1/H)                [H, E]       tensor_id 1
* w_gate, w_up ~ N(0, 1/H)            [E, H, I]    tensor_id 2, 3
* w_down ~ N(0, 1/I)                  [E, I, H]    tensor_id 4
* skewed workload only: logit_bias[e] = -s * ln(e + 1), s = 1.2 (float32, [E]): an additive
  gate-logit bias that makes expert popularity fall off as a power of the expert's rank.
* combine-alone input: y_slots ~ N(0, 1) [T*k, H]   tensor_id 5

CPU and CUDA generators produce different streams for the same seed, so a workload drawn on
the GPU is copied to the host before the oracle sees it.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch

SEED_BASE = 20261202


@dataclass(frozen=True)
class Workload:
    name: str
    index: int
    T: int
    H: int
    E: int
    k: int
    I: int
    dtype: str            # "f32" or "bf16": activations, weights and output
    capacity_factor: float  # <= 0: no capacity limit
    zipf_s: float = 0.0   # > 0: add the power-law gate-logit bias

    def with_tokens(self, T: int) -> "Workload":
        return replace(self, T=int(T))

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def describe(self) -> str:
        cf = "no capacity limit" if self.capacity_factor <= 0 else f"cf={self.capacity_factor}"
        z = f", Zipf-bias s={self.zipf_s}" if self.zipf_s > 0 else ""
        return (f"{self.name}: T={self.T} H={self.H} E={self.E} k={self.k} I={self.I} "
                f"{self.dtype} {cf}{z}")


# The five workloads: tiny fp32, Mixtral-8x7B-shaped, fine-grained E=256, decode-shaped
# (T swept over 1/16/64/256), and the skewed-load stress case.
WORKLOADS = {
    "tiny": Workload("tiny", 0, 64, 128, 8, 2, 256, "f32", 0.0),
    "mixtral": Workload("mixtral", 1, 4096, 4096, 8, 2, 14336, "bf16", 1.25),
    "fine": Workload("fine", 2, 4096, 4096, 256, 8, 2048, "bf16", 1.25),
    "decode": Workload("decode", 3, 16, 4096, 256, 8, 2048, "bf16", 0.0),
    "skewed": Workload("skewed", 4, 32768, 2048, 64, 6, 1408, "bf16", 1.25, zipf_s=1.2),
}
DECODE_TOKENS = (1, 16, 64, 256)

# Profiling stand-in for the fine-grained layer: same per-expert shapes and load (C = 160,
# about 128 tokens per expert) with 32 experts, so a profiler capture holds 1.6 GB of weights
# (still far larger than L2) instead of 12.9 GB.
PROFILE_WORKLOADS = {
    "fine_e32": Workload("fine_e32", 5, 512, 4096, 32, 8, 2048, "bf16", 1.25),
    # the fine-grained router (T, H, E, k identical) with a small expert FFN
    "route_fine": Workload("route_fine", 6, 4096, 4096, 256, 8, 128, "bf16", 1.25),
}


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _randn(shape, std, seed, device, dtype, chunk_dim0=False):
    g = _gen(device, seed)
    if not chunk_dim0:
        t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        if std != 1.0:
            t.mul_(std)
        return t.to(dtype)
    # Draw expert by expert (same generator, sequential) to bound the float32 temporary.
    out = torch.empty(shape, device=device, dtype=dtype)
    for e in range(shape[0]):
        t = torch.randn(shape[1:], generator=g, device=device, dtype=torch.float32)
        if std != 1.0:
            t.mul_(std)
        out[e].copy_(t.to(dtype))
    return out


def logit_bias(wl: Workload):
    if wl.zipf_s <= 0:
        return None
    return torch.tensor([-wl.zipf_s * math.log(e + 1) for e in range(wl.E)], dtype=torch.float32)


def make_inputs(wl: Workload, device="cpu", weights=True):
    """Draw the workload's tensors on ``device``. Returns a dict of tensors."""
    seed = SEED_BASE + 100 * wl.index
    dt = wl.torch_dtype
    out = {
        "x": _randn((wl.T, wl.H), 1.0, seed + 0, device, dt),
        "w_router": _randn((wl.H, wl.E), 1.0 / math.sqrt(wl.H), seed + 1, device, dt),
    }
    b = logit_bias(wl)
    out["logit_bias"] = None if b is None else b.to(device)
    if weights:
        big = wl.E * wl.H * wl.I > (1 << 26)
        out["w_gate"] = _randn((wl.E, wl.H, wl.I), 1.0 / math.sqrt(wl.H), seed + 2, device, dt, big)
        out["w_up"] = _randn((wl.E, wl.H, wl.I), 1.0 / math.sqrt(wl.H), seed + 3, device, dt, big)
        out["w_down"] = _randn((wl.E, wl.I, wl.H), 1.0 / math.sqrt(wl.I), seed + 4, device, dt, big)
    return out


def make_y_slots(wl: Workload, device="cpu"):
    """Synthetic expert outputs per slot, for timing or testing the combine alone."""
    seed = SEED_BASE + 100 * wl.index
    return _randn((wl.T * wl.k, wl.H), 1.0, seed + 5, device, wl.torch_dtype)


def random_logits(T, E, seed, device="cpu", ties=False):
    """Gate logits for selection-only tests; ``ties`` quantises them so equal values are common
    and plants signed zeros."""
    g = _gen(device, seed)
    l = torch.randn((T, E), generator=g, device=device, dtype=torch.float32)
    if ties:
        l = torch.round(l * 2.0) / 2.0
        z = torch.rand((T, E), generator=g, device=device) < 0.1
        l = torch.where(z, torch.where(torch.rand((T, E), generator=g, device=device) < 0.5,
                                       torch.tensor(-0.0, device=device),
                                       torch.tensor(0.0, device=device)), l)
    return l


def random_topk_idx(T, E, k, seed, device="cpu", mode="uniform"):
    """Expert choices (distinct within a token) for align-only tests.

    mode: "uniform" (random distinct experts), "one" (every token picks experts 0..k-1, so
    expert 0 gets all T), "zipf" (distinct experts drawn with probability ~ (e+1)^-1.2).
    """
    g = _gen("cpu", seed)
    if mode == "one":
        idx = torch.arange(k, dtype=torch.int32).repeat(T, 1)
    else:
        if mode == "zipf":
            w = torch.tensor([(e + 1) ** -1.2 for e in range(E)], dtype=torch.float64)
        else:
            w = torch.ones(E, dtype=torch.float64)
        idx = torch.multinomial(w.expand(T, E), k, replacement=False, generator=g).to(torch.int32)
    return idx.to(device)
