"""Seeded synthetic inputs for the zero-computation-expert MoE layer.

This module only draws tensors: token activations x, the router weight Wr, the routing bias b
and the SwiGLU expert weights W13 / W2, from one seeded ``torch.Generator`` in the fixed order
x, Wr, b, W13, W2. It holds no step of the layer's arithmetic, and it is the one module that
both the CUDA path's callers and the oracle's callers use. Nothing here loads the CUDA library.

Shapes and distributions follow the LongCat-Flash llm-wiki entity page (section 1 core-parameter
table: hidden 6144, FFN-expert width 2048, 512 FFN experts, 256 zero-computation experts,
12 experts per token including zero experts) for the three full-size workloads, plus two small
workloads for exhaustive checks. There is no dataset: every value is synthetic.
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int          # tokens per batch
    d: int          # hidden size
    N: int          # FFN experts
    Z: int          # zero-computation (identity) experts
    K: int          # experts picked per token, zero experts included
    K_e: int        # target number of FFN experts per token (bias controller)
    I: int          # FFN-expert intermediate width
    seed: int
    expert_std: float | None = None   # None: 1/sqrt(d)
    bias: str = "zero"                # "zero" | "uniform" (U(-0.1, 0.1))
    router: str = "uniform"           # "uniform" | "zipf"
    mu: float = 1e-3                  # bias adaptation rate
    steps: int = 1                    # batches (the bias-control loop draws a fresh x per step)

    @property
    def E(self) -> int:
        return self.N + self.Z

    def weight_bytes(self) -> int:
        return self.N * 3 * self.d * self.I * 2


WORKLOADS = {
    # tiny layer: frequent logit ties exercise the tie-break
    "tiny": Workload("tiny", T=64, d=128, N=8, Z=4, K=3, K_e=2, I=64, seed=0, expert_std=0.02),
    "small": Workload("small", T=4096, d=1024, N=64, Z=32, K=6, K_e=4, I=256, seed=1,
                      bias="uniform"),
    # LongCat-Flash shape, decode batch
    "decode": Workload("decode", T=128, d=6144, N=512, Z=256, K=12, K_e=8, I=2048, seed=2),
    # LongCat-Flash shape, prefill with Zipf(1.1) expert popularity
    "prefill": Workload("prefill", T=16384, d=6144, N=512, Z=256, K=12, K_e=8, I=2048, seed=3,
                        router="zipf"),
    # the prefill recipe with 32 FFN + 16 zero experts and 4096 tokens (~3.5 GB on the device):
    # same d, I, K and kernel tiles, small enough for profiler captures
    "prefill_ncu": Workload("prefill_ncu", T=4096, d=6144, N=32, Z=16, K=12, K_e=8, I=2048, seed=3,
                            router="zipf"),
    # LongCat-Flash router shape (E = 768) with 64-wide experts (~4 GB on the device): profiler
    # captures of the router GEMM, the top-K and the grouping at full routing width
    "route_ncu": Workload("route_ncu", T=8192, d=6144, N=512, Z=256, K=12, K_e=8, I=64, seed=3,
                          router="zipf"),
    # LongCat-Flash router shape at decode batch size (T = 128) with 64-wide experts (~0.8 GB on
    # the device): profiler captures of the small-batch routing and one-launch grouping
    "decode_ncu": Workload("decode_ncu", T=128, d=6144, N=512, Z=256, K=12, K_e=8, I=64, seed=2),
    # LongCat-Flash expert shape with 64 FFN + 32 zero experts and 512 tokens (~64 rows per FFN
    # expert, so every expert is cold: weight tiles only; ~4.9 GB on the device): profiler captures
    # of the expert GEMMs as weight streams
    "cold_ncu": Workload("cold_ncu", T=512, d=6144, N=64, Z=32, K=12, K_e=8, I=2048, seed=2),
    # bias-control loop: 200 fresh batches of 8192 tokens, routing only
    "bias_loop": Workload("bias_loop", T=8192, d=6144, N=512, Z=256, K=12, K_e=8, I=2048,
                          seed=4, steps=200),
}


def scaled(w: Workload, **changes) -> Workload:
    """A copy of a workload with some fields replaced (smaller cases of the same recipe)."""
    return dataclasses.replace(w, **changes)


def generator(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(seed)
    return g


def to_grid(x: torch.Tensor) -> torch.Tensor:
    """Quantise activations to k * 2^-4 with |k| <= 128 (exact in bf16). With router weights
    j * 2^-6, |j| <= 4, every product is a multiple of 2^-10 and every partial sum of a
    length-6144 dot product stays below 2^12, so any summation order is exact in fp32."""
    return (torch.clamp(torch.round(x.float() * 16.0), -128, 128) / 16.0).to(torch.bfloat16)


def draw_x(w: Workload, g: torch.Generator, device, grid: bool = False) -> torch.Tensor:
    x = torch.randn(w.T, w.d, generator=g, device=device, dtype=torch.float32)
    if w.router == "zipf":
        x[:, 0] = 1.0
    x = to_grid(x) if grid else x.to(torch.bfloat16)
    return x


def _zipf_column(w: Workload, g: torch.Generator, device) -> torch.Tensor:
    """Router column 0 = ln p_{pi(e)} rounded to 2^-4, with p_r proportional to r^-1.1 over the
    E experts and pi a seeded permutation: with x[:, 0] = 1 it gives Zipf(1.1) popularity."""
    r = torch.arange(1, w.E + 1, dtype=torch.float64)
    p = r.pow(-1.1)
    p = p / p.sum()
    perm = torch.randperm(w.E, generator=g, device=device).cpu()
    col = torch.log(p)[perm]
    return (torch.round(col * 16.0) / 16.0).to(torch.float32)


def draw_router(w: Workload, g: torch.Generator, device) -> torch.Tensor:
    wr = torch.randint(-4, 5, (w.E, w.d), generator=g, device=device, dtype=torch.int32)
    wr = wr.to(torch.float32) * (2.0 ** -6)
    if w.router == "zipf":
        wr[:, 0] = _zipf_column(w, g, device).to(device)
    return wr.to(torch.bfloat16)


def draw_bias(w: Workload, g: torch.Generator, device) -> torch.Tensor:
    if w.bias == "uniform":
        return (torch.rand(w.E, generator=g, device=device, dtype=torch.float32) * 0.2 - 0.1)
    return torch.zeros(w.E, device=device, dtype=torch.float32)


def draw_experts(w: Workload, g: torch.Generator, device):
    std = w.expert_std if w.expert_std is not None else 1.0 / math.sqrt(w.d)
    w13 = torch.empty(w.N, 2 * w.I, w.d, device=device, dtype=torch.bfloat16)
    w2 = torch.empty(w.N, w.d, w.I, device=device, dtype=torch.bfloat16)
    # one expert at a time keeps the fp32 staging small at the 38.6 GB full size
    for e in range(w.N):
        w13[e].copy_(torch.randn(2 * w.I, w.d, generator=g, device=device) * std)
    for e in range(w.N):
        w2[e].copy_(torch.randn(w.d, w.I, generator=g, device=device) * std)
    return w13, w2


def make(w: Workload, device="cpu", grid: bool = False, experts: bool = True) -> dict:
    """Draw one batch of a workload: dict(x, wr, bias[, w13, w2]) on ``device``."""
    g = generator(w.seed, device)
    out = dict(x=draw_x(w, g, device, grid=grid))
    out["wr"] = draw_router(w, g, device)
    out["bias"] = draw_bias(w, g, device)
    if experts:
        out["w13"], out["w2"] = draw_experts(w, g, device)
    out["generator"] = g
    return out


def bits(t: torch.Tensor):
    """A bf16 tensor's raw bits as a numpy uint16 array (host copy)."""
    assert t.dtype == torch.bfloat16
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view("uint16")


def from_bits(a, device="cpu") -> torch.Tensor:
    """numpy uint16 bf16 bits -> bf16 tensor."""
    import numpy as np
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)
