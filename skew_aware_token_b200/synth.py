"""Seeded synthetic inputs for the skew-aware MoE forward layer.

This module draws the inputs of one MoE layer (router logits, token activations, expert
weights) with the shapes and value distributions of the workloads below, and nothing
else: it holds none of the layer's arithmetic (no top-k, no histogram, no planning, no
FFN). Both the CUDA path and the CPU oracle consume what it produces.

Recipe (every draw is seeded; one generator per tensor, and one per expert for weights):
  * router logits  ~ N(0, 1) in fp32, plus a Zipf popularity bias alpha*log(1/(e+1))
    (popularity rank = expert id + 1, so the hot experts are the low ids);
  * hot-expert concentration (skew sweep): a Bernoulli(p) mask over tokens; a masked
    token gets the logit max_e(logits[t]) + 1 on one of the four fixed hot experts
    {0,1,2,3} ("one" mode, expert drawn uniformly) or on all four ("all4" mode);
  * x ~ N(0, 1) rounded to bf16 (round-to-nearest-even);
  * W1_e ~ N(0, 1/sqrt(d)) with shape [2f, d] (rows 0..f-1 gate G, f..2f-1 up U),
    W2_e ~ N(0, 1/sqrt(f)) with shape [d, f], both rounded to bf16 (std = 1/sqrt(fan_in)).

Logits and x are drawn on the host with torch's CPU generator; expert weights are drawn
on the device they will live on (CPU or CUDA), one seeded generator per expert, so any
single expert can be regenerated on its own.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch

# Tensor ids that key the per-tensor seed streams.
TID_LOGITS, TID_X, TID_W1, TID_W2, TID_HOT = 1, 2, 3, 4, 5
TID_DY = 6  # upstream gradient dL/dy of the backward pass
HOT_EXPERTS = (0, 1, 2, 3)


@dataclasses.dataclass(frozen=True)
class Workload:
    """One MoE layer configuration plus the recipe of its router logits."""

    name: str
    T: int          # tokens
    d: int          # model width
    E: int          # experts
    k: int          # experts per token
    f: int          # expert FFN width (SwiGLU: FC1 has 2f outputs)
    beta: int       # rows per token block
    P: int          # virtual execution slots
    s: int          # per-slot replica budget
    alpha: float = 0.0       # Zipf logit bias
    hot_p: float = 0.0       # fraction of tokens forced onto the hot experts
    hot_mode: str = "none"   # "none" | "one" | "all4"
    seed: int = 0

    @property
    def N(self) -> int:
        """Routed rows T*k."""
        return self.T * self.k

    @property
    def flops(self) -> int:
        """Algorithmic FFN flops 6*T*k*d*f (FC1 4*N*d*f, FC2 2*N*d*f; padding rows excluded)."""
        return 6 * self.T * self.k * self.d * self.f

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def _sweep(mode: str, p: float, beta: int, alpha: float = 0.0) -> Workload:
    tag = f"sweep_{mode}_p{p:g}_b{beta}" + (f"_zipf{alpha:g}" if alpha else "")
    return Workload(tag, T=16384, d=2048, E=128, k=8, f=768, beta=beta, P=8, s=2,
                    alpha=alpha, hot_p=p, hot_mode=mode)


def _build_workloads() -> dict[str, Workload]:
    w: list[Workload] = [
        Workload("tiny", T=256, d=512, E=8, k=2, f=1024, beta=64, P=4, s=1),
    ]
    for a in (0.0, 0.5, 1.0):
        w.append(Workload(f"olmoe_a{a:g}", T=4096, d=2048, E=64, k=8, f=1024, beta=128,
                          P=8, s=2, alpha=a))
    for a in (0.0, 0.5, 1.0, 1.5):
        w.append(Workload(f"qwen3_a{a:g}", T=8192, d=2048, E=128, k=8, f=768, beta=128,
                          P=8, s=2, alpha=a))
    for beta in (128, 64):
        for mode in ("one", "all4"):
            for p in (0.0, 0.1, 0.3, 0.5):
                w.append(_sweep(mode, p, beta))
        w.append(_sweep("all4", 1.0, beta))
        w.append(_sweep("all4", 1.0, beta, alpha=1.5))
    w.append(Workload("dsv3_a1", T=16384, d=7168, E=256, k=8, f=2048, beta=128, P=8, s=4,
                      alpha=1.0))
    # the DeepSeek-V3-shaped layer with 32 experts (2.8 GB of weights): small enough for
    # profilers that replay a kernel many times; at T = 2048 an expert averages 512 rows,
    # as in the full layer
    for T in (2048, 8192):
        w.append(Workload(f"dsv3_e32_t{T}", T=T, d=7168, E=32, k=8, f=2048, beta=128, P=8,
                          s=4, alpha=1.0))
    return {x.name: x for x in w}


WORKLOADS = _build_workloads()


def seed_for(seed: int, tid: int, e: int = 0) -> int:
    """64-bit seed of one tensor (or one expert of a tensor), from numpy's SeedSequence."""
    state = np.random.SeedSequence([seed, tid, e]).generate_state(2, dtype=np.uint32)
    return (int(state[0]) << 31) ^ int(state[1])


def _gen(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def make_logits(wl: Workload) -> torch.Tensor:
    """Router logits fp32 [T, E] on the host."""
    L = torch.randn(wl.T, wl.E, generator=_gen(seed_for(wl.seed, TID_LOGITS)),
                    dtype=torch.float32)
    if wl.alpha:
        bias = torch.tensor([wl.alpha * math.log(1.0 / (e + 1)) for e in range(wl.E)],
                            dtype=torch.float64).to(torch.float32)
        L += bias[None, :]
    if wl.hot_mode != "none" and wl.hot_p > 0:
        g = _gen(seed_for(wl.seed, TID_HOT))
        mask = torch.rand(wl.T, generator=g, dtype=torch.float64) < wl.hot_p
        which = torch.randint(0, len(HOT_EXPERTS), (wl.T,), generator=g)
        top = L.max(dim=1).values + 1.0
        rows = torch.nonzero(mask).flatten()
        if wl.hot_mode == "one":
            L[rows, which[rows]] = top[rows]
        elif wl.hot_mode == "all4":
            for e in HOT_EXPERTS:
                L[rows, e] = top[rows]
        else:
            raise ValueError(f"unknown hot_mode {wl.hot_mode!r}")
    return L


def make_x(wl: Workload) -> torch.Tensor:
    """Token activations bf16 [T, d] on the host."""
    return torch.randn(wl.T, wl.d, generator=_gen(seed_for(wl.seed, TID_X)),
                       dtype=torch.float32).to(torch.bfloat16)


def make_dy(wl: Workload) -> torch.Tensor:
    """Upstream gradient dL/dy fp32 [T, d] on the host, N(0, 1)."""
    return torch.randn(wl.T, wl.d, generator=_gen(seed_for(wl.seed, TID_DY)),
                       dtype=torch.float32)


def expert_weights(wl: Workload, e: int, device="cpu") -> tuple[torch.Tensor, torch.Tensor]:
    """(W1_e bf16 [2f, d], W2_e bf16 [d, f]) of expert e, drawn on `device`."""
    w1 = torch.randn(2 * wl.f, wl.d, generator=_gen(seed_for(wl.seed, TID_W1, e), device),
                     device=device, dtype=torch.float32)
    w1.mul_(1.0 / math.sqrt(wl.d))
    w2 = torch.randn(wl.d, wl.f, generator=_gen(seed_for(wl.seed, TID_W2, e), device),
                     device=device, dtype=torch.float32)
    w2.mul_(1.0 / math.sqrt(wl.f))
    return w1.to(torch.bfloat16), w2.to(torch.bfloat16)


def make_weights(wl: Workload, device="cpu") -> tuple[torch.Tensor, torch.Tensor]:
    """All expert weights: W1 bf16 [E, 2f, d] and W2 bf16 [E, d, f] on `device`."""
    W1 = torch.empty(wl.E, 2 * wl.f, wl.d, dtype=torch.bfloat16, device=device)
    W2 = torch.empty(wl.E, wl.d, wl.f, dtype=torch.bfloat16, device=device)
    for e in range(wl.E):
        W1[e], W2[e] = expert_weights(wl, e, device)
    return W1, W2
