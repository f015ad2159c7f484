"""Seeded synthetic inputs for MoE token dispatch / combine.

This module only draws inputs: router choices, route weights, token rows and
stand-in expert outputs. It holds none of the dispatch / combine arithmetic,
and both the CUDA library's tests and the CPU oracle consume exactly the
arrays it returns.

Shapes follow the workloads the pages describe:
  * "Экспертный параллелизм (EP)" glossary, section "Что подтверждено":
    num_experts=8 with ep_size=4 gives two local experts per rank (tiny case).
  * "DeepSeek开源周第二天：DeepEP深度分析", section "性能": 4096 tokens per batch,
    hidden 7168, top-4 groups, top-8 experts, FP8 dispatch, BF16 combine
    (prefill); 128 tokens per batch with top-8 for the low-latency case (decode).
  * "MoonEP核心功能深度剖析", section "快速上手" (Buffer(S=4096, H=7168, K=8,
    E=256, num_ep_ranks=8, token_padding=128)) and section "1. 完美负载平衡"
    (skewed routing, each rank receives S*K rows).

Router details the pages leave open (softmax, group score = max in group,
ties to the lower index, Zipf popularity over a seeded permutation, Dirichlet(1)
weights) are generator choices only: they shape the inputs, never the result
of the method on those inputs.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    R: int              # logical EP ranks
    S: int              # tokens per rank
    H: int              # hidden size
    E: int              # routed experts
    K: int              # experts per token
    pad: int = 1        # token_padding per expert group
    fp8: bool = False   # FP8 e4m3 dispatch with 1x128 scales
    routing: str = "softmax"   # softmax | group_limited | zipf
    zipf_s: float = 0.0
    n_groups: int = 8
    topk_groups: int = 4
    B: int = 0          # redundant-expert slots per rank (balanced plan)
    I: int = 0          # expert FFN intermediate size (balanced plan)
    seed: int = 0

    @property
    def N(self) -> int:
        return self.R * self.S

    @property
    def describe(self) -> str:
        s = (f"{self.name}: R={self.R} S={self.S} N={self.N} H={self.H} "
             f"E={self.E} K={self.K} pad={self.pad} "
             f"{'fp8-e4m3 1x128' if self.fp8 else 'bf16'} dispatch, "
             f"routing={self.routing}")
        if self.routing == "zipf":
            s += f"(s={self.zipf_s})"
        if self.B:
            s += f" B={self.B} I={self.I}"
        return s


WORKLOADS = {
    "tiny": Workload("tiny", R=4, S=64, H=256, E=8, K=2, routing="softmax",
                     seed=0),
    "prefill": Workload("prefill", R=8, S=4096, H=7168, E=256, K=8, fp8=True,
                        routing="group_limited", seed=1),
    "decode": Workload("decode", R=8, S=128, H=7168, E=256, K=8, fp8=True,
                       routing="group_limited", seed=2),
    "skewed": Workload("skewed", R=8, S=4096, H=7168, E=256, K=8, pad=128,
                       routing="zipf", zipf_s=1.2, seed=3),
    "balanced": Workload("balanced", R=8, S=4096, H=7168, E=256, K=8,
                         routing="zipf", zipf_s=1.5, B=4, I=2048, seed=4),
}


def scaled(w: Workload, S: Optional[int] = None, H: Optional[int] = None,
           **kw) -> Workload:
    """The same workload with fewer tokens per rank or a narrower row."""
    d = dataclasses.asdict(w)
    if S is not None:
        d["S"] = S
    if H is not None:
        d["H"] = H
    d.update(kw)
    return Workload(**d)


# --------------------------------------------------------------------------
# token rows and expert outputs (bf16 bit patterns)
# --------------------------------------------------------------------------

def bf16_normal(shape, seed: int, device="cpu") -> torch.Tensor:
    """N(0,1) samples rounded to bf16 (torch's own round-to-nearest cast).

    Large tensors are drawn in chunks so the fp32 temporaries stay small.
    """
    dev = torch.device(device)
    g = torch.Generator(device=dev).manual_seed(int(seed))
    out = torch.empty(shape, dtype=torch.bfloat16, device=dev)
    flat = out.view(-1)
    chunk = 1 << 26
    for i in range(0, flat.numel(), chunk):
        n = min(chunk, flat.numel() - i)
        flat[i:i + n] = torch.randn(n, generator=g, device=dev,
                                    dtype=torch.float32).to(torch.bfloat16)
    return out


def hidden_states(w: Workload, device="cpu") -> torch.Tensor:
    """hidden [N, H] bf16, N(0,1)."""
    return bf16_normal((w.N, w.H), seed=1000 + w.seed, device=device)


def expert_outputs(rows: int, H: int, seed: int, device="cpu") -> torch.Tensor:
    """Stand-in expert outputs y [rows, H] bf16, N(0,1)."""
    return bf16_normal((rows, H), seed=2000 + seed, device=device)


# --------------------------------------------------------------------------
# routing
# --------------------------------------------------------------------------

def _desc_stable_order(scores: np.ndarray) -> np.ndarray:
    """Per-row indices sorted by descending score, ties to the lower index."""
    return np.argsort(-scores, axis=1, kind="stable")


def _softmax(x: np.ndarray) -> np.ndarray:
    x = x.astype(np.float64)
    m = x.max(axis=1, keepdims=True)
    p = np.exp(x - m)
    return p / p.sum(axis=1, keepdims=True)


def route_softmax_topk(rng: np.random.Generator, N: int, E: int, K: int):
    """logits ~ N(0,1); softmax; top-K; weights renormalised to sum to 1."""
    logits = rng.standard_normal((N, E), dtype=np.float32)
    p = _softmax(logits)
    idx = _desc_stable_order(p)[:, :K]
    wk = np.take_along_axis(p, idx, axis=1)
    wk = wk / wk.sum(axis=1, keepdims=True)
    return idx.astype(np.int32), wk.astype(np.float32)


def route_group_limited(rng: np.random.Generator, N: int, E: int, K: int,
                        n_groups: int, topk_groups: int):
    """Group-limited gating: pick the top groups by their best expert score,
    then the top-K experts inside the picked groups; renormalised weights."""
    assert E % n_groups == 0
    logits = rng.standard_normal((N, E), dtype=np.float32)
    p = _softmax(logits)
    gsz = E // n_groups
    gscore = p.reshape(N, n_groups, gsz).max(axis=2)
    gsel = _desc_stable_order(gscore)[:, :topk_groups]
    gmask = np.zeros((N, n_groups), dtype=bool)
    np.put_along_axis(gmask, gsel, True, axis=1)
    emask = np.repeat(gmask, gsz, axis=1)
    masked = np.where(emask, p, -1.0)
    idx = _desc_stable_order(masked)[:, :K]
    wk = np.take_along_axis(p, idx, axis=1)
    wk = wk / wk.sum(axis=1, keepdims=True)
    return idx.astype(np.int32), wk.astype(np.float32)


def route_zipf(rng: np.random.Generator, N: int, E: int, K: int, s: float):
    """Zipf(s) popularity over a seeded permutation of experts; K distinct
    experts per token drawn without replacement (Gumbel top-K); route weights
    Dirichlet(1), i.e. normalised Exp(1) draws."""
    perm = rng.permutation(E)
    pop = np.empty(E, dtype=np.float64)
    pop[perm] = (np.arange(E, dtype=np.float64) + 1.0) ** (-s)
    pop /= pop.sum()
    keys = np.log(pop)[None, :] + rng.gumbel(size=(N, E))
    idx = _desc_stable_order(keys)[:, :K]
    g = rng.exponential(size=(N, K))
    wk = g / g.sum(axis=1, keepdims=True)
    return idx.astype(np.int32), wk.astype(np.float32)


def routing(w: Workload):
    """topk_experts [N, K] int32 and route_weights [N, K] fp32 (numpy)."""
    rng = np.random.default_rng(w.seed)
    if w.routing == "softmax":
        return route_softmax_topk(rng, w.N, w.E, w.K)
    if w.routing == "group_limited":
        return route_group_limited(rng, w.N, w.E, w.K, w.n_groups,
                                   w.topk_groups)
    if w.routing == "zipf":
        return route_zipf(rng, w.N, w.E, w.K, w.zipf_s)
    raise ValueError(w.routing)


def random_topk(rng: np.random.Generator, N: int, K: int, E: int,
                distinct: bool = False):
    """Uniform expert ids (duplicates within a token allowed unless
    `distinct`) and positive weights; used for small randomized cases."""
    if distinct:
        idx = np.argsort(rng.random((N, E)), axis=1)[:, :K]
    else:
        idx = rng.integers(0, E, size=(N, K))
    wk = rng.random((N, K)).astype(np.float32) + np.float32(0.05)
    return idx.astype(np.int32), wk.astype(np.float32)


def weight_buffer(E_rows: int, H: int, I: int, seed: int, device="cpu"):
    """Expert projection weights [E_rows, H, I] bf16 ~ N(0,1) * 0.02."""
    dev = torch.device(device)
    g = torch.Generator(device=dev).manual_seed(3000 + int(seed))
    out = torch.empty((E_rows, H, I), dtype=torch.bfloat16, device=dev)
    flat = out.view(-1)
    chunk = 1 << 26
    for i in range(0, flat.numel(), chunk):
        n = min(chunk, flat.numel() - i)
        flat[i:i + n] = (torch.randn(n, generator=g, device=dev,
                                     dtype=torch.float32) * 0.02
                         ).to(torch.bfloat16)
    return out
