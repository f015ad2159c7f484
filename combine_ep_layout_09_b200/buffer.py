"""EPBuffer: the call shape of the pages' Buffer API over the C ABI.

"MoonEP核心功能深度剖析", section "快速上手", builds Buffer(S, H, K, E,
num_ep_ranks, num_sms, token_padding) and calls dispatch(...),
prefetch_weight(plan, gate, up, down) and combine(plan, expert_output, ...)
on it. EPBuffer keeps that shape for one GPU with logical ranks. It allocates
every buffer once, at construction (static shapes: section "2. 高效通信机制"),
with PyTorch, and each method is one or more calls of the C library on the
current stream. Nothing is synchronised; `check()` reads the device status
word when the caller wants it.
"""
from __future__ import annotations

import torch

from . import _binding as B


class EPBuffer:
    def __init__(self, S: int, H: int, K: int, E: int, num_ep_ranks: int,
                 num_sms: int = 0, token_padding: int = 1, fp8: bool = False,
                 device=None):
        self.S, self.H, self.K, self.E = S, H, K, E
        self.R = num_ep_ranks
        self.N = self.R * S
        self.num_sms = num_sms
        self.pad = token_padding
        self.fp8 = fp8
        dev = torch.device(device if device is not None else "cuda")
        self.cap = B.ep_capacity_bound(self.N, K, E, token_padding)
        if self.cap < 0:
            raise ValueError("invalid buffer shape")
        i32 = dict(dtype=torch.int32, device=dev)
        self.tokens_per_expert = torch.zeros(E, **i32)
        self.expert_offsets = torch.zeros(E + 1, **i32)
        self.pos = torch.zeros(self.N, K, **i32)
        self.row_src = torch.zeros(max(self.cap, 1), **i32)
        ws = B.ep_layout_workspace_bytes(self.N, K, E)
        self.workspace = torch.zeros(max(ws, 16), dtype=torch.uint8, device=dev)
        self.status = torch.zeros(4, **i32)
        rows = max(self.cap, 1)
        if fp8:
            self.recv = torch.empty(rows, H, dtype=torch.float8_e4m3fn,
                                    device=dev)
            self.recv_scales = torch.empty(rows, H // 128,
                                           dtype=torch.float32, device=dev)
        else:
            self.recv = torch.empty(rows, H, dtype=torch.bfloat16, device=dev)
            self.recv_scales = None
        self.recv_weights = torch.empty(rows, dtype=torch.float32, device=dev)

    # -- dispatch ------------------------------------------------------------
    def layout(self, topk_experts: torch.Tensor, stream=None):
        B.ep_layout(topk_experts, self.R, self.S, self.K, self.E, self.pad,
                    self.tokens_per_expert, self.expert_offsets, self.pos,
                    self.row_src, self.workspace, self.status, cap=self.cap,
                    stream=stream)

    def dispatch(self, hidden: torch.Tensor, route_weights: torch.Tensor,
                 topk_experts: torch.Tensor, stream=None):
        """-> (recv, recv_scales, recv_weights, expert_offsets): rank r's
        rows are expert_offsets[r*E/R] .. expert_offsets[(r+1)*E/R]."""
        self.layout(topk_experts, stream)
        B.ep_dispatch(hidden, route_weights, self.pos, self.row_src,
                      self.expert_offsets, self.N, self.K, self.E, self.H,
                      self.fp8, self.recv, self.recv_scales,
                      self.recv_weights, self.num_sms, self.status,
                      cap=self.cap, stream=stream)
        return self.recv, self.recv_scales, self.recv_weights, \
            self.expert_offsets

    # -- balanced plan + prefetch -------------------------------------------
    def plan(self, slots_per_rank: int, stream=None) -> dict:
        """Balanced plan from the last layout's tokens_per_expert
        (token_padding must be 1)."""
        if self.pad != 1:
            raise ValueError("the balanced plan needs token_padding == 1")
        dev = self.pos.device
        R, E, Bs = self.R, self.E, slots_per_rank
        i32 = dict(dtype=torch.int32, device=dev)
        p = dict(cu=torch.empty(R, E + 1, **i32),
                 expert=torch.empty(R, E, **i32),
                 wrow=torch.empty(R, E, **i32),
                 nseg=torch.empty(R, **i32),
                 slot_expert=torch.empty(R, max(Bs, 1), **i32), B=Bs)
        B.ep_plan_balanced(self.tokens_per_expert, R, self.S, self.K, E, Bs,
                           p["cu"], p["expert"], p["wrow"], p["nseg"],
                           p["slot_expert"] if Bs > 0 else None, self.status,
                           stream=stream)
        return p

    def prefetch_weight(self, plan: dict, full_gate_weight, full_up_weight,
                        full_down_weight, stream=None):
        B.ep_prefetch_weights(plan["slot_expert"], self.R, self.E, plan["B"],
                              full_gate_weight, full_up_weight,
                              full_down_weight, self.num_sms, stream=stream)

    # -- combine -------------------------------------------------------------
    def combine(self, expert_output: torch.Tensor,
                route_weights: torch.Tensor, out: torch.Tensor | None = None,
                stream=None) -> torch.Tensor:
        if out is None:
            out = torch.empty(self.N, self.H, dtype=torch.bfloat16,
                              device=expert_output.device)
        # rows of expert_output bound the positions it may be read at
        B.ep_combine(expert_output, self.pos, route_weights, self.N, self.K,
                     self.H, out, self.num_sms, self.status,
                     cap=expert_output.shape[0], stream=stream)
        return out

    def check(self):
        """Synchronising read of the device status word; raises on error."""
        s = int(self.status[0].item())
        if s:
            raise B.EPError(s, "device status")
