"""EPBuffer: the call shape of the pages' Buffer API over the C ABI.

"MoonEP核心功能深度剖析", section "快速上手", builds Buffer(S, H, K, E,
num_ep_ranks, num_sms, token_padding) and calls

    hidden_nvsh, route_weights_nvs, cu_seqlens, plan = buffer.dispatch(
        hidden_sh, route_weights_sk, topk_experts_sk, ...)
    buffer.prefetch_weight(plan, gate, up, down)
    output_sh, gathered_route_weights_sk, _ = buffer.combine(
        plan, expert_output_nvsh, route_weights_nvs)

EPBuffer keeps that shape for one GPU with logical ranks. Every buffer is
allocated once, at construction: shapes are static (section "2. 高效通信机制"),
so no call synchronises with the host. Each method is one or more calls of
the C library on the current stream.

With double_buffer=True, two sets of receive buffers alternate between
dispatches (buffer index ^= 1, as in "DeepSeek开源周第二天：DeepEP深度分析",
section "代码解读", 双缓冲区). A dispatch's outputs then stay valid while the
next dispatch fills the other set, so one layer's expert work can overlap
the next layer's dispatch.
"""
from __future__ import annotations

import dataclasses

import torch

from . import _binding as B


@dataclasses.dataclass
class DispatchHandle:
    """What combine and the backward pass need from one dispatch: the
    layout of that batch and the buffer set it used (the pages' `plan`)."""
    index: int
    tokens_per_expert: torch.Tensor
    expert_offsets: torch.Tensor     # the pages' cu_seqlens, [E+1]
    pos: torch.Tensor
    row_src: torch.Tensor
    recv: torch.Tensor
    recv_scales: torch.Tensor | None
    recv_weights: torch.Tensor
    balanced: dict | None = None     # filled by plan()


class _Set:
    def __init__(self, owner: "EPBuffer", dev):
        N, K, E, H, cap = owner.N, owner.K, owner.E, owner.H, owner.cap
        i32 = dict(dtype=torch.int32, device=dev)
        rows = max(cap, 1)
        self.tokens_per_expert = torch.zeros(E, **i32)
        self.expert_offsets = torch.zeros(E + 1, **i32)
        self.pos = torch.zeros(max(N, 1), K, **i32)
        self.row_src = torch.zeros(rows, **i32)
        if owner.fp8:
            self.recv = torch.empty(rows, H, dtype=torch.float8_e4m3fn,
                                    device=dev)
            self.recv_scales = torch.empty(rows, H // 128, dtype=torch.float32,
                                           device=dev)
        else:
            self.recv = torch.empty(rows, H, dtype=torch.bfloat16, device=dev)
            self.recv_scales = None
        self.recv_weights = torch.empty(rows, dtype=torch.float32, device=dev)
        # combine's outputs, reused by every combine on this set
        self.out = torch.empty(max(N, 1), H, dtype=torch.bfloat16, device=dev)
        self.gathered = torch.empty(max(N, 1), K, dtype=torch.float32,
                                    device=dev)


class EPBuffer:
    def __init__(self, S: int, H: int, K: int, E: int, num_ep_ranks: int,
                 num_sms: int = 0, token_padding: int = 1, fp8: bool = False,
                 double_buffer: bool = False, device=None):
        self.S, self.H, self.K, self.E = S, H, K, E
        self.R = num_ep_ranks
        self.N = self.R * S
        self.num_sms = num_sms
        self.pad = token_padding
        self.fp8 = fp8
        dev = torch.device(device if device is not None else "cuda")
        self.device = dev
        self.cap = B.ep_capacity_bound(self.N, K, E, token_padding)
        if self.cap < 0:
            raise ValueError("invalid buffer shape")
        ws = B.ep_layout_workspace_bytes(self.N, K, E)
        self.workspace = torch.zeros(max(ws, 16), dtype=torch.uint8,
                                     device=dev)
        self.status = torch.zeros(4, dtype=torch.int32, device=dev)
        self.sets = [_Set(self, dev) for _ in range(2 if double_buffer else 1)]
        self.index = len(self.sets) - 1   # the next dispatch flips to 0

    # -- the current set (single-buffer convenience views) -------------------
    @property
    def pos(self):
        return self.sets[self.index].pos

    @property
    def tokens_per_expert(self):
        return self.sets[self.index].tokens_per_expert

    @property
    def expert_offsets(self):
        return self.sets[self.index].expert_offsets

    # -- dispatch --------------------------------------------------------------
    def dispatch(self, hidden_sh: torch.Tensor, route_weights_sk: torch.Tensor,
                 topk_experts_sk: torch.Tensor, stream=None):
        """-> (recv, recv_weights, expert_offsets, handle): recv holds rank
        r's rows in [expert_offsets[r*E/R], expert_offsets[(r+1)*E/R]);
        FP8 scales are handle.recv_scales."""
        self.index = (self.index + 1) % len(self.sets)   # idx ^= 1
        st = self.sets[self.index]
        B.ep_layout_dispatch(topk_experts_sk, hidden_sh, route_weights_sk,
                             self.R, self.S, self.K, self.E, self.H, self.pad,
                             self.fp8, st.tokens_per_expert,
                             st.expert_offsets, st.pos, st.row_src, st.recv,
                             st.recv_scales, st.recv_weights, self.workspace,
                             self.num_sms, self.status, cap=self.cap,
                             stream=stream)
        h = DispatchHandle(self.index, st.tokens_per_expert,
                           st.expert_offsets, st.pos, st.row_src, st.recv,
                           st.recv_scales, st.recv_weights)
        return st.recv, st.recv_weights, st.expert_offsets, h

    # -- balanced plan + prefetch ---------------------------------------------
    def plan(self, handle: DispatchHandle, slots_per_rank: int,
             stream=None) -> dict:
        """Balanced plan from the dispatch's tokens_per_expert (token_padding
        must be 1). Stored on the handle and returned."""
        if self.pad != 1:
            raise ValueError("the balanced plan needs token_padding == 1")
        R, E, Bs = self.R, self.E, slots_per_rank
        i32 = dict(dtype=torch.int32, device=self.device)
        p = dict(cu=torch.empty(R, E + 1, **i32),
                 expert=torch.empty(R, E, **i32),
                 wrow=torch.empty(R, E, **i32),
                 nseg=torch.empty(R, **i32),
                 slot_expert=torch.empty(R, max(Bs, 1), **i32), B=Bs)
        B.ep_plan_balanced(handle.tokens_per_expert, R, self.S, self.K, E, Bs,
                           p["cu"], p["expert"], p["wrow"], p["nseg"],
                           p["slot_expert"] if Bs > 0 else None, self.status,
                           stream=stream)
        handle.balanced = p
        return p

    def prefetch_weight(self, plan: dict, full_gate_weight, full_up_weight,
                        full_down_weight, stream=None):
        B.ep_prefetch_weights(plan["slot_expert"], self.R, self.E, plan["B"],
                              full_gate_weight, full_up_weight,
                              full_down_weight, self.num_sms, self.status,
                              stream=stream)

    def reduce_grads(self, plan: dict, grad_gate, grad_up, grad_down,
                     stream=None):
        """Fold the prefetched copies' fp32 gradients into the owners' rows."""
        B.ep_reduce_slot_grads(plan["slot_expert"], self.R, self.E, plan["B"],
                               grad_gate, grad_up, grad_down, self.num_sms,
                               stream=stream)

    # -- combine ---------------------------------------------------------------
    def combine(self, handle: DispatchHandle, expert_output: torch.Tensor,
                route_weights_nvs: torch.Tensor | None = None,
                out: torch.Tensor | None = None,
                gathered: torch.Tensor | None = None, stream=None):
        """-> (output_sh, gathered_route_weights_sk). Each entry's weight is
        the receive-side route_weights_nvs at its row (the dispatch's
        recv_weights when None); one launch computes the output and hands
        the weights back in token order. Unless `out` / `gathered` are
        given, the results are the handle's buffer set's own tensors,
        allocated at construction and overwritten by the next combine on
        that set."""
        st = self.sets[handle.index]
        rw = handle.recv_weights if route_weights_nvs is None else \
            route_weights_nvs
        out = st.out if out is None else out
        gathered = st.gathered if gathered is None else gathered
        # rows of expert_output (and of the weights) bound the positions
        # that may be read
        B.ep_combine_recv_weights(expert_output, handle.pos, rw, self.N,
                                  self.K, self.H, out, gathered,
                                  self.num_sms, self.status,
                                  cap=min(expert_output.shape[0], rw.numel()),
                                  stream=stream)
        return out[:self.N], gathered[:self.N]

    # -- backward --------------------------------------------------------------
    def combine_backward(self, handle: DispatchHandle, grad_out, expert_output,
                         route_weights_sk, stream=None):
        """-> (grad_expert_output [cap,H] bf16, grad_route_weights [N,K])."""
        gy = torch.empty(self.cap, self.H, dtype=torch.bfloat16,
                         device=grad_out.device)
        gw = torch.empty(self.N, self.K, dtype=torch.float32,
                         device=grad_out.device)
        B.ep_combine_backward(grad_out, expert_output, handle.pos,
                              handle.row_src, handle.expert_offsets,
                              route_weights_sk, self.N, self.K, self.E,
                              self.H, gy, gw, self.num_sms, self.status,
                              cap=self.cap, stream=stream)
        return gy, gw

    def dispatch_backward(self, handle: DispatchHandle, grad_recv,
                          stream=None):
        """-> grad_hidden [N,H] bf16: sum over k of the receive-row grads."""
        gx = torch.empty(self.N, self.H, dtype=torch.bfloat16,
                         device=grad_recv.device)
        B.ep_dispatch_backward(grad_recv, handle.pos, self.N, self.K, self.H,
                               gx, self.num_sms, self.status,
                               cap=grad_recv.shape[0], stream=stream)
        return gx

    def check(self):
        """Synchronising read of the device status word; raises on error."""
        s = int(self.status[0].item())
        if s:
            raise B.EPError(s, "device status")
