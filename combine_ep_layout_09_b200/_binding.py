"""ctypes binding of libeplayout.so.

Argument marshalling only: each function checks that the tensors it is given
are CUDA, contiguous and of the right dtype, turns them into device pointers
and sizes, calls the C entry point of the same name, and raises EPError on a
non-zero return. Every step of the computation runs in the library's CUDA
kernels; there is no fallback. If the library is missing and cannot be built,
importing this package fails.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

from . import build as _build

EP_OK = 0
EP_ERR_INVALID_ARG = -1
EP_ERR_ALIGNMENT = -2
EP_ERR_WORKSPACE = -3
EP_ERR_CAPACITY = -4
EP_ERR_CUDA = -5

EP_DEV_BAD_EXPERT = 1
EP_DEV_CAPACITY = 2
EP_DEV_TIMEOUT = 4
EP_DEV_SLOTS = 8
EP_DEV_PLAN_TOTAL = 16

EP_WAIT_SITE_LOOKBACK = 1
EP_WAIT_SITE_TILE_REDUCE = 2
EP_WAIT_SITE_DISPATCH = 4
EP_WAIT_SITE_COMBINE = 8
EP_WAIT_SITE_SMALL = 16
EP_WAIT_SITE_PREFETCH = 32
EP_WAIT_SITE_ALL = 63

_lock = threading.Lock()
_lib = None


class EPError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {strerror(code)} (code {code})")


def library_path() -> str:
    return _build.LIB


def lib() -> ctypes.CDLL:
    """Load libeplayout.so, building it first if it is missing or stale."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is None:
            if not _build.up_to_date():
                try:
                    _build.build()
                except Exception as e:  # fail loudly: no other code path
                    raise RuntimeError(
                        "libeplayout.so is missing or stale and could not be "
                        f"built: {e}") from e
            L = ctypes.CDLL(_build.LIB)
            _declare(L)
            _lib = L
    return _lib


def _declare(L):
    P, i32, i64, sz = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64,
                       ctypes.c_size_t)
    L.ep_abi_version.restype = i32
    L.ep_abi_version.argtypes = []
    L.ep_strerror.restype = ctypes.c_char_p
    L.ep_strerror.argtypes = [i32]
    L.ep_capacity_bound.restype = i64
    L.ep_capacity_bound.argtypes = [i64, i32, i32, i32]
    L.ep_layout_workspace_bytes.restype = sz
    L.ep_layout_workspace_bytes.argtypes = [i64, i32, i32]
    L.ep_layout.restype = i32
    L.ep_layout.argtypes = [P, i32, i32, i32, i32, i32, P, P, P, P, i64, P,
                            sz, P, P]
    L.ep_dispatch.restype = i32
    L.ep_dispatch.argtypes = [P, P, P, P, P, i64, i32, i32, i32, i64, i32, P,
                              P, P, i32, P, P]
    L.ep_layout_dispatch.restype = i32
    L.ep_layout_dispatch.argtypes = [P, P, P, i32, i32, i32, i32, i32, i32,
                                     i32, P, P, P, P, i64, P, P, P, P, sz,
                                     i32, P, P]
    L.ep_combine.restype = i32
    L.ep_combine.argtypes = [P, P, P, i64, i32, i32, i64, P, i32, P, P]
    L.ep_combine_recv_weights.restype = i32
    L.ep_combine_recv_weights.argtypes = [P, P, P, i64, i32, i32, i64, P, P,
                                          i32, P, P]
    L.ep_dispatch_backward.restype = i32
    L.ep_dispatch_backward.argtypes = [P, P, i64, i32, i32, i64, P, i32, P, P]
    L.ep_combine_backward.restype = i32
    L.ep_combine_backward.argtypes = [P, P, P, P, P, P, i64, i32, i32, i32,
                                      i64, P, P, i32, P, P]
    L.ep_gather_route_weights.restype = i32
    L.ep_gather_route_weights.argtypes = [P, P, i64, i32, i64, P, P]
    L.ep_plan_balanced.restype = i32
    L.ep_plan_balanced.argtypes = [P, i32, i32, i32, i32, i32, P, P, P, P, P,
                                   P, P]
    L.ep_prefetch_weights.restype = i32
    L.ep_prefetch_weights.argtypes = [P, i32, i32, i32, i64, P, P, P, i32, P,
                                      P]
    L.ep_reduce_slot_grads.restype = i32
    L.ep_reduce_slot_grads.argtypes = [P, i32, i32, i32, i64, P, P, P, i32, P]
    L.ep_debug_e4m3_encode.restype = i32
    L.ep_debug_e4m3_encode.argtypes = [P, P, i64, P]
    L.ep_debug_quantize.restype = i32
    L.ep_debug_quantize.argtypes = [P, P, P, i64, P]
    L.ep_debug_bounded_wait.restype = i32
    L.ep_debug_bounded_wait.argtypes = [P, i64, P, P]
    L.ep_debug_stream_read.restype = i32
    L.ep_debug_stream_read.argtypes = [P, i64, P, P]
    L.ep_debug_force_timeouts.restype = i32
    L.ep_debug_force_timeouts.argtypes = [ctypes.c_uint32, i64]


# --------------------------------------------------------------------------
# marshalling helpers
# --------------------------------------------------------------------------

def _ptr(t, name, dtypes=None, min_numel=None, optional=False):
    if t is None:
        if optional:
            return None
        raise ValueError(f"{name} is required")
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (got {t.device})")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtypes is not None and t.dtype not in dtypes:
        raise TypeError(f"{name}: dtype {t.dtype} not in {dtypes}")
    if min_numel is not None and t.numel() < min_numel:
        raise ValueError(f"{name} holds {t.numel()} elements, needs "
                         f">= {min_numel}")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _check(rc: int, where: str):
    if rc != EP_OK:
        raise EPError(rc, where)


_I32 = (torch.int32,)
_F32 = (torch.float32,)
_BF16 = (torch.bfloat16,)
_W16 = (torch.bfloat16, torch.float16, torch.int16)
_FP8 = (torch.float8_e4m3fn, torch.uint8)


# --------------------------------------------------------------------------
# entry points (same names as the C ABI)
# --------------------------------------------------------------------------

def ep_abi_version() -> int:
    return lib().ep_abi_version()


def strerror(code: int) -> str:
    return lib().ep_strerror(int(code)).decode()


ep_strerror = strerror


def ep_capacity_bound(num_tokens: int, K: int, E: int,
                      token_padding: int) -> int:
    return lib().ep_capacity_bound(num_tokens, K, E, token_padding)


def ep_layout_workspace_bytes(num_tokens: int, K: int, E: int) -> int:
    return lib().ep_layout_workspace_bytes(num_tokens, K, E)


def ep_layout(topk_experts, R, S, K, E, token_padding, tokens_per_expert,
              expert_offsets, pos, row_src, workspace, status=None,
              cap=None, stream=None):
    """Histogram, padded expert offsets and stable positions."""
    N = R * S
    cap = row_src.numel() if cap is None else int(cap)
    rc = lib().ep_layout(
        _ptr(topk_experts, "topk_experts", _I32, N * K),
        R, S, K, E, token_padding,
        _ptr(tokens_per_expert, "tokens_per_expert", _I32, E),
        _ptr(expert_offsets, "expert_offsets", _I32, E + 1),
        _ptr(pos, "pos", _I32, N * K),
        _ptr(row_src, "row_src", _I32, cap),
        cap,
        _ptr(workspace, "workspace"),
        workspace.numel() * workspace.element_size(),
        _ptr(status, "status", _I32, 1, optional=True),
        _stream(stream))
    _check(rc, "ep_layout")


def ep_dispatch(hidden, route_weights, pos, row_src, expert_offsets,
                num_tokens, K, E, H, fp8, recv, recv_scales=None,
                recv_weights=None, num_sms=0, status=None, cap=None,
                stream=None):
    """Copy (bf16) or quantise-and-copy (fp8) token rows to their K rows."""
    cap = recv.shape[0] if cap is None else int(cap)
    rc = lib().ep_dispatch(
        _ptr(hidden, "hidden", _BF16, num_tokens * H),
        _ptr(route_weights, "route_weights", _F32, num_tokens * K),
        _ptr(pos, "pos", _I32, num_tokens * K),
        _ptr(row_src, "row_src", _I32, cap),
        _ptr(expert_offsets, "expert_offsets", _I32, E + 1),
        num_tokens, K, E, H, cap, 1 if fp8 else 0,
        _ptr(recv, "recv", _FP8 if fp8 else _BF16, cap * H),
        _ptr(recv_scales, "recv_scales", _F32, cap * (H // 128),
             optional=not fp8),
        _ptr(recv_weights, "recv_weights", _F32, cap, optional=True),
        int(num_sms),
        _ptr(status, "status", _I32, 1, optional=True),
        _stream(stream))
    _check(rc, "ep_dispatch")


def ep_layout_dispatch(topk_experts, hidden, route_weights, R, S, K, E, H,
                       token_padding, fp8, tokens_per_expert, expert_offsets,
                       pos, row_src, recv, recv_scales=None,
                       recv_weights=None, workspace=None, num_sms=0,
                       status=None, cap=None, stream=None):
    """ep_layout then ep_dispatch; one launch for a small batch."""
    N = R * S
    cap = row_src.numel() if cap is None else int(cap)
    rc = lib().ep_layout_dispatch(
        _ptr(topk_experts, "topk_experts", _I32, N * K),
        _ptr(hidden, "hidden", _BF16, N * H),
        _ptr(route_weights, "route_weights", _F32, N * K),
        R, S, K, E, H, token_padding, 1 if fp8 else 0,
        _ptr(tokens_per_expert, "tokens_per_expert", _I32, E),
        _ptr(expert_offsets, "expert_offsets", _I32, E + 1),
        _ptr(pos, "pos", _I32, N * K),
        _ptr(row_src, "row_src", _I32, cap),
        cap,
        _ptr(recv, "recv", _FP8 if fp8 else _BF16, cap * H),
        _ptr(recv_scales, "recv_scales", _F32, cap * (H // 128),
             optional=not fp8),
        _ptr(recv_weights, "recv_weights", _F32, cap, optional=True),
        _ptr(workspace, "workspace"),
        workspace.numel() * workspace.element_size(),
        int(num_sms),
        _ptr(status, "status", _I32, 1, optional=True),
        _stream(stream))
    _check(rc, "ep_layout_dispatch")


def ep_combine(expert_out, pos, route_weights, num_tokens, K, H, out,
               num_sms=0, status=None, cap=None, stream=None):
    """out[t] = bf16(sum_k fma(w[t,k], y[pos[t,k]])) in fp32, k ascending."""
    cap = expert_out.shape[0] if cap is None else int(cap)
    rc = lib().ep_combine(
        _ptr(expert_out, "expert_out", _BF16, cap * H),
        _ptr(pos, "pos", _I32, num_tokens * K),
        _ptr(route_weights, "route_weights", _F32, num_tokens * K),
        num_tokens, K, H, cap,
        _ptr(out, "out", _BF16, num_tokens * H),
        int(num_sms),
        _ptr(status, "status", _I32, 1, optional=True),
        _stream(stream))
    _check(rc, "ep_combine")


def ep_combine_recv_weights(expert_out, pos, recv_weights, num_tokens, K, H,
                            out, gathered=None, num_sms=0, status=None,
                            cap=None, stream=None):
    """Combine with the receive-side weights recv_weights[pos[t,k]]; the
    weights also come back in token order in `gathered` (may be None)."""
    cap = expert_out.shape[0] if cap is None else int(cap)
    rc = lib().ep_combine_recv_weights(
        _ptr(expert_out, "expert_out", _BF16, cap * H),
        _ptr(pos, "pos", _I32, num_tokens * K),
        _ptr(recv_weights, "recv_weights", _F32, cap),
        num_tokens, K, H, cap,
        _ptr(out, "out", _BF16, num_tokens * H),
        _ptr(gathered, "gathered", _F32, num_tokens * K, optional=True),
        int(num_sms),
        _ptr(status, "status", _I32, 1, optional=True),
        _stream(stream))
    _check(rc, "ep_combine_recv_weights")


def ep_dispatch_backward(grad_recv, pos, num_tokens, K, H, grad_hidden,
                         num_sms=0, status=None, cap=None, stream=None):
    """grad_hidden[t] = bf16(sum_k grad_recv[pos[t,k]]) in fp32, k order."""
    cap = grad_recv.shape[0] if cap is None else int(cap)
    rc = lib().ep_dispatch_backward(
        _ptr(grad_recv, "grad_recv", _BF16, cap * H),
        _ptr(pos, "pos", _I32, num_tokens * K), num_tokens, K, H, cap,
        _ptr(grad_hidden, "grad_hidden", _BF16, num_tokens * H),
        int(num_sms), _ptr(status, "status", _I32, 1, optional=True),
        _stream(stream))
    _check(rc, "ep_dispatch_backward")


def ep_combine_backward(grad_out, expert_out, pos, row_src, expert_offsets,
                        route_weights, num_tokens, K, E, H, grad_expert_out,
                        grad_route_weights, num_sms=0, status=None, cap=None,
                        stream=None):
    """Gradients of combine: scaled rows and per-entry dot products."""
    cap = expert_out.shape[0] if cap is None else int(cap)
    rc = lib().ep_combine_backward(
        _ptr(grad_out, "grad_out", _BF16, num_tokens * H),
        _ptr(expert_out, "expert_out", _BF16, cap * H),
        _ptr(pos, "pos", _I32, num_tokens * K),
        _ptr(row_src, "row_src", _I32, cap),
        _ptr(expert_offsets, "expert_offsets", _I32, E + 1),
        _ptr(route_weights, "route_weights", _F32, num_tokens * K),
        num_tokens, K, E, H, cap,
        _ptr(grad_expert_out, "grad_expert_out", _BF16, cap * H),
        _ptr(grad_route_weights, "grad_route_weights", _F32, num_tokens * K),
        int(num_sms), _ptr(status, "status", _I32, 1, optional=True),
        _stream(stream))
    _check(rc, "ep_combine_backward")


def ep_gather_route_weights(row_values, pos, num_tokens, K, out, cap=None,
                            stream=None):
    """out[t,k] = row_values[pos[t,k]] (gathered_route_weights)."""
    cap = row_values.numel() if cap is None else int(cap)
    rc = lib().ep_gather_route_weights(
        _ptr(row_values, "row_values", _F32, cap),
        _ptr(pos, "pos", _I32, num_tokens * K), num_tokens, K, cap,
        _ptr(out, "out", _F32, num_tokens * K), _stream(stream))
    _check(rc, "ep_gather_route_weights")


def ep_plan_balanced(tokens_per_expert, R, S, K, E, B, plan_cu, plan_expert,
                     plan_wrow, plan_nseg, slot_expert, status=None,
                     stream=None):
    """Cut the expert-sorted rows into R chunks of S*K rows; assign slots."""
    rc = lib().ep_plan_balanced(
        _ptr(tokens_per_expert, "tokens_per_expert", _I32, E),
        R, S, K, E, B,
        _ptr(plan_cu, "plan_cu", _I32, R * (E + 1)),
        _ptr(plan_expert, "plan_expert", _I32, R * E),
        _ptr(plan_wrow, "plan_wrow", _I32, R * E),
        _ptr(plan_nseg, "plan_nseg", _I32, R),
        _ptr(slot_expert, "slot_expert", _I32, R * B, optional=(B == 0)),
        _ptr(status, "status", _I32, 1, optional=True),
        _stream(stream))
    _check(rc, "ep_plan_balanced")


def ep_prefetch_weights(slot_expert, R, E, B, gate, up, down, num_sms=0,
                        status=None, stream=None):
    """Copy the slot experts' gate/up/down rows into the prefetch slots."""
    rows = E + R * B
    elems = gate[0].numel() if gate.shape[0] > 0 else 0
    for name, t in (("gate", gate), ("up", up), ("down", down)):
        if t.shape[0] != rows or t[0].numel() != elems:
            raise ValueError(f"{name} must be [E + R*B, ...] like gate")
    rc = lib().ep_prefetch_weights(
        _ptr(slot_expert, "slot_expert", _I32, R * B, optional=(B == 0)),
        R, E, B, elems,
        _ptr(gate, "gate", _W16), _ptr(up, "up", _W16),
        _ptr(down, "down", _W16),
        int(num_sms), _ptr(status, "status", _I32, 1, optional=True),
        _stream(stream))
    _check(rc, "ep_prefetch_weights")


def ep_reduce_slot_grads(slot_expert, R, E, B, grad_gate, grad_up,
                         grad_down, num_sms=0, stream=None):
    """Add every prefetched copy's gradient into its expert's row."""
    rows = E + R * B
    elems = grad_gate[0].numel() if grad_gate.shape[0] > 0 else 0
    for name, t in (("grad_gate", grad_gate), ("grad_up", grad_up),
                    ("grad_down", grad_down)):
        if t.shape[0] != rows or t[0].numel() != elems:
            raise ValueError(f"{name} must be [E + R*B, ...] like grad_gate")
    rc = lib().ep_reduce_slot_grads(
        _ptr(slot_expert, "slot_expert", _I32, R * B, optional=(B == 0)),
        R, E, B, elems,
        _ptr(grad_gate, "grad_gate", _F32), _ptr(grad_up, "grad_up", _F32),
        _ptr(grad_down, "grad_down", _F32), int(num_sms), _stream(stream))
    _check(rc, "ep_reduce_slot_grads")


def ep_debug_e4m3_encode(x, out, stream=None):
    rc = lib().ep_debug_e4m3_encode(
        _ptr(x, "x", _F32), _ptr(out, "out", (torch.uint8,), x.numel()),
        x.numel(), _stream(stream))
    _check(rc, "ep_debug_e4m3_encode")


def ep_debug_quantize(x, group_scale, out, stream=None):
    n = x.numel()
    rc = lib().ep_debug_quantize(
        _ptr(x, "x", _F32), _ptr(group_scale, "group_scale", _F32, n // 16),
        _ptr(out, "out", (torch.uint8,), n), n, _stream(stream))
    _check(rc, "ep_debug_quantize")


def ep_debug_bounded_wait(flag, max_polls, status, stream=None):
    rc = lib().ep_debug_bounded_wait(
        _ptr(flag, "flag", _I32, 1), int(max_polls),
        _ptr(status, "status", _I32, 1), _stream(stream))
    _check(rc, "ep_debug_bounded_wait")


def ep_debug_stream_read(src, sink, stream=None):
    """Read all of `src` (a CUDA tensor, 32-byte aligned, a multiple of 32
    bytes) once; the XOR of its 32-bit words is XOR-ed into sink[0]."""
    nbytes = src.numel() * src.element_size()
    if not src.is_cuda or not src.is_contiguous():
        raise ValueError("src must be a contiguous CUDA tensor")
    rc = lib().ep_debug_stream_read(
        ctypes.c_void_p(src.data_ptr()), int(nbytes),
        _ptr(sink, "sink", (torch.int32,), 1), _stream(stream))
    _check(rc, "ep_debug_stream_read")


def ep_debug_force_timeouts(sites, budget_ns=0):
    """Make the waits at `sites` (EP_WAIT_SITE_* bits) give up after
    budget_ns on the current device; sites=0 restores normal waits."""
    rc = lib().ep_debug_force_timeouts(int(sites), int(budget_ns))
    _check(rc, "ep_debug_force_timeouts")
