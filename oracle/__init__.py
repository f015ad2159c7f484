"""CPU oracle for MoE token dispatch / combine (test infrastructure).

A plain, slow, single-threaded restatement of what the method computes,
written in C (oracle.c) and wrapped here with ctypes and numpy. Only the
tests, the package smoke check and the benchmark's CPU-baseline leg use it;
the CUDA library neither imports nor links it, and the two share no code.

Every function takes and returns numpy arrays; bf16 data travels as uint16
bit patterns, FP8 E4M3 codes as uint8.

Parity status of each function (what pins it, in tests/test_oracle_*.py):
  histogram / expert_offsets / positions  brute-force sort of (e, t, k),
                                          sum = N*K, E % R, goldens
  dispatch_bf16                           closed form recv[pos] == hidden[t]
  e4m3_encode / quantize_row              torch.float8_e4m3fn cast, all 256
                                          codes, ties, saturation, error bound
  combine / combine_f64                   identity experts give x exactly,
                                          1-ulp bound vs the double sum,
                                          brute-force per-element sum
  plan_balanced                           brute-force row-by-row planner,
                                          every rank exactly S*K rows
  prefetch                                slot rows equal source rows
  reduce_slot_grads                       brute force, exact on integer
                                          gradients, sum preserved (fp64)
  dispatch_backward                       adjoint of bf16 dispatch (fp64
                                          inner products), brute force
  combine_backward_rows / _weights        adjoint of combine, finite
                                          differences of combine_f64 in w,
                                          numpy einsum in fp64
  gather_row_values                       closed form, round trip with
                                          dispatch's recv_w
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

ST_BAD_EXPERT = 1
ST_CAPACITY = 2
ST_SLOTS = 8
ST_PLAN_TOTAL = 16

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i64 = ctypes.c_int64
        i32 = ctypes.c_int
        L.oracle_e4m3_encode.restype = ctypes.c_uint8
        L.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        L.oracle_e4m3_decode.restype = ctypes.c_double
        L.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_encode_array.argtypes = [P, i64, P]
        L.oracle_bf16_to_f32.restype = ctypes.c_float
        L.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.oracle_f32_to_bf16.restype = ctypes.c_uint16
        L.oracle_f32_to_bf16.argtypes = [ctypes.c_float]
        L.oracle_histogram.restype = i32
        L.oracle_histogram.argtypes = [P, i64, i32, i32, P]
        L.oracle_expert_offsets.restype = None
        L.oracle_expert_offsets.argtypes = [P, i32, i32, P]
        L.oracle_positions.restype = i32
        L.oracle_positions.argtypes = [P, i64, i32, i32, P, P, P, i64]
        L.oracle_layout.restype = i32
        L.oracle_layout.argtypes = [P, i64, i32, i32, i32, P, P, P, P, i64]
        L.oracle_dispatch_bf16.restype = None
        L.oracle_dispatch_bf16.argtypes = [P, P, P, P, P, i64, i32, i32, i32,
                                           i64, P, P]
        L.oracle_quantize_row.restype = None
        L.oracle_quantize_row.argtypes = [P, i32, P, P]
        L.oracle_quantize_by_scale.restype = None
        L.oracle_quantize_by_scale.argtypes = [P, P, i64, i32, P]
        L.oracle_dispatch_fp8.restype = None
        L.oracle_dispatch_fp8.argtypes = [P, P, P, P, P, i64, i32, i32, i32,
                                          i64, P, P, P]
        L.oracle_combine.restype = None
        L.oracle_combine.argtypes = [P, P, P, i64, i32, i32, i64, P]
        L.oracle_combine_f64.restype = None
        L.oracle_combine_f64.argtypes = [P, P, P, i64, i32, i32, i64, P]
        L.oracle_dispatch_backward.restype = None
        L.oracle_dispatch_backward.argtypes = [P, P, i64, i32, i32, i64, P]
        L.oracle_combine_backward_rows.restype = None
        L.oracle_combine_backward_rows.argtypes = [P, P, P, P, P, i64, i32,
                                                   i32, i32, i64, P]
        L.oracle_combine_backward_weights.restype = None
        L.oracle_combine_backward_weights.argtypes = [P, P, P, i64, i32, i32,
                                                      i64, P]
        L.oracle_gather_row_values.restype = None
        L.oracle_gather_row_values.argtypes = [P, P, i64, i32, i64, P]
        L.oracle_reduce_slot_grads.restype = None
        L.oracle_reduce_slot_grads.argtypes = [P, i32, i32, i32, i64, P]
        L.oracle_plan_balanced.restype = i32
        L.oracle_plan_balanced.argtypes = [P, i32, i32, i32, i32, i32, P, P,
                                           P, P, P]
        L.oracle_prefetch.restype = None
        L.oracle_prefetch.argtypes = [P, i32, i32, i32, i64, P]
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# --- scalar helpers ---------------------------------------------------------

def e4m3_encode(x) -> np.ndarray:
    x = _c(np.atleast_1d(x), np.float32)
    out = np.empty(x.shape, dtype=np.uint8)
    lib().oracle_e4m3_encode_array(_p(x), x.size, _p(out))
    return out


def e4m3_decode(codes) -> np.ndarray:
    c = np.atleast_1d(np.asarray(codes, dtype=np.uint8))
    return np.array([lib().oracle_e4m3_decode(int(v)) for v in c.ravel()],
                    dtype=np.float64).reshape(c.shape)


def bf16_to_f32(h) -> np.ndarray:
    h = np.atleast_1d(np.asarray(h, dtype=np.uint16))
    return np.array([lib().oracle_bf16_to_f32(int(v)) for v in h.ravel()],
                    dtype=np.float32).reshape(h.shape)


def f32_to_bf16(f) -> np.ndarray:
    f = np.atleast_1d(np.asarray(f, dtype=np.float32))
    return np.array([lib().oracle_f32_to_bf16(float(v)) for v in f.ravel()],
                    dtype=np.uint16).reshape(f.shape)


# --- layout -----------------------------------------------------------------

def capacity_bound(N: int, K: int, E: int, pad: int) -> int:
    """Rows any routing can need: N*K entries plus at most pad-1 padding rows
    per expert."""
    return N * K + E * (pad - 1)


def layout(topk: np.ndarray, E: int, pad: int, cap: int | None = None,
           row_src_fill: int = -7):
    """-> dict(counts[E], offsets[E+1], pos[N,K], row_src[cap], status).
    Rows of row_src the method leaves untouched keep `row_src_fill`."""
    topk = _c(topk, np.int32)
    N, K = topk.shape
    if cap is None:
        cap = capacity_bound(N, K, E, pad)
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    pos = np.empty((N, K), np.int32)
    row_src = np.full(max(cap, 1), row_src_fill, np.int32)
    st = lib().oracle_layout(_p(topk), N, K, E, pad, _p(counts), _p(offsets),
                             _p(pos), _p(row_src), cap)
    return dict(counts=counts, offsets=offsets, pos=pos,
                row_src=row_src[:cap], status=st)


# --- dispatch ---------------------------------------------------------------

def dispatch_bf16(hidden: np.ndarray, w: np.ndarray, lay: dict, E: int,
                  cap: int, recv_fill: int = 0x7FBF, recv_w_fill=-3.0):
    """-> (recv [cap,H] uint16, recv_w [cap] f32). Untouched rows keep the
    fill patterns."""
    hidden = _c(hidden, np.uint16)
    w = _c(w, np.float32)
    N, H = hidden.shape
    K = lay["pos"].shape[1]
    recv = np.full((cap, H), recv_fill, np.uint16)
    recv_w = np.full(cap, recv_w_fill, np.float32)
    lib().oracle_dispatch_bf16(_p(hidden), _p(w), _p(_c(lay["pos"], np.int32)),
                               _p(_c(lay["row_src"], np.int32)),
                               _p(_c(lay["offsets"], np.int32)), N, K, E, H,
                               cap, _p(recv), _p(recv_w))
    return recv, recv_w


def quantize_row(row: np.ndarray):
    """One bf16 row [H] -> (codes [H] uint8, scales [H/128] f32)."""
    row = _c(row, np.uint16)
    H = row.shape[0]
    q = np.empty(H, np.uint8)
    s = np.empty(H // 128, np.float32)
    lib().oracle_quantize_row(_p(row), H, _p(q), _p(s))
    return q, s


def quantize_rows(rows: np.ndarray):
    rows = _c(rows, np.uint16)
    n, H = rows.shape
    q = np.empty((n, H), np.uint8)
    s = np.empty((n, H // 128), np.float32)
    for i in range(n):
        q[i], s[i] = quantize_row(rows[i])
    return q, s


def quantize_by_scale(x: np.ndarray, scale: np.ndarray, group: int = 16):
    """codes[i] = e4m3(fp32(x[i] / scale[i // group])), 0 where scale == 0."""
    x = _c(x, np.float32).ravel()
    scale = _c(scale, np.float32).ravel()
    assert scale.size * group >= x.size
    out = np.empty(x.size, np.uint8)
    lib().oracle_quantize_by_scale(_p(x), _p(scale), x.size, group, _p(out))
    return out


def dispatch_fp8(hidden: np.ndarray, w: np.ndarray, lay: dict, E: int,
                 cap: int, recv_fill: int = 0xA5, scale_fill=-5.0,
                 recv_w_fill=-3.0):
    """-> (recv [cap,H] uint8, scales [cap,H/128] f32, recv_w [cap] f32)."""
    hidden = _c(hidden, np.uint16)
    w = _c(w, np.float32)
    N, H = hidden.shape
    K = lay["pos"].shape[1]
    recv = np.full((cap, H), recv_fill, np.uint8)
    scales = np.full((cap, H // 128), scale_fill, np.float32)
    recv_w = np.full(cap, recv_w_fill, np.float32)
    lib().oracle_dispatch_fp8(_p(hidden), _p(w), _p(_c(lay["pos"], np.int32)),
                              _p(_c(lay["row_src"], np.int32)),
                              _p(_c(lay["offsets"], np.int32)), N, K, E, H,
                              cap, _p(recv), _p(scales), _p(recv_w))
    return recv, scales, recv_w


# --- combine ----------------------------------------------------------------

def combine(y: np.ndarray, pos: np.ndarray, w: np.ndarray) -> np.ndarray:
    """-> out [N,H] uint16 (bf16 bits); fp32 fma chain in k order."""
    y = _c(y, np.uint16)
    pos = _c(pos, np.int32)
    w = _c(w, np.float32)
    cap, H = y.shape
    N, K = pos.shape
    out = np.empty((N, H), np.uint16)
    lib().oracle_combine(_p(y), _p(pos), _p(w), N, K, H, cap, _p(out))
    return out


def combine_f64(y: np.ndarray, pos: np.ndarray, w: np.ndarray) -> np.ndarray:
    y = _c(y, np.uint16)
    pos = _c(pos, np.int32)
    w = _c(w, np.float32)
    cap, H = y.shape
    N, K = pos.shape
    out = np.empty((N, H), np.float64)
    lib().oracle_combine_f64(_p(y), _p(pos), _p(w), N, K, H, cap, _p(out))
    return out


# --- backward pair ----------------------------------------------------------

def dispatch_backward(grad_recv: np.ndarray, pos: np.ndarray) -> np.ndarray:
    """grad_hidden [N,H] bf16 bits: sum over k of the receive-row grads."""
    g = _c(grad_recv, np.uint16)
    pos = _c(pos, np.int32)
    cap, H = g.shape
    N, K = pos.shape
    out = np.empty((N, H), np.uint16)
    lib().oracle_dispatch_backward(_p(g), _p(pos), N, K, H, cap, _p(out))
    return out


def combine_backward_rows(grad_out: np.ndarray, w: np.ndarray, lay: dict,
                          E: int, cap: int, fill: int = 0x7FBF) -> np.ndarray:
    """grad of the expert outputs [cap,H] bf16 bits (untouched rows keep
    `fill`)."""
    g = _c(grad_out, np.uint16)
    w = _c(w, np.float32)
    N, H = g.shape
    K = lay["pos"].shape[1]
    out = np.full((cap, H), fill, np.uint16)
    lib().oracle_combine_backward_rows(
        _p(g), _p(w), _p(_c(lay["pos"], np.int32)),
        _p(_c(lay["row_src"], np.int32)), _p(_c(lay["offsets"], np.int32)),
        N, K, E, H, cap, _p(out))
    return out


def combine_backward_weights(grad_out: np.ndarray, y: np.ndarray,
                             pos: np.ndarray) -> np.ndarray:
    """grad of the route weights [N,K], in double precision."""
    g = _c(grad_out, np.uint16)
    y = _c(y, np.uint16)
    pos = _c(pos, np.int32)
    N, H = g.shape
    K = pos.shape[1]
    out = np.empty((N, K), np.float64)
    lib().oracle_combine_backward_weights(_p(g), _p(y), _p(pos), N, K, H,
                                          y.shape[0], _p(out))
    return out


def gather_row_values(row_vals: np.ndarray, pos: np.ndarray) -> np.ndarray:
    v = _c(row_vals, np.float32)
    pos = _c(pos, np.int32)
    N, K = pos.shape
    out = np.empty((N, K), np.float32)
    lib().oracle_gather_row_values(_p(v), _p(pos), N, K, v.shape[0], _p(out))
    return out


# --- balanced plan and prefetch ---------------------------------------------

def plan_balanced(counts: np.ndarray, R: int, S: int, K: int, B: int):
    counts = _c(counts, np.int32)
    E = counts.shape[0]
    cu = np.full((R, E + 1), -9, np.int32)
    ex = np.full((R, E), -9, np.int32)
    wr = np.full((R, E), -9, np.int32)
    nseg = np.full(R, -9, np.int32)
    slots = np.full((R, max(B, 1)), -9, np.int32)[:, :B].copy()
    st = lib().oracle_plan_balanced(_p(counts), R, S, K, E, B, _p(cu), _p(ex),
                                    _p(wr), _p(nseg), _p(slots))
    return dict(cu=cu, expert=ex, wrow=wr, nseg=nseg, slot_expert=slots,
                status=st)


def reduce_slot_grads(slot_expert: np.ndarray, E: int,
                      G: np.ndarray) -> np.ndarray:
    """-> a copy of the fp32 gradient buffer G [E+R*B, ...] with every used
    slot's gradient added into its expert's row, in (d, b) order."""
    slot_expert = _c(slot_expert, np.int32)
    R, B = slot_expert.shape
    G = np.array(G, dtype=np.float32, order="C", copy=True)
    elems = int(np.prod(G.shape[1:]))
    lib().oracle_reduce_slot_grads(_p(slot_expert), R, E, B, elems, _p(G))
    return G


def prefetch(slot_expert: np.ndarray, E: int, W: np.ndarray) -> np.ndarray:
    """-> a copy of W [E+R*B, ...] (16-bit elements) with the slots filled."""
    slot_expert = _c(slot_expert, np.int32)
    R, B = slot_expert.shape
    W = np.array(W, dtype=np.uint16, order="C", copy=True)
    elems = int(np.prod(W.shape[1:]))
    lib().oracle_prefetch(_p(slot_expert), R, E, B, elems, _p(W))
    return W
