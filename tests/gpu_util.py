"""Helpers for the GPU parity tests: run the CUDA library through its Python
binding on numpy inputs and bring the results back as numpy arrays.

Output buffers are pre-filled with sentinels so that the tests can check
which rows the library wrote and which it left alone. The layout workspace
is pre-filled with garbage: the library must not rely on it being zero.
"""
import numpy as np
import torch

import combine_ep_layout_09_b200 as ep

DEV = torch.device("cuda:0")

ROW_SRC_FILL = -7
RECV_BF16_FILL = 0x7FBF      # a NaN bf16 pattern, never written by dispatch
RECV_FP8_FILL = 0xA5
SCALE_FILL = -5.0
RECV_W_FILL = -3.0


def u16(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> uint16 bit patterns (host)."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(
        np.uint16)


def to_bf16_dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(
        DEV).view(torch.bfloat16)


def to_dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def status_tensor():
    return torch.zeros(4, dtype=torch.int32, device=DEV)


def gpu_layout(topk: np.ndarray, R: int, S: int, E: int, pad: int,
               cap: int | None = None, topk_dev=None):
    N, K = topk.shape
    assert N == R * S
    if cap is None:
        cap = ep.ep_capacity_bound(N, K, E, pad)
    i32 = dict(dtype=torch.int32, device=DEV)
    counts = torch.full((E,), -9, **i32)
    offsets = torch.full((E + 1,), -9, **i32)
    pos = torch.full((max(N, 1), K), -9, **i32)
    row_src = torch.full((max(cap, 1),), ROW_SRC_FILL, **i32)
    wsb = ep.ep_layout_workspace_bytes(N, K, E)
    ws = torch.randint(0, 255, (max(wsb, 16),), dtype=torch.uint8,
                       device=DEV)
    st = status_tensor()
    t = topk_dev if topk_dev is not None else to_dev(
        topk.astype(np.int32) if N > 0 else np.zeros((1, K), np.int32))
    ep.ep_layout(t, R, S, K, E, pad, counts, offsets, pos, row_src, ws, st,
                 cap=cap)
    torch.cuda.synchronize()
    return dict(counts=counts.cpu().numpy(), offsets=offsets.cpu().numpy(),
                pos=pos[:N].cpu().numpy(), row_src=row_src[:cap].cpu().numpy(),
                status=int(st[0].item()),
                dev=dict(counts=counts, offsets=offsets, pos=pos,
                         row_src=row_src, topk=t, cap=cap))


def gpu_dispatch(hidden_dev: torch.Tensor, w: np.ndarray, lay: dict, E: int,
                 fp8: bool, with_weights: bool = True, num_sms: int = 0,
                 w_dev=None):
    d = lay["dev"]
    cap = d["cap"]
    N, H = hidden_dev.shape
    K = w.shape[1]
    rows = max(cap, 1)
    if fp8:
        recv = torch.full((rows, H), RECV_FP8_FILL, dtype=torch.uint8,
                          device=DEV)
        scales = torch.full((rows, H // 128), SCALE_FILL,
                            dtype=torch.float32, device=DEV)
    else:
        recv = torch.full((rows, H), RECV_BF16_FILL, dtype=torch.int16,
                          device=DEV).view(torch.bfloat16)
        scales = None
    recv_w = torch.full((rows,), RECV_W_FILL, dtype=torch.float32,
                        device=DEV) if with_weights else None
    st = status_tensor()
    wd = w_dev if w_dev is not None else to_dev(w.astype(np.float32))
    ep.ep_dispatch(hidden_dev, wd, d["pos"], d["row_src"], d["offsets"], N,
                   K, E, H, fp8, recv, scales, recv_w, num_sms=num_sms,
                   status=st, cap=cap)
    torch.cuda.synchronize()
    return dict(recv=recv, scales=scales, recv_w=recv_w,
                status=int(st[0].item()))


def gpu_combine(y_dev: torch.Tensor, pos_dev: torch.Tensor, w_dev, N: int,
                K: int, num_sms: int = 0):
    H = y_dev.shape[1]
    out = torch.full((max(N, 1), H), RECV_BF16_FILL, dtype=torch.int16,
                     device=DEV).view(torch.bfloat16)
    st = status_tensor()
    ep.ep_combine(y_dev, pos_dev, w_dev, N, K, H, out, num_sms=num_sms,
                  status=st)
    torch.cuda.synchronize()
    return out[:N], int(st[0].item())


def rows_to_host(t: torch.Tensor, rows: np.ndarray) -> np.ndarray:
    """Selected rows of a device tensor, as host numpy (uint8/uint16/f32)."""
    idx = torch.from_numpy(np.asarray(rows, np.int64)).to(DEV)
    sel = t.index_select(0, idx)
    if sel.dtype == torch.bfloat16:
        return u16(sel)
    if sel.dtype in (torch.uint8, torch.float8_e4m3fn):
        return sel.view(torch.uint8).cpu().numpy()
    return sel.cpu().numpy()


def gpu_layout_dispatch(topk: np.ndarray, hidden_dev: torch.Tensor,
                        w: np.ndarray, R: int, S: int, E: int, pad: int,
                        fp8: bool, num_sms: int = 0, with_weights: bool = True,
                        cap: int | None = None):
    """ep_layout_dispatch with sentinel-filled outputs (garbage workspace)."""
    N, K = topk.shape
    H = hidden_dev.shape[1]
    if cap is None:
        cap = ep.ep_capacity_bound(N, K, E, pad)
    rows = max(cap, 1)
    i32 = dict(dtype=torch.int32, device=DEV)
    counts = torch.full((E,), -9, **i32)
    offsets = torch.full((E + 1,), -9, **i32)
    pos = torch.full((max(N, 1), K), -9, **i32)
    row_src = torch.full((rows,), ROW_SRC_FILL, **i32)
    if fp8:
        recv = torch.full((rows, H), RECV_FP8_FILL, dtype=torch.uint8,
                          device=DEV)
        scales = torch.full((rows, H // 128), SCALE_FILL,
                            dtype=torch.float32, device=DEV)
    else:
        recv = torch.full((rows, H), RECV_BF16_FILL, dtype=torch.int16,
                          device=DEV).view(torch.bfloat16)
        scales = None
    recv_w = torch.full((rows,), RECV_W_FILL, dtype=torch.float32,
                        device=DEV) if with_weights else None
    wsb = ep.ep_layout_workspace_bytes(N, K, E)
    ws = torch.randint(0, 255, (max(wsb, 16),), dtype=torch.uint8,
                       device=DEV)
    st = status_tensor()
    t = to_dev(topk.astype(np.int32) if N > 0 else np.zeros((1, K), np.int32))
    wd = to_dev(w.astype(np.float32) if N > 0 else np.zeros((1, K), np.float32))
    ep.ep_layout_dispatch(t, hidden_dev, wd, R, S, K, E, H, pad, fp8, counts,
                          offsets, pos, row_src, recv, scales, recv_w,
                          workspace=ws, num_sms=num_sms, status=st, cap=cap)
    torch.cuda.synchronize()
    return dict(counts=counts.cpu().numpy(), offsets=offsets.cpu().numpy(),
                pos=pos[:N].cpu().numpy(), row_src=row_src[:cap].cpu().numpy(),
                recv=recv, scales=scales, recv_w=recv_w,
                status=int(st[0].item()), cap=cap)


ROW_CHUNK = 16384     # receive rows per device -> host copy


def host_rows(t: torch.Tensor, lo: int, hi: int) -> np.ndarray:
    """Rows [lo, hi) of a device tensor as host numpy bit patterns."""
    part = t[lo:hi]
    if part.dtype == torch.bfloat16:
        return u16(part)
    if part.dtype in (torch.uint8, torch.float8_e4m3fn):
        return part.view(torch.uint8).cpu().numpy()
    return part.cpu().numpy()


def assert_rows_equal(dev: torch.Tensor, ref: np.ndarray, what: str):
    """Every row of a device tensor equal to `ref`, compared in chunks of
    ROW_CHUNK rows so that the host holds one chunk of the device data."""
    assert dev.shape[0] == ref.shape[0], what
    for lo in range(0, ref.shape[0], ROW_CHUNK):
        hi = min(lo + ROW_CHUNK, ref.shape[0])
        got = host_rows(dev, lo, hi)
        if not np.array_equal(got, ref[lo:hi]):
            bad = np.nonzero((got != ref[lo:hi]).reshape(hi - lo, -1).any(1))[0]
            raise AssertionError(f"{what}: {len(bad)} rows differ in "
                                 f"[{lo}, {hi}), first {lo + int(bad[0])}")
