"""Every wait site the kernels ship gives up cleanly.

ep_debug_force_timeouts makes the waits at one site ignore their condition,
as if nothing ever set it, for a short budget; the kernel must then take its
give-up path: report EP_DEV_TIMEOUT, drain the copies it has in flight and
return. Nothing faults or hangs: the stall is made inside the wait, not by a
missing producer. Each test checks the status, that no byte outside the
call's buffers (guard rows past `cap`) was written, and that the next normal
call on the same context is bit-exact against the oracle.
"""
import contextlib

import numpy as np
import pytest
import torch

import combine_ep_layout_09_b200 as ep
import oracle
import workloads
from gpu_util import (DEV, RECV_BF16_FILL, RECV_FP8_FILL, ROW_SRC_FILL,
                      gpu_layout, status_tensor, to_bf16_dev, to_dev, u16)

pytestmark = pytest.mark.gpu

BUDGET_NS = 200_000   # 0.2 ms per forced wait
GUARD = 64            # rows past cap that no call may touch


@contextlib.contextmanager
def forced(sites):
    torch.cuda.synchronize()
    ep.ep_debug_force_timeouts(sites, BUDGET_NS)
    try:
        yield
    finally:
        torch.cuda.synchronize()
        ep.ep_debug_force_timeouts(0)


def layout_bufs(N, K, E, cap):
    i32 = dict(dtype=torch.int32, device=DEV)
    return dict(counts=torch.full((E,), -9, **i32),
                offsets=torch.full((E + 1,), -9, **i32),
                pos=torch.full((N, K), -9, **i32),
                row_src=torch.full((cap + GUARD,), ROW_SRC_FILL, **i32),
                ws=torch.randint(0, 255, (ep.ep_layout_workspace_bytes(N, K, E),),
                                 dtype=torch.uint8, device=DEV),
                status=status_tensor())


def run_layout(topk_dev, R, S, K, E, pad, cap):
    b = layout_bufs(R * S, K, E, cap)
    ep.ep_layout(topk_dev, R, S, K, E, pad, b["counts"], b["offsets"],
                 b["pos"], b["row_src"], b["ws"], b["status"], cap=cap)
    torch.cuda.synchronize()
    return b


def check_layout(b, topk, E, pad, cap):
    o = oracle.layout(topk, E, pad, cap)
    np.testing.assert_array_equal(b["counts"].cpu().numpy(), o["counts"])
    np.testing.assert_array_equal(b["offsets"].cpu().numpy(), o["offsets"])
    np.testing.assert_array_equal(b["pos"].cpu().numpy(), o["pos"])
    np.testing.assert_array_equal(b["row_src"][:cap].cpu().numpy(),
                                  o["row_src"])
    return o


@pytest.mark.parametrize("site,R,S", [
    # more tiles of 4096 entries than can be resident: histogram + look-back
    (ep.EP_WAIT_SITE_LOOKBACK, 8, 128000),
    # every tile resident: one cooperative launch waiting for all tiles
    (ep.EP_WAIT_SITE_TILE_REDUCE, 8, 4096),
])
def test_layout_waits_give_up(site, R, S):
    K, E, pad = 8, 256, 1
    rng = np.random.default_rng(site)
    topk = rng.integers(0, E, size=(R * S, K)).astype(np.int32)
    t = to_dev(topk)
    cap = ep.ep_capacity_bound(R * S, K, E, pad)
    with forced(site):
        b = run_layout(t, R, S, K, E, pad, cap)
    st = int(b["status"][0].item())
    assert st & ep.EP_DEV_TIMEOUT
    assert not st & ep.EP_DEV_BAD_EXPERT
    assert bool((b["row_src"][cap:] == ROW_SRC_FILL).all())
    pos = b["pos"]
    assert int(pos.min().item()) >= 0 and int(pos.max().item()) < cap
    # the same context, normal waits: exact again
    b = run_layout(t, R, S, K, E, pad, cap)
    assert int(b["status"][0].item()) == 0
    check_layout(b, topk, E, pad, cap)


def dispatch_case(fp8, N=4000, K=8, E=64, H=1024, pad=4, seed=5):
    rng = np.random.default_rng(seed)
    topk, w = workloads.random_topk(rng, N, K, E)
    h = u16(workloads.bf16_normal((N, H), seed).to(torch.bfloat16))
    return topk, w, h


def dispatch_bufs(cap, H, fp8):
    rows = cap + GUARD
    if fp8:
        recv = torch.full((rows, H), RECV_FP8_FILL, dtype=torch.uint8,
                          device=DEV)
        scales = torch.full((rows, H // 128), -5.0, dtype=torch.float32,
                            device=DEV)
    else:
        recv = torch.full((rows, H), RECV_BF16_FILL, dtype=torch.int16,
                          device=DEV).view(torch.bfloat16)
        scales = None
    recv_w = torch.full((rows,), -3.0, dtype=torch.float32, device=DEV)
    return recv, scales, recv_w


def guards_intact(recv, scales, recv_w, cap, fp8):
    if fp8:
        tail, fill = recv[cap:].view(torch.uint8), RECV_FP8_FILL
    else:
        tail = recv[cap:].view(torch.int16)
        fill = int(np.array(RECV_BF16_FILL, np.uint16).view(np.int16))
    ok = bool((tail == fill).all())
    ok &= bool((recv_w[cap:] == -3.0).all())
    if fp8:
        ok &= bool((scales[cap:] == -5.0).all())
    return ok


def check_dispatch(recv, scales, recv_w, topk, w, h, E, pad, cap, fp8):
    o = oracle.layout(topk, E, pad, cap)
    if fp8:
        r, s, rw = oracle.dispatch_fp8(h, w, o, E, cap, recv_fill=RECV_FP8_FILL,
                                       scale_fill=-5.0, recv_w_fill=-3.0)
        np.testing.assert_array_equal(recv[:cap].cpu().numpy(), r)
        np.testing.assert_array_equal(scales[:cap].cpu().numpy(), s)
    else:
        r, rw = oracle.dispatch_bf16(h, w, o, E, cap, recv_fill=RECV_BF16_FILL,
                                     recv_w_fill=-3.0)
        np.testing.assert_array_equal(u16(recv[:cap]), r)
    np.testing.assert_array_equal(recv_w[:cap].cpu().numpy(), rw)


@pytest.mark.parametrize("fp8", [False, True])
def test_dispatch_waits_give_up(fp8):
    E, pad, H = 64, 4, 1024
    topk, w, h = dispatch_case(fp8, E=E, H=H, pad=pad)
    N, K = topk.shape
    g = gpu_layout(topk, 1, N, E, pad)
    cap = g["dev"]["cap"]
    hid, wd = to_bf16_dev(h), to_dev(w)

    def run():
        recv, scales, recv_w = dispatch_bufs(cap, H, fp8)
        st = status_tensor()
        # on fewer SMs than the device has the dispatch runs its persistent
        # kernels, the ones with waits (on every SM it runs one CTA per
        # token, which waits on nothing)
        ep.ep_dispatch(hid, wd, g["dev"]["pos"], g["dev"]["row_src"],
                       g["dev"]["offsets"], N, K, E, H, fp8, recv, scales,
                       recv_w, num_sms=100, status=st, cap=cap)
        torch.cuda.synchronize()
        return recv, scales, recv_w, int(st[0].item())

    with forced(ep.EP_WAIT_SITE_DISPATCH):
        recv, scales, recv_w, st = run()
    assert st & ep.EP_DEV_TIMEOUT
    assert guards_intact(recv, scales, recv_w, cap, fp8)
    recv, scales, recv_w, st = run()
    assert st == 0
    check_dispatch(recv, scales, recv_w, topk, w, h, E, pad, cap, fp8)


@pytest.mark.parametrize("fp8,num_sms", [(False, 0), (True, 0), (False, 100),
                                         (True, 100)])
def test_layout_dispatch_large_batch_gives_up(fp8, num_sms):
    # the layout kernel, then the dispatch kernel launched as its programmatic
    # dependent; both sites forced at once
    E, pad, H, R = 64, 1, 1024, 4
    topk, w, h = dispatch_case(fp8, N=4096 * R, E=E, H=H, pad=pad, seed=6)
    N, K = topk.shape
    S = N // R
    cap = ep.ep_capacity_bound(N, K, E, pad)
    hid, wd, t = to_bf16_dev(h), to_dev(w), to_dev(topk)

    def run():
        b = layout_bufs(N, K, E, cap)
        recv, scales, recv_w = dispatch_bufs(cap, H, fp8)
        ep.ep_layout_dispatch(t, hid, wd, R, S, K, E, H, pad, fp8, b["counts"],
                              b["offsets"], b["pos"], b["row_src"], recv,
                              scales, recv_w, workspace=b["ws"],
                              num_sms=num_sms, status=b["status"], cap=cap)
        torch.cuda.synchronize()
        return b, recv, scales, recv_w

    with forced(ep.EP_WAIT_SITE_DISPATCH | ep.EP_WAIT_SITE_TILE_REDUCE):
        b, recv, scales, recv_w = run()
    assert int(b["status"][0].item()) & ep.EP_DEV_TIMEOUT
    assert guards_intact(recv, scales, recv_w, cap, fp8)
    assert bool((b["row_src"][cap:] == ROW_SRC_FILL).all())
    b, recv, scales, recv_w = run()
    assert int(b["status"][0].item()) == 0
    check_layout(b, topk, E, pad, cap)
    check_dispatch(recv, scales, recv_w, topk, w, h, E, pad, cap, fp8)


@pytest.mark.parametrize("fp8,num_sms", [
    (True, 0),      # decode shape: one chunk of ~7 tokens per SM
    (False, 0),
    (False, 8),     # 128 tokens per CTA: several batches of staged rows
    (True, 8),
])
def test_small_batch_waits_give_up(fp8, num_sms):
    wl = workloads.WORKLOADS["decode"]
    topk, w = workloads.routing(wl)
    h = u16(workloads.hidden_states(wl))
    R, S, K, E, H, pad = wl.R, wl.S, wl.K, wl.E, wl.H, 1
    N = R * S
    cap = ep.ep_capacity_bound(N, K, E, pad)
    hid, wd, t = to_bf16_dev(h), to_dev(w), to_dev(topk)

    def run():
        b = layout_bufs(N, K, E, cap)
        recv, scales, recv_w = dispatch_bufs(cap, H, fp8)
        ep.ep_layout_dispatch(t, hid, wd, R, S, K, E, H, pad, fp8, b["counts"],
                              b["offsets"], b["pos"], b["row_src"], recv,
                              scales, recv_w, workspace=b["ws"],
                              num_sms=num_sms, status=b["status"], cap=cap)
        torch.cuda.synchronize()
        return b, recv, scales, recv_w

    with forced(ep.EP_WAIT_SITE_SMALL):
        b, recv, scales, recv_w = run()
    assert int(b["status"][0].item()) & ep.EP_DEV_TIMEOUT
    assert guards_intact(recv, scales, recv_w, cap, fp8)
    b, recv, scales, recv_w = run()
    assert int(b["status"][0].item()) == 0
    check_layout(b, topk, E, pad, cap)
    check_dispatch(recv, scales, recv_w, topk, w, h, E, pad, cap, fp8)


# the persistent pipeline on every SM (0) and on fewer (100)
@pytest.mark.parametrize("num_sms", [0, 100])
def test_combine_waits_give_up(num_sms):
    # enough (token, part) units per SM for the bulk-copy kernels
    N, K, H, rows = 2500, 8, 1024, 9000
    rng = np.random.default_rng(8)
    y = u16(workloads.bf16_normal((rows, H), 9))
    pos = rng.integers(0, rows, size=(N, K)).astype(np.int32)
    w = rng.standard_normal((N, K)).astype(np.float32)
    yd, pd, wd = to_bf16_dev(y), to_dev(pos), to_dev(w)

    def run():
        out = torch.full((N + GUARD, H), RECV_BF16_FILL, dtype=torch.int16,
                         device=DEV).view(torch.bfloat16)
        st = status_tensor()
        ep.ep_combine(yd, pd, wd, N, K, H, out, num_sms=num_sms, status=st)
        torch.cuda.synchronize()
        return out, int(st[0].item())

    with forced(ep.EP_WAIT_SITE_COMBINE):
        out, st = run()
    assert st & ep.EP_DEV_TIMEOUT
    fill = int(np.array(RECV_BF16_FILL, np.uint16).view(np.int16))
    assert bool((out[N:].view(torch.int16) == fill).all())
    out, st = run()
    assert st == 0
    np.testing.assert_array_equal(u16(out[:N]), oracle.combine(y, pos, w))


def test_prefetch_waits_give_up():
    rng = np.random.default_rng(10)
    R, B, E = 8, 4, 64
    rows = E + R * B
    shape = (rows + GUARD, 3, 5000)
    W = [rng.integers(0, 65535, size=shape, dtype=np.uint16)
         for _ in range(3)]
    slots = rng.integers(0, E, size=(R, B)).astype(np.int32)
    slots[rng.random(slots.shape) < 0.3] = -1

    def run():
        dev = [to_dev(x.view(np.int16)).view(torch.bfloat16) for x in W]
        st = status_tensor()
        ep.ep_prefetch_weights(to_dev(slots), R, E, B,
                               *[d[:rows] for d in dev], status=st)
        torch.cuda.synchronize()
        return dev, int(st[0].item())

    with forced(ep.EP_WAIT_SITE_PREFETCH):
        dev, st = run()
    assert st & ep.EP_DEV_TIMEOUT
    for x, d in zip(W, dev):
        got = d.view(torch.int16).cpu().numpy().view(np.uint16)
        np.testing.assert_array_equal(got[rows:], x[rows:])
        np.testing.assert_array_equal(got[:E], x[:E])
    dev, st = run()
    assert st == 0
    for x, d in zip(W, dev):
        got = d.view(torch.int16).cpu().numpy().view(np.uint16)
        np.testing.assert_array_equal(got[:rows],
                                      oracle.prefetch(slots, E, x[:rows]))
        np.testing.assert_array_equal(got[rows:], x[rows:])


def test_forcing_off_by_default_and_cleared():
    # sites = 0 is the default: a call after clearing takes no forced wait
    ep.ep_debug_force_timeouts(0)
    topk = np.random.default_rng(11).integers(0, 8, (64, 2)).astype(np.int32)
    assert gpu_layout(topk, 2, 32, 8, 1)["status"] == 0
