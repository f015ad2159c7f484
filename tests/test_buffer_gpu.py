"""EPBuffer, the pages' Buffer call shape: dispatch -> (recv,
route_weights_nvs, cu_seqlens, plan), prefetch_weight(plan, ...), combine(plan,
expert_output, route_weights_nvs) -> (output, gathered_route_weights), with
double-buffered receive sets and the backward helpers."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from combine_ep_layout_09_b200 import EPBuffer
from gpu_util import DEV, to_dev, u16

pytestmark = pytest.mark.gpu


def test_double_buffer_keeps_the_previous_dispatch():
    wl = workloads.WORKLOADS["tiny"]
    topk, w = workloads.routing(wl)
    topk2 = np.roll(topk, 1, axis=0)
    buf = EPBuffer(wl.S, wl.H, wl.K, wl.E, wl.R, double_buffer=True)
    h1 = workloads.hidden_states(wl, device=DEV)
    h2 = workloads.bf16_normal((wl.N, wl.H), 99, device=DEV)
    r1, _, off1, hd1 = buf.dispatch(h1, to_dev(w), to_dev(topk))
    snap = r1.clone()
    pos1 = hd1.pos.clone()
    r2, _, off2, hd2 = buf.dispatch(h2, to_dev(w), to_dev(topk2))
    torch.cuda.synchronize()
    assert hd1.index != hd2.index and r1.data_ptr() != r2.data_ptr()
    assert torch.equal(r1.view(torch.int16), snap.view(torch.int16))
    assert torch.equal(hd1.pos, pos1)
    # a third dispatch reuses the first set (idx ^= 1)
    _, _, _, hd3 = buf.dispatch(h1, to_dev(w), to_dev(topk))
    assert hd3.index == hd1.index
    # each handle still combines its own batch: identity experts give x back
    out2, g2 = buf.combine(hd2, r2)
    torch.cuda.synchronize()
    assert torch.equal(out2.view(torch.int16), h2.view(torch.int16))
    np.testing.assert_array_equal(g2.cpu().numpy(), w)


def test_combine_uses_receive_side_weights():
    wl = workloads.WORKLOADS["tiny"]
    topk, w = workloads.routing(wl)
    buf = EPBuffer(wl.S, wl.H, wl.K, wl.E, wl.R)
    hid = workloads.hidden_states(wl, device=DEV)
    recv, recv_w, off, hd = buf.dispatch(hid, to_dev(w), to_dev(topk))
    y = workloads.expert_outputs(buf.cap, wl.H, 3, device=DEV)
    nvs = (recv_w * 0.5).contiguous()        # weights changed on the rows
    out, gathered = buf.combine(hd, y, nvs)
    torch.cuda.synchronize()
    lay = oracle.layout(topk, wl.E, wl.pad)
    np.testing.assert_array_equal(gathered.cpu().numpy(), w * np.float32(0.5))
    ref = oracle.combine(u16(y), lay["pos"], w * np.float32(0.5))
    np.testing.assert_array_equal(u16(out), ref)


def test_plan_prefetch_reduce_and_backward_through_the_buffer():
    wl = workloads.scaled(workloads.WORKLOADS["balanced"], S=256, H=512, I=16)
    topk, w = workloads.routing(wl)
    buf = EPBuffer(wl.S, wl.H, wl.K, wl.E, wl.R)
    hid = workloads.hidden_states(wl, device=DEV)
    recv, recv_w, off, hd = buf.dispatch(hid, to_dev(w), to_dev(topk))
    plan = buf.plan(hd, wl.B)
    rows = wl.E + wl.R * wl.B
    Ws = [workloads.weight_buffer(rows, wl.H, wl.I, j, device=DEV)
          for j in range(3)]
    buf.prefetch_weight(plan, *Ws)
    Gs = [torch.randn(rows, wl.H, wl.I, device=DEV) for _ in range(3)]
    G0 = [g.cpu().numpy() for g in Gs]
    buf.reduce_grads(plan, *Gs)
    torch.cuda.synchronize()
    buf.check()
    slots = plan["slot_expert"].cpu().numpy()[:, :wl.B]
    for g, g0 in zip(Gs, G0):
        np.testing.assert_array_equal(g.cpu().numpy(),
                                      oracle.reduce_slot_grads(slots, wl.E, g0))
    # backward of the round trip with identity experts returns the gradient
    grad_out = workloads.bf16_normal((wl.N, wl.H), 5, device=DEV)
    gy, gw = buf.combine_backward(hd, grad_out, recv, to_dev(w))
    gx = buf.dispatch_backward(hd, gy)
    torch.cuda.synchronize()
    a, b = gx.float(), grad_out.float()
    assert bool(((a - b).abs() <= b.abs() * 2.0 ** -7 + 1e-30).all())


def test_double_buffer_on_the_large_batch_kernels():
    # 4800 tokens x top-8: layout and dispatch are two kernels, the dispatch a
    # programmatic dependent of the layout; two batches in flight on the two
    # receive sets, each checked against the oracle afterwards
    wl = workloads.scaled(workloads.WORKLOADS["prefill"], S=600, H=512)
    topk, w = workloads.routing(wl)
    topk2 = np.roll(topk, 7, axis=0)
    buf = EPBuffer(wl.S, wl.H, wl.K, wl.E, wl.R, fp8=True, double_buffer=True)
    h1 = workloads.hidden_states(wl, device=DEV)
    h2 = workloads.bf16_normal((wl.N, wl.H), 77, device=DEV)
    r1, rw1, _, hd1 = buf.dispatch(h1, to_dev(w), to_dev(topk))
    r2, rw2, _, hd2 = buf.dispatch(h2, to_dev(w), to_dev(topk2))
    torch.cuda.synchronize()
    buf.check()
    for hid, tk, r, hd in ((h1, topk, r1, hd1), (h2, topk2, r2, hd2)):
        lay = oracle.layout(tk, wl.E, wl.pad, buf.cap)
        used = int(lay["offsets"][-1])
        np.testing.assert_array_equal(hd.pos.cpu().numpy(), lay["pos"])
        q, s, _ = oracle.dispatch_fp8(u16(hid), w, lay, wl.E, buf.cap)
        np.testing.assert_array_equal(r.view(torch.uint8).cpu().numpy()[:used],
                                      q[:used])
        np.testing.assert_array_equal(hd.recv_scales.cpu().numpy()[:used],
                                      s[:used])
