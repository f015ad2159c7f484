"""num_sms partitioning ("DeepSeek开源周第二天：DeepEP深度分析", "DeepEP介绍":
SM-count control, so that communication overlaps computation): the dispatch
and combine limited to part of the SMs run on one stream while a GEMM runs
on another, and their results are still exact."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_util import DEV, to_dev, u16
import combine_ep_layout_09_b200 as ep

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("fp8", [False, True])
def test_dispatch_and_combine_beside_a_gemm(fp8):
    wl = workloads.scaled(workloads.WORKLOADS["prefill"], S=600, H=1024,
                          fp8=fp8)
    topk, w = workloads.routing(wl)
    hid = workloads.hidden_states(wl, device=DEV)
    buf = ep.EPBuffer(wl.S, wl.H, wl.K, wl.E, wl.R, num_sms=74, fp8=fp8,
                      device=DEV)
    a = torch.randn(4096, 4096, device=DEV, dtype=torch.bfloat16)
    y = workloads.expert_outputs(buf.cap, wl.H, 5, device=DEV)
    s_gemm, s_ep = torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()
    with torch.cuda.stream(s_gemm):
        for _ in range(4):
            c = a @ a
    with torch.cuda.stream(s_ep):
        recv, recv_w, off, hd = buf.dispatch(hid, to_dev(w), to_dev(topk))
        out, _ = buf.combine(hd, y)
    torch.cuda.synchronize()
    buf.check()
    # the GEMM that ran beside them gives what it gives alone
    c_alone = a @ a
    torch.cuda.synchronize()
    assert torch.allclose(c.float(), c_alone.float(), rtol=1e-2, atol=1e-2)
    lay = oracle.layout(topk, wl.E, wl.pad, buf.cap)
    used = int(lay["offsets"][-1])
    np.testing.assert_array_equal(hd.pos.cpu().numpy(), lay["pos"])
    h = u16(hid)
    if fp8:
        q, s, rw = oracle.dispatch_fp8(h, w, lay, wl.E, buf.cap)
        np.testing.assert_array_equal(recv.view(torch.uint8).cpu().numpy()[:used], q[:used])
        np.testing.assert_array_equal(hd.recv_scales.cpu().numpy()[:used], s[:used])
    else:
        r, rw = oracle.dispatch_bf16(h, w, lay, wl.E, buf.cap)
        np.testing.assert_array_equal(u16(recv)[:used], r[:used])
    np.testing.assert_array_equal(recv_w.cpu().numpy()[:used], rw[:used])
    np.testing.assert_array_equal(u16(out), oracle.combine(u16(y), lay["pos"], w))
