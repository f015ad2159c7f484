"""The whole path on the five workloads: layout -> dispatch -> combine
through EPBuffer, at full size, with identity experts: for bf16 dispatch and
weights summing to one, combine(dispatch(x)) must return x bit for bit (the
round trip the pages describe), for FP8 within the E4M3 error bound. The
layout is compared with the oracle here as well; every receive row, scale
and combined token of the same workloads is compared with the oracle in
test_fullsize_gpu.py."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from combine_ep_layout_09_b200 import EPBuffer
from gpu_util import to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["tiny", "prefill", "decode", "skewed",
                                  "balanced"])
def test_round_trip(name):
    wl = workloads.WORKLOADS[name]
    topk, w = workloads.routing(wl)
    hid = workloads.hidden_states(wl, device="cuda:0")
    buf = EPBuffer(wl.S, wl.H, wl.K, wl.E, wl.R, token_padding=wl.pad,
                   fp8=wl.fp8)
    wd = to_dev(w)
    recv, recv_w, offsets, handle = buf.dispatch(hid, wd, to_dev(topk))
    scales = handle.recv_scales
    o = oracle.layout(topk, wl.E, wl.pad, buf.cap)
    np.testing.assert_array_equal(buf.pos.cpu().numpy(), o["pos"])
    np.testing.assert_array_equal(offsets.cpu().numpy(), o["offsets"])
    used = int(o["offsets"][-1])
    if wl.fp8:
        # identity experts on the dequantised rows
        y = (recv[:used].float() *
             scales[:used].repeat_interleave(128, dim=1)).to(torch.bfloat16)
    else:
        y = recv[:used]
    out, gathered = buf.combine(handle, y.contiguous())
    np.testing.assert_array_equal(gathered.cpu().numpy(), w)
    buf.check()
    x = hid.float()
    if wl.fp8:
        err = (out.float() - x).abs()
        amax = x.abs().view(wl.N, wl.H // 128, 128).amax(-1)
        amax = amax.repeat_interleave(128, dim=1)
        bound = x.abs() * (2.0 ** -4 + 2.0 ** -7) + amax / 448 * 2.0 ** -9
        assert bool((err <= bound * 1.01 + 1e-30).all())
    else:
        assert torch.equal(out.view(torch.int16), hid.view(torch.int16))
