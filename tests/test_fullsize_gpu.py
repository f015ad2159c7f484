"""Parity at full size on all five workloads, in the launch configuration the
benchmark times.

One step of bench.Path on the benchmark's own inputs: ep_layout_dispatch
(the one-launch kernel for the decode batch, the cooperative layout and the
dispatch kernel as its programmatic dependent otherwise), the balanced plan
and the weight prefetch on the balanced workload, then ep_combine on the
stand-in expert outputs. Every output is compared with the oracle on every
row and every token, not a sample:
  * layout: tokens_per_expert, expert_offsets, pos, row_src (bit-exact);
  * dispatch: the whole receive buffer (bf16 rows or E4M3 codes), the FP8
    scales and the receive weights, including the padding rows and the
    untouched rows past off[E] ("MoonEP核心功能深度剖析", "2. 高效通信机制":
    final expert-grouped positions; "DeepSeek开源周第二天：DeepEP深度分析",
    "性能": FP8 dispatch, BF16 combine);
  * combine: every token's output (bit-exact, so within the 1-ulp bar);
  * balanced: the plan, and every slot row of the three projections against
    its source expert row, every other row unchanged ("MoonEP核心功能深度剖析",
    "1. 完美负载平衡", "3. 智能内存管理").
Device buffers are brought to the host in row chunks.
"""
import gc

import numpy as np
import pytest
import torch

import bench
import oracle
import workloads
from gpu_util import (DEV, RECV_BF16_FILL, RECV_FP8_FILL, RECV_W_FILL,
                      ROW_SRC_FILL, SCALE_FILL, assert_rows_equal, host_rows,
                      rows_to_host, u16)

pytestmark = pytest.mark.gpu

TOKEN_CHUNK = 2048    # tokens per combine comparison


def row_checksums(W: torch.Tensor) -> torch.Tensor:
    return W.view(W.shape[0], -1).view(torch.int64).sum(1)


@pytest.mark.parametrize("name", ["tiny", "prefill", "decode", "skewed",
                                  "balanced"])
def test_bench_step_matches_oracle_at_full_size(name):
    wl = workloads.WORKLOADS[name]
    path = bench.Path(wl, DEV)
    cap = path.cap
    # sentinels: rows the method must not touch keep them
    path.row_src.fill_(ROW_SRC_FILL)
    if wl.fp8:
        path.recv.view(torch.uint8).fill_(RECV_FP8_FILL)
        path.scales.fill_(SCALE_FILL)
    else:
        fill = int(np.array(RECV_BF16_FILL, np.uint16).view(np.int16))
        path.recv.view(torch.int16).fill_(fill)
    path.recv_w.fill_(RECV_W_FILL)
    path.out.view(torch.int16).fill_(-1)
    before = ([row_checksums(W) for W in path.W] if wl.B else None)
    path.status.zero_()
    path.step()
    torch.cuda.synchronize()
    assert int(path.status[0].item()) == 0

    topk, w = path.topk_np, path.w_np
    N, K, E, H = wl.N, wl.K, wl.E, wl.H

    # ---- layout -----------------------------------------------------------
    o = oracle.layout(topk, E, wl.pad, cap)
    assert o["status"] == 0
    np.testing.assert_array_equal(path.counts.cpu().numpy(), o["counts"])
    np.testing.assert_array_equal(path.offsets.cpu().numpy(), o["offsets"])
    np.testing.assert_array_equal(path.pos.cpu().numpy(), o["pos"])
    np.testing.assert_array_equal(path.row_src.cpu().numpy(), o["row_src"])

    # ---- dispatch: every receive row, scale and weight ----------------------
    h = u16(path.hidden)
    if wl.fp8:
        r, s, rw = oracle.dispatch_fp8(h, w, o, E, cap)
        assert_rows_equal(path.recv, r, "e4m3 codes")
        del r
        assert_rows_equal(path.scales, s, "scales")
    else:
        r, rw = oracle.dispatch_bf16(h, w, o, E, cap)
        assert_rows_equal(path.recv, r, "bf16 rows")
        del r
    np.testing.assert_array_equal(path.recv_w.cpu().numpy(), rw)
    del h
    gc.collect()

    # ---- combine: every token ----------------------------------------------
    # oracle.combine over each chunk's gathered rows: the K rows token t
    # reads are y[pos[t, :]], handed to the oracle in the same order
    for t0 in range(0, N, TOKEN_CHUNK):
        t1 = min(N, t0 + TOKEN_CHUNK)
        rows = o["pos"][t0:t1].ravel()
        ysel = rows_to_host(path.y, rows)
        local = np.arange(len(rows), dtype=np.int32).reshape(t1 - t0, K)
        ref = oracle.combine(ysel, local, w[t0:t1])
        got = host_rows(path.out, t0, t1)
        np.testing.assert_array_equal(got, ref, err_msg=f"tokens {t0}..{t1}")

    # ---- balanced plan and weight prefetch ---------------------------------
    if wl.B:
        p = oracle.plan_balanced(o["counts"], wl.R, wl.S, K, wl.B)
        assert p["status"] == 0
        np.testing.assert_array_equal(path.plan["cu"].cpu().numpy(), p["cu"])
        np.testing.assert_array_equal(path.plan["expert"].cpu().numpy(),
                                      p["expert"])
        np.testing.assert_array_equal(path.plan["wrow"].cpu().numpy(),
                                      p["wrow"])
        np.testing.assert_array_equal(path.plan["nseg"].cpu().numpy(),
                                      p["nseg"])
        slots = p["slot_expert"]
        np.testing.assert_array_equal(path.plan["slot"].cpu().numpy(), slots)
        assert (slots >= 0).sum() >= 1
        for W, b in zip(path.W, before):
            after = row_checksums(W)
            for d in range(wl.R):
                for j in range(wl.B):
                    row = E + d * wl.B + j
                    if slots[d, j] >= 0:
                        assert torch.equal(W[row], W[int(slots[d, j])])
                    else:
                        assert int(after[row]) == int(b[row])
            assert torch.equal(after[:E], b[:E])
    del path
    gc.collect()
    torch.cuda.empty_cache()
