"""GPU ep_layout_dispatch (layout and dispatch of a small batch in one
launch, or the two separate launches above its size limit) against the
oracle: counts, offsets, pos and row_src, the bf16 or FP8 payload, scales
and receive weights bit-exact; padding rows zero; rows past the used region
untouched."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_util import (RECV_BF16_FILL, RECV_FP8_FILL, RECV_W_FILL,
                      ROW_SRC_FILL, SCALE_FILL, gpu_dispatch, gpu_layout,
                      gpu_layout_dispatch, to_bf16_dev, u16)

pytestmark = pytest.mark.gpu


def make(seed, N, K, E, H, distinct=False):
    rng = np.random.default_rng(seed)
    topk, w = workloads.random_topk(rng, N, K, E, distinct=distinct)
    hid = workloads.bf16_normal((max(N, 1), H), seed)
    return topk, w, u16(hid.to(torch.bfloat16))


def check(topk, w, hidden, R, S, E, pad, fp8, num_sms=0, with_weights=True,
          cap=None, expect_status=0):
    N, K = topk.shape
    H = hidden.shape[1]
    g = gpu_layout_dispatch(topk, to_bf16_dev(hidden), w, R, S, E, pad, fp8,
                            num_sms=num_sms, with_weights=with_weights,
                            cap=cap)
    cap = g["cap"]
    o = oracle.layout(topk, E, pad, cap=cap, row_src_fill=ROW_SRC_FILL)
    np.testing.assert_array_equal(g["counts"], o["counts"])
    np.testing.assert_array_equal(g["offsets"], o["offsets"])
    np.testing.assert_array_equal(g["pos"], o["pos"])
    np.testing.assert_array_equal(g["row_src"], o["row_src"])
    assert g["status"] == expect_status
    hid = hidden[:N]
    if fp8:
        r, s, rw = oracle.dispatch_fp8(hid, w, o, E, cap,
                                       recv_fill=RECV_FP8_FILL,
                                       scale_fill=SCALE_FILL,
                                       recv_w_fill=RECV_W_FILL)
        np.testing.assert_array_equal(g["recv"].cpu().numpy()[:cap], r)
        np.testing.assert_array_equal(g["scales"].cpu().numpy()[:cap], s)
    else:
        r, rw = oracle.dispatch_bf16(hid, w, o, E, cap,
                                     recv_fill=RECV_BF16_FILL,
                                     recv_w_fill=RECV_W_FILL)
        np.testing.assert_array_equal(u16(g["recv"])[:cap], r)
    if with_weights:
        np.testing.assert_array_equal(g["recv_w"].cpu().numpy()[:cap], rw)
    return g


# R, S, K, E, H, pad: one launch (N*K <= 32768); chunks of ceil(N/148)
# tokens per CTA with a ragged last chunk, fewer tokens than SMs, padding,
# H not a multiple of 512 (scales stored by lanes), the widest rows, K = 32,
# E = 1024.
SMALL = [
    (4, 64, 2, 8, 256, 1),
    (8, 128, 8, 256, 7168, 1),
    (8, 128, 8, 256, 7168, 128),
    (1, 5, 8, 16, 512, 1),
    (1, 149, 4, 32, 384, 3),
    (3, 111, 5, 9, 640, 7),
    (2, 8, 8, 16, 32768, 1),
    (1, 300, 32, 64, 1024, 2),
    (2, 200, 8, 1024, 256, 1),
    (8, 512, 8, 256, 1024, 1),       # N*K = 32768 exactly
    (1, 1, 1, 1, 128, 1),
]


@pytest.mark.parametrize("R,S,K,E,H,pad", SMALL)
@pytest.mark.parametrize("fp8", [False, True])
def test_small_batch_one_launch(R, S, K, E, H, pad, fp8):
    topk, w, h = make(R * 7 + S + K + E + H + pad, R * S, K, E, H,
                      distinct=K <= E)
    check(topk, w, h, R, S, E, pad, fp8)


@pytest.mark.parametrize("fp8", [False, True])
def test_above_limit_two_launches(fp8):
    # N*K = 32776 > 32768: ep_layout then ep_dispatch inside the same call
    R, S, K, E, H = 1, 4097, 8, 64, 256
    topk, w, h = make(41, R * S, K, E, H, distinct=True)
    check(topk, w, h, R, S, E, 4, fp8)


@pytest.mark.parametrize("num_sms", [1, 3, 7, 200])
@pytest.mark.parametrize("fp8", [False, True])
def test_num_sms(num_sms, fp8):
    # fewer CTAs: longer chunks per CTA, rows staged through a reused ring;
    # 1 SM: the whole batch (64 tokens x 8 = 512 entries) in one CTA
    R, S, K, E, H = 2, 32, 8, 32, 2048
    topk, w, h = make(num_sms, R * S, K, E, H, distinct=True)
    check(topk, w, h, R, S, E, 2, fp8, num_sms=num_sms)


@pytest.mark.parametrize("fp8", [False, True])
def test_long_chunk_reuses_stages(fp8):
    # 3 SMs for 300 tokens of 16 KB: 100 rows per CTA through a ring of
    # 10 (fp8) or 12 (bf16) staged rows
    R, S, K, E, H = 1, 300, 3, 8, 8192
    topk, w, h = make(77, R * S, K, E, H, distinct=True)
    check(topk, w, h, R, S, E, 1, fp8, num_sms=3)


def test_decode_workload_matches_separate_calls():
    # the decode shape (1024 tokens, H=7168, FP8, group-limited top-8) in one
    # launch equals ep_layout followed by ep_dispatch, bit for bit
    wl = workloads.WORKLOADS["decode"]
    topk, w = workloads.routing(wl)
    hid = workloads.bf16_normal((wl.N, wl.H), 1000 + wl.seed)
    h = u16(hid.to(torch.bfloat16))
    g = check(topk, w, h, wl.R, wl.S, wl.E, wl.pad, wl.fp8)
    lay = gpu_layout(topk, wl.R, wl.S, wl.E, wl.pad)
    d = gpu_dispatch(to_bf16_dev(h), w, lay, wl.E, wl.fp8)
    np.testing.assert_array_equal(lay["pos"], g["pos"])
    np.testing.assert_array_equal(d["recv"].view(torch.uint8).cpu().numpy(),
                                  g["recv"].view(torch.uint8).cpu().numpy())
    np.testing.assert_array_equal(d["scales"].cpu().numpy(),
                                  g["scales"].cpu().numpy())


def test_without_weights_and_spare_capacity():
    R, S, K, E, H = 2, 50, 4, 8, 256
    topk, w, h = make(5, R * S, K, E, H, distinct=True)
    cap = 1000
    g = check(topk, w, h, R, S, E, 8, True, with_weights=False, cap=cap)
    used = g["offsets"][-1]
    assert np.all(g["row_src"][used:] == ROW_SRC_FILL)
    assert np.all(g["recv"].cpu().numpy()[used:] == RECV_FP8_FILL)


def test_bad_ids_flagged_and_skipped():
    R, S, K, E, H = 2, 100, 4, 16, 256
    topk, w, h = make(9, R * S, K, E, H)
    topk[3, 1] = 16
    topk[150, 0] = -1
    topk[199, 3] = 1 << 30
    g = check(topk, w, h, R, S, E, 2, True, expect_status=1)
    assert g["pos"][3, 1] == -1 and g["pos"][150, 0] == -1


def test_empty_batch():
    topk = np.zeros((0, 4), np.int32)
    w = np.zeros((0, 4), np.float32)
    h = np.zeros((1, 256), np.uint16)
    g = gpu_layout_dispatch(topk, to_bf16_dev(h), w, 4, 0, 8, 16, True)
    assert np.all(g["counts"] == 0) and np.all(g["offsets"] == 0)
    assert g["status"] == 0


@pytest.mark.parametrize("fp8", [False, True])
def test_widest_rows_single_stage_ring(fp8):
    # H = 32768 on 2 SMs: 4 tokens per CTA through one FP8 stage (rows of
    # 64 KB plus a 33 KB output) or three bf16 stages
    R, S, K, E, H = 1, 8, 4, 8, 32768
    topk, w, h = make(13, R * S, K, E, H, distinct=True)
    check(topk, w, h, R, S, E, 2, fp8, num_sms=2)


@pytest.mark.parametrize("fp8", [False, True])
def test_duplicate_ids_single_expert_and_wide_padding(fp8):
    # ids repeat inside a token (K > E), one expert takes every entry, and
    # a padding of 1000 rows per expert dwarfs the batch
    R, S, K, E, H = 2, 60, 4, 2, 256
    rng = np.random.default_rng(17)
    topk = rng.integers(0, E, size=(R * S, K)).astype(np.int32)
    w = rng.random((R * S, K)).astype(np.float32)
    h = u16(workloads.bf16_normal((R * S, H), 17).to(torch.bfloat16))
    check(topk, w, h, R, S, E, 1, fp8)
    check(np.full((R * S, K), 1, np.int32), w, h, R, S, E, 7, fp8)
    check(topk, w, h, R, S, E, 1000, fp8)


@pytest.mark.parametrize("fp8", [False, True])
def test_small_batch_on_one_sm_takes_two_launches(fp8):
    # 256 tokens x 8 on one SM would put 2048 entries on one CTA, above its
    # limit of 1024: the call runs the layout and dispatch kernels instead
    R, S, K, E, H = 2, 128, 8, 32, 1024
    topk, w, h = make(23, R * S, K, E, H, distinct=True)
    check(topk, w, h, R, S, E, 2, fp8, num_sms=1)
