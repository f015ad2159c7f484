"""GPU dispatch (bf16 copy and fused FP8 quantisation) against the oracle:
bit-exact payload, scales and weights; padding rows zero; rows past the used
region untouched."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_util import (DEV, RECV_BF16_FILL, RECV_FP8_FILL, RECV_W_FILL,
                      SCALE_FILL, gpu_dispatch, gpu_layout, status_tensor,
                      to_bf16_dev, to_dev, u16)

import combine_ep_layout_09_b200 as ep

pytestmark = pytest.mark.gpu


def make(seed, R, S, K, E, H, scale=1.0, distinct=False):
    rng = np.random.default_rng(seed)
    topk, w = workloads.random_topk(rng, R * S, K, E, distinct=distinct)
    hid = workloads.bf16_normal((R * S, H), seed) * scale
    return topk, w, u16(hid.to(torch.bfloat16))


def check_full(topk, w, hidden, R, S, E, H, pad, fp8, num_sms=0,
               with_weights=True):
    N, K = topk.shape
    g = gpu_layout(topk, R, S, E, pad)
    cap = g["dev"]["cap"]
    d = gpu_dispatch(to_bf16_dev(hidden), w, g, E, fp8,
                     with_weights=with_weights, num_sms=num_sms)
    assert d["status"] == 0
    o_lay = oracle.layout(topk, E, pad, cap)
    if fp8:
        r, s, rw = oracle.dispatch_fp8(hidden, w, o_lay, E, cap,
                                       recv_fill=RECV_FP8_FILL,
                                       scale_fill=SCALE_FILL,
                                       recv_w_fill=RECV_W_FILL)
        np.testing.assert_array_equal(d["recv"].cpu().numpy()[:cap], r)
        np.testing.assert_array_equal(d["scales"].cpu().numpy()[:cap], s)
    else:
        r, rw = oracle.dispatch_bf16(hidden, w, o_lay, E, cap,
                                     recv_fill=RECV_BF16_FILL,
                                     recv_w_fill=RECV_W_FILL)
        np.testing.assert_array_equal(u16(d["recv"])[:cap], r)
    if with_weights:
        np.testing.assert_array_equal(d["recv_w"].cpu().numpy()[:cap], rw)


# num_sms 0: one CTA per token; 100 (fewer SMs than the device has): the
# persistent kernels
@pytest.mark.parametrize("num_sms", [0, 100])
@pytest.mark.parametrize("R,S,K,E,H,pad", [
    (4, 64, 2, 8, 256, 1),          # tiny shape
    (2, 700, 8, 16, 7168, 1),       # several tiles, full row width
    (3, 333, 5, 9, 520, 3),         # row not a multiple of 512 channels
    (2, 257, 3, 8, 8, 4),           # one 16-byte vector per row
    (4, 100, 4, 16, 24, 128),       # odd vector count, heavy padding
    (1, 1, 1, 1, 16, 1),
])
def test_bf16(R, S, K, E, H, pad, num_sms):
    topk, w, h = make(R + S + K + E + H, R, S, K, E, H)
    check_full(topk, w, h, R, S, E, H, pad, fp8=False, num_sms=num_sms)


@pytest.mark.parametrize("num_sms", [0, 100])
@pytest.mark.parametrize("R,S,K,E,H,pad", [
    (4, 64, 2, 8, 256, 1),
    (2, 700, 8, 16, 7168, 1),
    (3, 333, 5, 9, 384, 3),
    (2, 301, 8, 32, 640, 128),
    (1, 1, 1, 1, 128, 1),
])
def test_fp8(R, S, K, E, H, pad, num_sms):
    topk, w, h = make(7 * (R + S + K + E + H), R, S, K, E, H)
    check_full(topk, w, h, R, S, E, H, pad, fp8=True, num_sms=num_sms)


@pytest.mark.parametrize("num_sms", [0, 100])
def test_fp8_extreme_values(num_sms):
    # huge, tiny, subnormal and zero groups, signed zeros, exact ties
    R, S, K, E, H = 2, 40, 3, 4, 512
    rng = np.random.default_rng(3)
    topk, w = workloads.random_topk(rng, R * S, K, E)
    x = rng.standard_normal((R * S, H)).astype(np.float32)
    x[0] *= 1e30
    x[1] *= 1e-30
    x[2, :128] = 0.0
    x[2, 128:256] = -0.0
    x[3] = 0.0
    x[4, 0] = 1.0
    x[4, 1:128] = 1.0 / 448 * 1.0625       # exact ties after scaling
    x[5, :] = 3e-39                        # bf16 subnormal group
    x[6, ::2] = -x[6, ::2]
    h = (x.view(np.uint32) >> 16).astype(np.uint16)   # truncate to bf16
    check_full(topk, w, h, R, S, E, H, 1, fp8=True, num_sms=num_sms)


@pytest.mark.parametrize("num_sms", [0, 100])
def test_fp8_scale_for_every_bf16_amax(num_sms):
    # one 128-channel group per finite non-negative bf16 value v: its largest
    # magnitude is v (signs alternate), so the kernels' scale RN(v/448) is
    # checked against the oracle's division for every amax a bf16 row can
    # have, and the group's codes with it
    H, G = 7168, 56
    vals = (np.arange(0, 0x7f80, dtype=np.uint32) << 16).view(np.float32)
    n_groups = -(-len(vals) // G) * G
    amax = np.resize(vals, n_groups)
    rng = np.random.default_rng(11)
    x = amax[:, None] * rng.uniform(-1.0, 1.0, (n_groups, 128)).astype(np.float32)
    x[:, 0] = amax * np.where(np.arange(n_groups) % 2 == 0, 1.0, -1.0)
    # truncate to bf16: magnitudes never rise above the group's amax
    h = (np.ascontiguousarray(x, np.float32).view(np.uint32) >> 16).astype(np.uint16)
    h = h.reshape(-1, H)
    N = h.shape[0]
    topk = np.zeros((N, 1), np.int32)
    w = rng.random((N, 1)).astype(np.float32)
    check_full(topk, w, h, 1, N, 1, H, 1, fp8=True, num_sms=num_sms)


@pytest.mark.parametrize("fp8", [False, True])
def test_rows_16_byte_aligned_only(fp8):
    # hidden and the receive rows start 16 bytes past a 32-byte boundary, so
    # the per-token kernels take their 16-byte access forms
    R, S, K, E, H, pad = 2, 300, 8, 16, 7168, 1
    topk, w, h = make(404, R, S, K, E, H)
    N = R * S
    g = gpu_layout(topk, R, S, E, pad)
    cap = g["dev"]["cap"]
    base = torch.empty(N * H + 8, dtype=torch.int16, device=DEV)
    hid = base[8:].view(N, H)
    hid.copy_(torch.from_numpy(h.view(np.int16)).to(DEV))
    hid = hid.view(torch.bfloat16)
    assert hid.data_ptr() % 32 == 16
    if fp8:
        rbase = torch.full((cap * H + 16,), RECV_FP8_FILL, dtype=torch.uint8,
                           device=DEV)
        recv = rbase[16:].view(cap, H)
        scales = torch.full((cap, H // 128), SCALE_FILL, dtype=torch.float32,
                            device=DEV)
    else:
        rbase = torch.full((cap * H + 8,), RECV_BF16_FILL, dtype=torch.int16,
                           device=DEV)
        recv = rbase[8:].view(cap, H).view(torch.bfloat16)
        scales = None
    assert recv.data_ptr() % 32 == 16
    recv_w = torch.full((cap,), RECV_W_FILL, dtype=torch.float32, device=DEV)
    st = status_tensor()
    ep.ep_dispatch(hid, to_dev(w), g["dev"]["pos"], g["dev"]["row_src"],
                   g["dev"]["offsets"], N, K, E, H, fp8, recv, scales, recv_w,
                   status=st, cap=cap)
    torch.cuda.synchronize()
    assert int(st[0].item()) == 0
    o_lay = oracle.layout(topk, E, pad, cap)
    if fp8:
        r, sc, rw = oracle.dispatch_fp8(h, w, o_lay, E, cap,
                                        recv_fill=RECV_FP8_FILL,
                                        scale_fill=SCALE_FILL,
                                        recv_w_fill=RECV_W_FILL)
        np.testing.assert_array_equal(recv.cpu().numpy(), r)
        np.testing.assert_array_equal(scales.cpu().numpy(), sc)
    else:
        r, rw = oracle.dispatch_bf16(h, w, o_lay, E, cap,
                                     recv_fill=RECV_BF16_FILL,
                                     recv_w_fill=RECV_W_FILL)
        np.testing.assert_array_equal(u16(recv), r)
    np.testing.assert_array_equal(recv_w.cpu().numpy(), rw)


@pytest.mark.parametrize("fp8", [False, True])
def test_without_weights_and_limited_sms(fp8):
    topk, w, h = make(99, 2, 500, 4, 8, 1024)
    check_full(topk, w, h, 2, 500, 8, 1024, 16, fp8=fp8, num_sms=3,
               with_weights=False)


def test_decode_full_size():
    wl = workloads.WORKLOADS["decode"]
    topk, w = workloads.routing(wl)
    h = u16(workloads.hidden_states(wl))
    check_full(topk, w, h, wl.R, wl.S, wl.E, wl.H, wl.pad, fp8=True)


@pytest.mark.parametrize("fp8", [False, True])
def test_k32(fp8):
    topk, w, h = make(321, 2, 200, 32, 64, 256, distinct=True)
    check_full(topk, w, h, 2, 200, 64, 256, 1, fp8=fp8)


@pytest.mark.parametrize("num_sms", [0, 100])
@pytest.mark.parametrize("fp8", [False, True])
def test_widest_row(fp8, num_sms):
    # H = 32768, the largest the ABI accepts: two input stages of 64 KB in
    # the persistent kernels, several passes of a CTA's warps per token
    topk, w, h = make(322, 1, 48, 3, 4, 32768)
    check_full(topk, w, h, 1, 48, 4, 32768, 1, fp8=fp8, num_sms=num_sms)


@pytest.mark.parametrize("fp8", [False, True])
def test_capacity_smaller_than_layout_is_reported(fp8):
    # dispatch told about fewer rows than the layout used: rows past cap
    # are skipped (never written) and EP_DEV_CAPACITY is raised
    topk, w, h = make(323, 2, 100, 4, 8, 256)
    g = gpu_layout(topk, 2, 100, 8, 1)
    half = g["dev"]["cap"] // 2
    g["dev"]["cap"] = half
    d = gpu_dispatch(to_bf16_dev(h), w, g, 8, fp8)
    assert d["status"] & 2                     # EP_DEV_CAPACITY
    assert d["recv"].shape[0] == half
    o = oracle.layout(topk, 8, 1)
    keep = o["pos"] < half
    rows = o["pos"][keep]
    toks = np.nonzero(keep)[0]
    if fp8:
        q, s = oracle.quantize_rows(h)
        np.testing.assert_array_equal(d["recv"].cpu().numpy()[rows], q[toks])
    else:
        np.testing.assert_array_equal(u16(d["recv"])[rows], h[toks])
