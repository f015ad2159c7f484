"""GPU backward pair against the oracle: dispatch backward bit-exact (it is
combine with unit weights), combine backward's row gradients bit-exact, its
route-weight gradients within the fp32 summation bound H * 2^-24 * sum|terms|
of the double-precision sum, gathered route weights bit-exact."""
import numpy as np
import pytest
import torch

import combine_ep_layout_09_b200 as ep
import oracle
import workloads
from gpu_util import (DEV, RECV_BF16_FILL, assert_rows_equal, gpu_layout,
                      host_rows, rows_to_host, status_tensor, to_bf16_dev,
                      to_dev, u16)

pytestmark = pytest.mark.gpu


def as_f32(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32)


@pytest.mark.parametrize("N,K,H,rows", [
    (40, 3, 64, 200), (700, 8, 7168, 6000), (2500, 8, 1024, 21000),
    (3000, 2, 520, 7000), (50, 9, 24, 600),
])
def test_dispatch_backward(N, K, H, rows):
    rng = np.random.default_rng(N + K)
    g = u16(workloads.bf16_normal((rows, H), N))
    pos = rng.integers(0, rows, size=(N, K)).astype(np.int32)
    pos[rng.random(pos.shape) < 0.05] = -1
    out = torch.full((N, H), RECV_BF16_FILL, dtype=torch.int16,
                     device=DEV).view(torch.bfloat16)
    st = status_tensor()
    ep.ep_dispatch_backward(to_bf16_dev(g), to_dev(pos), N, K, H, out,
                            status=st)
    torch.cuda.synchronize()
    assert int(st[0].item()) == 0
    np.testing.assert_array_equal(u16(out), oracle.dispatch_backward(g, pos))


def run_combine_backward(topk, w, R, S, E, H, pad, seed, num_sms=0):
    N, K = topk.shape
    lay = gpu_layout(topk, R, S, E, pad)
    cap = lay["dev"]["cap"]
    y = workloads.expert_outputs(cap, H, seed, device=DEV)
    g = workloads.bf16_normal((N, H), seed + 1, device=DEV)
    rows = torch.full((cap, H), RECV_BF16_FILL, dtype=torch.int16,
                      device=DEV).view(torch.bfloat16)
    gw = torch.full((N, K), -7.0, dtype=torch.float32, device=DEV)
    st = status_tensor()
    ep.ep_combine_backward(g, y, lay["dev"]["pos"], lay["dev"]["row_src"],
                           lay["dev"]["offsets"], to_dev(w), N, K, E, H, rows,
                           gw, num_sms=num_sms, status=st)
    torch.cuda.synchronize()
    assert int(st[0].item()) == 0
    return lay, cap, y, g, rows, gw


def weight_grad_ok(got, g_bits, y_rows_bits, K, H):
    """|got - exact| <= H * 2^-24 * sum|y*g| (+ a tiny absolute floor)."""
    gf = as_f32(g_bits).astype(np.float64)
    yf = as_f32(y_rows_bits).astype(np.float64).reshape(len(gf), K, -1)
    exact = np.einsum("tkh,th->tk", yf, gf)
    mag = np.einsum("tkh,th->tk", np.abs(yf), np.abs(gf))
    assert np.all(np.abs(got - exact) <= H * 2.0 ** -24 * mag + 1e-30)


# num_sms 0: one CTA per token; 100: persistent CTAs on fewer SMs
@pytest.mark.parametrize("num_sms", [0, 100])
@pytest.mark.parametrize("R,S,K,E,H,pad", [
    (4, 64, 2, 8, 256, 1), (2, 300, 8, 16, 7168, 4), (3, 200, 5, 9, 520, 128),
])
def test_combine_backward_small(R, S, K, E, H, pad, num_sms):
    rng = np.random.default_rng(R * S + K)
    topk, w = workloads.random_topk(rng, R * S, K, E)
    w = (w * rng.choice([-1.0, 1.0], w.shape) * 2).astype(np.float32)
    lay, cap, y, g, rows, gw = run_combine_backward(topk, w, R, S, E, H, pad,
                                                     R + S, num_sms=num_sms)
    o = oracle.layout(topk, E, pad, cap)
    ref_rows = oracle.combine_backward_rows(u16(g), w, o, E, cap,
                                            fill=RECV_BF16_FILL)
    np.testing.assert_array_equal(u16(rows), ref_rows)
    got = gw.cpu().numpy().astype(np.float64)
    y_rows = u16(y)[o["pos"].ravel()]
    weight_grad_ok(got, u16(g), y_rows, K, H)
    ref_w = oracle.combine_backward_weights(u16(g), u16(y), o["pos"])
    assert np.all(np.abs(got - ref_w) <= 1e-2 * np.abs(ref_w).max() + 1e-6)


@pytest.mark.parametrize("name", ["skewed", "prefill"])
def test_backward_full_size(name):
    # every row of the expert-output gradient (padding rows included) and
    # every token's route-weight gradient and token gradient, at full size
    wl = workloads.WORKLOADS[name]
    topk, w = workloads.routing(wl)
    lay, cap, y, g, rows, gw = run_combine_backward(topk, w, wl.R, wl.S, wl.E,
                                                     wl.H, wl.pad, 9)
    o = oracle.layout(topk, wl.E, wl.pad, cap)
    g_host = u16(g)
    ref_rows = oracle.combine_backward_rows(g_host, w, o, wl.E, cap,
                                            fill=RECV_BF16_FILL)
    assert_rows_equal(rows, ref_rows, "grad rows")
    del ref_rows
    gx = torch.empty(wl.N, wl.H, dtype=torch.bfloat16, device=DEV)
    st = status_tensor()
    ep.ep_dispatch_backward(rows, lay["dev"]["pos"], wl.N, wl.K, wl.H, gx,
                            status=st)
    torch.cuda.synchronize()
    assert int(st[0].item()) == 0
    gw_host = gw.cpu().numpy()
    chunk = 2048
    for t0 in range(0, wl.N, chunk):
        t1 = min(wl.N, t0 + chunk)
        r = o["pos"][t0:t1].ravel()
        local = np.arange(len(r), dtype=np.int32).reshape(t1 - t0, wl.K)
        y_rows = rows_to_host(y, r)
        weight_grad_ok(gw_host[t0:t1].astype(np.float64), g_host[t0:t1],
                       y_rows, wl.K, wl.H)
        gr_rows = rows_to_host(rows, r)
        np.testing.assert_array_equal(host_rows(gx, t0, t1),
                                      oracle.dispatch_backward(gr_rows, local))


def test_gather_route_weights():
    rng = np.random.default_rng(1)
    vals = rng.standard_normal(5000).astype(np.float32)
    pos = rng.integers(-1, 5000, size=(900, 7)).astype(np.int32)
    out = torch.zeros(900, 7, dtype=torch.float32, device=DEV)
    ep.ep_gather_route_weights(to_dev(vals), to_dev(pos), 900, 7, out)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(out.cpu().numpy(),
                                  oracle.gather_row_values(vals, pos))


def test_gradient_round_trip_identity_experts():
    # forward: out = combine(dispatch(x)) with identity experts; backward of
    # both with grad_out = g gives grad_x = sum_k w_k * g = g (weights sum to
    # one), up to two bf16 roundings
    wl = workloads.WORKLOADS["tiny"]
    topk, w = workloads.routing(wl)
    lay = gpu_layout(topk, wl.R, wl.S, wl.E, wl.pad)
    cap = lay["dev"]["cap"]
    g = workloads.bf16_normal((wl.N, wl.H), 77, device=DEV)
    y = workloads.expert_outputs(cap, wl.H, 1, device=DEV)   # unused by rows
    rows = torch.empty(cap, wl.H, dtype=torch.bfloat16, device=DEV)
    gw = torch.empty(wl.N, wl.K, dtype=torch.float32, device=DEV)
    ep.ep_combine_backward(g, y, lay["dev"]["pos"], lay["dev"]["row_src"],
                           lay["dev"]["offsets"], to_dev(w), wl.N, wl.K, wl.E,
                           wl.H, rows, gw)
    gx = torch.empty(wl.N, wl.H, dtype=torch.bfloat16, device=DEV)
    ep.ep_dispatch_backward(rows, lay["dev"]["pos"], wl.N, wl.K, wl.H, gx)
    torch.cuda.synchronize()
    a, b = gx.float(), g.float()
    assert bool(((a - b).abs() <= b.abs() * 2.0 ** -7 + 1e-30).all())
