"""Pins for the oracle's backward pair (dispatch backward, combine backward)
and for gathering row values back into token order.

Dispatch backward is pinned as the adjoint of dispatch (fp64 inner products)
and against numpy's fancy-index sum. Combine backward's row gradient is
pinned against numpy fp32 multiplication + torch's bf16 cast. Its weight
gradient is pinned against finite differences of the double-precision
combine in each weight (combine is linear in w) and against numpy einsum.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def as_f32(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32)


def torch_bf16_bits(x: np.ndarray) -> np.ndarray:
    return bf16_bits(torch.from_numpy(np.asarray(x, np.float32)).to(
        torch.bfloat16))


def case(seed, N=48, K=3, E=7, H=64, pad=4):
    rng = np.random.default_rng(seed)
    topk, w = workloads.random_topk(rng, N, K, E)
    lay = oracle.layout(topk, E, pad)
    cap = oracle.capacity_bound(N, K, E, pad) + 3
    return rng, topk, w, lay, cap


def ulp_bf16(v):
    a = np.abs(v)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.exp2(np.maximum(e, -126) - 7)


@pytest.mark.parametrize("seed", range(4))
def test_dispatch_backward_is_the_adjoint(seed):
    rng, topk, w, lay, cap = case(seed)
    N, K = topk.shape
    H = 64
    x = bf16_bits(workloads.bf16_normal((N, H), seed))
    g = bf16_bits(workloads.bf16_normal((cap, H), seed + 100))
    recv, _ = oracle.dispatch_bf16(x, w, lay, 7, cap, recv_fill=0)
    gx = oracle.dispatch_backward(g, lay["pos"])
    # exact fp64 value of the backward: sum of the K receive-row grads
    exact = as_f32(g)[lay["pos"]].astype(np.float64).sum(axis=1)
    got = as_f32(gx).astype(np.float64)
    mag = np.abs(as_f32(g)[lay["pos"]].astype(np.float64)).sum(axis=1)
    assert np.all(np.abs(got - exact) <= ulp_bf16(exact) + K * 2.0 ** -23 * mag)
    # <dispatch(x), g> == <x, exact backward>, both in fp64
    used = lay["offsets"][-1]
    lhs = float((as_f32(recv[:used]).astype(np.float64) *
                 as_f32(g[:used]).astype(np.float64)).sum())
    rhs = float((as_f32(x).astype(np.float64) * exact).sum())
    assert abs(lhs - rhs) <= 1e-9 * (1 + abs(lhs))


def test_dispatch_backward_exact_on_small_integers():
    pos = np.array([[0, 2, 3], [1, -1, 2]], np.int32)
    g = torch_bf16_bits(np.arange(4 * 8, dtype=np.float32).reshape(4, 8))
    out = as_f32(oracle.dispatch_backward(g, pos))
    gf = as_f32(g)
    np.testing.assert_array_equal(out[0], gf[0] + gf[2] + gf[3])
    np.testing.assert_array_equal(out[1], gf[1] + gf[2])


@pytest.mark.parametrize("seed", range(3))
def test_combine_backward_rows_closed_form(seed):
    rng, topk, w, lay, cap = case(seed)
    N, K = topk.shape
    H = 64
    g = bf16_bits(workloads.bf16_normal((N, H), seed + 7))
    w = (rng.standard_normal((N, K)) * 3).astype(np.float32)
    rows = oracle.combine_backward_rows(g, w, lay, 7, cap)
    for k in range(K):
        prod = (as_f32(g) * w[:, k:k + 1]).astype(np.float32)
        np.testing.assert_array_equal(rows[lay["pos"][:, k]],
                                      torch_bf16_bits(prod))
    used = lay["offsets"][-1]
    padrows = np.where(lay["row_src"][:used] < 0)[0]
    assert np.all(rows[padrows] == 0)
    assert np.all(rows[used:] == 0x7FBF)


@pytest.mark.parametrize("seed", range(3))
def test_combine_backward_weights_by_finite_differences(seed):
    rng = np.random.default_rng(seed)
    N, K, H, rows = 6, 4, 32, 20
    y = bf16_bits(workloads.bf16_normal((rows, H), seed))
    g = bf16_bits(workloads.bf16_normal((N, H), seed + 1))
    pos = rng.integers(0, rows, size=(N, K)).astype(np.int32)
    pos[2, 1] = -1
    # dyadic weights so that w + 1 is exact in fp32
    w = (rng.integers(-8, 8, size=(N, K)) / 4.0).astype(np.float32)
    gw = oracle.combine_backward_weights(g, y, pos)
    gf = as_f32(g).astype(np.float64)
    base = oracle.combine_f64(y, pos, w)
    for t in range(N):
        for k in range(K):
            w2 = w.copy()
            w2[t, k] += 1.0
            d = oracle.combine_f64(y, pos, w2) - base
            fd = float((d * gf).sum())
            assert abs(gw[t, k] - fd) <= 1e-9 * (1 + abs(fd))
    assert gw[2, 1] == 0.0
    ref = np.einsum("tkh,th->tk",
                    as_f32(y)[np.where(pos >= 0, pos, 0)].astype(np.float64),
                    gf) * (pos >= 0)
    np.testing.assert_allclose(gw, ref, rtol=1e-12, atol=1e-12)


def test_gather_row_values_round_trip():
    rng, topk, w, lay, cap = case(5)
    H = 16
    x = bf16_bits(workloads.bf16_normal((topk.shape[0], H), 5))
    _, recv_w = oracle.dispatch_bf16(x, w, lay, 7, cap)
    np.testing.assert_array_equal(oracle.gather_row_values(recv_w,
                                                           lay["pos"]), w)
    pos = lay["pos"].copy()
    pos[0, 0] = -1
    out = oracle.gather_row_values(recv_w, pos)
    assert out[0, 0] == 0.0
