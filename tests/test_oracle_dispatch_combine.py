"""Pins for the oracle's dispatch copies and its combine reduction.

Dispatch is pinned by its closed form (every destination row is the source
row, bit for bit; padding rows are zero). Combine is pinned by the identity
round trip (identity experts and weights that sum to one give x back
exactly), by a brute-force double-precision sum with math.fsum, and by the
rigorous error bound of an fp32 fused multiply-add chain.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def as_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


def small_case(seed, N=40, H=256, E=9, K=3, pad=4):
    rng = np.random.default_rng(seed)
    topk, w = workloads.random_topk(rng, N, K, E)
    hidden = bf16_bits(workloads.bf16_normal((N, H), seed))
    return topk, w, hidden, E, pad


@pytest.mark.parametrize("seed", range(6))
def test_dispatch_bf16_closed_form(seed):
    topk, w, hidden, E, pad = small_case(seed)
    N, K = topk.shape
    cap = oracle.capacity_bound(N, K, E, pad) + 5
    lay = oracle.layout(topk, E, pad, cap)
    recv, recv_w = oracle.dispatch_bf16(hidden, w, lay, E, cap)
    pos = lay["pos"]
    for k in range(K):
        np.testing.assert_array_equal(recv[pos[:, k]], hidden)
        np.testing.assert_array_equal(recv_w[pos[:, k]], w[:, k])
    used = lay["offsets"][-1]
    padrows = np.where(lay["row_src"][:used] == -1)[0]
    assert np.all(recv[padrows] == 0) and np.all(recv_w[padrows] == 0)
    assert np.all(recv[used:] == 0x7FBF) and np.all(recv_w[used:] == -3.0)


@pytest.mark.parametrize("seed", range(4))
def test_dispatch_fp8_closed_form(seed):
    topk, w, hidden, E, pad = small_case(seed, H=384)
    N, K = topk.shape
    cap = oracle.capacity_bound(N, K, E, pad)
    lay = oracle.layout(topk, E, pad, cap)
    recv, scales, recv_w = oracle.dispatch_fp8(hidden, w, lay, E, cap)
    q, s = oracle.quantize_rows(hidden)
    pos = lay["pos"]
    for k in range(K):
        np.testing.assert_array_equal(recv[pos[:, k]], q)
        np.testing.assert_array_equal(scales[pos[:, k]], s)
        np.testing.assert_array_equal(recv_w[pos[:, k]], w[:, k])
    used = lay["offsets"][-1]
    padrows = np.where(lay["row_src"][:used] == -1)[0]
    assert len(padrows) > 0
    assert np.all(recv[padrows] == 0) and np.all(scales[padrows] == 0)
    assert np.all(recv_w[padrows] == 0)


def test_identity_round_trip_is_exact():
    # combine(dispatch(x)) with identity experts and sum_k w = 1 returns x
    w_ = workloads.WORKLOADS["tiny"]
    topk, w = workloads.routing(w_)
    hidden = bf16_bits(workloads.hidden_states(w_))
    lay = oracle.layout(topk, w_.E, w_.pad)
    cap = lay["offsets"][-1]
    recv, _ = oracle.dispatch_bf16(hidden, w, lay, w_.E, cap)
    out = oracle.combine(recv, lay["pos"], w)
    np.testing.assert_array_equal(out, hidden)


def test_identity_round_trip_skewed_padded():
    w_ = workloads.scaled(workloads.WORKLOADS["skewed"], S=32, H=512)
    topk, w = workloads.routing(w_)
    hidden = bf16_bits(workloads.hidden_states(w_))
    lay = oracle.layout(topk, w_.E, w_.pad)
    cap = oracle.capacity_bound(w_.N, w_.K, w_.E, w_.pad)
    recv, _ = oracle.dispatch_bf16(hidden, w, lay, w_.E, cap)
    out = oracle.combine(recv, lay["pos"], w)
    np.testing.assert_array_equal(out, hidden)


def _ulp_bf16(v):
    a = np.abs(v)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -126)
    return np.exp2(e - 7)


@pytest.mark.parametrize("seed", range(3))
def test_combine_against_fsum(seed):
    rng = np.random.default_rng(seed)
    N, K, H, rows = 24, 8, 64, 100
    y = bf16_bits(workloads.bf16_normal((rows, H), seed))
    pos = rng.integers(0, rows, size=(N, K)).astype(np.int32)
    pos[0, 3] = -1                                   # a skipped entry
    w = rng.random((N, K)).astype(np.float32)
    out = as_f32(oracle.combine(y, pos, w)).astype(np.float64)
    ref64 = oracle.combine_f64(y, pos, w)
    yf = as_f32(y).astype(np.float64)
    for t in range(N):
        for h in range(H):
            terms = [float(w[t, k]) * yf[pos[t, k], h] for k in range(K)
                     if pos[t, k] >= 0]
            exact = math.fsum(terms)
            assert abs(ref64[t, h] - exact) <= 1e-12 * (1 + abs(exact))
            mag = math.fsum(abs(x) for x in terms)
            # fp32 fma chain: <= K unit roundoffs of the magnitude sum, then
            # one rounding to bf16 (at most one bf16 ulp of the result)
            bound = _ulp_bf16(exact) + K * 2.0 ** -23 * mag
            assert abs(out[t, h] - exact) <= bound


def test_combine_stated_tolerance_on_workload():
    # the combine bound: |err| <= 1e-2 * max|y|, and 1 bf16 ulp where the
    # terms do not cancel
    w_ = workloads.scaled(workloads.WORKLOADS["prefill"], S=8, H=1024)
    topk, w = workloads.routing(w_)
    lay = oracle.layout(topk, w_.E, 1)
    cap = lay["offsets"][-1]
    y = bf16_bits(workloads.expert_outputs(cap, w_.H, 1))
    out = as_f32(oracle.combine(y, lay["pos"], w)).astype(np.float64)
    ref = oracle.combine_f64(y, lay["pos"], w)
    maxabs = np.abs(as_f32(y)).max()
    assert np.abs(out - ref).max() <= 1e-2 * maxabs
    # non-cancelling outputs are within one bf16 ulp of the exact sum
    yf = as_f32(y).astype(np.float64)
    mag = np.zeros_like(ref)
    for k in range(w_.K):
        mag += np.abs(w[:, k:k + 1].astype(np.float64) * yf[lay["pos"][:, k]])
    ok = mag <= 2 * np.abs(ref)
    assert ok.sum() > 1000
    assert np.all(np.abs(out - ref)[ok] <= _ulp_bf16(ref[ok]))


def test_combine_accumulates_in_k_order():
    # 1 - 1 + 2^-30 in k order keeps the 2^-30; any order that adds 2^-30 to
    # one of the unit terms first loses it in fp32 and returns 0.
    one, minus_one, tiny = 0x3F80, 0xBF80, 0x3080       # 1, -1, 2^-30
    assert as_f32(np.array([tiny], np.uint16))[0] == 2.0 ** -30
    y = np.array([[one], [minus_one], [tiny]], np.uint16)
    w = np.ones((1, 3), np.float32)
    fwd = oracle.combine(y, np.array([[0, 1, 2]], np.int32), w)
    assert as_f32(fwd)[0, 0] == 2.0 ** -30
    rev = oracle.combine(y, np.array([[2, 1, 0]], np.int32), w)
    assert as_f32(rev)[0, 0] == 0.0


def test_combine_uses_fused_multiply_add():
    # p = (1 + 2^-23)(1 + 2^-7) = 1 + 2^-7 + 2^-23 + 2^-30 needs 31 bits.
    # k=0 adds -p rounded to fp32 (the 2^-30 is lost); k=1 fuses +p exactly
    # into that accumulator, leaving 2^-30. Rounding the product before the
    # add would give 0 instead.
    y = np.array([[0x3F81], [0x3F81]], np.uint16)          # 1 + 2^-7
    w = np.array([[-(1 + 2.0 ** -23), 1 + 2.0 ** -23]], np.float32)
    out = oracle.combine(y, np.array([[0, 1]], np.int32), w)
    assert as_f32(out)[0, 0] == 2.0 ** -30


def test_combine_empty_and_single():
    y = np.zeros((4, 16), np.uint16)
    out = oracle.combine(y, np.zeros((0, 2), np.int32),
                         np.zeros((0, 2), np.float32))
    assert out.shape == (0, 16)
    y = bf16_bits(workloads.bf16_normal((3, 16), 9))
    out = oracle.combine(y, np.array([[2]], np.int32),
                         np.array([[1.0]], np.float32))
    np.testing.assert_array_equal(out[0], y[2])
