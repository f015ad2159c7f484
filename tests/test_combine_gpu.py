"""GPU combine against the oracle: the same fp32 fused-multiply-add chain in
k order, so results are bit-identical; the stated bar (within 1 bf16 ulp of
the exact sum, absolute error <= 1e-2 * max|y|) is checked as well."""
import numpy as np
import pytest
import torch

import combine_ep_layout_09_b200 as ep
import oracle
import workloads
from gpu_util import gpu_combine, to_bf16_dev, to_dev, u16

pytestmark = pytest.mark.gpu


def as_f32(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32)


def ulp_bf16(v):
    a = np.abs(v)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.exp2(np.maximum(e, -126) - 7)


def check(y_bits, pos, w, num_sms=0):
    N, K = pos.shape
    out, st = gpu_combine(to_bf16_dev(y_bits), to_dev(pos), to_dev(w), N, K,
                          num_sms=num_sms)
    assert st == 0
    got = u16(out)
    ref = oracle.combine(y_bits, pos, w)
    np.testing.assert_array_equal(got, ref)          # bit-exact
    # the stated tolerance against the exact (double) sum
    exact = oracle.combine_f64(y_bits, pos, w)
    err = np.abs(as_f32(got).astype(np.float64) - exact)
    # the stated bar is relative to max|y| for weights summing to one; for
    # other weights it scales with the largest per-token sum of |w|
    maxabs = float(np.abs(as_f32(y_bits)).max()) if y_bits.size else 0.0
    wsum = float(np.abs(w).sum(axis=1).max()) if w.size else 0.0
    assert np.all(err <= 1e-2 * maxabs * max(1.0, wsum) + 1e-30)
    return got


@pytest.mark.parametrize("N,K,H,rows", [
    (1, 1, 8, 1), (256, 2, 256, 600), (1000, 8, 7168, 9000),
    (333, 3, 520, 1200), (77, 5, 24, 400), (129, 9, 1024, 2000),
    (64, 32, 64, 3000), (500, 6, 4096, 3100), (40, 4, 16, 100),
])
def test_random(N, K, H, rows):
    rng = np.random.default_rng(N + K + H)
    y = u16(workloads.bf16_normal((rows, H), N + H))
    pos = rng.integers(0, rows, size=(N, K)).astype(np.int32)
    w = rng.random((N, K)).astype(np.float32)
    check(y, pos, w)


def test_skipped_entries_and_limited_sms():
    rng = np.random.default_rng(2)
    y = u16(workloads.bf16_normal((300, 512), 3))
    pos = rng.integers(0, 300, size=(200, 8)).astype(np.int32)
    pos[rng.random(pos.shape) < 0.2] = -1
    pos[5] = -1                                   # a token with no entries
    w = (rng.standard_normal((200, 8))).astype(np.float32)
    got = check(y, pos, w, num_sms=2)
    assert np.all(got[5] == 0)


def test_k_order_and_fma_cases():
    # 1 - 1 + 2^-30 (order) and the 31-bit product case (fusion)
    y = np.array([[0x3F80] * 8, [0xBF80] * 8, [0x3080] * 8, [0x3F81] * 8],
                 np.uint16)
    pos = np.array([[0, 1, 2], [2, 1, 0]], np.int32)
    w = np.ones((2, 3), np.float32)
    got = check(y, pos, w)
    assert as_f32(got)[0, 0] == 2.0 ** -30 and as_f32(got)[1, 0] == 0.0
    pos = np.array([[3, 3]], np.int32)
    w = np.array([[-(1 + 2.0 ** -23), 1 + 2.0 ** -23]], np.float32)
    got = check(y, pos, w)
    assert as_f32(got)[0, 0] == 2.0 ** -30


@pytest.mark.parametrize("N,K,H,rows", [
    (2500, 8, 7176, 4000),    # two parts per row, the last one shorter
    (5000, 3, 520, 6000),     # one part per row
    (2400, 32, 2056, 9000),   # K=32: three parts of 688 / 688 / 680 channels
    (2400, 1, 32768, 2600),   # K=1, the widest row: one 64 KB part per stage
])
# the persistent pipeline on every SM (0) and on fewer (100)
@pytest.mark.parametrize("num_sms", [0, 100])
def test_large_batches_tma_path(N, K, H, rows, num_sms):
    # enough (token, part) units per SM that the bulk-copy pipeline runs
    rng = np.random.default_rng(N + K)
    y = u16(workloads.bf16_normal((rows, H), K))
    pos = rng.integers(0, rows, size=(N, K)).astype(np.int32)
    pos[rng.random(pos.shape) < 0.05] = -1
    pos[7] = -1                                  # a token with no rows
    w = rng.standard_normal((N, K)).astype(np.float32)
    got = check(y, pos, w, num_sms=num_sms)
    assert np.all(got[7] == 0)


def test_widest_row_and_k32():
    rng = np.random.default_rng(11)
    y = u16(workloads.bf16_normal((300, 32768), 12))
    pos = rng.integers(0, 300, size=(40, 2)).astype(np.int32)
    w = rng.random((40, 2)).astype(np.float32)
    check(y, pos, w)
    y = u16(workloads.bf16_normal((600, 1024), 13))
    pos = rng.integers(0, 600, size=(2600, 32)).astype(np.int32)
    w = rng.random((2600, 32)).astype(np.float32) / 32
    check(y, pos, w)


@pytest.mark.parametrize("N,K,H,rows", [
    (300, 8, 7168, 3000),     # register-gather kernel, K = 8
    (200, 5, 520, 1500),      # runtime-K kernel
    (2500, 8, 1024, 9000),    # bulk-copy pipeline
    (2400, 8, 7176, 4000),    # bulk-copy pipeline, two parts per row
])
@pytest.mark.parametrize("num_sms", [0, 100])
def test_receive_side_weights(N, K, H, rows, num_sms):
    # weight of (t,k) = recv_weights[pos[t,k]], handed back in token order
    rng = np.random.default_rng(N * K + H)
    y = u16(workloads.bf16_normal((rows, H), N + 7))
    pos = rng.integers(0, rows, size=(N, K)).astype(np.int32)
    pos[rng.random(pos.shape) < 0.05] = -1
    rw = rng.standard_normal(rows).astype(np.float32)
    gw_ref = oracle.gather_row_values(rw, pos)
    out = torch.full((N, H), 0x7FBF, dtype=torch.int16,
                     device="cuda:0").view(torch.bfloat16)
    gathered = torch.full((N, K), -7.0, dtype=torch.float32, device="cuda:0")
    st = torch.zeros(4, dtype=torch.int32, device="cuda:0")
    ep.ep_combine_recv_weights(to_bf16_dev(y), to_dev(pos), to_dev(rw), N, K,
                               H, out, gathered, num_sms=num_sms, status=st)
    assert int(st[0].item()) == 0
    np.testing.assert_array_equal(gathered.cpu().numpy(), gw_ref)
    np.testing.assert_array_equal(u16(out), oracle.combine(y, pos, gw_ref))
    # without the gathered output: the same result
    out2 = torch.empty_like(out)
    ep.ep_combine_recv_weights(to_bf16_dev(y), to_dev(pos), to_dev(rw), N, K,
                               H, out2, None, num_sms=num_sms)
    assert torch.equal(out2.view(torch.int16), out.view(torch.int16))
