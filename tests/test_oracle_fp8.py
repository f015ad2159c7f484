"""Pins for the oracle's FP8 E4M3 encoder and its 1x128 row quantisation.

The encoder is written from the OCP OFP8 definition of E4M3. It is pinned
here against torch's float8_e4m3fn cast (a library routine), the format's
textbook values, exact ties and the half-step error bound. The quantisation
is pinned against an independent composition of library routines (numpy
fp32 division + the torch cast) and against the property that fixes the
scale: the largest magnitude of every group lands on +-448.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads


def torch_e4m3(x: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.asarray(x, np.float32))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_textbook_values():
    dec = oracle.e4m3_decode
    assert dec(0x7E)[0] == 448.0          # largest finite
    assert dec(0x01)[0] == 2.0 ** -9      # smallest subnormal
    assert dec(0x07)[0] == 7 * 2.0 ** -9  # largest subnormal
    assert dec(0x08)[0] == 2.0 ** -6      # smallest normal
    assert dec(0x38)[0] == 1.0
    assert np.isnan(dec(0x7F)[0]) and np.isnan(dec(0xFF)[0])
    assert dec(0x80)[0] == 0.0 and np.signbit(dec(0x80)[0])


def test_all_codes_round_trip():
    for c in range(256):
        if c in (0x7F, 0xFF):
            continue
        v = oracle.e4m3_decode(c)[0]
        assert oracle.e4m3_encode(np.float32(v))[0] == c, hex(c)


def test_matches_torch_cast_random():
    rng = np.random.default_rng(0)
    # magnitudes spread over the whole e4m3 range and below it
    mag = np.exp2(rng.uniform(-14, np.log2(448.0), size=200_000))
    x = (mag * rng.choice([-1.0, 1.0], size=mag.size)).astype(np.float32)
    x = x[np.abs(x) <= 448.0]
    np.testing.assert_array_equal(oracle.e4m3_encode(x), torch_e4m3(x))


def test_matches_torch_cast_on_ties_and_neighbours():
    # every midpoint between adjacent codes, and the fp32 values one ulp on
    # either side of it
    vals = [oracle.e4m3_decode(c)[0] for c in range(0x7F)]
    mids = np.array([(a + b) / 2 for a, b in zip(vals[:-1], vals[1:])],
                    np.float32)
    up = np.nextafter(mids, np.float32(np.inf))
    dn = np.nextafter(mids, np.float32(0))
    for arr in (mids, up, dn, -mids, -up, -dn):
        np.testing.assert_array_equal(oracle.e4m3_encode(arr),
                                      torch_e4m3(arr))


def test_ties_go_to_even():
    # 1 + 1/16 lies halfway between 1.0 (mantissa 0) and 1.125 (mantissa 1)
    assert oracle.e4m3_encode(np.float32(1.0625))[0] == 0x38
    # 1 + 3/16 lies halfway between 1.125 and 1.25 -> mantissa 2
    assert oracle.e4m3_encode(np.float32(1.1875))[0] == 0x3A
    # 1.5 * 2^-9 lies halfway between subnormal codes 1 and 2 -> 2
    assert oracle.e4m3_encode(np.float32(1.5 * 2 ** -9))[0] == 0x02
    # 0.5 * 2^-9 lies halfway between 0 and the smallest subnormal -> 0
    assert oracle.e4m3_encode(np.float32(0.5 * 2 ** -9))[0] == 0x00
    # 7.5 * 2^-9 rounds up across the subnormal/normal border to 2^-6
    assert oracle.e4m3_encode(np.float32(7.5 * 2 ** -9))[0] == 0x08


def test_saturation_and_signed_zero():
    enc = oracle.e4m3_encode
    for v, c in [(448.0, 0x7E), (449.0, 0x7E), (464.0, 0x7E), (1e30, 0x7E),
                 (np.inf, 0x7E), (-448.0, 0xFE), (-1000.0, 0xFE),
                 (-np.inf, 0xFE), (0.0, 0x00), (-0.0, 0x80),
                 (-1e-9, 0x80), (1e-9, 0x00)]:
        assert enc(np.float32(v))[0] == c, v


def test_half_step_error_bound():
    rng = np.random.default_rng(1)
    x = (rng.uniform(-448, 448, 100_000)).astype(np.float32)
    x = np.concatenate([x, (rng.uniform(-1, 1, 20_000) * 2.0 ** -6)
                        .astype(np.float32)])
    q = oracle.e4m3_decode(oracle.e4m3_encode(x))
    err = np.abs(q - x.astype(np.float64))
    normal = np.abs(x) >= 2.0 ** -6
    assert np.all(err[normal] <= np.abs(x[normal]) * 2.0 ** -4)
    assert np.all(err[~normal] <= 2.0 ** -10)


def _bf16_rows(n, H, seed, scale=1.0):
    t = workloads.bf16_normal((n, H), seed) * scale
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_quantize_row_matches_library_composition():
    rows = _bf16_rows(16, 1024, 5)
    q, s = oracle.quantize_rows(rows)
    x = rows.astype(np.uint32) << 16
    x = x.view(np.float32).reshape(16, 8, 128)
    amax = np.abs(x).max(axis=2)
    scale = (amax / np.float32(448.0)).astype(np.float32)
    np.testing.assert_array_equal(s, scale)
    quot = (x / scale[:, :, None]).astype(np.float32)
    np.testing.assert_array_equal(q, torch_e4m3(quot).reshape(16, 1024))


def test_quantize_group_max_hits_448():
    rows = _bf16_rows(32, 512, 6, scale=3.0)
    q, s = oracle.quantize_rows(rows)
    x = (rows.astype(np.uint32) << 16).view(np.float32).reshape(32, 4, 128)
    qg = q.reshape(32, 4, 128)
    for i in range(32):
        for g in range(4):
            j = int(np.argmax(np.abs(x[i, g])))
            assert qg[i, g, j] in (0x7E, 0xFE)
            assert (qg[i, g, j] == 0xFE) == (x[i, g, j] < 0)


def test_quantize_dequant_error_bound():
    rows = _bf16_rows(8, 2048, 7, scale=0.01)
    q, s = oracle.quantize_rows(rows)
    x = (rows.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    deq = oracle.e4m3_decode(q) * np.repeat(s.astype(np.float64), 128, axis=1)
    err = np.abs(deq - x)
    step = np.repeat(s.astype(np.float64), 128, axis=1)
    bound = np.maximum(np.abs(x) * 2.0 ** -4, step * 2.0 ** -10) * 1.0001
    assert np.all(err <= bound)


def test_quantize_zero_and_tiny_groups():
    row = np.zeros(384, np.uint16)
    row[128:256] = 0x8000                     # a group of -0.0
    row[256] = 0x0001                         # smallest bf16 subnormal
    row[300] = 0x8003
    q, s = oracle.quantize_row(row)
    assert s[0] == 0 and s[1] == 0 and np.all(q[:256] == 0)
    assert s[2] > 0                           # a subnormal fp32 scale
    assert q[300] == 0xFE                     # |x| = amax -> -448
    assert 0 < q[256] < 0x7E                  # a third of amax


@pytest.mark.parametrize("H", [128, 7168])
def test_quantize_row_widths(H):
    rows = _bf16_rows(3, H, 8)
    q, s = oracle.quantize_rows(rows)
    assert q.shape == (3, H) and s.shape == (3, H // 128)


def test_quantize_by_scale_matches_row_quantisation_and_library():
    rows = _bf16_rows(6, 512, 11)
    q, s = oracle.quantize_rows(rows)
    x = (rows.astype(np.uint32) << 16).view(np.float32)
    got = oracle.quantize_by_scale(x, s, group=128).reshape(6, 512)
    np.testing.assert_array_equal(got, q)
    rng = np.random.default_rng(12)
    xs = (rng.standard_normal(4096) * 10).astype(np.float32)
    sc = np.exp2(rng.uniform(-20, 20, 256)).astype(np.float32)
    sc[3] = 0.0
    got = oracle.quantize_by_scale(xs, sc, group=16)
    quot = (xs / np.repeat(sc, 16)).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        ref = torch_e4m3(np.clip(quot, -448, 448))
    ref[48:64] = 0
    np.testing.assert_array_equal(got, ref)
