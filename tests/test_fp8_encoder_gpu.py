"""The device E4M3 conversion the FP8 dispatch uses, against the oracle's
encoder written from the OCP definition: every fp32 bit pattern whose
exponent lies where E4M3 rounding happens (2^-12 .. 2^9, both signs), plus
random patterns from the rest of the fp32 range."""
import numpy as np
import pytest
import torch

import combine_ep_layout_09_b200 as ep
import oracle
from gpu_util import DEV

pytestmark = pytest.mark.gpu


def gpu_encode(x: np.ndarray) -> np.ndarray:
    xd = torch.from_numpy(x).to(DEV)
    out = torch.empty(x.size, dtype=torch.uint8, device=DEV)
    ep.ep_debug_e4m3_encode(xd, out)
    torch.cuda.synchronize()
    return out.cpu().numpy()


@pytest.mark.parametrize("exp", list(range(-12, 10)))
def test_exhaustive_binade(exp):
    m = np.arange(1 << 23, dtype=np.uint32)
    biased = np.uint32(exp + 127)
    pos = (biased << np.uint32(23)) | m
    bits = np.concatenate([pos, pos | np.uint32(0x80000000)])
    x = bits.view(np.float32)
    np.testing.assert_array_equal(gpu_encode(x), oracle.e4m3_encode(x))


def test_random_rest_and_specials():
    rng = np.random.default_rng(0)
    bits = rng.integers(0, 1 << 32, size=4_000_000, dtype=np.uint64)
    x = bits.astype(np.uint32).view(np.float32)
    x = x[np.isfinite(x)]
    specials = np.array([0.0, -0.0, 448.0, -448.0, 464.0, 480.0, 1e38,
                         -1e38, 1e-45, -1e-45, 2.0 ** -149, 2.0 ** -126],
                        np.float32)
    x = np.concatenate([x, specials])
    np.testing.assert_array_equal(gpu_encode(x), oracle.e4m3_encode(x))


def gpu_quantize(x: np.ndarray, scale: np.ndarray) -> np.ndarray:
    xd = torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(DEV)
    sd = torch.from_numpy(np.ascontiguousarray(scale, np.float32)).to(DEV)
    out = torch.empty(x.size, dtype=torch.uint8, device=DEV)
    ep.ep_debug_quantize(xd, sd, out)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def _midpoints():
    v = np.array([oracle.e4m3_decode(c)[0] for c in range(0x7F)])
    return (v[:-1] + v[1:]) / 2


def test_quantize_random_scales():
    rng = np.random.default_rng(1)
    G = 1 << 18
    scale = np.exp2(rng.uniform(-130, 30, G)).astype(np.float32)
    scale[::97] = 0.0
    mag = np.exp2(rng.uniform(-12, 9.5, G * 16))
    x = (np.repeat(scale.astype(np.float64), 16) * mag *
         rng.choice([-1.0, 1.0], G * 16)).astype(np.float32)
    x[::1001] = 0.0
    x[5::1003] = -0.0
    np.testing.assert_array_equal(gpu_quantize(x, scale),
                                  oracle.quantize_by_scale(x, scale))


def test_quantize_quotients_on_rounding_boundaries():
    # x/s lands on, or one fp32 step either side of, every E4M3 midpoint, so
    # the bracket disagrees and the correctly rounded division decides
    rng = np.random.default_rng(2)
    mids = _midpoints()
    G = 1 << 16
    scale = np.exp2(rng.uniform(-20, 20, G)).astype(np.float32)
    m = rng.choice(mids, G * 16) * rng.choice([-1.0, 1.0], G * 16)
    x = (np.repeat(scale.astype(np.float64), 16) * m).astype(np.float32)
    nudge = rng.integers(-2, 3, G * 16)
    x = np.nextafter(x, np.where(nudge > 0, np.inf, -np.inf).astype(
        np.float32)) * (nudge != 0) + x * (nudge == 0)
    x = x.astype(np.float32)
    got = gpu_quantize(x, scale)
    np.testing.assert_array_equal(got, oracle.quantize_by_scale(x, scale))
    # exact ties with scale 1: the midpoints themselves
    xm = np.concatenate([mids, -mids]).astype(np.float32)
    xm = np.resize(xm, ((xm.size + 15) // 16) * 16)
    sm = np.ones(xm.size // 16, np.float32)
    np.testing.assert_array_equal(gpu_quantize(xm, sm),
                                  oracle.quantize_by_scale(xm, sm))
