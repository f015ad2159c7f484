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
