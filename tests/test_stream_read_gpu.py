"""ep_debug_stream_read reads every byte it is given: the XOR of all 32-bit
words comes back (the bench's read ceiling relies on it)."""
import numpy as np
import pytest
import torch

import combine_ep_layout_09_b200 as ep

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("nbytes", [32, 32 * 1024 + 32, 3 * 2 ** 20 + 96,
                                    64 * 2 ** 20])
def test_xor_of_every_word(nbytes):
    rng = np.random.default_rng(nbytes % 1000)
    words = rng.integers(0, 2 ** 32, size=nbytes // 4, dtype=np.uint64)
    words = words.astype(np.uint32)
    src = torch.from_numpy(words.view(np.int32)).to("cuda:0")
    sink = torch.zeros(1, dtype=torch.int32, device="cuda:0")
    ep.ep_debug_stream_read(src, sink)
    torch.cuda.synchronize()
    want = np.bitwise_xor.reduce(words)
    assert np.uint32(sink.cpu().numpy().view(np.uint32)[0]) == want
