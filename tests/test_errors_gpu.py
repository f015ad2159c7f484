"""Failure detection without a GPU fault: bad inputs are reported through
the device status word, bounded waits give up and report, and the context
stays usable afterwards."""
import numpy as np
import pytest
import torch

import combine_ep_layout_09_b200 as ep
from gpu_util import DEV, gpu_layout, status_tensor

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_on_a_flag_nothing_sets():
    flag = torch.zeros(4, dtype=torch.int32, device=DEV)
    st = status_tensor()
    ep.ep_debug_bounded_wait(flag, 20000, st)     # ~2 ms of polling
    torch.cuda.synchronize()
    assert int(st[0].item()) == ep.EP_DEV_TIMEOUT
    # the context is still usable
    topk = np.random.default_rng(0).integers(0, 8, (64, 2)).astype(np.int32)
    assert gpu_layout(topk, 2, 32, 8, 1)["status"] == 0


def test_bounded_wait_returns_when_flag_set():
    flag = torch.ones(4, dtype=torch.int32, device=DEV)
    st = status_tensor()
    ep.ep_debug_bounded_wait(flag, 1 << 40, st)
    torch.cuda.synchronize()
    assert int(st[0].item()) == 0


def test_host_side_errors_raise():
    t = torch.zeros(64, dtype=torch.int32, device=DEV)
    ws = torch.zeros(1 << 16, dtype=torch.uint8, device=DEV)
    with pytest.raises(ep.EPError) as e:
        ep.ep_layout(t, 3, 8, 2, 8, 1, t, t, t, t, ws)   # E % R != 0
    assert e.value.code == ep.EP_ERR_INVALID_ARG
    with pytest.raises(ep.EPError) as e:
        ep.ep_layout(t, 4, 8, 2, 8, 1, t[:8], t[:9], t, t[:31], ws)
    assert e.value.code == ep.EP_ERR_CAPACITY
    small = torch.zeros(16, dtype=torch.uint8, device=DEV)
    with pytest.raises(ep.EPError) as e:
        ep.ep_layout(t, 4, 8, 2, 8, 1, t[:8], t[:9], t, t, small)
    assert e.value.code == ep.EP_ERR_WORKSPACE
    with pytest.raises(ep.EPError) as e:
        ep.ep_layout(t, 4, 8, 2, 8, 1, t[:8], t[1:10], t, t, ws)
    assert e.value.code == ep.EP_ERR_ALIGNMENT
