"""ep_layout_static: the layout entry point for callers that cannot allocate
device memory (a plugin inside a framework that owns every allocation, a
runtime that forbids allocation on its serving path, code running during a
global-mode graph capture). Its scratch is a fixed array inside the library.

Checked through the C ABI against ep_layout with a caller-provided workspace
on two calls in a row with different inputs, so anything the first call left
in the shared array would show up in the second. Results must be bit-exact,
as for every layout test. This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import combine_ep_layout_09_b200 as ep
from combine_ep_layout_09_b200 import build as epbuild

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")
SCRATCH_BYTES = 1 << 20          # EP_LAYOUT_STATIC_SCRATCH_BYTES


def _static_fn():
    lib = ctypes.CDLL(epbuild.LIB)
    f = lib.ep_layout_static
    P, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    f.restype = i32
    f.argtypes = [P, i32, i32, i32, i32, i32, P, P, P, P, i64, P, P]
    return f


def _buffers(N, K, E, cap):
    i32 = dict(dtype=torch.int32, device=DEV)
    return dict(counts=torch.full((E,), -9, **i32),
                offsets=torch.full((E + 1,), -9, **i32),
                pos=torch.full((N, K), -9, **i32),
                row_src=torch.full((cap,), -7, **i32),
                status=torch.zeros(4, **i32))


def _run_static(f, topk, R, S, K, E, pad, cap):
    b = _buffers(R * S, K, E, cap)
    stream = torch.cuda.current_stream().cuda_stream
    rc = f(topk.data_ptr(), R, S, K, E, pad, b["counts"].data_ptr(),
           b["offsets"].data_ptr(), b["pos"].data_ptr(),
           b["row_src"].data_ptr(), cap, b["status"].data_ptr(), stream)
    assert rc == 0, ep.strerror(rc)
    return b


def _run_workspace(topk, R, S, K, E, pad, cap):
    b = _buffers(R * S, K, E, cap)
    ws = torch.randint(0, 255, (ep.ep_layout_workspace_bytes(R * S, K, E),),
                       dtype=torch.uint8, device=DEV)
    ep.ep_layout(topk, R, S, K, E, pad, b["counts"], b["offsets"], b["pos"],
                 b["row_src"], ws, b["status"], cap=cap)
    return b


@pytest.mark.parametrize("first,second", [
    # (R, S, K, E, pad): a large call followed by a smaller one, and back
    ((8, 4096, 8, 256, 1), (4, 300, 6, 64, 16)),
    ((4, 300, 6, 64, 16), (8, 2048, 8, 256, 128)),
])
def test_static_scratch_matches_workspace_entry_point(first, second):
    f = _static_fn()
    rng = np.random.default_rng(sum(first) + sum(second))
    for (R, S, K, E, pad) in (first, second):
        topk = torch.from_numpy(
            rng.integers(0, E, size=(R * S, K)).astype(np.int32)).to(DEV)
        cap = ep.ep_capacity_bound(R * S, K, E, pad)
        a = _run_static(f, topk, R, S, K, E, pad, cap)
        b = _run_workspace(topk, R, S, K, E, pad, cap)
        torch.cuda.synchronize()
        for k in ("counts", "offsets", "pos", "row_src", "status"):
            assert torch.equal(a[k], b[k]), k
        assert int(a["status"][0].item()) == 0


def test_static_scratch_refuses_problems_beyond_its_size():
    f = _static_fn()
    R, K, E = 8, 8, 1024
    S = 256 * 1024                     # needs far more than 1 MiB of scratch
    assert ep.ep_layout_workspace_bytes(R * S, K, E) > SCRATCH_BYTES
    dummy = torch.zeros(16, dtype=torch.int32, device=DEV)
    p = dummy.data_ptr()
    rc = f(p, R, S, K, E, 1, p, p, p, p, R * S * K, p,
           torch.cuda.current_stream().cuda_stream)
    assert rc == ep.EP_ERR_WORKSPACE
