"""ep_layout_static: the layout entry point for callers that cannot allocate
device memory (a plugin inside a framework that owns every allocation, a
runtime that forbids allocation on its serving path, code running during a
global-mode graph capture). Its scratch is a fixed array inside the library.

Checked through the C ABI against ep_layout with a caller-provided workspace
on two calls in a row with different inputs and sizes, both large enough to
use the array (the cooperative kernel and the histogram + look-back pair), so
anything the first call left in the shared array would show up in the
second; and at the array's size limit, where the largest accepted problem
runs and one entry more is refused. Results must be bit-exact, as for every
layout test. This file is collected last on purpose.
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
    # (R, S, K, E, pad). Every call here has more than 32768 entries, so it
    # uses the array (smaller batches take a kernel that needs no scratch).
    # Cooperative layout (64 tiles, E=256), then another with E=64 and
    # padding: the second reads descriptors the first left behind.
    ((8, 4096, 8, 256, 1), (8, 2048, 8, 64, 128)),
    # Cooperative, then 700 tiles at E=256 (more than can be resident):
    # the histogram + look-back path runs on the array after a fused call.
    ((8, 4096, 8, 256, 1), (8, 44800, 8, 256, 1)),
    # The other way round, with a different E.
    ((8, 44800, 8, 256, 4), (4, 3000, 8, 32, 1)),
])
def test_static_scratch_matches_workspace_entry_point(first, second):
    f = _static_fn()
    rng = np.random.default_rng(sum(first) + sum(second))
    for (R, S, K, E, pad) in (first, second):
        assert R * S * K > 32768
        assert ep.ep_layout_workspace_bytes(R * S, K, E) <= SCRATCH_BYTES
        topk = torch.from_numpy(
            rng.integers(0, E, size=(R * S, K)).astype(np.int32)).to(DEV)
        cap = ep.ep_capacity_bound(R * S, K, E, pad)
        a = _run_static(f, topk, R, S, K, E, pad, cap)
        b = _run_workspace(topk, R, S, K, E, pad, cap)
        torch.cuda.synchronize()
        for k in ("counts", "offsets", "pos", "row_src", "status"):
            assert torch.equal(a[k], b[k]), k
        assert int(a["status"][0].item()) == 0


def test_static_scratch_at_its_size_limit():
    # E=256: 256 + 1024 + tiles * 1024 bytes, so 1022 tiles of 4096 entries
    # (N*K = 4,186,112) is the largest problem the 1 MiB array holds
    f = _static_fn()
    R, S, K, E, pad = 8, 65408, 8, 256, 1
    assert R * S * K == 1022 * 4096
    assert ep.ep_layout_workspace_bytes(R * S, K, E) <= SCRATCH_BYTES
    assert ep.ep_layout_workspace_bytes(R * S * K + 1, 1, E) > SCRATCH_BYTES
    rng = np.random.default_rng(12)
    topk = torch.from_numpy(
        rng.integers(0, E, size=(R * S, K)).astype(np.int32)).to(DEV)
    cap = ep.ep_capacity_bound(R * S, K, E, pad)
    a = _run_static(f, topk, R, S, K, E, pad, cap)
    b = _run_workspace(topk, R, S, K, E, pad, cap)
    torch.cuda.synchronize()
    for k in ("counts", "offsets", "pos", "row_src", "status"):
        assert torch.equal(a[k], b[k]), k
    # one entry more needs a 1023rd tile: refused before any CUDA call
    p = topk.data_ptr()
    rc = f(p, 1, R * S * K + 1, 1, E, 1, p, p, p, p, R * S * K + 1, p,
           torch.cuda.current_stream().cuda_stream)
    assert rc == ep.EP_ERR_WORKSPACE


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
