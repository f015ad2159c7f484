"""The C ABI library loads, exports every entry point its header declares,
and rejects bad arguments on the host before touching the GPU. No compute
call is made here: these tests run without a GPU."""
import ctypes
import os
import re

import pytest

import combine_ep_layout_09_b200 as ep
from combine_ep_layout_09_b200 import build as epbuild

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include",
                      "eplayout.h")


def declared_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^EP_API [^;(]*?\b(ep_\w+)\s*\(", src,
                                 flags=re.M)))


def test_header_declares_the_path():
    names = declared_functions()
    for n in ["ep_layout", "ep_dispatch", "ep_combine", "ep_plan_balanced",
              "ep_prefetch_weights", "ep_capacity_bound",
              "ep_layout_workspace_bytes", "ep_strerror", "ep_abi_version"]:
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(epbuild.LIB)
    for n in declared_functions():
        assert hasattr(lib, n), n


def test_library_is_the_in_tree_build():
    assert os.path.dirname(ep.library_path()) == os.path.dirname(
        os.path.abspath(ep.__file__))
    assert epbuild.up_to_date()


def test_pure_host_entry_points():
    assert ep.ep_abi_version() == 5
    assert ep.ep_capacity_bound(32768, 8, 256, 128) == 32768 * 8 + 256 * 127
    assert ep.ep_capacity_bound(10, 2, 4, 1) == 20
    assert ep.ep_capacity_bound(-1, 2, 4, 1) < 0
    assert ep.ep_layout_workspace_bytes(32768, 8, 256) > 0
    assert ep.ep_layout_workspace_bytes(10, 0, 4) == 0
    assert ep.ep_layout_workspace_bytes(10, 2, 4096) == 0   # E too large
    for code in [0, -1, -2, -3, -4, -5, 1, 2, 4, 8, 16]:
        assert ep.strerror(code) != "unknown code"


def _raw():
    return ctypes.CDLL(epbuild.LIB)


def test_layout_rejects_on_host():
    lib = _raw()
    lib.ep_layout.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                              ctypes.c_int, ctypes.c_int, ctypes.c_int,
                              ctypes.c_void_p, ctypes.c_void_p,
                              ctypes.c_void_p, ctypes.c_void_p,
                              ctypes.c_int64, ctypes.c_void_p,
                              ctypes.c_size_t, ctypes.c_void_p,
                              ctypes.c_void_p]
    fake = ctypes.c_void_p(1 << 20)        # aligned, never dereferenced
    args = dict(R=4, S=8, K=2, E=8, pad=1, cap=64)

    def call(**kw):
        a = dict(args, **kw)
        return lib.ep_layout(fake, a["R"], a["S"], a["K"], a["E"], a["pad"],
                             fake, fake, fake, fake, a["cap"], fake, 1 << 20,
                             None, None)
    assert call(E=10) == ep.EP_ERR_INVALID_ARG      # E % R != 0
    assert call(K=0) == ep.EP_ERR_INVALID_ARG
    assert call(K=33) == ep.EP_ERR_INVALID_ARG
    assert call(pad=0) == ep.EP_ERR_INVALID_ARG
    assert call(cap=63) == ep.EP_ERR_CAPACITY       # below N*K
    assert call(pad=4, cap=64) == ep.EP_ERR_CAPACITY
    assert call(cap=2 ** 31) == ep.EP_ERR_CAPACITY
    assert call(S=1 << 28, cap=1 << 31) == ep.EP_ERR_INVALID_ARG


def test_dispatch_combine_reject_on_host():
    lib = _raw()
    P, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    lib.ep_dispatch.argtypes = [P, P, P, P, P, i64, i32, i32, i32, i64, i32,
                                P, P, P, i32, P, P]
    lib.ep_combine.argtypes = [P, P, P, i64, i32, i32, i64, P, i32, P, P]
    ok = ctypes.c_void_p(1 << 20)
    bad = ctypes.c_void_p((1 << 20) + 8)
    # fp8 needs H % 128 == 0
    assert lib.ep_dispatch(ok, ok, ok, ok, ok, 4, 2, 8, 200, 16, 1, ok, ok,
                           ok, 0, None, None) == ep.EP_ERR_INVALID_ARG
    # misaligned receive buffer
    assert lib.ep_dispatch(ok, ok, ok, ok, ok, 4, 2, 8, 256, 16, 0, bad, None,
                           None, 0, None, None) == ep.EP_ERR_ALIGNMENT
    # fp8 without scales
    assert lib.ep_dispatch(ok, ok, ok, ok, ok, 4, 2, 8, 256, 16, 1, ok, None,
                           None, 0, None, None) == ep.EP_ERR_ALIGNMENT
    assert lib.ep_combine(ok, ok, ok, 4, 2, 12, 16, ok, 0, None,
                          None) == ep.EP_ERR_INVALID_ARG   # H % 8
    assert lib.ep_combine(ok, ok, ok, 4, 2, 16, 16, bad, 0, None,
                          None) == ep.EP_ERR_ALIGNMENT
    assert lib.ep_combine(ok, ok, ok, 0, 2, 16, 16, ok, 0, None,
                          None) == ep.EP_OK                # nothing to do


def test_layout_dispatch_rejects_on_host():
    lib = _raw()
    P, i32, i64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    lib.ep_layout_dispatch.argtypes = [P, P, P, i32, i32, i32, i32, i32, i32,
                                       i32, P, P, P, P, i64, P, P, P, P, sz,
                                       i32, P, P]
    ok = ctypes.c_void_p(1 << 20)
    bad = ctypes.c_void_p((1 << 20) + 8)
    args = dict(R=4, S=8, K=2, E=8, H=256, pad=1, fp8=0, cap=64, recv=ok,
                scales=ok, ws=1 << 20, sms=0)

    def call(**kw):
        a = dict(args, **kw)
        return lib.ep_layout_dispatch(ok, ok, ok, a["R"], a["S"], a["K"],
                                      a["E"], a["H"], a["pad"], a["fp8"], ok,
                                      ok, ok, ok, a["cap"], a["recv"],
                                      a["scales"], None, ok, a["ws"],
                                      a["sms"], None, None)
    assert call(E=10) == ep.EP_ERR_INVALID_ARG        # E % R != 0
    assert call(fp8=1, H=200) == ep.EP_ERR_INVALID_ARG
    assert call(H=12) == ep.EP_ERR_INVALID_ARG
    assert call(sms=-1) == ep.EP_ERR_INVALID_ARG
    assert call(cap=63) == ep.EP_ERR_CAPACITY
    assert call(recv=bad) == ep.EP_ERR_ALIGNMENT
    assert call(fp8=1, scales=None) == ep.EP_ERR_ALIGNMENT
    assert call(ws=0) == ep.EP_ERR_WORKSPACE


def test_plan_prefetch_reject_on_host():
    lib = _raw()
    P, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    lib.ep_plan_balanced.argtypes = [P, i32, i32, i32, i32, i32, P, P, P, P,
                                     P, P, P]
    lib.ep_prefetch_weights.argtypes = [P, i32, i32, i32, i64, P, P, P, i32, P,
                                        P]
    ok = ctypes.c_void_p(1 << 20)
    assert lib.ep_plan_balanced(ok, 0, 4, 2, 8, 1, ok, ok, ok, ok, ok, None,
                                None) == ep.EP_ERR_INVALID_ARG
    assert lib.ep_plan_balanced(ok, 2, 4, 2, 8, 1, ok, ok, ok, ok, None, None,
                                None) == ep.EP_ERR_ALIGNMENT
    assert lib.ep_prefetch_weights(ok, 2, 8, 1, 7, ok, ok, ok, 0, None,
                                   None) == ep.EP_ERR_INVALID_ARG
    assert lib.ep_prefetch_weights(ok, 2, 8, 0, 8, ok, ok, ok, 0, None,
                                   None) == ep.EP_OK
    assert lib.ep_prefetch_weights(ok, 2, 8, 1, 8, ok, ok, ok, 0,
                                   ctypes.c_void_p(2), None) == ep.EP_ERR_ALIGNMENT


def test_force_timeouts_rejects_on_host():
    lib = _raw()
    lib.ep_debug_force_timeouts.argtypes = [ctypes.c_uint32, ctypes.c_int64]
    assert lib.ep_debug_force_timeouts(64, 1000) == ep.EP_ERR_INVALID_ARG
    assert lib.ep_debug_force_timeouts(ep.EP_WAIT_SITE_DISPATCH, 0) == \
        ep.EP_ERR_INVALID_ARG
    assert lib.ep_debug_force_timeouts(ep.EP_WAIT_SITE_DISPATCH,
                                       3_000_000_000) == ep.EP_ERR_INVALID_ARG


def test_stream_read_rejects_on_host():
    lib = _raw()
    P = ctypes.c_void_p
    lib.ep_debug_stream_read.argtypes = [P, ctypes.c_int64, P, P]
    ok = P(1 << 20)                       # aligned; never dereferenced
    assert lib.ep_debug_stream_read(ok, 33, ok, None) == ep.EP_ERR_INVALID_ARG
    assert lib.ep_debug_stream_read(ok, -32, ok, None) == ep.EP_ERR_INVALID_ARG
    assert lib.ep_debug_stream_read(ok, 64, None, None) == ep.EP_ERR_INVALID_ARG
    assert lib.ep_debug_stream_read(P((1 << 20) + 16), 64, ok, None) == \
        ep.EP_ERR_ALIGNMENT
    assert lib.ep_debug_stream_read(ok, 0, ok, None) == ep.EP_OK


def test_binding_rejects_host_tensors():
    import torch
    t = torch.zeros(8, dtype=torch.int32)
    with pytest.raises(ValueError):
        ep.ep_layout(t, 1, 4, 2, 2, 1, t, t, t, t, torch.zeros(
            64, dtype=torch.uint8))
    h = torch.zeros(4, 8, dtype=torch.bfloat16)
    wt = torch.zeros(4, 2, dtype=torch.float32)
    with pytest.raises(ValueError):
        ep.ep_layout_dispatch(t, h, wt, 1, 4, 2, 2, 8, 1, False, t, t, t, t,
                              h, workspace=torch.zeros(64, dtype=torch.uint8))


def test_static_layout_refuses_beyond_its_array_on_host():
    # refused before any CUDA call, so this runs without a GPU: with E=256
    # the 1 MiB array holds 1022 tiles of 4096 entries, and one entry more
    # needs a 1023rd
    lib = _raw()
    P, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    lib.ep_layout_static.argtypes = [P, i32, i32, i32, i32, i32, P, P, P, P,
                                     i64, P, P]
    E, limit = 256, 1022 * 4096
    assert ep.ep_layout_workspace_bytes(limit, 1, E) <= 1 << 20
    assert ep.ep_layout_workspace_bytes(limit + 1, 1, E) > 1 << 20
    ok = ctypes.c_void_p(1 << 20)
    assert lib.ep_layout_static(ok, 1, limit + 1, 1, E, 1, ok, ok, ok, ok,
                                limit + 1, None, None) == ep.EP_ERR_WORKSPACE
