"""combine_ep_layout_09_b200 -- MoE token dispatch / combine with an
expert-grouped layout, as hand-written sm_100a CUDA kernels behind a C ABI
(include/eplayout.h, built into libeplayout.so), with a thin ctypes binding.
"""
from ._binding import (  # noqa: F401
    EP_DEV_BAD_EXPERT, EP_DEV_CAPACITY, EP_DEV_PLAN_TOTAL, EP_DEV_SLOTS,
    EP_DEV_TIMEOUT, EP_ERR_ALIGNMENT, EP_WAIT_SITE_ALL, EP_WAIT_SITE_COMBINE,
    EP_WAIT_SITE_DISPATCH, EP_WAIT_SITE_LOOKBACK, EP_WAIT_SITE_PREFETCH,
    EP_WAIT_SITE_SMALL, EP_WAIT_SITE_TILE_REDUCE, EP_ERR_CAPACITY, EP_ERR_CUDA,
    EP_ERR_INVALID_ARG, EP_ERR_WORKSPACE, EP_OK, EPError, ep_abi_version,
    ep_capacity_bound, ep_combine, ep_combine_backward, ep_combine_recv_weights, ep_debug_bounded_wait,
    ep_debug_e4m3_encode, ep_debug_force_timeouts, ep_debug_quantize,
    ep_debug_stream_read, ep_dispatch,
    ep_dispatch_backward, ep_gather_route_weights, ep_layout, ep_layout_dispatch,
    ep_layout_workspace_bytes,
    ep_plan_balanced, ep_prefetch_weights, ep_reduce_slot_grads, ep_strerror, lib, library_path,
    strerror)
from .buffer import EPBuffer  # noqa: F401

lib()  # load (and if needed build) the CUDA library at import: no fallback
