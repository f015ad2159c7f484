"""Benchmark: MoE token dispatch / combine on B200, one JSON line on rank 0.

A step is one pass of the hot path over one batch: ep_layout (histogram,
padded offsets, stable positions) -> ep_dispatch (FP8 E4M3 1x128 for the
prefill and decode workloads, bf16 otherwise) -> ep_combine (fp32 fma, bf16
out). The balanced workload adds ep_plan_balanced and ep_prefetch_weights.
Inputs are seeded synthetic tensors resident in HBM before timing starts;
every workload's inputs are larger than L2, so no flush runs between steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   # the CPU oracle on a bounded sample

value = algorithmic bytes of all steps on all ranks / max-over-ranks time.
With N > 1 (torchrun, one process per GPU) every rank runs an independent
replica of the workload on its own batch: the path has no exchange between
logical ranks on one GPU, so the scaling is weak.
"""
from __future__ import annotations

import argparse
import contextlib
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = ("dispatch/combine GB/s and µs per call on 1 B200; "
          "fraction of HBM peak")
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0


# --------------------------------------------------------------------------
# byte accounting (algorithmic bytes: each input read once, each output
# written once)
# --------------------------------------------------------------------------

def bytes_layout(N, K, E, used_rows):
    # topk read by the histogram and by the position scan, pos written,
    # row_src written over the used rows, counts / offsets
    return 2 * N * K * 4 + N * K * 4 + used_rows * 4 + (2 * E + 1) * 4


def bytes_dispatch(N, K, H, fp8, used_rows):
    rd = N * H * 2 + N * K * 4 * 2 + used_rows * 4   # hidden, pos, w, row_src
    if fp8:
        wr = used_rows * (H + (H // 128) * 4 + 4)      # codes, scales, weight
    else:
        wr = used_rows * (H * 2 + 4)
    return rd + wr


def payload_dispatch(N, K, H, fp8):
    """Bytes that land in the receive buffer for real tokens (the analogue
    of the pages' per-link GB/s)."""
    return N * K * (H + (H // 128) * 4 if fp8 else H * 2)


def bytes_combine(N, K, H):
    return N * K * H * 2 + N * K * 4 * 2 + N * H * 2


def bytes_prefetch(n_slots, H, I):
    return 3 * n_slots * H * I * 2 * 2


def bytes_combine_backward(N, K, H, used_rows):
    # grad_out and the K gathered expert-output rows read, every used
    # receive row's gradient written (padding rows zeroed), grad_w written
    return (N * H * 2 + N * K * H * 2 + N * K * 8 + used_rows * 4 +
            used_rows * H * 2 + N * K * 4)


def bytes_dispatch_backward(N, K, H):
    return N * K * H * 2 + N * K * 4 + N * H * 2


def bytes_reduce_slot_grads(slots, H, I):
    """fp32 gradients: per expert with n slots, its row read and written and
    its n slot rows read, for three projections."""
    import collections
    groups = collections.Counter(int(e) for e in slots.ravel() if e >= 0)
    return 3 * sum(n + 2 for n in groups.values()) * H * I * 4


# --------------------------------------------------------------------------
# environment helpers
# --------------------------------------------------------------------------

def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def dist_info():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(x: float, device) -> float:
    """Max of a per-rank time over all ranks (identity without a group)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return x
    if dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def total_value_gbs(bytes_per_step: int, steps: int, world: int,
                    ms_max: float) -> float:
    """Whole-job throughput: bytes of all steps on all ranks / max time."""
    return bytes_per_step * steps * world / (ms_max * 1e-3) / 1e9


class ClockSampler:
    """Samples SM clock and throttle reasons with NVML every millisecond."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting",
        0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x10: "sync_boost",
        0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int):
        self.samples, self.reasons = [], 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            h = None
            try:
                uuid = str(torch.cuda.get_device_properties(device_index).uuid)
                h = pynvml.nvmlDeviceGetHandleByUUID(
                    uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            except Exception:
                h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.h = h
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(
                h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(
                    self.h, nv.NVML_CLOCK_SM))
                self.reasons |= int(
                    nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
            except Exception:
                pass
            time.sleep(0.001)

    def __enter__(self):
        if self.nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()

    def summary(self):
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit
                 and n != "gpu_idle"]
        return {"sm_mhz": (statistics.median(self.samples)
                           if self.samples else None),
                "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(self.samples), "source": "nvml"}


def traffic_from_profiles(kernel: str, workload: str, src_file: str):
    """DRAM bytes per launch recorded by ncu, if the profile summary names
    the current source of the kernel (else None)."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(p):
        return None
    sha = hashlib.sha256(open(src_file, "rb").read()).hexdigest()[:16]
    for line in open(p):
        if line.startswith("#") or not line.strip():
            continue
        f = dict(kv.split("=", 1) for kv in line.split())
        if (f.get("kernel") == kernel and f.get("workload") == workload
                and f.get("src_sha") == sha):
            return float(f["dram_bytes_per_launch"])
    return None


# --------------------------------------------------------------------------
# the GPU path
# --------------------------------------------------------------------------

def layout_dispatch_kernels(wl, sms=148):
    """Kernels one ep_layout_dispatch call launches, by the library's size
    rule: one for N*K <= 32768 with at most 1024 entries per CTA; else the
    cooperative layout kernel (tiles of 4096 entries all resident) or the
    histogram + scan pair, then the dispatch kernel."""
    entries = wl.N * wl.K
    chunk = -(-wl.N // sms)
    if entries <= 32768 and chunk * wl.K <= 1024:
        return 1
    tiles = -(-entries // 4096)
    return (1 if tiles <= sms else 2) + 1


def combine_kernel(wl, sms=148):
    """Kernel one ep_combine launch runs, by the library's size rule: the
    bulk-copy pipeline k_combine_tma when the row splits into parts whose K
    part-rows fill a stage of at most 64 KB, its shared memory stays within
    200 KB, and there are at least 16 (token, part) units per SM; else the
    register gather k_combine<K>."""
    al = lambda x: (x + 127) & ~127  # noqa: E731
    max_ch = max(8, (65536 // (wl.K * 2)) & ~7)
    parts = -(-wl.H // max_ch)
    part_ch = (-(-wl.H // parts) + 7) & ~7
    smem = 3 * al(wl.K * part_ch * 2) + 3 * (16 + 4 + 4 * 32) + 64
    if smem <= 200 * 1024 and wl.N * parts >= 16 * sms:
        return "k_combine_tma"
    return f"k_combine<{wl.K}>"


class Path:
    """All device buffers of one replica, allocated once."""

    def __init__(self, wl, dev, seed_offset=0):
        import combine_ep_layout_09_b200 as ep
        self.ep = ep
        self.wl = wl
        self.dev = dev
        topk, w = workloads.routing(workloads.scaled(
            wl, seed=wl.seed + seed_offset))
        self.topk_np, self.w_np = topk, w
        i32 = dict(dtype=torch.int32, device=dev)
        self.topk = torch.from_numpy(topk).to(dev)
        self.w = torch.from_numpy(w).to(dev)
        self.hidden = workloads.bf16_normal((wl.N, wl.H), 1000 + wl.seed +
                                            seed_offset, device=dev)
        self.cap = ep.ep_capacity_bound(wl.N, wl.K, wl.E, wl.pad)
        self.counts = torch.zeros(wl.E, **i32)
        self.offsets = torch.zeros(wl.E + 1, **i32)
        self.pos = torch.zeros(wl.N, wl.K, **i32)
        self.row_src = torch.zeros(self.cap, **i32)
        self.ws = torch.zeros(ep.ep_layout_workspace_bytes(wl.N, wl.K, wl.E),
                              dtype=torch.uint8, device=dev)
        self.status = torch.zeros(4, **i32)
        if wl.fp8:
            self.recv = torch.empty(self.cap, wl.H, dtype=torch.float8_e4m3fn,
                                    device=dev)
            self.scales = torch.empty(self.cap, wl.H // 128,
                                      dtype=torch.float32, device=dev)
        else:
            self.recv = torch.empty(self.cap, wl.H, dtype=torch.bfloat16,
                                    device=dev)
            self.scales = None
        self.recv_w = torch.empty(self.cap, dtype=torch.float32, device=dev)
        # stand-in expert outputs, one bf16 row per receive row
        self.y = workloads.expert_outputs(self.cap, wl.H, wl.seed +
                                          seed_offset, device=dev)
        self.out = torch.empty(wl.N, wl.H, dtype=torch.bfloat16, device=dev)
        if wl.B > 0:
            R, E, B = wl.R, wl.E, wl.B
            self.plan = dict(cu=torch.empty(R, E + 1, **i32),
                             expert=torch.empty(R, E, **i32),
                             wrow=torch.empty(R, E, **i32),
                             nseg=torch.empty(R, **i32),
                             slot=torch.empty(R, B, **i32))
            rows = E + R * B
            self.W = [workloads.weight_buffer(rows, wl.H, wl.I, wl.seed + j,
                                              device=dev) for j in range(3)]
        self.launches_per_step = (layout_dispatch_kernels(wl) + 1 +
                                  (2 if wl.B > 0 else 0))
        self.backward = False

    def enable_backward(self, seed_offset=0):
        """Buffers of the backward pair: a synthetic gradient of the
        combined output, gradients of the expert outputs / route weights /
        token rows."""
        wl, dev = self.wl, self.dev
        self.backward = True
        self.grad_out = workloads.bf16_normal((wl.N, wl.H), 4000 + wl.seed +
                                              seed_offset, device=dev)
        self.grad_rows = torch.empty(self.cap, wl.H, dtype=torch.bfloat16,
                                     device=dev)
        self.grad_w = torch.empty(wl.N, wl.K, dtype=torch.float32, device=dev)
        self.grad_hidden = torch.empty(wl.N, wl.H, dtype=torch.bfloat16,
                                       device=dev)
        self.launches_per_step += 2
        if wl.B > 0:
            rows = wl.E + wl.R * wl.B
            self.GW = [torch.zeros(rows, wl.H, wl.I, dtype=torch.float32,
                                   device=dev) for _ in range(3)]
            self.launches_per_step += 1

    def reduce_slot_grads(self, io=None):
        wl = self.wl
        self.ep.ep_reduce_slot_grads(self.plan["slot"], wl.R, wl.E, wl.B,
                                     *self.GW)

    def combine_backward(self, io=None):
        wl = self.wl
        io = io or self.io()
        self.ep.ep_combine_backward(self.grad_out, self.y, self.pos,
                                    self.row_src, self.offsets, io["w"], wl.N,
                                    wl.K, wl.E, wl.H, self.grad_rows,
                                    self.grad_w, status=self.status,
                                    cap=self.cap)

    def dispatch_backward(self, io=None):
        wl = self.wl
        self.ep.ep_dispatch_backward(self.grad_rows, self.pos, wl.N, wl.K,
                                     wl.H, self.grad_hidden,
                                     status=self.status, cap=self.cap)

    def io(self):
        """The buffers a user hands in and gets back (one set)."""
        return dict(hidden=self.hidden, topk=self.topk, w=self.w,
                    out=self.out)

    def layout(self, io=None):
        wl = self.wl
        topk = (io or self.io())["topk"]
        self.ep.ep_layout(topk, wl.R, wl.S, wl.K, wl.E, wl.pad,
                          self.counts, self.offsets, self.pos, self.row_src,
                          self.ws, self.status, cap=self.cap)

    def plan_prefetch(self):
        wl, p = self.wl, self.plan
        self.ep.ep_plan_balanced(self.counts, wl.R, wl.S, wl.K, wl.E, wl.B,
                                 p["cu"], p["expert"], p["wrow"], p["nseg"],
                                 p["slot"], self.status)
        self.ep.ep_prefetch_weights(p["slot"], wl.R, wl.E, wl.B, *self.W,
                                    status=self.status)

    def layout_dispatch(self, io=None):
        """The user's dispatch call: layout and copy (one launch for a small
        batch, ep_layout + ep_dispatch otherwise)."""
        wl = self.wl
        io = io or self.io()
        self.ep.ep_layout_dispatch(io["topk"], io["hidden"], io["w"], wl.R,
                                   wl.S, wl.K, wl.E, wl.H, wl.pad, wl.fp8,
                                   self.counts, self.offsets, self.pos,
                                   self.row_src, self.recv, self.scales,
                                   self.recv_w, workspace=self.ws,
                                   status=self.status, cap=self.cap)

    def dispatch(self, io=None):
        wl = self.wl
        io = io or self.io()
        self.ep.ep_dispatch(io["hidden"], io["w"], self.pos, self.row_src,
                            self.offsets, wl.N, wl.K, wl.E, wl.H, wl.fp8,
                            self.recv, self.scales, self.recv_w,
                            status=self.status, cap=self.cap)

    def combine(self, io=None):
        wl = self.wl
        io = io or self.io()
        self.ep.ep_combine(self.y, self.pos, io["w"], wl.N, wl.K, wl.H,
                           io["out"], status=self.status, cap=self.cap)

    def combine_recv_weights(self, io=None):
        """The combine with receive-side weights (the EPBuffer call)."""
        wl = self.wl
        io = io or self.io()
        if not hasattr(self, "gathered"):
            self.gathered = torch.empty(wl.N, wl.K, dtype=torch.float32,
                                        device=self.dev)
        self.ep.ep_combine_recv_weights(self.y, self.pos, self.recv_w, wl.N,
                                        wl.K, wl.H, io["out"], self.gathered,
                                        status=self.status, cap=self.cap)

    def step(self, io=None):
        self.layout_dispatch(io)
        if self.wl.B > 0:
            self.plan_prefetch()
        self.combine(io)
        if self.backward:
            self.combine_backward(io)
            self.dispatch_backward(io)
            if self.wl.B > 0:
                self.reduce_slot_grads(io)


@contextlib.contextmanager
def nvtx(name: str):
    """NVTX range around a phase of the benchmark (seen by nsys / ncu)."""
    torch.cuda.nvtx.range_push(name)
    try:
        yield
    finally:
        torch.cuda.nvtx.range_pop()


def capture(fn, n):
    """One CUDA graph of n calls of fn (the library allocates nothing and
    never synchronises, so its calls capture as they are)."""
    cs = torch.cuda.Stream()
    cs.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cs):
        for i in range(n):
            fn(i)
    torch.cuda.synchronize()
    return g


def replay_ms(g):
    a_, b_ = (torch.cuda.Event(enable_timing=True),
              torch.cuda.Event(enable_timing=True))
    a_.record()
    g.replay()
    b_.record()
    torch.cuda.synchronize()
    return a_.elapsed_time(b_)


def step_bytes(path, backward):
    """Algorithmic bytes of one step of `path` and of each of its calls
    (after a warm-up step: padding makes the used rows data-dependent)."""
    wl = path.wl
    used = int(path.offsets[-1].item())
    n_slots = int((path.plan["slot"] >= 0).sum().item()) if wl.B else 0
    b = {"layout": bytes_layout(wl.N, wl.K, wl.E, used),
         "dispatch": bytes_dispatch(wl.N, wl.K, wl.H, wl.fp8, used),
         "combine": bytes_combine(wl.N, wl.K, wl.H),
         "plan_prefetch": bytes_prefetch(n_slots, wl.H, wl.I) if wl.B else 0,
         "combine_backward": (bytes_combine_backward(wl.N, wl.K, wl.H, used)
                              if backward else 0),
         "dispatch_backward": (bytes_dispatch_backward(wl.N, wl.K, wl.H)
                               if backward else 0),
         "reduce_slot_grads": (bytes_reduce_slot_grads(
             path.plan["slot"].cpu().numpy(), wl.H, wl.I)
             if backward and wl.B else 0),
         "used_rows": used}
    b["layout_dispatch"] = b["layout"] + b["dispatch"]
    b["step"] = (b["layout_dispatch"] + b["combine"] + b["plan_prefetch"] +
                 b["combine_backward"] + b["dispatch_backward"] +
                 b["reduce_slot_grads"])
    return b


def percentiles(us):
    return {"p10": round(float(np.percentile(us, 10)), 2),
            "p50": round(float(np.percentile(us, 50)), 2),
            "p90": round(float(np.percentile(us, 90)), 2),
            "calls": len(us)}


def measure(paths, K, warmup, backward, device_index, flush, barrier=None,
            rank_max=None, kernels=True):
    """Time one workload on the input sets `paths` (one Path each).

    The K timed steps are captured once into a CUDA graph and replayed once,
    so no host launch gap sits between kernels; step i runs on input set
    i % len(paths), so that with several sets a set's data has left the
    126 MB L2 before it is used again. Each call's own average comes the
    same way from a graph of K launches of that call alone (events between
    kernels inside one graph would add their own gaps). Then each call is
    timed alone with CUDA events (eager launches, so the interval includes
    the launch), after writing the 512 MB `flush` buffer so that no call
    finds its inputs in L2 (p10 / p50 / p90); steps smaller than the flush
    are also timed L2-hot, calls back to back on one set."""
    barrier = barrier or (lambda: None)
    rank_max = rank_max or (lambda x: x)
    n = len(paths)
    wl = paths[0].wl
    with nvtx(f"{wl.name}: warm-up"):
        for _ in range(warmup):
            for p in paths:
                p.step()
        torch.cuda.synchronize()
    for p in paths:
        st = int(p.status[0].item())
        if st:
            raise RuntimeError(f"device status after warm-up: {st}")
    bts = [step_bytes(p, backward) for p in paths]
    b_total = sum(bts[i % n]["step"] for i in range(K))

    graph = capture(lambda i: paths[i % n].step(), K)
    start = torch.cuda.Event(enable_timing=True)
    stop = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with nvtx(f"{wl.name}: timed steps"), ClockSampler(device_index) as clk:
        start.record()
        graph.replay()
        stop.record()
        torch.cuda.synchronize()
    barrier()
    del graph
    ms = rank_max(start.elapsed_time(stop))

    calls = ["layout_dispatch", "combine"]
    if kernels:
        calls += ["layout", "dispatch", "combine_recv_weights"]
    if wl.B:
        calls.append("plan_prefetch")
    if backward:
        calls += ["combine_backward", "dispatch_backward"]
        if wl.B:
            calls.append("reduce_slot_grads")
    avg = {}
    with nvtx(f"{wl.name}: per-call graphs"):
        for name in calls:
            g = capture(lambda i: getattr(paths[i % n], name)(), K)
            avg[name] = replay_ms(g) / K * 1e3     # us per launch
            del g
    per_call = {}
    timed = ["layout_dispatch", "combine"] + (["plan_prefetch"] if wl.B else [])
    # l2_flushed: 512 MB written before each call, so L2 holds none of the
    # call's data but is full of dirty lines the call's own traffic must
    # write back first; l2_clean: the same write, then a read of the 512 MB,
    # so L2 holds none of the call's data and only clean lines
    modes = [("l2_flushed", "write"), ("l2_clean", "write+read")]
    if bts[0]["step"] < flush.numel():
        modes.append(("l2_hot", None))
    flush64 = flush.view(torch.int64)
    with nvtx(f"{wl.name}: per-call distribution"):
        for mode, how in modes:
            for name in timed:
                n_calls = 10 if name == "plan_prefetch" else 50
                evs = []
                if how is None:
                    # keep the GPU busy while the host enqueues the calls,
                    # so that they run back to back and each interval is
                    # GPU time
                    torch.cuda._sleep(4_000_000)
                for c in range(n_calls):
                    p = paths[c % n] if how else paths[0]
                    if how:
                        flush.fill_(1)
                    if how == "write+read":
                        flush64.max()
                    a_, b_ = (torch.cuda.Event(enable_timing=True),
                              torch.cuda.Event(enable_timing=True))
                    a_.record()
                    getattr(p, name)()
                    b_.record()
                    evs.append((a_, b_))
                torch.cuda.synchronize()
                us = np.array([a_.elapsed_time(b_) * 1e3 for a_, b_ in evs])
                per_call.setdefault(mode, {})[name] = percentiles(us)
    for p in paths:
        st = int(p.status[0].item())
        if st:
            raise RuntimeError(f"device status after timing: {st}")
    # bytes per call averaged over the sets
    mean_b = {k: sum(b[k] for b in bts) / n for k in bts[0]}
    return {"ms": ms, "K": K, "bytes_total": b_total, "bytes": mean_b,
            "avg_us": avg, "per_call_us": per_call, "clocks": clk.summary(),
            "sets": n}


def gbps(nbytes, us):
    return nbytes / (us * 1e-6) / 1e9 if us > 0 else None


def kernel_names(wl, sms=148):
    """Kernels the step launches, by the library's size rules (mirrored
    here; tests/test_bench_accounting.py pins the mirror)."""
    one_launch = layout_dispatch_kernels(wl, sms) == 1
    prec = "fp8" if wl.fp8 else "bf16"
    if one_launch:
        disp = f"k_layout_small<{prec}>"
    else:
        # a grid of one CTA per token when every SM is in use
        disp = f"k_dispatch_{prec}_tok"
    return {"one_launch": one_launch, "dispatch": disp,
            "combine": combine_kernel(wl, sms)}


def arithmetic(wl):
    return (("fp8-e4m3 dispatch (1x128 fp32 scales, x/scale in fp32)"
             if wl.fp8 else "bf16 dispatch (bit copy)") +
            ", bf16 combine with fp32 fma accumulation")


def workload_summary(wl, m, peak):
    """The line for a workload other than the headline one."""
    avg, b = m["avg_us"], m["bytes"]
    names = kernel_names(wl)
    out = {
        "workload": wl.describe,
        "arithmetic": arithmetic(wl),
        "input_sets": m["sets"],
        "l2": (f"{m['sets']} input sets rotated, {m['sets']} x "
               f"{b['step'] / 1e6:.0f} MB per rotation > the 126 MB L2"
               if m["sets"] > 1 else
               f"one input set; every step moves {b['step'] / 1e6:.0f} MB, "
               "more than the 126 MB L2"),
        "step_us": round(m["ms"] / m["K"] * 1e3, 2),
        "step_GBps": round(m["bytes_total"] / (m["ms"] * 1e-3) / 1e9, 1),
        "graph_us": {k: round(v, 2) for k, v in avg.items()},
        "per_call_us": m["per_call_us"],
        "kernels": names,
        "clocks": m["clocks"],
    }
    rates = {}
    for k in ("layout_dispatch", "combine", "plan_prefetch"):
        if k in avg and b[k]:
            r = gbps(b[k], avg[k])
            rates[k] = {"bytes": int(b[k]), "GBps": round(r, 1),
                        "frac_of_measured": round(r / peak, 4),
                        "frac_of_8TBps": round(r / NOMINAL_HBM_GBS, 4)}
            fl = m["per_call_us"].get("l2_flushed", {}).get(k)
            if fl:
                r50 = gbps(b[k], fl["p50"])
                rates[k]["flushed_p50_GBps"] = round(r50, 1)
                rates[k]["flushed_p50_frac_of_measured"] = round(r50 / peak, 4)
    out["rates"] = rates
    return out


def time_epbuffer(path, K, dev):
    """One pass of the pages' Buffer call shape (EPBuffer.dispatch, then
    EPBuffer.combine on stand-in expert outputs), timed beside the raw-call
    step: a graph of K passes, and K eager passes with the Python of the
    binding and of EPBuffer on the host side."""
    from combine_ep_layout_09_b200 import EPBuffer
    wl = path.wl
    buf = EPBuffer(wl.S, wl.H, wl.K, wl.E, wl.R, token_padding=wl.pad,
                   fp8=wl.fp8, device=dev)

    def one(_i=0):
        _, _, _, h = buf.dispatch(path.hidden, path.w, path.topk)
        buf.combine(h, path.y)

    for _ in range(3):
        one()
    torch.cuda.synchronize()
    g = capture(one, K)
    graph_us = replay_ms(g) / K * 1e3
    del g
    a_, b_ = (torch.cuda.Event(enable_timing=True),
              torch.cuda.Event(enable_timing=True))
    a_.record()
    for _ in range(K):
        one()
    b_.record()
    torch.cuda.synchronize()
    eager_us = a_.elapsed_time(b_) / K * 1e3
    buf.check()
    del buf
    return {"graph_us_per_pass": round(graph_us, 2),
            "eager_us_per_pass": round(eager_us, 2),
            "calls": "EPBuffer.dispatch (ep_layout_dispatch) + "
                     "EPBuffer.combine (ep_combine_recv_weights: receive-"
                     "side weights, gathered weights written, no allocation)",
            "launches_per_pass": layout_dispatch_kernels(wl) + 1}


EXTRA_WORKLOADS = {"decode": 4, "skewed": 1, "balanced": 1}


def run_gpu(args, wl):
    ws, rank, local = dist_info()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(
            seconds=120), device_id=dev)

    def barrier():
        if ws > 1:
            import torch.distributed as dist
            dist.barrier()

    def rank_max(x: float) -> float:
        return max_over_ranks(x, dev)

    K = args.steps
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    # the headline workload: one input set (every step moves more than L2)
    # unless the step is smaller than the 512 MB flush, then four
    n_sets = 1
    path = Path(wl, dev, seed_offset=rank)
    if args.backward:
        path.enable_backward(seed_offset=rank)
    paths = [path]
    torch.cuda.synchronize()
    path.step()
    torch.cuda.synchronize()
    if step_bytes(path, args.backward)["step"] < flush.numel():
        n_sets = 4
        for j in range(1, n_sets):
            p = Path(wl, dev, seed_offset=rank + 100 * j)
            if args.backward:
                p.enable_backward(seed_offset=rank + 100 * j)
            paths.append(p)
    m = measure(paths, K, args.warmup, args.backward, local, flush, barrier,
                rank_max)
    avg, b = m["avg_us"], m["bytes"]
    ms_max = m["ms"]

    # ---- end to end: host buffers in, host result out, every step -------
    e2e = None
    if not args.no_e2e:
        with nvtx(f"{wl.name}: end to end"):
            e2e = run_e2e(args, path, b["step"], rank_max, barrier)

    # a streaming read and a streaming write of 4 GiB, timed here as
    # context: a read-heavy call such as combine can pass the copy peak, a
    # write-heavy one such as dispatch is bounded by the write rate. The read
    # is the library's 256-bit streaming read (faster than torch's
    # reduction on this part), the write torch's fill (faster than plain
    # grid-stride stores).
    read_probe = write_probe = None
    if rank == 0 and not args.no_read_probe:
        with nvtx("read / write probes"):
            x = torch.empty(4 << 30, dtype=torch.uint8, device=dev).view(
                torch.int64)

            def rate(fn):
                for _ in range(2):
                    fn()
                a_, b_ = (torch.cuda.Event(enable_timing=True),
                          torch.cuda.Event(enable_timing=True))
                a_.record()
                for _ in range(5):
                    fn()
                b_.record()
                torch.cuda.synchronize()
                return (4 << 30) * 5 / (a_.elapsed_time(b_) * 1e-3) / 1e9

            write_probe = rate(lambda: x.fill_(1))
            sink = torch.zeros(1, dtype=torch.int32, device=dev)
            read_probe = rate(lambda: path.ep.ep_debug_stream_read(x, sink))
            del x

    epbuf = None
    if ws == 1 and not args.no_epbuffer:
        with nvtx(f"{wl.name}: EPBuffer pass"):
            epbuf = time_epbuffer(path, K, dev)

    result = None
    if rank == 0:
        peak, peak_src = measured_peak()
        value = total_value_gbs(m["bytes_total"] / K, K, ws, ms_max)
        names = kernel_names(wl)
        one_launch = names["one_launch"]
        comb_gbs = gbps(b["combine"], avg["combine"])
        dis_gbs = gbps(b["dispatch"], avg["dispatch"])
        ld_gbs = gbps(b["layout_dispatch"], avg["layout_dispatch"])
        # the dominant kernel: combine, or the dispatch side's longest kernel
        # (the single layout+dispatch kernel of a small batch)
        if one_launch:
            cand = ("layout_dispatch", names["dispatch"], "layout_small.cu",
                    b["layout_dispatch"], ld_gbs)
        else:
            cand = ("dispatch", names["dispatch"], "dispatch.cu",
                    b["dispatch"], dis_gbs)
        if avg["combine"] >= avg[cand[0]]:
            cand = ("combine", names["combine"], "combine.cu", b["combine"],
                    comb_gbs)
        dom, kname, ksrc, dom_bytes, dom_gbs = cand
        src = os.path.join(ROOT, "combine_ep_layout_09_b200", "csrc", ksrc)
        traffic = traffic_from_profiles(kname, wl.name, src)
        clocks = m["clocks"]
        per_call = m["per_call_us"]
        result = {
            "metric": METRIC,
            "value": round(value, 1),
            "unit": "GB/s",
            "n_gpus": ws,
            "steps": K,
            "warmup": args.warmup,
            "ms_per_step": round(ms_max / K, 4),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": ("e4m3+bf16, fp32 accumulate" if wl.fp8 else
                      "bf16, fp32 accumulate"),
            "data": "synthetic",
            "config": {
                "workload": wl.describe,
                "arithmetic": arithmetic(wl),
                "step": ("ep_layout_dispatch (" +
                         ("one launch" if one_launch else
                          "ep_layout + ep_dispatch") + ") + " +
                         ("ep_plan_balanced + ep_prefetch_weights + "
                          if wl.B else "") + "ep_combine" +
                         (" + ep_combine_backward + ep_dispatch_backward"
                          if args.backward else "") +
                         (" + ep_reduce_slot_grads"
                          if args.backward and wl.B else "")),
                "bytes_per_step": int(b["step"]),
                "used_rows": int(b["used_rows"]),
                "input_sets": m["sets"],
                "l2": (f"no flush: every step moves {b['step'] / 1e6:.0f} MB,"
                       " more than the 126 MB L2" if m["sets"] == 1 else
                       f"{m['sets']} input sets rotated, "
                       f"{m['sets'] * b['step'] / 1e6:.0f} MB per rotation, "
                       "more than the 126 MB L2"),
                "parallelism": f"{ws} independent replica(s), one per GPU",
                "timing": "K steps captured in one CUDA graph, replayed "
                          "once, CUDA events around the replay; per-call "
                          "averages from a graph of K launches of that call",
            },
            "per_call_us": per_call,
            "breakdown": {
                "layout_dispatch_us": round(avg["layout_dispatch"], 2),
                "layout_dispatch_GBps": round(ld_gbs, 1),
                "layout_dispatch_one_launch": one_launch,
                "layout_us": round(avg["layout"], 2),
                "dispatch_us": round(avg["dispatch"], 2),
                "combine_us": round(avg["combine"], 2),
                "combine_recv_weights_us": round(
                    avg.get("combine_recv_weights", 0.0), 2),
                "plan_prefetch_us": round(avg.get("plan_prefetch", 0.0), 2),
                "layout_plus_dispatch_us": round(avg["layout"] +
                                                 avg["dispatch"], 2),
                "dispatch_GBps": round(dis_gbs, 1),
                "combine_GBps": round(comb_gbs, 1),
                "dispatch_payload_GBps": round(
                    payload_dispatch(wl.N, wl.K, wl.H, wl.fp8) /
                    (avg["dispatch"] * 1e-6) / 1e9, 1),
                "combine_backward_us": round(avg.get("combine_backward", 0), 2),
                "dispatch_backward_us": round(avg.get("dispatch_backward", 0),
                                              2),
                "combine_backward_GBps": round(gbps(
                    b["combine_backward"], avg["combine_backward"]), 1)
                if args.backward else None,
                "dispatch_backward_GBps": round(gbps(
                    b["dispatch_backward"], avg["dispatch_backward"]), 1)
                if args.backward else None,
                "reduce_slot_grads_us": round(avg.get("reduce_slot_grads", 0),
                                              2),
                "reduce_slot_grads_GBps": round(gbps(
                    b["reduce_slot_grads"], avg["reduce_slot_grads"]), 1)
                if b["reduce_slot_grads"] else None,
                "dispatch_bytes": int(b["dispatch"]),
                "combine_bytes": int(b["combine"]),
                "layout_bytes": int(b["layout"]),
                "prefetch_bytes": int(b["plan_prefetch"]),
                "kernels": names,
                "frac_of_8TBps": {
                    "dispatch": round(dis_gbs / NOMINAL_HBM_GBS, 4),
                    "layout_dispatch": round(ld_gbs / NOMINAL_HBM_GBS, 4),
                    "combine": round(comb_gbs / NOMINAL_HBM_GBS, 4)},
                "frac_of_measured": {
                    "dispatch": round(dis_gbs / peak, 4),
                    "layout_dispatch": round(ld_gbs / peak, 4),
                    "combine": round(comb_gbs / peak, 4)},
            },
            "roofline": {
                "bound": "hbm",
                "kernel": kname,
                "call": dom,
                "achieved": round(dom_gbs, 1),
                "peak": peak,
                "unit": "GB/s",
                "frac": round(dom_gbs / peak, 4),
                "traffic": traffic,
                "algorithmic_bytes": int(dom_bytes),
                "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)"
                if peak_src == "measured" else "fallback 6.65 TB/s",
                "read_probe_GBps": (round(read_probe, 1) if read_probe
                                    else None),
                "frac_of_read_probe": (round(dom_gbs / read_probe, 4)
                                       if read_probe else None),
                "write_probe_GBps": (round(write_probe, 1) if write_probe
                                     else None),
                "dispatch_frac_of_write_probe": (
                    round(dis_gbs / write_probe, 4) if write_probe else None),
                "note": "peak is a copy (half reads, half writes); a "
                        "read-heavy call such as combine (89% reads) can "
                        "pass it, so the same call is also given against a "
                        "4 GiB streaming read timed in this run (256-bit "
                        "loads, ep_debug_stream_read), and the write-heavy "
                        "dispatch (80% writes) against a 4 GiB streaming "
                        "write (torch fill)",
            },
            "clocks": clocks,
            "e2e": e2e,
            "epbuffer": epbuf,
            "gpu_launches": path.launches_per_step * K,
            "gpu_launches_note": "kernels of libeplayout.so in the timed "
                                 "region" + ("" if one_launch else
                                             "; ep_layout adds one "
                                             "cudaMemsetAsync per step"),
        }
    del paths, path
    torch.cuda.empty_cache()

    # ---- the other workloads, in the same process (one GPU only) --------
    extras = {}
    if ws == 1 and not args.no_extra_workloads and wl.name == "prefill" \
            and args.tokens_per_rank is None:
        peak, _ = measured_peak()
        for name, sets in EXTRA_WORKLOADS.items():
            xw = workloads.WORKLOADS[name]
            with nvtx(f"{name}: setup"):
                xp = [Path(xw, dev, seed_offset=100 * j) for j in range(sets)]
                torch.cuda.synchronize()
            xm = measure(xp, K, args.warmup, False, local, flush,
                         kernels=False)
            extras[name] = workload_summary(xw, xm, peak)
            del xp
            torch.cuda.empty_cache()
    if result is not None and extras:
        # the decode step's receive rows stay in L2: its layout + dispatch
        # call is given against an L2-resident write as well (a graph of
        # 20 fills of one 64 MB buffer)
        if "decode" in extras and not args.no_read_probe:
            x = torch.empty(64 << 20, dtype=torch.uint8, device=dev)
            x.fill_(1)
            g = capture(lambda i: x.fill_(i & 1), 20)
            replay_ms(g)
            l2w = (64 << 20) * 20 / (replay_ms(g) * 1e-3) / 1e9
            del g, x
            dec = extras["decode"]
            ld = dec["rates"]["layout_dispatch"]
            dec["l2_write_probe_GBps"] = round(l2w, 1)
            ld["frac_of_l2_write_probe"] = round(ld["GBps"] / l2w, 4)
        result["workloads"] = extras
    del flush
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return result


def run_e2e(args, path, b_step, max_over_ranks, barrier):
    """Same step with the user's inputs in pinned host memory: every step
    copies hidden, topk and route weights in (H2D) and the combined output
    out (D2H) inside the timed region. Copies in, compute and copies out
    run on three streams with two buffer sets, so step i's D2H overlaps
    step i+1's H2D (PCIe is full duplex) and the kernels of either."""
    wl = path.wl
    h_hidden = path.hidden.cpu().pin_memory()
    h_topk = path.topk.cpu().pin_memory()
    h_w = path.w.cpu().pin_memory()
    h_out = [torch.empty(path.out.shape, dtype=path.out.dtype).pin_memory()
             for _ in range(2)]
    sets = [path.io(), dict(hidden=torch.empty_like(path.hidden),
                            topk=torch.empty_like(path.topk),
                            w=torch.empty_like(path.w),
                            out=torch.empty_like(path.out))]
    # The first step's H2D and the last step's D2H overlap nothing; the run
    # is long enough (default 40 steps) that this fill and drain weigh
    # little against the steady state.
    steps = max(1, args.e2e_steps)
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    s_comp = torch.cuda.current_stream()
    ev = lambda: torch.cuda.Event()  # noqa: E731
    done_in = [ev(), ev()]
    done_comp = [ev(), ev()]
    done_out = [ev(), ev()]
    used = [False, False]

    def one(j):
        b = j % 2
        io = sets[b]
        if used[b]:
            s_in.wait_event(done_comp[b])    # its inputs were consumed
        with torch.cuda.stream(s_in):
            io["hidden"].copy_(h_hidden, non_blocking=True)
            io["topk"].copy_(h_topk, non_blocking=True)
            io["w"].copy_(h_w, non_blocking=True)
            done_in[b].record(s_in)
        s_comp.wait_event(done_in[b])
        if used[b]:
            s_comp.wait_event(done_out[b])   # its output was read back
        path.step(io)
        done_comp[b].record(s_comp)
        s_out.wait_event(done_comp[b])
        with torch.cuda.stream(s_out):
            h_out[b].copy_(io["out"], non_blocking=True)
            done_out[b].record(s_out)
        used[b] = True

    for j in range(2):
        one(j)
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    stop = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    start.record(s_in)
    for j in range(steps):
        one(j)
    s_in.wait_stream(s_out)
    stop.record(s_in)
    torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(start.elapsed_time(stop))
    ws, _, _ = dist_info()
    h2d = (h_hidden.numel() * h_hidden.element_size() + h_topk.numel() * 4 +
           h_w.numel() * 4)
    d2h = h_out[0].numel() * h_out[0].element_size()
    return {"value": round(b_step * steps * ws / (ms * 1e-3) / 1e9, 1),
            "unit": "GB/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": steps,
            "ms_per_step": round(ms / steps, 3),
            "note": "H2D, kernels and D2H on three streams, two buffer "
                    "sets, fill and drain of the pipeline inside the timed "
                    "steps; expert outputs (combine input) stay "
                    "device-resident"}


# --------------------------------------------------------------------------
# the CPU oracle (baseline / reference arm)
# --------------------------------------------------------------------------

def oracle_sample(wl, n_tok, seed_offset=0):
    """Inputs for the first n_tok tokens of the workload (host)."""
    topk, w = workloads.routing(workloads.scaled(wl, seed=wl.seed +
                                                 seed_offset))
    hid = workloads.bf16_normal((n_tok, wl.H), 1000 + wl.seed + seed_offset)
    h = hid.view(torch.int16).numpy().view(np.uint16)
    y = workloads.expert_outputs(n_tok * wl.K, wl.H, wl.seed + seed_offset)
    y = y.view(torch.int16).numpy().view(np.uint16)
    return topk[:n_tok], w[:n_tok], h, y


def time_oracle_step(wl, topk, w, h, y):
    """One oracle pass over the sample: layout, dispatch, combine. Returns
    (seconds, algorithmic bytes of the sample)."""
    import oracle
    n = topk.shape[0]
    t0 = time.perf_counter()
    lay = oracle.layout(topk, wl.E, wl.pad)
    cap = int(lay["offsets"][-1])
    if wl.fp8:
        oracle.dispatch_fp8(h, w, lay, wl.E, max(cap, 1))
    else:
        oracle.dispatch_bf16(h, w, lay, wl.E, max(cap, 1))
    pos = np.arange(n * wl.K, dtype=np.int32).reshape(n, wl.K)
    oracle.combine(y, pos, w)
    dt = time.perf_counter() - t0
    b = (bytes_layout(n, wl.K, wl.E, cap) +
         bytes_dispatch(n, wl.K, wl.H, wl.fp8, cap) +
         bytes_combine(n, wl.K, wl.H))
    return dt, b


def cpu_baseline(wl, n_tok):
    topk, w, h, y = oracle_sample(wl, n_tok)
    dt, b = time_oracle_step(wl, topk, w, h, y)
    return {"value": round(b / dt / 1e9, 3), "unit": "GB/s", "cores": 1,
            "kind": "oracle", "seconds": round(dt, 2),
            "sample": f"tokens 0..{n_tok - 1} of {wl.N}: layout, "
                      f"{'FP8' if wl.fp8 else 'bf16'} dispatch and combine "
                      "of the sample, single-threaded C"}


def _oracle_worker(job):
    """One process of the multi-core baseline: an independent synthetic
    sample of the workload, timed after every process has built its inputs
    (the barrier), on the wall clock shared by the processes."""
    wl_name, scale_kw, n_tok, seed_offset, barrier = job
    wl = workloads.WORKLOADS[wl_name]
    if scale_kw:
        wl = workloads.scaled(wl, **scale_kw)
    topk, w, h, y = oracle_sample(wl, n_tok, seed_offset=seed_offset)
    barrier.wait()
    t0 = time.time()
    dt, b = time_oracle_step(wl, topk, w, h, y)
    return t0, t0 + dt, b


def cpu_baseline_parallel(wl, n_tok, scale_kw):
    """The same oracle step, unmodified, run by one process per available
    core (capped at 32) on independent samples at once."""
    import multiprocessing as mp
    cores = len(os.sched_getaffinity(0))
    procs = max(1, min(32, cores))
    ctx = mp.get_context("spawn")   # the parent holds a CUDA context
    with ctx.Manager() as mgr:
        barrier = mgr.Barrier(procs)
        with ctx.Pool(procs) as pool:
            res = pool.map(_oracle_worker,
                           [(wl.name, scale_kw, n_tok, 100 + i, barrier)
                            for i in range(procs)])
    t0 = min(r[0] for r in res)
    t1 = max(r[1] for r in res)
    b = sum(r[2] for r in res)
    return {"value": round(b / (t1 - t0) / 1e9, 3), "unit": "GB/s",
            "cores": procs, "kind": "oracle",
            "seconds": round(t1 - t0, 2),
            "sample": f"{procs} processes at once, each the single-threaded "
                      f"oracle step on its own {n_tok}-token sample"}


def run_reference(args, wl):
    ws, rank, _ = dist_info()
    if rank != 0:
        return None
    # about a minute of oracle work for the whole warm-up + timed run
    per_tok = 0.8e-3
    n_tok = int(max(1, min(4096, wl.N, 60.0 / (args.steps + args.warmup) /
                           per_tok)))
    topk, w, h, y = oracle_sample(wl, n_tok)
    for _ in range(args.warmup):
        time_oracle_step(wl, topk, w, h, y)
    tot_t, tot_b = 0.0, 0
    for _ in range(args.steps):
        dt, b = time_oracle_step(wl, topk, w, h, y)
        tot_t += dt
        tot_b += b
    value = tot_b / tot_t / 1e9
    sample = (f"each step: tokens 0..{n_tok - 1} of {wl.N}: layout, "
              f"{'FP8' if wl.fp8 else 'bf16'} dispatch and combine of the "
              "sample, single-threaded C oracle")
    return {
        "impl": "reference",
        "metric": METRIC, "value": round(value, 3), "unit": "GB/s",
        "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(tot_t / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        # the oracle computes the same codes and sums (fp32 quotients and
        # fp32 fma chains) as the GPU path
        "dtype": ("e4m3+bf16, fp32 accumulate" if wl.fp8 else
                  "bf16, fp32 accumulate"), "data": "synthetic",
        "config": {"workload": wl.describe,
                   "step": "oracle layout + dispatch + combine"},
        "cpu_baseline": {"value": round(value, 3), "unit": "GB/s",
                         "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 3), "unit": "GB/s",
                "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="prefill",
                    choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=40)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-epbuffer", action="store_true",
                    help="skip timing the EPBuffer pass")
    ap.add_argument("--no-extra-workloads", action="store_true",
                    help="time only the selected workload")
    ap.add_argument("--no-read-probe", action="store_true",
                    help="skip the 4 GiB streaming read and write probes")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--backward", action="store_true",
                    help="add the backward pair to the step")
    ap.add_argument("--cpu-sample-tokens", type=int, default=8192)
    ap.add_argument("--tokens-per-rank", type=int, default=None,
                    help="override S (smaller cases for profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    wl = workloads.WORKLOADS[args.workload]
    if args.tokens_per_rank:
        wl = workloads.scaled(wl, S=args.tokens_per_rank)

    if args.impl == "reference":
        res = run_reference(args, wl)
        if res is not None:
            print(json.dumps(res), flush=True)
        return

    res = run_gpu(args, wl)
    ws, rank, _ = dist_info()
    if rank == 0:
        if ws == 1 and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline(
                wl, min(wl.N, args.cpu_sample_tokens))
            scale_kw = ({"S": args.tokens_per_rank}
                        if args.tokens_per_rank else None)
            res["cpu_baseline_all_cores"] = cpu_baseline_parallel(
                wl, min(wl.N, 1024), scale_kw)
        else:
            res["cpu_baseline"] = None
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
