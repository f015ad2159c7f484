"""bench.py's byte accounting against the figures it is defined by, and its
launch count against the library's size rule (host only)."""
import os
import re

import pytest

import bench
import workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_prefill_and_decode_bytes():
    # each input read once, each output written once: hidden 2 B/channel,
    # FP8 codes 1 B/channel + one fp32 scale per 128 channels + a weight per
    # row; combine reads K bf16 rows and writes one
    N, K, H = 32768, 8, 7168
    rows = N * K
    disp = bench.bytes_dispatch(N, K, H, True, rows)
    assert disp == (N * H * 2 + N * K * 8 + rows * 4 +
                    rows * (H + H // 128 * 4 + 4))
    assert abs(disp / 1e6 - 2411.7) < 0.1
    assert abs(bench.bytes_combine(N, K, H) / 1e6 - 4230.0) < 0.1
    dec = workloads.WORKLOADS["decode"]
    d = bench.bytes_dispatch(dec.N, dec.K, dec.H, True, dec.N * dec.K)
    assert abs(d / 1e6 - 75.37) < 0.01
    # bf16 rows are twice as wide; padding rows count as written rows
    assert (bench.bytes_dispatch(N, K, H, False, rows + 100) -
            bench.bytes_dispatch(N, K, H, False, rows)) == 100 * (2 * H + 4) + 100 * 4


def test_reduce_bytes_per_slot_group():
    import numpy as np
    slots = np.array([[3, -1], [3, 7]], np.int32)   # expert 3 twice, 7 once
    H, I = 8, 4
    # expert 3: own row read + written, 2 slot rows read; expert 7: 1 slot
    assert bench.bytes_reduce_slot_grads(slots, H, I) == 3 * (4 + 3) * H * I * 4


def _header_constant(name):
    src = open(os.path.join(ROOT, "combine_ep_layout_09_b200", "csrc",
                            "ep_launch.h")).read()
    m = re.search(r"constexpr\s+int64_t\s+%s\s*=\s*(\d+)\s*;" % name, src)
    assert m, name
    return int(m.group(1))


@pytest.mark.parametrize("S,K,expect", [
    (128, 8, 1),      # decode: 8192 entries, 7 tokens per CTA
    (512, 8, 1),      # 32768 entries exactly
    (513, 8, 2),      # one tile more: cooperative layout + dispatch
    (4096, 8, 2),     # prefill: 64 tiles, all resident
    (49152, 8, 3),    # 768 tiles: histogram + scan + dispatch
])
def test_launch_count_follows_the_library_rule(S, K, expect):
    limit = _header_constant("kSmallMaxEntries")
    per_cta = _header_constant("kSmallMaxChunkEntries")
    assert (limit, per_cta) == (32768, 1024)   # the numbers bench.py mirrors
    wl = workloads.scaled(workloads.WORKLOADS["prefill"], S=S, K=K)
    assert bench.layout_dispatch_kernels(wl) == expect


def _combine_constants():
    src = open(os.path.join(ROOT, "combine_ep_layout_09_b200", "csrc",
                            "combine.cu")).read()
    stage = re.search(r"kTmaStageTarget\s*=\s*(\d+)\s*\*\s*1024", src)
    rule = re.search(r"sh\.smem\s*<=\s*(\d+)\s*\*\s*1024\s*&&\s*N\s*\*\s*"
                     r"sh\.parts\s*>=\s*(\d+)\s*\*", src)
    assert stage and rule
    return int(stage.group(1)), int(rule.group(1)), int(rule.group(2))


@pytest.mark.parametrize("N,K,H,expect", [
    (32768, 8, 7168, "k_combine_tma"),    # prefill: 2 parts per row
    (1024, 8, 7168, "k_combine<8>"),      # decode: 2048 units < 16 per SM
    (2500, 8, 1024, "k_combine_tma"),     # one part, 2500 units
    (300, 8, 7168, "k_combine<8>"),
    (100000, 1, 32768, "k_combine_tma"),  # one 64 KB part: 192 KB of stages
    (100000, 2, 32768, "k_combine_tma"),  # two 64 KB parts
    (2000, 1, 32768, "k_combine<1>"),     # 2000 units < 16 per SM
])
def test_combine_kernel_follows_the_library_rule(N, K, H, expect):
    assert _combine_constants() == (64, 200, 16)   # what bench.py mirrors
    wl = workloads.scaled(workloads.WORKLOADS["prefill"], S=N // 8, K=K, H=H)
    wl = workloads.scaled(wl, R=1, S=N)
    assert bench.combine_kernel(wl) == expect


def test_dispatch_kernel_names_follow_the_library_rule():
    src = open(os.path.join(ROOT, "combine_ep_layout_09_b200", "csrc",
                            "dispatch.cu")).read()
    # with every SM in use the dispatch launches one CTA per token
    assert re.search(r"all_sms\s*=\s*num_sms\s*>=\s*device_sm_count\(\)", src)
    assert re.search(r"if\s*\(all_sms\s*&&\s*!fp8\)", src)
    assert re.search(r"if\s*\(all_sms\s*&&\s*fp8\)", src)
    for name in ("k_dispatch_bf16_tok", "k_dispatch_fp8_tok"):
        assert re.search(r"auto kern = \w+ \? " + name + r"<true> : " + name +
                         r"<false>;", src)
    names = {w: bench.kernel_names(workloads.WORKLOADS[w])["dispatch"]
             for w in ("prefill", "skewed", "decode")}
    assert names == {"prefill": "k_dispatch_fp8_tok",
                     "skewed": "k_dispatch_bf16_tok",
                     "decode": "k_layout_small<fp8>"}
