"""GPU layout (histogram, padded offsets, stable positions) against the
oracle: bit-exact on counts, offsets, pos and row_src, including the rows the
method must leave untouched."""
import numpy as np
import pytest

import oracle
import workloads
from gpu_util import ROW_SRC_FILL, gpu_layout

pytestmark = pytest.mark.gpu


def compare(topk, R, S, E, pad, cap=None):
    N, K = topk.shape
    g = gpu_layout(topk, R, S, E, pad, cap=cap)
    o = oracle.layout(topk, E, pad, cap=g["dev"]["cap"],
                      row_src_fill=ROW_SRC_FILL)
    np.testing.assert_array_equal(g["counts"], o["counts"])
    np.testing.assert_array_equal(g["offsets"], o["offsets"])
    np.testing.assert_array_equal(g["pos"], o["pos"])
    np.testing.assert_array_equal(g["row_src"], o["row_src"])
    assert bool(g["status"] & 1) == bool(o["status"] & oracle.ST_BAD_EXPERT)
    assert g["status"] & ~1 == 0      # no timeout, no capacity error
    return g, o


CASES = [
    # R, S, K, E, pad   (N*K spans several 4096-entry tiles, ragged tails)
    (1, 1, 1, 1, 1),
    (4, 64, 2, 8, 1),
    (2, 1000, 8, 16, 1),
    (8, 513, 8, 256, 1),
    (8, 513, 8, 256, 128),
    (3, 777, 5, 9, 3),
    (4, 301, 9, 1024, 7),
    (1, 5000, 32, 64, 1),
    (16, 100, 1, 16, 4),
]


@pytest.mark.parametrize("R,S,K,E,pad", CASES)
def test_random_uniform(R, S, K, E, pad):
    rng = np.random.default_rng(R * 1000 + S + K + E + pad)
    topk = rng.integers(0, E, size=(R * S, K)).astype(np.int32)
    compare(topk, R, S, E, pad)


@pytest.mark.parametrize("seed", range(4))
def test_random_skewed_duplicates(seed):
    rng = np.random.default_rng(seed)
    E, K, R, S = 64, 6, 4, 1200
    p = rng.dirichlet(np.full(E, 0.05))
    topk = rng.choice(E, size=(R * S, K), p=p).astype(np.int32)
    compare(topk, R, S, E, int(rng.choice([1, 16, 128])))


def test_single_expert_gets_everything():
    R, S, K, E = 2, 3000, 4, 8
    topk = np.full((R * S, K), 5, np.int32)
    compare(topk, R, S, E, 128)


@pytest.mark.parametrize("name", ["tiny", "prefill", "decode", "skewed",
                                  "balanced"])
def test_workloads_full_size(name):
    w = workloads.WORKLOADS[name]
    topk, _ = workloads.routing(w)
    g, o = compare(topk, w.R, w.S, w.E, w.pad)
    assert g["counts"].sum() == w.N * w.K
    # rank r's region = experts [r*E/R, (r+1)*E/R)
    L = w.E // w.R
    for r in range(w.R):
        lo, hi = g["offsets"][r * L], g["offsets"][(r + 1) * L]
        src = g["row_src"][lo:hi]
        e = topk.ravel()[src[src >= 0]]
        assert np.all((e >= r * L) & (e < (r + 1) * L))


def test_capacity_above_bound_leaves_tail():
    rng = np.random.default_rng(11)
    topk = rng.integers(0, 8, size=(400, 3)).astype(np.int32)
    g, o = compare(topk, 4, 100, 8, 4, cap=2000)
    used = g["offsets"][-1]
    assert np.all(g["row_src"][used:] == ROW_SRC_FILL)


def test_empty_batch():
    topk = np.zeros((0, 4), np.int32)
    g = gpu_layout(topk, 4, 0, 8, 16)
    assert np.all(g["counts"] == 0) and np.all(g["offsets"] == 0)
    assert g["status"] == 0


def test_bad_ids_flagged_and_skipped():
    rng = np.random.default_rng(5)
    topk = rng.integers(0, 16, size=(2000, 4)).astype(np.int32)
    topk[3, 1] = 16
    topk[1500, 0] = -1
    topk[1999, 3] = 1 << 30
    g, o = compare(topk, 4, 500, 16, 2)
    assert g["status"] & 1
    assert g["pos"][3, 1] == -1 and g["pos"][1500, 0] == -1


def test_repeat_calls_reuse_workspace():
    # the same buffers twice in a row give the same answer
    rng = np.random.default_rng(6)
    topk = rng.integers(0, 32, size=(4096, 8)).astype(np.int32)
    a = gpu_layout(topk, 8, 512, 32, 1)
    b = gpu_layout(topk, 8, 512, 32, 1)
    np.testing.assert_array_equal(a["pos"], b["pos"])


@pytest.mark.parametrize("E,pad", [(256, 1), (64, 128)])
def test_large_input_takes_two_kernel_path(E, pad):
    # 3 M entries: more 4096-entry tiles than can be co-resident, so the
    # histogram + look-back scan pair runs instead of the fused kernel
    R, S, K = 8, 49152, 8
    rng = np.random.default_rng(E + pad)
    topk = rng.integers(0, E, size=(R * S, K)).astype(np.int32)
    compare(topk, R, S, E, pad)


@pytest.mark.parametrize("E", [2, 96, 128, 192, 256, 320, 512, 768])
def test_expert_counts_across_thread_mappings(E):
    # E values that map experts to threads differently (pairs of look-back
    # threads, chunks of warps per expert), with several tiles
    R = 2 if E % 2 == 0 else 1
    rng = np.random.default_rng(E)
    S = 9000 // R
    topk = rng.integers(0, E, size=(R * S, 8)).astype(np.int32)
    g, _ = compare(topk, R, S, E, 4)
    assert g["status"] == 0
