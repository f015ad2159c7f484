"""Pins for the oracle's layout (histogram, padded offsets, stable positions).

The oracle is checked against things other than itself: a brute-force
construction of the receive buffer from sorted (expert, token, k) tuples,
numpy's bincount, the invariants the pages state, and the golden values the
pages print.
"""
import os

import numpy as np
import pytest

import oracle
import workloads


def brute_force_layout(topk, E, pad):
    """Build the receive buffer row by row: sort all (e, t, k) tuples, then
    lay each expert's tuples out in order, followed by filler rows until the
    group length is a multiple of pad."""
    N, K = topk.shape
    tuples = sorted((int(topk[t, k]), t, k) for t in range(N) for k in range(K)
                    if 0 <= topk[t, k] < E)
    rows = []          # each row: (t, k) or None for padding
    starts = []
    for e in range(E):
        starts.append(len(rows))
        mine = [(t, k) for (ee, t, k) in tuples if ee == e]
        rows.extend(mine)
        while (len(rows) - starts[-1]) % pad:
            rows.append(None)
    starts.append(len(rows))
    pos = np.full((N, K), -1, np.int64)
    row_src = np.full(len(rows), -1, np.int64)
    for r, tk in enumerate(rows):
        if tk is not None:
            pos[tk] = r
            row_src[r] = tk[0] * K + tk[1]
    return np.array(starts), pos, row_src


def check_against_brute_force(topk, E, pad):
    N, K = topk.shape
    lay = oracle.layout(topk, E, pad)
    starts, pos, row_src = brute_force_layout(topk, E, pad)
    valid = topk[(topk >= 0) & (topk < E)]
    np.testing.assert_array_equal(lay["counts"],
                                  np.bincount(valid, minlength=E)[:E])
    np.testing.assert_array_equal(lay["offsets"], starts)
    np.testing.assert_array_equal(lay["pos"], pos)
    used = int(starts[-1])
    np.testing.assert_array_equal(lay["row_src"][:used], row_src)
    # rows past the used region are not written
    assert np.all(lay["row_src"][used:] == -7)
    return lay


@pytest.mark.parametrize("seed", range(40))
def test_brute_force_random(seed):
    rng = np.random.default_rng(seed)
    N = int(rng.integers(0, 65))
    E = int(rng.integers(1, 17))
    K = int(rng.integers(1, 5))
    pad = int(rng.choice([1, 2, 3, 4, 128]))
    topk = rng.integers(0, E, size=(N, K)).astype(np.int32)
    check_against_brute_force(topk, E, pad)


def test_brute_force_tiny_workload():
    w = workloads.WORKLOADS["tiny"]
    topk, _ = workloads.routing(w)
    lay = check_against_brute_force(topk, w.E, w.pad)
    assert lay["status"] == 0


@pytest.mark.parametrize("pad", [1, 128])
def test_brute_force_skewed_small(pad):
    w = workloads.scaled(workloads.WORKLOADS["skewed"], S=16, pad=pad)
    topk, _ = workloads.routing(w)
    check_against_brute_force(topk, w.E, pad)


def test_invariants_per_rank():
    # "1. 完美负载平衡": each rank contributes S*K entries; the histogram over
    # all ranks therefore sums to R*S*K.
    w = workloads.scaled(workloads.WORKLOADS["prefill"], S=64)
    topk, _ = workloads.routing(w)
    lay = oracle.layout(topk, w.E, w.pad)
    assert lay["counts"].sum() == w.R * w.S * w.K
    per_rank = topk.reshape(w.R, w.S * w.K)
    for r in range(w.R):
        assert np.bincount(per_rank[r], minlength=w.E).sum() == w.S * w.K
    # pos is a bijection onto the non-padding rows; row_src inverts it
    flat = lay["pos"].ravel()
    assert len(np.unique(flat)) == flat.size
    assert np.all(lay["row_src"][flat] == np.arange(flat.size))


def test_padding_regions():
    rng = np.random.default_rng(7)
    E, K, N, pad = 12, 3, 50, 8
    topk = rng.integers(0, E, size=(N, K)).astype(np.int32)
    topk[topk == 5] = 4            # an expert with no entries
    lay = oracle.layout(topk, E, pad)
    off, cnt = lay["offsets"], lay["counts"]
    assert np.all(np.diff(off) % pad == 0)
    assert cnt[5] == 0 and off[6] == off[5]   # empty expert -> no rows
    for e in range(E):
        used = lay["row_src"][off[e]:off[e] + cnt[e]]
        fill = lay["row_src"][off[e] + cnt[e]:off[e + 1]]
        assert np.all(used >= 0) and np.all(fill == -1)
        assert len(fill) < pad
        # rows inside a group are ordered by (t, k)
        assert np.all(np.diff(used) > 0)


def test_rank_regions_golden(golden_dir):
    # "Экспертный параллелизм (EP)": 8 experts, ep_size 4 -> 2 per rank.
    rows = [l.split() for l in open(os.path.join(golden_dir,
                                                 "local_experts.txt"))
            if l.strip() and not l.startswith("#")]
    E, R, L = map(int, rows[0])
    assert E % R == 0 and E // R == L
    E2, R2, ok = map(int, rows[1])
    assert (E2 % R2 == 0) == bool(ok)
    # with contiguous ownership, rank r's region spans experts 2r, 2r+1
    w = workloads.WORKLOADS["tiny"]
    assert (w.E, w.R) == (E, R)
    topk, _ = workloads.routing(w)
    lay = oracle.layout(topk, E, 1)
    for r in range(R):
        lo, hi = lay["offsets"][r * L], lay["offsets"][(r + 1) * L]
        src = lay["row_src"][lo:hi]
        experts = topk.ravel()[src]
        assert set(experts.tolist()) <= {r * L + j for j in range(L)}


def test_invalid_ids_are_skipped():
    topk = np.array([[0, 9], [-1, 2], [2, 1]], np.int32)
    lay = oracle.layout(topk, 3, 1)
    assert lay["status"] & oracle.ST_BAD_EXPERT
    np.testing.assert_array_equal(lay["counts"], [1, 1, 2])
    np.testing.assert_array_equal(lay["pos"], [[0, -1], [-1, 2], [3, 1]])
    np.testing.assert_array_equal(lay["row_src"][:4], [0, 5, 3, 4])


def test_empty_input():
    topk = np.zeros((0, 4), np.int32)
    lay = oracle.layout(topk, 16, 4)
    assert lay["status"] == 0
    assert np.all(lay["counts"] == 0) and np.all(lay["offsets"] == 0)


def test_duplicate_expert_in_token_ordered_by_k():
    topk = np.array([[1, 1, 0], [1, 0, 1]], np.int32)
    lay = oracle.layout(topk, 2, 1)
    # expert 0 rows: (0,2),(1,1); expert 1 rows: (0,0),(0,1),(1,0),(1,2)
    np.testing.assert_array_equal(lay["row_src"], [2, 4, 0, 1, 3, 5])


def test_capacity_bound_formula():
    # worst case: every entry on one expert, all others padded from 1 row
    rng = np.random.default_rng(3)
    for _ in range(20):
        E, K, pad = int(rng.integers(1, 9)), int(rng.integers(1, 4)), \
            int(rng.integers(1, 9))
        N = int(rng.integers(0, 20))
        topk = rng.integers(0, E, size=(N, K)).astype(np.int32)
        lay = oracle.layout(topk, E, pad)
        assert lay["offsets"][-1] <= oracle.capacity_bound(N, K, E, pad)
    # the bound is reached when every count is 1 modulo pad
    E, pad = 4, 5
    topk = np.array([[0], [1], [2]] + [[3]] * 6, np.int32)
    lay = oracle.layout(topk, E, pad)
    assert lay["offsets"][-1] == 25 == oracle.capacity_bound(9, 1, E, pad)
