"""Pins for the oracle's balanced plan and weight prefetch.

The plan is checked against a brute-force planner that labels every one of
the R*S*K expert-sorted rows with its expert and its chunk and reads the
segments off run by run, against the pages' invariant that every rank
receives exactly S*K rows, and against the golden example size.
"""
import os

import numpy as np
import pytest

import oracle
import workloads


def brute_force_plan(counts, R, S, K, B):
    E = len(counts)
    T = S * K
    labels = np.repeat(np.arange(E), counts)         # expert of every row
    assert len(labels) == R * T
    first_row = {e: int(np.argmax(labels == e)) for e in range(E)
                 if counts[e] > 0}
    plan = []
    for d in range(R):
        chunk = labels[d * T:(d + 1) * T]
        segs = []
        j = 0
        nslot = 0
        slots = [-1] * B
        while j < T:
            e = int(chunk[j])
            n = 1
            while j + n < T and chunk[j + n] == e:
                n += 1
            if first_row[e] >= d * T:
                wrow = e
            else:
                assert nslot < B
                slots[nslot] = e
                wrow = E + d * B + nslot
                nslot += 1
            segs.append((j, n, e, wrow))
            j += n
        plan.append((segs, slots))
    return plan


def check(counts, R, S, K, B):
    E = len(counts)
    T = S * K
    got = oracle.plan_balanced(counts, R, S, K, B)
    assert got["status"] == 0
    ref = brute_force_plan(counts, R, S, K, B)
    for d, (segs, slots) in enumerate(ref):
        n = got["nseg"][d]
        assert n == len(segs)
        for j, (start, length, e, wrow) in enumerate(segs):
            assert got["cu"][d, j] == start
            assert got["cu"][d, j + 1] - got["cu"][d, j] == length
            assert got["expert"][d, j] == e
            assert got["wrow"][d, j] == wrow
        assert np.all(got["cu"][d, n:] == T)
        assert np.all(got["expert"][d, n:] == -1)
        assert np.all(got["wrow"][d, n:] == -1)
        np.testing.assert_array_equal(got["slot_expert"][d], slots)
    return got


def random_counts(rng, R, S, K, E, skew):
    p = rng.dirichlet(np.full(E, skew))
    c = rng.multinomial(R * S * K, p)
    return c.astype(np.int32)


@pytest.mark.parametrize("seed", range(30))
def test_brute_force_random(seed):
    rng = np.random.default_rng(seed)
    R = int(rng.integers(1, 9))
    S = int(rng.integers(1, 9))
    K = int(rng.integers(1, 5))
    E = R * int(rng.integers(1, 5))
    counts = random_counts(rng, R, S, K, E, float(rng.choice([0.1, 1, 10])))
    got = check(counts, R, S, K, B=R)
    # every rank receives exactly S*K rows ("1. 完美负载平衡")
    for d in range(R):
        assert got["cu"][d, got["nseg"][d]] == S * K
    # each expert's segments add up to its count
    tot = np.zeros(E, np.int64)
    for d in range(R):
        for j in range(got["nseg"][d]):
            tot[got["expert"][d, j]] += got["cu"][d, j + 1] - got["cu"][d, j]
    np.testing.assert_array_equal(tot, counts)


def test_expert_spanning_many_chunks():
    # T = 4: expert 0 holds rows 0-2, expert 1 rows 3-16, expert 3 rows
    # 17-19. Expert 1 starts in chunk 0 and reaches chunks 1..4.
    R, S, K = 5, 2, 2
    counts = np.array([3, 14, 0, 3], np.int32)
    got = check(counts, R, S, K, B=2)
    assert got["slot_expert"][:, 0].tolist() == [-1, 1, 1, 1, 1]
    assert got["wrow"][0, 1] == 1                   # first chunk of expert 1
    assert got["wrow"][2, 0] == 4 + 2 * 2 + 0       # E + d*B + slot
    assert got["wrow"][4, 0] == 4 + 4 * 2 + 0
    assert got["wrow"][4, 1] == 3                   # expert 3 starts here


def test_workload_skew_needs_at_most_one_slot_per_rank():
    w = workloads.scaled(workloads.WORKLOADS["balanced"], S=256)
    topk, _ = workloads.routing(w)
    lay = oracle.layout(topk, w.E, 1)
    got = check(lay["counts"], w.R, w.S, w.K, w.B)
    used = got["slot_expert"] >= 0
    assert used.sum(axis=1).max() <= 1
    assert used.sum() <= w.R - 1


def test_golden_rows_per_rank(golden_dir):
    rows = [l.split() for l in open(os.path.join(golden_dir,
                                                 "balanced_rows.txt"))
            if l.strip() and not l.startswith("#")]
    S, K, R, E, T = map(int, rows[0])
    assert S * K == T
    w = workloads.WORKLOADS["balanced"]
    assert (w.S, w.K, w.R, w.E) == (S, K, R, E)
    # a hot expert holding well over one rank's rows still gives T per rank
    counts = np.full(E, (R * T - 3 * T) // (E - 1), np.int32)
    counts[0] = R * T - counts[1:].sum()
    got = oracle.plan_balanced(counts, R, S, K, w.B)
    assert got["status"] == 0
    for d in range(R):
        assert got["cu"][d, got["nseg"][d]] == T


def test_total_mismatch_and_slot_overflow():
    got = oracle.plan_balanced(np.array([3, 4], np.int32), 2, 2, 2, 1)
    assert got["status"] & oracle.ST_PLAN_TOTAL
    got = oracle.plan_balanced(np.array([3, 5], np.int32), 2, 2, 2, 0)
    assert got["status"] & oracle.ST_SLOTS
    assert got["wrow"][1, 0] == -1


def test_prefetch_copies_slots_only():
    rng = np.random.default_rng(4)
    R, B, E, elems = 3, 2, 6, 10
    W = rng.integers(0, 65535, size=(E + R * B, 2, elems // 2),
                     dtype=np.uint16)
    slots = np.array([[4, -1], [-1, -1], [0, 5]], np.int32)
    out = oracle.prefetch(slots, E, W)
    ref = W.copy()
    for d in range(R):
        for b in range(B):
            if slots[d, b] >= 0:
                ref[E + d * B + b] = W[slots[d, b]]
    np.testing.assert_array_equal(out, ref)
    assert np.array_equal(out[:E], W[:E])
    assert np.array_equal(out[E + 2], W[E + 2])     # unused slots untouched


def test_reduce_slot_grads_exact_on_integers():
    # integer-valued fp32 gradients: every sum is exact, so the result is
    # the brute-force sum whatever the order
    R, B, E = 4, 2, 6
    rng = np.random.default_rng(8)
    G = rng.integers(-1000, 1000, size=(E + R * B, 3, 5)).astype(np.float32)
    slots = np.array([[2, -1], [2, 5], [-1, -1], [0, 2]], np.int32)
    out = oracle.reduce_slot_grads(slots, E, G)
    ref = G.copy()
    for d in range(R):
        for b in range(B):
            if slots[d, b] >= 0:
                ref[slots[d, b]] += G[E + d * B + b]
    np.testing.assert_array_equal(out, ref)
    np.testing.assert_array_equal(out[E:], G[E:])        # slot rows kept
    assert np.array_equal(out[1], G[1]) and np.array_equal(out[3], G[3])


def test_reduce_slot_grads_preserves_the_total_and_order():
    R, B, E = 3, 2, 4
    rng = np.random.default_rng(9)
    G = rng.standard_normal((E + R * B, 64)).astype(np.float32)
    slots = np.array([[1, 3], [1, -1], [0, 1]], np.int32)
    out = oracle.reduce_slot_grads(slots, E, G)
    used = [(d, b) for d in range(R) for b in range(B) if slots[d, b] >= 0]
    total_before = G[:E].astype(np.float64).sum(0) + sum(
        G[E + d * B + b].astype(np.float64) for d, b in used)
    total_after = out[:E].astype(np.float64).sum(0)
    np.testing.assert_allclose(total_after, total_before, rtol=0, atol=1e-5)
    # expert 1 gets slots (0,0), (1,0), (2,1) added left to right in fp32
    acc = G[1].copy()
    for d, b in [(0, 0), (1, 0), (2, 1)]:
        acc = (acc + G[E + d * B + b]).astype(np.float32)
    np.testing.assert_array_equal(out[1], acc)
