"""Properties of the seeded input generators (shapes, determinism, routing
structure). Nothing here depends on the method under test."""
import numpy as np
import pytest

import workloads


@pytest.mark.parametrize("name", ["tiny", "prefill", "decode", "skewed",
                                  "balanced"])
def test_routing_shapes_and_weights(name):
    w = workloads.WORKLOADS[name]
    if w.N > 4096:
        w = workloads.scaled(w, S=256)
    topk, wk = workloads.routing(w)
    assert topk.shape == (w.N, w.K) and topk.dtype == np.int32
    assert wk.shape == (w.N, w.K) and wk.dtype == np.float32
    assert topk.min() >= 0 and topk.max() < w.E
    # K distinct experts per token
    s = np.sort(topk, axis=1)
    assert np.all(np.diff(s, axis=1) > 0)
    assert np.all(wk > 0)
    np.testing.assert_allclose(wk.sum(axis=1), 1.0, atol=1e-6)
    topk2, wk2 = workloads.routing(w)
    assert np.array_equal(topk, topk2) and np.array_equal(wk, wk2)


def test_group_limited_stays_in_top_groups():
    w = workloads.scaled(workloads.WORKLOADS["prefill"], S=64)
    topk, _ = workloads.routing(w)
    groups = topk // (w.E // w.n_groups)
    for row in groups:
        assert len(set(row.tolist())) <= w.topk_groups


def test_zipf_is_skewed():
    w = workloads.scaled(workloads.WORKLOADS["skewed"], S=512)
    topk, _ = workloads.routing(w)
    c = np.bincount(topk.ravel(), minlength=w.E)
    assert c.max() > 20 * np.median(c)


def test_bf16_normal_deterministic():
    a = workloads.bf16_normal((7, 33), 5)
    b = workloads.bf16_normal((7, 33), 5)
    assert a.dtype.is_floating_point and a.shape == (7, 33)
    assert bool((a == b).all())
    assert abs(float(a.float().std()) - 1.0) < 0.3
