"""GPU balanced plan and weight prefetch against the oracle (bit-exact)."""
import numpy as np
import pytest
import torch

import combine_ep_layout_09_b200 as ep
import oracle
import workloads
from gpu_util import DEV, gpu_layout, status_tensor, to_dev

pytestmark = pytest.mark.gpu


def gpu_plan(counts, R, S, K, B):
    E = len(counts)
    i32 = dict(dtype=torch.int32, device=DEV)
    p = dict(cu=torch.full((R, E + 1), -9, **i32),
             expert=torch.full((R, E), -9, **i32),
             wrow=torch.full((R, E), -9, **i32),
             nseg=torch.full((R,), -9, **i32),
             slot_expert=torch.full((R, max(B, 1)), -9, **i32))
    st = status_tensor()
    ep.ep_plan_balanced(to_dev(counts.astype(np.int32)), R, S, K, E, B,
                        p["cu"], p["expert"], p["wrow"], p["nseg"],
                        p["slot_expert"] if B > 0 else None, st)
    torch.cuda.synchronize()
    out = {k: v.cpu().numpy() for k, v in p.items()}
    out["slot_expert"] = out["slot_expert"][:, :B]
    out["status"] = int(st[0].item())
    out["dev_slots"] = p["slot_expert"]
    return out


def compare(counts, R, S, K, B):
    g = gpu_plan(counts, R, S, K, B)
    o = oracle.plan_balanced(counts, R, S, K, B)
    assert g["status"] == o["status"] == 0
    for k in ["cu", "expert", "wrow", "nseg", "slot_expert"]:
        np.testing.assert_array_equal(g[k], o[k], err_msg=k)
    return g


@pytest.mark.parametrize("seed", range(12))
def test_random_counts(seed):
    rng = np.random.default_rng(seed)
    R = int(rng.integers(1, 17))
    S = int(rng.integers(1, 300))
    K = int(rng.integers(1, 9))
    E = R * int(rng.integers(1, 33))
    p = rng.dirichlet(np.full(E, float(rng.choice([0.05, 1.0, 20.0]))))
    counts = rng.multinomial(R * S * K, p).astype(np.int32)
    compare(counts, R, S, K, int(rng.integers(1, 5)))


def test_expert_over_many_chunks_and_empty_experts():
    counts = np.array([3, 14, 0, 3], np.int32)
    g = compare(counts, 5, 2, 2, 2)
    assert g["slot_expert"][:, 0].tolist() == [-1, 1, 1, 1, 1]


def test_large_E():
    rng = np.random.default_rng(9)
    E, R, S, K = 1024, 8, 2048, 8
    counts = rng.multinomial(R * S * K, rng.dirichlet(np.full(E, 0.3)))
    compare(counts.astype(np.int32), R, S, K, 4)


def test_balanced_workload_from_gpu_layout():
    w = workloads.WORKLOADS["balanced"]
    topk, _ = workloads.routing(w)
    lay = gpu_layout(topk, w.R, w.S, w.E, 1)
    g = compare(lay["counts"], w.R, w.S, w.K, w.B)
    T = w.S * w.K
    for d in range(w.R):
        assert g["cu"][d, g["nseg"][d]] == T        # exactly S*K rows


def test_errors_reported():
    g = gpu_plan(np.array([3, 4], np.int32), 2, 2, 2, 1)
    assert g["status"] & ep.EP_DEV_PLAN_TOTAL
    g = gpu_plan(np.array([3, 5], np.int32), 2, 2, 2, 0)
    assert g["status"] & ep.EP_DEV_SLOTS
    assert g["wrow"][1, 0] == -1


def test_prefetch_small_against_oracle():
    rng = np.random.default_rng(4)
    R, B, E = 4, 2, 8
    shape = (E + R * B, 24, 40)
    W = [rng.integers(0, 65535, size=shape, dtype=np.uint16)
         for _ in range(3)]
    slots = np.array([[-1, -1], [3, -1], [7, 0], [-1, 5]], np.int32)
    dev = [to_dev(x.view(np.int16)).view(torch.bfloat16) for x in W]
    ep.ep_prefetch_weights(to_dev(slots), R, E, B, *dev)
    torch.cuda.synchronize()
    for x, d in zip(W, dev):
        got = d.view(torch.int16).cpu().numpy().view(np.uint16)
        np.testing.assert_array_equal(got, oracle.prefetch(slots, E, x))


def test_prefetch_balanced_full_size():
    w = workloads.WORKLOADS["balanced"]
    topk, _ = workloads.routing(w)
    lay = gpu_layout(topk, w.R, w.S, w.E, 1)
    g = compare(lay["counts"], w.R, w.S, w.K, w.B)
    rows = w.E + w.R * w.B
    Ws = [workloads.weight_buffer(rows, w.H, w.I, w.seed + j, device="cuda:0")
          for j in range(3)]
    def rowsum(x):  # per-row checksum, reinterpreting 4 bf16 as one int64
        return x.view(rows, -1).view(torch.int64).sum(1)
    before = [rowsum(x) for x in Ws]
    ep.ep_prefetch_weights(g["dev_slots"], w.R, w.E, w.B, *Ws)
    torch.cuda.synchronize()
    slots = g["slot_expert"]
    assert (slots >= 0).sum() >= 1
    for x, b in zip(Ws, before):
        after = rowsum(x)
        for d in range(w.R):
            for s in range(w.B):
                r = w.E + d * w.B + s
                e = slots[d, s]
                if e >= 0:
                    assert torch.equal(x[r], x[e])
                else:
                    assert after[r] == b[r]
        assert torch.equal(after[:w.E], b[:w.E])


@pytest.mark.parametrize("R,B,E,shape", [
    (8, 4, 256, (3, 5000)),      # chunked copy, last chunk shorter
    (64, 20, 128, (2, 40)),      # more slots than the compacted list holds
])
def test_prefetch_forms_against_oracle(R, B, E, shape):
    rng = np.random.default_rng(R * B)
    rows = E + R * B
    W = [rng.integers(0, 65535, size=(rows, *shape), dtype=np.uint16)
         for _ in range(3)]
    slots = rng.integers(-1, E, size=(R, B)).astype(np.int32)
    slots[rng.random(slots.shape) < 0.5] = -1
    dev = [to_dev(x.view(np.int16)).view(torch.bfloat16) for x in W]
    ep.ep_prefetch_weights(to_dev(slots), R, E, B, *dev)
    torch.cuda.synchronize()
    for x, d in zip(W, dev):
        got = d.view(torch.int16).cpu().numpy().view(np.uint16)
        np.testing.assert_array_equal(got, oracle.prefetch(slots, E, x))


def gpu_reduce(slots, E, Gs):
    dev = [torch.from_numpy(np.ascontiguousarray(g)).to(DEV) for g in Gs]
    R, B = slots.shape
    ep.ep_reduce_slot_grads(to_dev(slots), R, E, B, *dev)
    torch.cuda.synchronize()
    return [d.cpu().numpy() for d in dev]


@pytest.mark.parametrize("seed", range(3))
def test_reduce_slot_grads_against_oracle(seed):
    rng = np.random.default_rng(seed)
    R, B, E = 6, 3, 10
    shape = (E + R * B, 7, 12)
    Gs = [rng.standard_normal(shape).astype(np.float32) for _ in range(3)]
    slots = rng.integers(-1, E, size=(R, B)).astype(np.int32)
    slots[0, 0] = slots[1, 0] = slots[2, 2] = 4      # one expert, three slots
    got = gpu_reduce(slots, E, Gs)
    for g, G in zip(got, Gs):
        np.testing.assert_array_equal(g, oracle.reduce_slot_grads(slots, E, G))


def test_reduce_slot_grads_balanced_plan():
    w = workloads.WORKLOADS["balanced"]
    topk, _ = workloads.routing(w)
    lay = gpu_layout(topk, w.R, w.S, w.E, 1)
    g = compare(lay["counts"], w.R, w.S, w.K, w.B)
    slots = g["slot_expert"]
    assert (slots >= 0).sum() >= 1
    rng = np.random.default_rng(5)
    shape = (w.E + w.R * w.B, w.H, 16)               # narrow I for the test
    Gs = [rng.standard_normal(shape).astype(np.float32) for _ in range(3)]
    got = gpu_reduce(slots, w.E, Gs)
    for gg, G in zip(got, Gs):
        np.testing.assert_array_equal(gg, oracle.reduce_slot_grads(slots, w.E,
                                                                   G))


def test_reduce_slot_grads_rejects_large_tables():
    t = torch.zeros(8, dtype=torch.float32, device=DEV)
    s = torch.zeros(2048, dtype=torch.int32, device=DEV)
    with pytest.raises(ep.EPError) as e:
        ep.ep_reduce_slot_grads(s, 1024, 8, 2, t.view(1, 8).expand(2056, 8)
                                .contiguous(), t.view(1, 8).expand(2056, 8)
                                .contiguous(), t.view(1, 8).expand(2056, 8)
                                .contiguous())
    assert e.value.code == ep.EP_ERR_INVALID_ARG
