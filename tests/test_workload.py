"""The seeded input recipe: shapes, determinism and the load distributions."""
import numpy as np
import pytest
import torch

from grouped_gemm_plan_b200 import workload as wl


def test_registry_shapes():
    W = wl.WORKLOADS
    assert (W["mixtral"].M, W["mixtral"].H, W["mixtral"].F, W["mixtral"].E, W["mixtral"].topk) == (4096, 4096, 14336, 8, 2)
    assert (W["qwen2"].H, W["qwen2"].F, W["qwen2"].E, W["qwen2"].topk) == (2048, 1408, 64, 4)
    assert (W["phi35"].M, W["phi35"].H, W["phi35"].F, W["phi35"].E) == (16384, 4096, 6400, 16)
    assert [W[f"wide{m}"].M for m in (16, 128, 512, 2048)] == [16, 128, 512, 2048]
    assert W["tiny"].flops() == 6 * 512 * 256 * 512


@pytest.mark.parametrize("routing", ["uniform", "balanced", "skewed"])
def test_routing_deterministic_and_distinct(routing):
    w = wl.Workload("t", 300, 8, 8, 16, 4, routing, 0.05, 42)
    a, wa = wl.make_routing(w)
    b, wb = wl.make_routing(w)
    assert np.array_equal(a, b) and np.array_equal(wa, wb)
    assert a.shape == (300, 4) and a.dtype == np.int32
    assert a.min() >= 0 and a.max() < 16
    assert all(len(set(r)) == 4 for r in a.tolist())
    np.testing.assert_allclose(wa.sum(1), 1.0, rtol=1e-6)
    assert np.all(wa > 0)
    c, _ = wl.make_routing(w.with_(seed=43))
    assert not np.array_equal(a, c)


def test_skewed_load_is_skewed():
    w = wl.WORKLOADS["phi35"]
    ids = wl.make_topk_ids(w)
    counts = np.bincount(ids.reshape(-1), minlength=w.E)
    p = wl.expert_probabilities(w)
    assert abs(p.sum() - 1) < 1e-12 and p.min() >= 1e-4 / p.sum() - 1e-12
    # heavy skew: the heaviest expert gets several times the lightest one
    assert counts.max() > 3 * max(counts.min(), 1)
    # the empirical load follows p (first-choice marginals are exactly p)
    first = np.bincount(ids[:, 0], minlength=w.E) / w.M
    np.testing.assert_allclose(first, p, atol=0.02)


def test_uniform_load_is_roughly_uniform():
    w = wl.WORKLOADS["tiny"]
    ids = wl.make_topk_ids(w)
    counts = np.bincount(ids.reshape(-1), minlength=w.E)
    assert counts.sum() == w.R
    assert counts.min() > 0.5 * w.R / w.E


def test_weights_scale_and_bf16():
    w = wl.Workload("t", 4, 256, 128, 2, 1, "uniform", 0, 3)
    W1, W2 = wl.make_weights(w)
    assert W1.dtype == torch.bfloat16 and W1.shape == (2, 256, 256)
    assert W2.shape == (2, 128, 256)
    assert abs(W1.float().std().item() - 1 / 16) < 0.01      # N(0,1)/sqrt(H)
    assert abs(W2.float().std().item() - 1 / np.sqrt(128)) < 0.01
    x = wl.make_x(w)
    assert x.shape == (4, 256) and x.dtype == torch.bfloat16
    # experts are independent streams
    assert not torch.equal(W1[0], W1[1])
    assert torch.equal(wl.make_expert_w1(w, 1), W1[1])


def test_rank_workload_changes_seed_only():
    base = wl.WORKLOADS["mixtral"]
    r1 = wl.rank_workload(base, 1)
    assert (r1.M, r1.H, r1.F, r1.E) == (base.M, base.H, base.F, base.E)
    assert r1.seed != base.seed and wl.rank_workload(base, 0) == base
