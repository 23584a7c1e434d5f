"""GPU parity of the router (moe_route) with the oracle: expert ids bit for bit,
softmax weights within 1e-6 (fp32 softmax of at most 32 terms against fp64), and
the routed layer end to end."""
import numpy as np
import pytest
import torch

import oracle
from grouped_gemm_plan_b200 import binding as B
from helpers import check_close, layer_case

pytestmark = pytest.mark.gpu


def _route_gpu(dev, logits_np, topk):
    M, E = logits_np.shape
    logits = torch.from_numpy(logits_np).to(dev)
    ids = torch.full((M, topk), -9, dtype=torch.int32, device=dev)
    w = torch.full((M, topk), -9.0, dtype=torch.float32, device=dev)
    ws = B.alloc_workspace(B.OP_ROUTE, M, 0, 0, E, topk, dev)
    B.moe_route(logits, topk, ids, w, ws)
    assert B.moe_get_device_status(ws) == B.MOE_OK
    return ids.cpu().numpy(), w.cpu().numpy()


@pytest.mark.parametrize("M,E,topk", [(1, 1, 1), (300, 8, 2), (1000, 64, 4), (77, 16, 8),
                                      (50, 100, 32), (513, 1024, 8), (20, 33, 33 - 1)])
def test_route_matches_oracle(cuda_dev, M, E, topk):
    rng = np.random.default_rng(M * 7 + E)
    logits = rng.standard_normal((M, E)).astype(np.float32)
    ids, w = _route_gpu(cuda_dev, logits, topk)
    rid, rw = oracle.route(logits, topk)
    assert np.array_equal(ids, rid)
    np.testing.assert_allclose(w, rw, rtol=0, atol=1e-6)


def test_route_ties_go_to_the_lower_index(cuda_dev):
    rng = np.random.default_rng(3)
    logits = (np.round(rng.standard_normal((400, 40)) * 2) / 2).astype(np.float32)  # many ties
    logits[0] = 1.0
    logits[1, ::2] = -np.inf
    ids, w = _route_gpu(cuda_dev, logits, 6)
    rid, rw = oracle.route(logits, 6)
    assert np.array_equal(ids, rid)
    assert ids[0].tolist() == [0, 1, 2, 3, 4, 5]
    np.testing.assert_allclose(w, rw, rtol=0, atol=1e-6)


def test_routed_layer(cuda_dev):
    dev = cuda_dev
    w_, x, W1, W2, _, _ = layer_case(300, 256, 384, 16, 2, "uniform", seed=31)
    logits = np.random.default_rng(31).standard_normal((300, 16)).astype(np.float32)
    M, H = x.shape
    ids = torch.empty(M, 2, dtype=torch.int32, device=dev)
    tw = torch.empty(M, 2, dtype=torch.float32, device=dev)
    rws = B.alloc_workspace(B.OP_ROUTE, M, 0, 0, 16, 2, dev)
    B.moe_route(torch.from_numpy(logits).to(dev), 2, ids, tw, rws)
    out = torch.empty(M, H, dtype=torch.bfloat16, device=dev)
    counts = torch.empty(16, dtype=torch.int32, device=dev)
    offsets = torch.empty(17, dtype=torch.int32, device=dev)
    perm = torch.empty(2 * M, dtype=torch.int32, device=dev)
    ws = B.alloc_workspace(B.OP_FFN_FUSED, M, H, 384, 16, 2, dev)
    B.moe_ffn_fused(x.to(dev), W1.to(dev), W2.to(dev), ids, tw, out, counts, offsets, perm, ws)
    assert B.moe_get_device_status(ws) == B.MOE_OK
    rid, rw = oracle.route(logits, 2)
    assert np.array_equal(ids.cpu().numpy(), rid)
    ref = oracle.moe_ffn(x, W1, W2, rid, rw.astype(np.float32))
    check_close(out, ref, "routed layer")


@pytest.mark.parametrize("M,E,topk", [(0, 8, 2), (1, 1, 1), (300, 8, 2), (4096, 8, 2),
                                      (8192, 64, 4), (1000, 16, 3), (77, 16, 8), (513, 1024, 8),
                                      (16384, 16, 2), (20, 33, 32)])
def test_route_plan_matches_oracle(cuda_dev, M, E, topk):
    """moe_route_plan: ids/weights exactly as moe_route writes them (ids bit-exact vs
    the oracle router, weights within 1e-6), and the plan of those ids bit-exact vs
    the oracle plan (counts, offsets, perm, inv, w_sorted) -- also for a topk that
    does not divide the plan's chunk size."""
    dev = cuda_dev
    rng = np.random.default_rng(M * 11 + E)
    logits_np = rng.standard_normal((M, E)).astype(np.float32)
    logits = torch.from_numpy(logits_np).to(dev)
    R = M * topk
    ids = torch.full((M, topk), -9, dtype=torch.int32, device=dev)
    w = torch.full((M, topk), -9.0, dtype=torch.float32, device=dev)
    counts = torch.full((E,), -1, dtype=torch.int32, device=dev)
    offsets = torch.full((E + 1,), -1, dtype=torch.int32, device=dev)
    perm = torch.full((max(R, 1),), -1, dtype=torch.int32, device=dev)
    inv = torch.full((max(R, 1),), -1, dtype=torch.int32, device=dev)
    ws_ = torch.full((max(R, 1),), -1.0, dtype=torch.float32, device=dev)
    ws = B.alloc_workspace(B.OP_PLAN, M, 0, 0, E, topk, dev)
    B.moe_route_plan(logits, topk, ids, w, counts, offsets, perm[:R], inv[:R], ws_[:R], ws)
    assert B.moe_get_device_status(ws) == B.MOE_OK
    assert counts.cpu().tolist() == [0] * E if M == 0 else True
    if M == 0:
        assert offsets.cpu().tolist() == [0] * (E + 1)
        return
    rid, rw = oracle.route(logits_np, topk)
    assert np.array_equal(ids.cpu().numpy(), rid)
    np.testing.assert_allclose(w.cpu().numpy(), rw, rtol=0, atol=1e-6)
    # the same ids and weights as the separate router call, bit for bit
    ids2, w2 = _route_gpu(dev, logits_np, topk)
    assert np.array_equal(ids.cpu().numpy(), ids2)
    assert np.array_equal(w.cpu().numpy().view(np.int32), w2.view(np.int32))
    rc, ro, rp, ri, rws = oracle.plan(rid, w.cpu().numpy(), E)
    assert np.array_equal(counts.cpu().numpy(), rc)
    assert np.array_equal(offsets.cpu().numpy(), ro)
    assert np.array_equal(perm[:R].cpu().numpy(), rp)
    assert np.array_equal(inv[:R].cpu().numpy(), ri)
    assert np.array_equal(ws_[:R].cpu().numpy(), rws)
