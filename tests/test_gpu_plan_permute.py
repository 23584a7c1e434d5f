"""GPU parity of the routing plan, dispatch and combine (through the C ABI).

Plan and dispatch are integer / bit-copy work: compared bit for bit with the
oracle.  Combine is floating point: compared with the fp64 oracle within the
layer tolerance."""
import numpy as np
import pytest
import torch

import oracle
from grouped_gemm_plan_b200 import binding as B
from helpers import check_close, guarded_empty, routing_case

pytestmark = pytest.mark.gpu


def _plan_gpu(ids_np, w_np, E, dev):
    M, topk = ids_np.shape
    R = M * topk
    ids = torch.from_numpy(ids_np).to(dev)
    w = torch.from_numpy(w_np).to(dev) if w_np is not None else None
    counts = torch.full((E,), -7, dtype=torch.int32, device=dev)
    offsets = torch.full((E + 1,), -7, dtype=torch.int32, device=dev)
    perm = torch.full((max(R, 1),), -7, dtype=torch.int32, device=dev)
    inv = torch.full((max(R, 1),), -7, dtype=torch.int32, device=dev)
    ws_sorted = torch.full((max(R, 1),), -7.0, dtype=torch.float32, device=dev) if w is not None else None
    ws = B.alloc_workspace(B.OP_PLAN, M, 0, 0, E, topk, dev)
    B.moe_plan(ids, w, E, counts, offsets, perm[:R] if R else perm, inv[:R] if R else inv,
               (ws_sorted[:R] if R else ws_sorted) if ws_sorted is not None else None, ws)
    status = B.moe_get_device_status(ws)
    out = (counts.cpu().numpy(), offsets.cpu().numpy(), perm[:R].cpu().numpy(),
           inv[:R].cpu().numpy(), ws_sorted[:R].cpu().numpy() if ws_sorted is not None else None)
    return status, out


PLAN_CASES = [
    # (M, E, topk, routing)
    (256, 8, 2, "uniform"),       # the tiny layer's shape
    (1, 1, 1, "uniform"),
    (1000, 1, 1, "uniform"),      # single expert
    (8192, 64, 4, "skewed"),      # Qwen2-MoE shape: many chunks
    (16384, 16, 2, "skewed"),     # Phi-3.5-MoE shape, heavy skew
    (4096, 8, 2, "balanced"),     # Mixtral shape, exact balance
    (12345, 17, 3, "skewed"),     # ragged tail of the last chunk
    (3000, 1024, 8, "uniform"),   # largest expert count
    (37, 300, 4, "uniform"),      # most experts empty
]


@pytest.mark.parametrize("M,E,topk,kind", PLAN_CASES)
def test_plan_bit_exact(cuda_dev, M, E, topk, kind):
    ids, w = routing_case(M, E, topk, kind, seed=M + E)
    status, (c, o, p, i, ws) = _plan_gpu(ids, w, E, cuda_dev)
    assert status == B.MOE_OK
    rc, ro, rp, ri, rws = oracle.plan(ids, w, E)
    assert np.array_equal(c, rc)
    assert np.array_equal(o, ro)
    assert np.array_equal(p, rp)
    assert np.array_equal(i, ri)
    assert np.array_equal(ws.view(np.uint32), rws.view(np.uint32))


def test_plan_duplicates_and_single_expert(cuda_dev):
    rng = np.random.default_rng(3)
    ids = rng.integers(0, 5, size=(999, 4), dtype=np.int32)   # duplicates within a token
    ids[:100] = 2
    w = rng.random((999, 4)).astype(np.float32)
    status, got = _plan_gpu(ids, w, 5, cuda_dev)
    assert status == B.MOE_OK
    for g, r in zip(got, oracle.plan(ids, w, 5)):
        assert np.array_equal(g, r)
    ids_all = np.full((513, 3), 6, np.int32)
    status, got = _plan_gpu(ids_all, None, 7, cuda_dev)
    assert status == B.MOE_OK
    rc, ro, rp, ri, _ = oracle.plan(ids_all, None, 7)
    assert np.array_equal(got[0], rc) and np.array_equal(got[2], rp)


def test_plan_empty(cuda_dev):
    ids = np.zeros((0, 2), np.int32)
    status, (c, o, p, i, _) = _plan_gpu(ids, None, 6, cuda_dev)
    assert status == B.MOE_OK
    assert c.tolist() == [0] * 6 and o.tolist() == [0] * 7


def test_plan_bad_id_is_a_defined_failure(cuda_dev):
    ids, w = routing_case(700, 8, 2, "uniform", seed=1)
    ids = ids.copy()
    ids[345, 1] = 8
    status, (c, o, p, i, ws) = _plan_gpu(ids, w, 8, cuda_dev)
    assert status == B.MOE_ERR_BAD_EXPERT_ID
    assert c.tolist() == [0] * 8 and o.tolist() == [0] * 9
    assert np.array_equal(p, np.arange(1400)) and np.array_equal(i, np.arange(1400))
    ids[345, 1] = -1
    status, _ = _plan_gpu(ids, w, 8, cuda_dev)
    assert status == B.MOE_ERR_BAD_EXPERT_ID


@pytest.mark.parametrize("M,H,E,topk", [(256, 256, 8, 2), (1000, 4096, 16, 2), (77, 7168, 16, 8),
                                         (5, 64, 3, 3)])
def test_dispatch_bit_exact(cuda_dev, M, H, E, topk):
    ids, _ = routing_case(M, E, topk, "skewed", seed=H)
    _, _, perm, inv, _ = oracle.plan(ids, None, E)
    x = torch.randn(M, H).to(torch.bfloat16)
    xp_ref = oracle.dispatch(x, perm, topk)
    xp, check = guarded_empty((M * topk, H), torch.bfloat16, cuda_dev)
    ws = B.alloc_workspace(B.OP_DISPATCH, M, H, 0, E, topk, cuda_dev)
    B.moe_dispatch(x.to(cuda_dev), torch.from_numpy(perm).to(cuda_dev), topk, xp, ws)
    assert B.moe_get_device_status(ws) == B.MOE_OK
    check()
    got = xp.cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, xp_ref)
    # unpermute of the permute is the identity
    back = oracle.unpermute_rows(got, inv)
    xb = x.view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(back, np.repeat(xb, topk, axis=0))


def test_dispatch_bad_index(cuda_dev):
    M, H, topk = 10, 64, 2
    perm = torch.arange(M * topk, dtype=torch.int32)
    perm[3] = 10_000
    x = torch.randn(M, H).to(torch.bfloat16).to(cuda_dev)
    xp = torch.empty(M * topk, H, dtype=torch.bfloat16, device=cuda_dev)
    ws = B.alloc_workspace(B.OP_DISPATCH, M, H, 0, 1, topk, cuda_dev)
    B.moe_dispatch(x, perm.to(cuda_dev), topk, xp, ws)
    assert B.moe_get_device_status(ws) == B.MOE_ERR_BAD_INDEX
    assert bool((xp[3] == 0).all())


@pytest.mark.parametrize("M,H,E,topk,token_major,ydt", [
    (256, 256, 8, 2, False, torch.bfloat16), (333, 2048, 64, 4, False, torch.bfloat16),
    (64, 7168, 16, 8, True, torch.float32), (1000, 4096, 16, 2, True, torch.float32),
    (9, 64, 40, 32, False, torch.float32), (50, 128, 8, 3, True, torch.bfloat16)])
def test_combine(cuda_dev, M, H, E, topk, token_major, ydt):
    ids, w = routing_case(M, E, topk, "uniform", seed=M)
    _, _, perm, inv, _ = oracle.plan(ids, w, E)
    R = M * topk
    y = torch.randn(R, H).to(ydt)
    yd = y.double().numpy()
    out, check = guarded_empty((M, H), torch.bfloat16, cuda_dev)
    ws = B.alloc_workspace(B.OP_COMBINE, M, H, 0, E, topk, cuda_dev)
    if token_major:
        # rows already weighted and in token order (the fused GEMM2 epilogue's output)
        B.moe_combine(y.to(cuda_dev), None, None, M, topk, out, ws)
        ref = yd.reshape(M, topk, H).sum(1)
    else:
        B.moe_combine(y.to(cuda_dev), torch.from_numpy(inv).to(cuda_dev),
                      torch.from_numpy(w).to(cuda_dev), M, topk, out, ws)
        ref = oracle.combine(yd, inv, w)
    assert B.moe_get_device_status(ws) == B.MOE_OK
    check()
    check_close(out, ref, "combine")
