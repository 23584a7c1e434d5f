"""GPU parity of the whole MoE SwiGLU FFN layer (moe_ffn_fused and the chain of
separate calls) against the fp64 oracle.

Small and medium shapes are compared element by element with the full oracle.
The five workload shapes are run at full size in the launch configuration the
benchmark times; there the plan is compared bit for bit, a sample of output rows
is compared with the oracle's per-token brute force, and the fused output is
compared with the chain of separate calls over every element.

Bar (the stated layer tolerance, read for a bf16 output): relative Frobenius <= 1e-2
and per element |err| <= 2e-2 * rms(ref) + half a bf16 ulp of ref per bf16
rounding on the path after the last GEMM (see helpers.check_close)."""
import numpy as np
import pytest
import torch

import oracle
from grouped_gemm_plan_b200 import binding as B
from grouped_gemm_plan_b200 import workload as wl
from helpers import check_close, guarded_empty, layer_case

pytestmark = pytest.mark.gpu


def run_fused(dev, x, W1, W2, ids, tw, n_c=0, W_on_dev=False):
    M, H = x.shape
    E, _, F2 = W1.shape
    topk = ids.shape[1]
    R = M * topk
    out, check = guarded_empty((M, H), torch.bfloat16, dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(max(R, 1), dtype=torch.int32, device=dev)
    ws = B.alloc_workspace(B.OP_FFN_FUSED, M, H, F2 // 2, E, topk, dev)
    W1d = W1 if W_on_dev else W1.to(dev)
    W2d = W2 if W_on_dev else W2.to(dev)
    B.moe_ffn_fused(x.to(dev), W1d, W2d, torch.from_numpy(ids).to(dev),
                    torch.from_numpy(tw).to(dev), out, counts, offsets, perm[:R] if R else perm,
                    ws, n_c=n_c)
    st = B.moe_get_device_status(ws)
    check()
    assert st == B.MOE_OK, B.STATUS_NAMES.get(st)
    return out, counts, offsets, perm[:R]


def run_chain(dev, x, W1, W2, ids, tw):
    """plan -> dispatch -> GEMM1+SwiGLU -> GEMM2 (plain store) -> weighted combine."""
    M, H = x.shape
    E, _, F2 = W1.shape
    F = F2 // 2
    topk = ids.shape[1]
    R = M * topk
    ids_d, tw_d = torch.from_numpy(ids).to(dev), torch.from_numpy(tw).to(dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(R, dtype=torch.int32, device=dev)
    inv = torch.empty(R, dtype=torch.int32, device=dev)
    ws = B.alloc_workspace(B.OP_PLAN, M, H, F, E, topk, dev)
    B.moe_plan(ids_d, tw_d, E, counts, offsets, perm, inv, None, ws)
    xp = torch.empty(R, H, dtype=torch.bfloat16, device=dev)
    B.moe_dispatch(x.to(dev), perm, topk, xp, ws)
    h = torch.empty(R, F, dtype=torch.bfloat16, device=dev)
    B.moe_grouped_gemm(xp, W1 if W1.is_cuda else W1.to(dev), offsets, B.EPI_SWIGLU, h, ws)
    y = torch.empty(R, H, dtype=torch.bfloat16, device=dev)
    B.moe_grouped_gemm(h, W2 if W2.is_cuda else W2.to(dev), offsets, B.EPI_STORE, y, ws)
    out = torch.empty(M, H, dtype=torch.bfloat16, device=dev)
    B.moe_combine(y, inv, tw_d, M, topk, out, ws)
    assert B.moe_get_device_status(ws) == B.MOE_OK
    return out


MEDIUM = [
    # (M, H, F, E, topk, routing)
    (256, 256, 512, 8, 2, "uniform"),     # the tiny layer, whole
    (300, 256, 384, 6, 2, "skewed"),
    (129, 512, 192, 3, 3, "skewed"),      # F = 192: GEMM1 half tile
    (1000, 128, 256, 64, 4, "skewed"),    # many small experts, most tiles ragged
    (64, 1024, 512, 16, 8, "skewed"),     # wide top-k, tiny M
    (513, 256, 128, 1, 1, "uniform"),     # dense special case E = 1, topk = 1
    (300, 64, 64, 1024, 8, "uniform"),    # the largest expert count: most experts hold 0-5 rows
]


@pytest.mark.parametrize("M,H,F,E,topk,kind", MEDIUM)
def test_layer_matches_oracle(cuda_dev, M, H, F, E, topk, kind):
    w, x, W1, W2, ids, tw = layer_case(M, H, F, E, topk, kind, seed=M + H)
    ref = oracle.moe_ffn(x, W1, W2, ids, tw)
    out, counts, offsets, perm = run_fused(cuda_dev, x, W1, W2, ids, tw)
    check_close(out, ref, "fused layer")
    rc, ro, rp, _, _ = oracle.plan(ids, tw, E)
    assert np.array_equal(counts.cpu().numpy(), rc)
    assert np.array_equal(offsets.cpu().numpy(), ro)
    assert np.array_equal(perm.cpu().numpy(), rp)
    chain = run_chain(cuda_dev, x, W1, W2, ids, tw)
    # the chain stores the expert outputs in bf16 before combining: one rounding more
    check_close(chain, ref, "chain of calls", ulps=2.0)


def test_layer_empty_batch(cuda_dev):
    x = torch.zeros(0, 128, dtype=torch.bfloat16)
    W1 = torch.zeros(4, 128, 256, dtype=torch.bfloat16)
    W2 = torch.zeros(4, 128, 128, dtype=torch.bfloat16)
    ids = np.zeros((0, 2), np.int32)
    tw = np.zeros((0, 2), np.float32)
    out, counts, offsets, _ = run_fused(cuda_dev, x, W1, W2, ids, tw)
    assert out.numel() == 0
    assert counts.cpu().tolist() == [0] * 4 and offsets.cpu().tolist() == [0] * 5


def test_layer_bad_expert_id(cuda_dev):
    w, x, W1, W2, ids, tw = layer_case(100, 128, 128, 4, 2, "uniform", seed=1)
    ids = ids.copy()
    ids[17, 0] = 4
    M, H = x.shape
    out = torch.empty(M, H, dtype=torch.bfloat16, device=cuda_dev)
    counts = torch.empty(4, dtype=torch.int32, device=cuda_dev)
    offsets = torch.empty(5, dtype=torch.int32, device=cuda_dev)
    perm = torch.empty(200, dtype=torch.int32, device=cuda_dev)
    ws = B.alloc_workspace(B.OP_FFN_FUSED, M, H, 128, 4, 2, cuda_dev)
    B.moe_ffn_fused(x.to(cuda_dev), W1.to(cuda_dev), W2.to(cuda_dev),
                    torch.from_numpy(ids).to(cuda_dev), torch.from_numpy(tw).to(cuda_dev), out,
                    counts, offsets, perm, ws)
    assert B.moe_get_device_status(ws) == B.MOE_ERR_BAD_EXPERT_ID
    assert counts.cpu().tolist() == [0] * 4


@pytest.mark.parametrize("pair", ["0", "1"])
def test_layer_both_gemm_kernels(cuda_dev, monkeypatch, pair):
    monkeypatch.setenv("MOE_GEMM_PAIR", pair)
    w, x, W1, W2, ids, tw = layer_case(700, 512, 384, 4, 2, "skewed", seed=12)
    out = run_fused(cuda_dev, x, W1, W2, ids, tw)[0]
    check_close(out, oracle.moe_ffn(x, W1, W2, ids, tw), f"layer, pair kernel={pair}")


def test_layer_deterministic(cuda_dev):
    w, x, W1, W2, ids, tw = layer_case(777, 512, 384, 16, 2, "skewed", seed=5)
    a = run_fused(cuda_dev, x, W1, W2, ids, tw)[0]
    b = run_fused(cuda_dev, x, W1, W2, ids, tw)[0]
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("n_c", [0, 2])
def test_stage_events(cuda_dev, n_c):
    """moe_set_stage_events: six events around the stages of one call, in order, the
    stage times summing to the call's time; the output is unchanged by timing."""
    w, x, W1, W2, ids, tw = layer_case(700, 512, 384, 8, 2, "skewed", seed=21)
    ref = run_fused(cuda_dev, x, W1, W2, ids, tw, n_c=n_c)[0]
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
    outer = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    B.moe_set_stage_events(evs)
    try:
        outer[0].record()
        got = run_fused(cuda_dev, x, W1, W2, ids, tw, n_c=n_c)[0]
        outer[1].record()
    finally:
        B.moe_set_stage_events(None)
    torch.cuda.synchronize()
    assert torch.equal(got.view(torch.int16), ref.view(torch.int16))
    stages = [evs[i].elapsed_time(evs[i + 1]) for i in range(5)]
    assert all(t >= 0.0 for t in stages), stages
    assert stages[2] > 0.0 and stages[3] > 0.0 or n_c > 0
    total = evs[0].elapsed_time(evs[5])
    assert abs(sum(stages) - total) < 1e-3 + 1e-3 * total
    assert total <= outer[0].elapsed_time(outer[1]) + 1e-3
    # off again: a later call records nothing (the events keep their times)
    run_fused(cuda_dev, x, W1, W2, ids, tw, n_c=n_c)
    torch.cuda.synchronize()
    assert evs[0].elapsed_time(evs[5]) == total


def _sample_tokens(ids, perm, offsets, n, seed):
    """Tokens whose output rows are compared with the oracle at full size.

    Every expert's first and last slot; for the heaviest and the lightest expert
    the slots on both sides of every 128-row and 256-row m-tile boundary (the
    single-CTA and the CTA-pair kernels' tiles); the first and last token; then
    random tokens until there are n (or all M).
    """
    M, topk = ids.shape
    rng = np.random.default_rng(seed)
    counts = np.diff(offsets)
    picks = {0, M - 1}

    def slot_token(s):
        picks.add(int(perm[s]) // topk)

    nz = np.flatnonzero(counts)
    for e in nz:
        slot_token(offsets[e])
        slot_token(offsets[e + 1] - 1)
    for e in {int(nz[np.argmax(counts[nz])]), int(nz[np.argmin(counts[nz])])}:
        for bm in (128, 256):
            for b in range(bm, int(counts[e]), bm):
                slot_token(offsets[e] + b - 1)
                slot_token(offsets[e] + b)
    rest = np.setdiff1d(np.arange(M), np.fromiter(picks, np.int64))
    extra = max(0, min(n, M) - len(picks))
    picks.update(rng.choice(rest, size=min(extra, rest.size), replace=False).tolist())
    return np.array(sorted(picks), np.int64)


@pytest.mark.parametrize("name", ["tiny", "mixtral", "qwen2", "phi35", "wide16", "wide128",
                                  "wide512", "wide2048"])
def test_workload_full_size(cuda_dev, name):
    w = wl.WORKLOADS[name]
    x = wl.make_x(w)
    W1 = torch.empty((w.E, w.H, 2 * w.F), dtype=torch.bfloat16, device=cuda_dev)
    W2 = torch.empty((w.E, w.F, w.H), dtype=torch.bfloat16, device=cuda_dev)
    wl.make_weights(w, W1, W2)
    ids, tw = wl.make_routing(w)
    out, counts, offsets, perm = run_fused(cuda_dev, x, W1, W2, ids, tw, W_on_dev=True)
    rc, ro, rp, _, _ = oracle.plan(ids, tw, w.E)
    assert np.array_equal(counts.cpu().numpy(), rc)
    assert np.array_equal(offsets.cpu().numpy(), ro)
    assert np.array_equal(perm.cpu().numpy(), rp)
    tokens = _sample_tokens(ids, rp, ro, 256, w.seed)
    assert tokens.size >= min(256, w.M)
    W1c, W2c = W1.cpu(), W2.cpu()
    ref_rows = oracle.bruteforce_tokens(x, W1c, W2c, ids, tw, tokens)
    check_close(out.cpu()[torch.from_numpy(tokens)], ref_rows, f"{name} sampled rows")
    chain = run_chain(cuda_dev, x, W1, W2, ids, tw)
    chain_rows = chain.cpu()[torch.from_numpy(tokens)]
    check_close(chain_rows, ref_rows, f"{name} chain sampled rows", ulps=2.0)
    # two bf16 results of the same layer: within the bar of each other, one
    # rounding of each allowed
    check_close(out, chain.double().cpu().numpy(), f"{name} fused vs chain", ulps=3.0)
