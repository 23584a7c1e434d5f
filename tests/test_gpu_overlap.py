"""The single-kernel layer (moe_ffn_fused with n_c >= 1): memory CTAs dispatch and
combine while GEMM CTAs run GEMM1 and GEMM2, handing off through ready flags.

It performs the same arithmetic in the same order as the five-launch sequence
(n_c = 0), so its output must be bit-identical for every n_c, and within the
layer bar of the fp64 oracle.  Failure detection is tested without any GPU
fault: a test hook withholds one ready flag, the bounded waits run out, the call
reports MOE_ERR_TIMEOUT and the context stays usable."""
import numpy as np
import pytest
import torch

import oracle
from grouped_gemm_plan_b200 import binding as B
from grouped_gemm_plan_b200 import workload as wl
from helpers import check_close, layer_case
from test_gpu_layer import run_fused

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def single_cta_sequence(monkeypatch):
    """The single-kernel layer uses 128-row tiles; the five-launch reference it is
    compared with bit for bit is pinned to the single-CTA GEMM (same tiles)."""
    monkeypatch.setenv("MOE_GEMM_PAIR", "0")

CASES = [
    (256, 256, 512, 8, 2, "uniform"),
    (129, 512, 192, 3, 3, "skewed"),
    (1000, 128, 256, 64, 4, "skewed"),
    (64, 1024, 512, 16, 8, "skewed"),
    (513, 256, 128, 1, 1, "uniform"),
    (7, 256, 256, 4, 2, "uniform"),     # fewer tokens than memory CTAs
]


@pytest.mark.parametrize("M,H,F,E,topk,kind", CASES)
def test_overlap_bit_identical_to_sequence_and_matches_oracle(cuda_dev, M, H, F, E, topk, kind):
    w, x, W1, W2, ids, tw = layer_case(M, H, F, E, topk, kind, seed=3 * M + H)
    ref_seq, c0, o0, p0 = run_fused(cuda_dev, x, W1, W2, ids, tw, n_c=0)
    for n_c in (1, 4, 16):
        out, counts, offsets, perm = run_fused(cuda_dev, x, W1, W2, ids, tw, n_c=n_c)
        assert torch.equal(out.view(torch.int16), ref_seq.view(torch.int16)), f"n_c={n_c}"
        assert torch.equal(counts, c0) and torch.equal(offsets, o0) and torch.equal(perm, p0)
    check_close(out, oracle.moe_ffn(x, W1, W2, ids, tw), "single-kernel layer")


def test_overlap_repeatable(cuda_dev):
    w, x, W1, W2, ids, tw = layer_case(900, 512, 384, 16, 2, "skewed", seed=9)
    a = run_fused(cuda_dev, x, W1, W2, ids, tw, n_c=8)[0]
    for _ in range(3):
        b = run_fused(cuda_dev, x, W1, W2, ids, tw, n_c=8)[0]
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("name", ["mixtral", "qwen2", "wide16"])
def test_overlap_full_size_matches_sequence(cuda_dev, name):
    w = wl.WORKLOADS[name]
    x = wl.make_x(w)
    W1 = torch.empty((w.E, w.H, 2 * w.F), dtype=torch.bfloat16, device=cuda_dev)
    W2 = torch.empty((w.E, w.F, w.H), dtype=torch.bfloat16, device=cuda_dev)
    wl.make_weights(w, W1, W2)
    ids, tw = wl.make_routing(w)
    seq = run_fused(cuda_dev, x, W1, W2, ids, tw, n_c=0, W_on_dev=True)[0]
    for n_c in (4, 16):
        out = run_fused(cuda_dev, x, W1, W2, ids, tw, n_c=n_c, W_on_dev=True)[0]
        assert torch.equal(out.view(torch.int16), seq.view(torch.int16)), f"{name} n_c={n_c}"


def test_withheld_flag_times_out_and_context_survives(cuda_dev):
    w, x, W1, W2, ids, tw = layer_case(300, 256, 256, 4, 2, "uniform", seed=4)
    M, H = x.shape
    E, _, F2 = W1.shape
    dev = cuda_dev
    args = [x.to(dev), W1.to(dev), W2.to(dev), torch.from_numpy(ids).to(dev),
            torch.from_numpy(tw).to(dev)]
    out = torch.empty(M, H, dtype=torch.bfloat16, device=dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(M * 2, dtype=torch.int32, device=dev)
    ws = B.alloc_workspace(B.OP_FFN_FUSED, M, H, F2 // 2, E, 2, dev)
    try:
        B.moe_set_wait_timeout_ns(200_000_000)            # 0.2 s without progress
        B.moe_set_fault_injection(1, 0)                   # m-tile 0 is never published
        B.moe_ffn_fused(*args, out, counts, offsets, perm, ws, n_c=4)
        assert B.moe_get_device_status(ws) == B.MOE_ERR_TIMEOUT
    finally:
        B.moe_set_fault_injection(0)
        B.moe_set_wait_timeout_ns(2_000_000_000)
    # the context is still usable and the next call is correct
    B.moe_ffn_fused(*args, out, counts, offsets, perm, ws, n_c=4)
    assert B.moe_get_device_status(ws) == B.MOE_OK
    check_close(out, oracle.moe_ffn(x, W1, W2, ids, tw), "after a timed-out call")


def test_overlap_bad_expert_id_ends_without_waiting(cuda_dev):
    w, x, W1, W2, ids, tw = layer_case(100, 128, 128, 4, 2, "uniform", seed=1)
    ids = ids.copy()
    ids[5, 1] = 11
    dev = cuda_dev
    out = torch.empty(100, 128, dtype=torch.bfloat16, device=dev)
    counts = torch.empty(4, dtype=torch.int32, device=dev)
    offsets = torch.empty(5, dtype=torch.int32, device=dev)
    perm = torch.empty(200, dtype=torch.int32, device=dev)
    ws = B.alloc_workspace(B.OP_FFN_FUSED, 100, 128, 128, 4, 2, dev)
    import time
    t0 = time.perf_counter()
    B.moe_ffn_fused(x.to(dev), W1.to(dev), W2.to(dev), torch.from_numpy(ids).to(dev),
                    torch.from_numpy(tw).to(dev), out, counts, offsets, perm, ws, n_c=4)
    assert B.moe_get_device_status(ws) == B.MOE_ERR_BAD_EXPERT_ID
    assert time.perf_counter() - t0 < 1.0      # the kernel saw the failed plan and left
