"""moe_ffn_fused_noalloc: the layer for callers that cannot allocate device memory.

A C or plugin caller that only holds its input and output buffers, or a process
whose device memory is reserved up front by another allocator, cannot provide
the workspace moe_ffn_fused needs.  moe_ffn_fused_noalloc keeps its intermediates
in the library's own fixed device array instead.  These tests call it through
the C ABI and check it against moe_ffn_fused on the same inputs.  The file sorts
last so that a run stopping at the first failure has run every other test first.
"""
import ctypes

import numpy as np
import pytest
import torch

from grouped_gemm_plan_b200 import binding as B
from helpers import check_close, layer_case


def _dev_ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _noalloc_c(lib, dev, x, W1, W2, ids, tw, out, counts, offsets, perm, status):
    M, H = x.shape
    E, _, F2 = W1.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    return lib.moe_ffn_fused_noalloc(_dev_ptr(x), _dev_ptr(W1), _dev_ptr(W2), _dev_ptr(ids),
                                     _dev_ptr(tw), M, H, F2 // 2, E, ids.shape[1], _dev_ptr(out),
                                     _dev_ptr(counts), _dev_ptr(offsets), _dev_ptr(perm),
                                     _dev_ptr(status), stream)


def _existing(dev, x, W1, W2, ids, tw):
    M, H = x.shape
    E, _, F2 = W1.shape
    topk = ids.shape[1]
    out = torch.empty(M, H, dtype=torch.bfloat16, device=dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(M * topk, dtype=torch.int32, device=dev)
    ws = B.alloc_workspace(B.OP_FFN_FUSED, M, H, F2 // 2, E, topk, dev)
    B.moe_ffn_fused(x, W1, W2, ids, tw, out, counts, offsets, perm, ws, n_c=0)
    assert B.moe_get_device_status(ws) == B.MOE_OK
    return out, counts, offsets, perm


CASES = [
    # (M, H, F, E, topk, routing): the second call is smaller than the first, so it
    # runs on scratch that still holds the first call's intermediates
    (150, 1024, 512, 8, 2, "skewed"),
    (40, 512, 384, 16, 4, "uniform"),
]


@pytest.mark.gpu
def test_noalloc_matches_fused_on_two_calls_in_a_row(cuda_dev):
    lib = B.load()
    inputs, results = [], []
    for i, (M, H, F, E, topk, kind) in enumerate(CASES):
        w, x, W1, W2, ids, tw = layer_case(M, H, F, E, topk, kind, seed=100 + i)
        d = [x.to(cuda_dev), W1.to(cuda_dev), W2.to(cuda_dev),
             torch.from_numpy(ids).to(cuda_dev), torch.from_numpy(tw).to(cuda_dev)]
        inputs.append(d)
    # two calls of the new entry point back to back
    for d in inputs:
        x, W1, W2, ids, tw = d
        M, H = x.shape
        E = W1.shape[0]
        out = torch.full((M, H), 7.0, dtype=torch.bfloat16, device=cuda_dev)
        counts = torch.empty(E, dtype=torch.int32, device=cuda_dev)
        offsets = torch.empty(E + 1, dtype=torch.int32, device=cuda_dev)
        perm = torch.empty(ids.numel(), dtype=torch.int32, device=cuda_dev)
        status = torch.full((1,), -1, dtype=torch.int32, device=cuda_dev)
        st = _noalloc_c(lib, cuda_dev, x, W1, W2, ids, tw, out, counts, offsets, perm, status)
        assert st == B.MOE_OK, B.moe_last_error()
        results.append((out, counts, offsets, perm, status))
    torch.cuda.synchronize()
    for d, (out, counts, offsets, perm, status) in zip(inputs, results):
        assert int(status.item()) == B.MOE_OK
        ref_out, ref_counts, ref_offsets, ref_perm = _existing(cuda_dev, *d)
        assert torch.equal(counts, ref_counts) and torch.equal(offsets, ref_offsets)
        assert torch.equal(perm, ref_perm)
        check_close(out, ref_out.double().cpu().numpy(), "noalloc vs moe_ffn_fused")


@pytest.mark.gpu
def test_noalloc_reports_device_status(cuda_dev):
    lib = B.load()
    w, x, W1, W2, ids, tw = layer_case(32, 256, 128, 4, 2, "uniform", seed=7)
    ids = ids.copy()
    ids[3, 1] = 9                              # expert id outside [0, E)
    d = [x.to(cuda_dev), W1.to(cuda_dev), W2.to(cuda_dev), torch.from_numpy(ids).to(cuda_dev),
         torch.from_numpy(tw).to(cuda_dev)]
    out = torch.empty(32, 256, dtype=torch.bfloat16, device=cuda_dev)
    counts = torch.empty(4, dtype=torch.int32, device=cuda_dev)
    offsets = torch.empty(5, dtype=torch.int32, device=cuda_dev)
    perm = torch.empty(64, dtype=torch.int32, device=cuda_dev)
    status = torch.zeros(1, dtype=torch.int32, device=cuda_dev)
    assert _noalloc_c(lib, cuda_dev, *d, out, counts, offsets, perm, status) == B.MOE_OK
    torch.cuda.synchronize()
    assert int(status.item()) == B.MOE_ERR_BAD_EXPERT_ID
    assert counts.cpu().tolist() == [0] * 4


def test_noalloc_rejects_shapes_beyond_its_scratch():
    # Checked on the host before any device work: no GPU needed.
    lib = B.load()
    fake = ctypes.c_void_p(0x10000)
    st = lib.moe_ffn_fused_noalloc(fake, fake, fake, fake, fake, 4096, 4096, 14336, 8, 2, fake,
                                   fake, fake, fake, None, None)
    assert st == B.MOE_ERR_WORKSPACE_TOO_SMALL
    assert "static scratch" in B.moe_last_error()
