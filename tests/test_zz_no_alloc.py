"""moe_ffn_fused_noalloc: the layer for callers that cannot allocate device memory.

A C or plugin caller that only holds its input and output buffers, or a process
whose device memory is reserved up front by another allocator, cannot provide
the workspace moe_ffn_fused needs.  moe_ffn_fused_noalloc keeps its intermediates
in the library's own fixed device array instead.  These tests call it through
the C ABI and check it against moe_ffn_fused on the same inputs (the same
kernels in the same order, so the outputs must be bit-identical) and against the
CPU oracle.  The file sorts last so that a run stopping at the first failure has
run every other test first.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from grouped_gemm_plan_b200 import binding as B
from helpers import check_close, layer_case

# Largest token counts whose intermediates fit the 64 MiB scratch:
# 256 + 256*(E+1)*4 + R*H*2 + R*F*2 + R*H*4 + R*4 bytes, each part rounded up to 256.
MIXTRAL = dict(H=4096, F=14336, E=8, topk=2)   # fits up to M = 630
WIDE = dict(H=7168, F=4096, E=16, topk=8)      # fits up to M = 163


def _needed_bytes(M, H, F, E, topk):
    a = lambda v: (v + 255) // 256 * 256  # noqa: E731
    R = M * topk
    return 256 + a(256 * (E + 1) * 4) + a(R * H * 2) + a(R * F * 2) + a(R * H * 4) + a(R * 4)


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
    cpu_inputs, inputs, results = [], [], []
    for i, (M, H, F, E, topk, kind) in enumerate(CASES):
        w, x, W1, W2, ids, tw = layer_case(M, H, F, E, topk, kind, seed=100 + i)
        cpu_inputs.append((x, W1, W2, ids, tw))
        inputs.append([x.to(cuda_dev), W1.to(cuda_dev), W2.to(cuda_dev),
                       torch.from_numpy(ids).to(cuda_dev), torch.from_numpy(tw).to(cuda_dev)])
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
        assert B.moe_last_error() == ""
        results.append((out, counts, offsets, perm, status))
    torch.cuda.synchronize()
    for d, c, (out, counts, offsets, perm, status) in zip(inputs, cpu_inputs, results):
        assert int(status.item()) == B.MOE_OK
        ref_out, ref_counts, ref_offsets, ref_perm = _existing(cuda_dev, *d)
        assert torch.equal(counts, ref_counts) and torch.equal(offsets, ref_offsets)
        assert torch.equal(perm, ref_perm)
        # same kernels, same arithmetic order: bit-identical to moe_ffn_fused
        assert torch.equal(out.view(torch.int16), ref_out.view(torch.int16)), \
            "noalloc output differs from moe_ffn_fused"
        x, W1, W2, ids, tw = c
        check_close(out, oracle.moe_ffn(x, W1, W2, ids, tw), "noalloc vs the oracle")


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


@pytest.mark.gpu
def test_noalloc_empty_batch(cuda_dev):
    # M = 0: a defined plan (zero counts and offsets), nothing else runs
    lib = B.load()
    E = 6
    x = torch.empty(0, 256, dtype=torch.bfloat16, device=cuda_dev)
    W1 = torch.empty(E, 256, 256, dtype=torch.bfloat16, device=cuda_dev)
    W2 = torch.empty(E, 128, 256, dtype=torch.bfloat16, device=cuda_dev)
    ids = torch.empty(0, 2, dtype=torch.int32, device=cuda_dev)
    tw = torch.empty(0, 2, dtype=torch.float32, device=cuda_dev)
    out = torch.empty(0, 256, dtype=torch.bfloat16, device=cuda_dev)
    counts = torch.full((E,), -1, dtype=torch.int32, device=cuda_dev)
    offsets = torch.full((E + 1,), -1, dtype=torch.int32, device=cuda_dev)
    perm = torch.empty(0, dtype=torch.int32, device=cuda_dev)
    status = torch.full((1,), -1, dtype=torch.int32, device=cuda_dev)
    st = _noalloc_c(lib, cuda_dev, x, W1, W2, ids, tw, out, counts, offsets, perm, status)
    assert st == B.MOE_OK, B.moe_last_error()
    torch.cuda.synchronize()
    assert int(status.item()) == B.MOE_OK
    assert counts.cpu().tolist() == [0] * E
    assert offsets.cpu().tolist() == [0] * (E + 1)


# ---------------------------------------------------------------- host-side checks
# Each of these returns before any device work, so they run without a GPU: the
# pointers below are never dereferenced.

def _call_host(lib, M, H, F, E, topk, x_ptr):
    fake = ctypes.c_void_p(0x10000)
    return lib.moe_ffn_fused_noalloc(x_ptr, fake, fake, fake, fake, M, H, F, E, topk, fake,
                                     fake, fake, fake, None, None)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    lib = B.load()
    fake = ctypes.c_void_p(0x10000)
    st = _call_host(lib, 4096, 4096, 14336, 8, 2, fake)
    assert st == B.MOE_ERR_WORKSPACE_TOO_SMALL
    assert "static scratch" in B.moe_last_error()


@pytest.mark.parametrize("shape,m_max", [(MIXTRAL, 630), (WIDE, 163)])
def test_noalloc_scratch_limit_boundary(shape, m_max):
    # The documented limit, checked against the byte formula of the header: M = m_max
    # passes the scratch check (and then fails on its NULL x, still on the host), one
    # more token is rejected for scratch.
    lib = B.load()
    limit = B.NOALLOC_SCRATCH_BYTES
    assert _needed_bytes(m_max, **shape) <= limit < _needed_bytes(m_max + 1, **shape)
    H, F, E, topk = shape["H"], shape["F"], shape["E"], shape["topk"]
    assert _call_host(lib, m_max, H, F, E, topk, None) == B.MOE_ERR_INVALID_ARG
    assert "must not be NULL" in B.moe_last_error()
    assert _call_host(lib, m_max + 1, H, F, E, topk, None) == B.MOE_ERR_WORKSPACE_TOO_SMALL


def test_noalloc_rejects_sizes_that_would_overflow():
    # M * topk beyond int32 (here M = 2^61, which wraps the byte counts of the
    # scratch layout to small numbers) must be refused by the shape checks with the
    # same code as moe_ffn_fused, before the scratch limit is looked at.
    lib = B.load()
    fake = ctypes.c_void_p(0x10000)
    assert _call_host(lib, 2 ** 61, 64, 64, 8, 2, fake) == B.MOE_ERR_UNSUPPORTED_SHAPE
    assert "2^31-1" in B.moe_last_error()
    assert _call_host(lib, 2 ** 30, 64, 64, 8, 2, fake) == B.MOE_ERR_UNSUPPORTED_SHAPE


def test_noalloc_error_codes_match_the_fused_call():
    lib = B.load()
    fake = ctypes.c_void_p(0x10000)
    cases = [  # (M, H, F, E, topk)
        (4, 64, 64, 0, 1),      # E < 1
        (4, 64, 64, 4, 5),      # topk > E
        (-1, 64, 64, 4, 2),     # M < 0
        (4, 96, 64, 4, 2),      # H not a multiple of 64
        (4, 64, 32, 4, 2),      # F not a multiple of 64
        (4, 64, 64, 2048, 2),   # E > MOE_MAX_EXPERTS
    ]
    for M, H, F, E, topk in cases:
        st_noalloc = _call_host(lib, M, H, F, E, topk, fake)
        msg_noalloc = B.moe_last_error()
        st_fused = lib.moe_ffn_fused(fake, fake, fake, fake, fake, M, H, F, E, topk, 0, fake,
                                     fake, fake, fake, fake, 1 << 40, None)
        assert st_noalloc == st_fused != B.MOE_OK, (M, H, F, E, topk, st_noalloc, st_fused)
        assert msg_noalloc == B.moe_last_error()
