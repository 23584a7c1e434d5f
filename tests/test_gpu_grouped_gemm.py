"""GPU parity of the tcgen05 grouped GEMM and its three epilogues (through the C ABI).

Structured one-hot operands make the result exact in bf16, so the operand
layouts (A K-major, B N-major, swizzle, descriptors) are checked bit for bit;
random operands are compared with the fp64 oracle within the layer tolerance."""
import numpy as np
import pytest
import torch

import oracle
from grouped_gemm_plan_b200 import binding as B
from helpers import check_stage, guarded_empty

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, params=["single", "pair"])
def gemm_kernel(request, monkeypatch):
    """Run every test on both grouped GEMM kernels: single-CTA 128-row tiles and
    CTA-pair (tcgen05 cta_group::2) 256-row tiles."""
    monkeypatch.setenv("MOE_GEMM_PAIR", "1" if request.param == "pair" else "0")
    return request.param


def _offsets(counts):
    return np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)


def _run(dev, A, Bw, offsets, epi, n_out, w_sorted=None, perm=None):
    R = A.shape[0]
    E = Bw.shape[0]
    dt = torch.float32 if epi == B.EPI_WEIGHT_SCATTER else torch.bfloat16
    C, check = guarded_empty((R, n_out), dt, dev)
    C.zero_()
    ws = B.alloc_workspace(B.OP_GROUPED_GEMM, R, 0, 0, E, 1, dev)
    B.moe_grouped_gemm(A.to(dev), Bw.to(dev), torch.from_numpy(offsets).to(dev), epi, C, ws,
                       w_sorted=None if w_sorted is None else torch.from_numpy(w_sorted).to(dev),
                       perm=None if perm is None else torch.from_numpy(perm).to(dev))
    st = B.moe_get_device_status(ws)
    check()
    assert st == B.MOE_OK, B.STATUS_NAMES.get(st)
    return C.cpu()


def _explain(got, ref, k=8):
    bad = np.argwhere(got != ref)
    return f"{len(bad)} mismatches, first: " + ", ".join(
        f"[{r},{c}] got {got[r, c]} want {ref[r, c]}" for r, c in bad[:k])


@pytest.mark.parametrize("counts,K,N", [([128], 64, 256), ([200, 0, 57], 256, 512)])
def test_one_hot_rows_select_b_rows(cuda_dev, counts, K, N):
    # A[s, k] = 1 iff k == (7 s + 3) mod K  =>  C[s, :] = B[e(s), (7 s + 3) mod K, :] exactly.
    off = _offsets(counts)
    R, E = int(off[-1]), len(counts)
    sel = (7 * np.arange(R) + 3) % K
    A = torch.zeros(R, K)
    A[np.arange(R), sel] = 1
    A = A.to(torch.bfloat16)
    Bw = torch.randn(E, K, N).to(torch.bfloat16)
    got = _run(cuda_dev, A, Bw, off, B.EPI_STORE, N).float().numpy()
    ref = np.zeros((R, N), np.float32)
    for e in range(E):
        for s in range(off[e], off[e + 1]):
            ref[s] = Bw[e, sel[s]].float().numpy()
    assert np.array_equal(got, ref), _explain(got, ref)


@pytest.mark.parametrize("counts,K,N", [([130], 64, 256), ([3, 140], 128, 320)])
def test_one_hot_columns_select_a_columns(cuda_dev, counts, K, N):
    # B[e, k, n] = 1 iff k == (5 n + e) mod K  =>  C[s, n] = A[s, (5 n + e) mod K] exactly.
    off = _offsets(counts)
    R, E = int(off[-1]), len(counts)
    A = torch.randn(R, K).to(torch.bfloat16)
    Bw = torch.zeros(E, K, N)
    for e in range(E):
        Bw[e, (5 * np.arange(N) + e) % K, np.arange(N)] = 1
    Bw = Bw.to(torch.bfloat16)
    got = _run(cuda_dev, A, Bw, off, B.EPI_STORE, N).float().numpy()
    ref = np.zeros((R, N), np.float32)
    Af = A.float().numpy()
    for e in range(E):
        cols = (5 * np.arange(N) + e) % K
        ref[off[e]:off[e + 1]] = Af[off[e]:off[e + 1]][:, cols]
    assert np.array_equal(got, ref), _explain(got, ref)


GEMM_CASES = [
    ([130, 0, 1, 300, 77], 256, 512),   # ragged: one-row expert, empty expert, multi-tile
    ([128, 256], 64, 64),               # whole tiles, smallest K and N
    ([1000], 1024, 256),
    ([5] * 16, 512, 768),               # N not a multiple of the 256-column tile
    ([700, 33, 0, 0, 411], 2048, 256),  # long K
]


def _rand_case(counts, K, N, seed):
    g = torch.Generator().manual_seed(seed)
    off = _offsets(counts)
    R, E = int(off[-1]), len(counts)
    A = torch.randn(R, K, generator=g).to(torch.bfloat16)
    Bw = (torch.randn(E, K, N, generator=g) / np.sqrt(K)).to(torch.bfloat16)
    return off, A, Bw


@pytest.mark.parametrize("counts,K,N", GEMM_CASES)
def test_store_epilogue(cuda_dev, counts, K, N):
    off, A, Bw = _rand_case(counts, K, N, 1)
    got = _run(cuda_dev, A, Bw, off, B.EPI_STORE, N)
    check_stage(got, oracle.grouped_gemm(A, Bw, off), "grouped GEMM store")


SWIGLU_CASES = [c for c in GEMM_CASES if (c[2] // 2) % 64 == 0] + [([90, 250], 256, 384)]  # F=192


@pytest.mark.parametrize("counts,K,N", SWIGLU_CASES)
def test_swiglu_epilogue(cuda_dev, counts, K, N):
    off, A, Bw = _rand_case(counts, K, N, 2)
    got = _run(cuda_dev, A, Bw, off, B.EPI_SWIGLU, N // 2)
    ref = oracle.swiglu(oracle.grouped_gemm(A, Bw, off))
    check_stage(got, ref, "grouped GEMM swiglu")


@pytest.mark.parametrize("counts,K,N", GEMM_CASES)
def test_weight_scatter_epilogue(cuda_dev, counts, K, N):
    off, A, Bw = _rand_case(counts, K, N, 3)
    R = int(off[-1])
    rng = np.random.default_rng(4)
    perm = rng.permutation(R).astype(np.int32)
    w_sorted = rng.random(R).astype(np.float32)
    got = _run(cuda_dev, A, Bw, off, B.EPI_WEIGHT_SCATTER, N, w_sorted=w_sorted, perm=perm)
    G = oracle.grouped_gemm(A, Bw, off)
    ref = np.zeros_like(G)
    ref[perm] = w_sorted[:, None].astype(np.float64) * G
    assert got.dtype == torch.float32
    check_stage(got, ref, "grouped GEMM weight scatter", kind="fp32")


def test_bad_offsets_are_refused_on_device(cuda_dev):
    A = torch.randn(64, 64).to(torch.bfloat16)
    Bw = torch.randn(2, 64, 64).to(torch.bfloat16)
    off = np.array([0, 50, 70], np.int32)          # offsets[E] > R
    C = torch.full((64, 64), 7.0, dtype=torch.bfloat16, device=cuda_dev)
    ws = B.alloc_workspace(B.OP_GROUPED_GEMM, 64, 0, 0, 2, 1, cuda_dev)
    B.moe_grouped_gemm(A.to(cuda_dev), Bw.to(cuda_dev), torch.from_numpy(off).to(cuda_dev),
                       B.EPI_STORE, C, ws)
    assert B.moe_get_device_status(ws) == B.MOE_ERR_BAD_INDEX
    assert bool((C == 7.0).all())            # nothing written


def test_repeat_is_bitwise_deterministic(cuda_dev):
    off, A, Bw = _rand_case([300, 20, 900], 512, 512, 5)
    a = _run(cuda_dev, A, Bw, off, B.EPI_SWIGLU, 256)
    b = _run(cuda_dev, A, Bw, off, B.EPI_SWIGLU, 256)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    rng = np.random.default_rng(6)
    R = int(off[-1])
    perm, w_sorted = rng.permutation(R).astype(np.int32), rng.random(R).astype(np.float32)
    c = _run(cuda_dev, A, Bw, off, B.EPI_WEIGHT_SCATTER, 512, w_sorted=w_sorted, perm=perm)
    d = _run(cuda_dev, A, Bw, off, B.EPI_WEIGHT_SCATTER, 512, w_sorted=w_sorted, perm=perm)
    assert torch.equal(c.view(torch.int32), d.view(torch.int32))


@pytest.mark.parametrize("epi", [B.EPI_STORE, B.EPI_SWIGLU, B.EPI_WEIGHT_SCATTER])
def test_many_tiles_mixed_shapes(cuda_dev, epi):
    """More tiles than CTA pairs, experts whose last m-tile holds 1..128 rows (the
    pair kernel's M = 128 tiles), 129..255 rows (padded 256-row tiles) and whole
    tiles, so the tile queue hands out whole tiles first and N halves at the end;
    one-hot A rows make every output exact."""
    counts = [600, 129, 1000, 0, 1, 383, 255, 256, 128, 64]
    K, N = 64, 4096
    off = _offsets(counts)
    R, E = int(off[-1]), len(counts)
    sel = (3 * np.arange(R) + 1) % K
    A = torch.zeros(R, K)
    A[np.arange(R), sel] = 1
    A = A.to(torch.bfloat16)
    Bw = torch.randn(E, K, N, generator=torch.Generator().manual_seed(8)).to(torch.bfloat16)
    G = np.zeros((R, N), np.float64)
    for e in range(E):
        for s in range(off[e], off[e + 1]):
            G[s] = Bw[e, sel[s]].double().numpy()
    if epi == B.EPI_STORE:
        got = _run(cuda_dev, A, Bw, off, epi, N).double().numpy()
        assert np.array_equal(got, G), _explain(got, G)
    elif epi == B.EPI_SWIGLU:
        got = _run(cuda_dev, A, Bw, off, epi, N // 2)
        check_stage(got, oracle.swiglu(G), "swiglu, many tiles")
    else:
        rng = np.random.default_rng(9)
        perm = rng.permutation(R).astype(np.int32)
        w_sorted = np.exp2(rng.integers(-3, 3, R)).astype(np.float32)   # exact scaling
        got = _run(cuda_dev, A, Bw, off, epi, N, w_sorted=w_sorted, perm=perm).double().numpy()
        ref = np.zeros_like(G)
        ref[perm] = w_sorted[:, None].astype(np.float64) * G
        assert np.array_equal(got, ref), _explain(got, ref)


def test_workspace_reused_back_to_back(cuda_dev):
    """Consecutive launches on one workspace (the layer's GEMM1 then GEMM2 pattern):
    each launch leaves the tile queue in the control block at zero for the next, and
    the results equal those of launches on fresh workspaces bit for bit."""
    off, A, Bw = _rand_case([300, 20, 900, 5], 256, 512, 12)
    R, E = int(off[-1]), len(off) - 1
    ws = B.alloc_workspace(B.OP_GROUPED_GEMM, R, 0, 0, E, 1, cuda_dev)
    A_d, B_d, off_d = A.to(cuda_dev), Bw.to(cuda_dev), torch.from_numpy(off).to(cuda_dev)
    outs = []
    for epi, n_out in [(B.EPI_SWIGLU, 256), (B.EPI_STORE, 512), (B.EPI_SWIGLU, 256),
                       (B.EPI_STORE, 512)]:
        C = torch.zeros(R, n_out, dtype=torch.bfloat16, device=cuda_dev)
        B.moe_grouped_gemm(A_d, B_d, off_d, epi, C, ws)
        outs.append(C)
    torch.cuda.synchronize()
    assert int(ws[128:136].view(torch.int32).abs().sum().item()) == 0, "tile queue not reset"
    assert B.moe_get_device_status(ws) == B.MOE_OK
    fresh_swiglu = _run(cuda_dev, A, Bw, off, B.EPI_SWIGLU, 256)
    fresh_store = _run(cuda_dev, A, Bw, off, B.EPI_STORE, 512)
    for i, ref in enumerate([fresh_swiglu, fresh_store, fresh_swiglu, fresh_store]):
        assert torch.equal(outs[i].cpu().view(torch.int16), ref.view(torch.int16)), i
