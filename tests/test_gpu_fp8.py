"""GPU parity of the FP8 (E4M3) down projection with the oracle: the two quantisers
bit for bit (codes and scales), the FP8 grouped GEMM within the fp32 summation
bound, the FP8 layer against the oracle's FP8 layer (same bar as the bf16 layer)
and bit for bit against the chain of separate calls."""
import numpy as np
import pytest
import torch

import oracle
from grouped_gemm_plan_b200 import binding as B
from helpers import check_close, guarded_empty, layer_case

pytestmark = pytest.mark.gpu


def _codes(t):
    return t.cpu().numpy()


@pytest.mark.parametrize("E,K,N", [(3, 144, 96), (2, 1408, 320), (1, 64, 16)])
def test_quantize_weights_matches_oracle(cuda_dev, E, K, N):
    g = torch.Generator().manual_seed(E * K + N)
    W = (torch.randn(E, K, N, generator=g) * torch.rand(1, 1, N, generator=g) / 8).to(torch.bfloat16)
    W[0, :, 1] = 0                                               # an all-zero column
    Wq, check_q = guarded_empty((E, N, K), torch.uint8, cuda_dev)
    sc, check_s = guarded_empty((E, N), torch.float32, cuda_dev)
    B.moe_quantize_weights_e4m3(W.to(cuda_dev), Wq, sc)
    torch.cuda.synchronize()
    check_q()
    check_s()
    rq, rsc = oracle.quantize_cols_e4m3(W)
    assert np.array_equal(_codes(Wq), rq)
    assert np.array_equal(sc.cpu().numpy(), rsc)


@pytest.mark.parametrize("R,K", [(5, 64), (300, 1408), (64, 14336), (9, 32768), (130, 6400)])
def test_quantize_rows_matches_oracle(cuda_dev, R, K):
    g = torch.Generator().manual_seed(R + K)
    A = (torch.randn(R, K, generator=g) * torch.exp(torch.randn(R, 1, generator=g) * 3)).to(torch.bfloat16)
    A[R // 2] = 0
    Aq, check_q = guarded_empty((R, K), torch.uint8, cuda_dev)
    sc, check_s = guarded_empty((R,), torch.float32, cuda_dev)
    ws = B.alloc_workspace(B.OP_GROUPED_GEMM, R, K, K, 1, 1, cuda_dev)
    B.moe_quantize_rows_e4m3(A.to(cuda_dev), Aq, sc, ws)
    assert B.moe_get_device_status(ws) == B.MOE_OK
    check_q()
    check_s()
    rq, rsc = oracle.quantize_rows_e4m3(A)
    assert np.array_equal(_codes(Aq), rq)
    assert np.array_equal(sc.cpu().numpy(), rsc)


def _random_codes(rng, shape):
    c = rng.integers(0, 256, shape).astype(np.uint8)
    c[(c & 0x7F) == 0x7F] ^= 0x01                                # no NaN codes
    return c


@pytest.mark.parametrize("pair", ["0", "1"])
@pytest.mark.parametrize("counts,K,N,scatter", [([100, 0, 300, 29], 192, 576, True),
                                                 ([128, 256], 1408, 256, False),
                                                 ([1, 2, 3], 128, 64, True),
                                                 ([700, 513, 0, 256], 384, 320, True),
                                                 ([i % 4 for i in range(1024)], 128, 64, True)])
def test_grouped_gemm_e4m3_matches_oracle(cuda_dev, monkeypatch, pair, counts, K, N, scatter):
    """Both kernels (single CTA, CTA pair): ragged experts, an empty one, K not a
    multiple of the stage depth (zero-filled tail), a partial last column tile."""
    monkeypatch.setenv("MOE_GEMM_PAIR", pair)
    rng = np.random.default_rng(K + N)
    E = len(counts)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    R = int(offsets[-1])
    Aq = _random_codes(rng, (R, K))
    Bq = _random_codes(rng, (E, N, K))
    sa = rng.uniform(1e-3, 1e-2, R).astype(np.float32)
    sb = rng.uniform(1e-3, 1e-2, (E, N)).astype(np.float32)
    perm = rng.permutation(R).astype(np.int32) if scatter else None
    w = rng.uniform(0.1, 1, R).astype(np.float32) if scatter else None
    d = lambda a: torch.from_numpy(a).to(cuda_dev) if a is not None else None
    C, check_c = guarded_empty((R, N), torch.float32, cuda_dev, fill=0x7F)
    ws = B.alloc_workspace(B.OP_GROUPED_GEMM, R, N, K, E, 1, cuda_dev)
    B.moe_grouped_gemm_e4m3(d(Aq), d(sa), d(Bq), d(sb), d(offsets), C, ws, w_sorted=d(w), perm=d(perm))
    assert B.moe_get_device_status(ws) == B.MOE_OK
    check_c()
    ref = oracle.grouped_gemm_e4m3(Aq, sa, Bq, sb, offsets)
    absref = oracle.grouped_gemm_e4m3(np.where(Aq & 0x80, Aq ^ 0x80, Aq).astype(np.uint8), sa,
                                      np.where(Bq & 0x80, Bq ^ 0x80, Bq).astype(np.uint8), sb, offsets)
    if scatter:
        ref = ref * w[:, None]
        absref = absref * w[:, None]
        out = np.empty_like(ref)
        out[perm] = ref
        ref = out
        out = np.empty_like(absref)
        out[perm] = absref
        absref = out
    got = C.cpu().numpy().astype(np.float64)
    # fp32 products of E4M3 values are exact; K-term fp32 sums and three fp32
    # scalings are within (K + 3) * 2^-24 of the sum of magnitudes
    bound = (K + 3) * 2.0 ** -24 * absref + 1e-30
    assert np.isfinite(got).all()
    assert (np.abs(got - ref) <= bound).all(), np.max(np.abs(got - ref) / (bound + 1e-30))


def _fp8_inputs(dev, W2):
    E, F, H = W2.shape
    W2q = torch.empty(E, H, F, dtype=torch.uint8, device=dev)
    w2s = torch.empty(E, H, dtype=torch.float32, device=dev)
    B.moe_quantize_weights_e4m3(W2.to(dev), W2q, w2s)
    return W2q, w2s


def _run_fp8(dev, x, W1, W2q, w2s, ids, tw):
    M, H = x.shape
    E, _, F2 = W1.shape
    topk = ids.shape[1]
    R = M * topk
    out = torch.full((M, H), float("nan"), dtype=torch.bfloat16, device=dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(max(R, 1), dtype=torch.int32, device=dev)
    ws = B.alloc_workspace(B.OP_FFN_FP8, M, H, F2 // 2, E, topk, dev)
    B.moe_ffn_fused_fp8(x.to(dev), W1.to(dev), W2q, w2s, torch.from_numpy(ids).to(dev),
                        torch.from_numpy(tw).to(dev), out, counts, offsets, perm, ws)
    assert B.moe_get_device_status(ws) == B.MOE_OK
    return out


def _gpu_h(dev, x, W1, offsets, perm, topk):
    """The GPU's bf16 h (dispatch + GEMM1 with the SwiGLU epilogue), on the CPU."""
    R = perm.shape[0]
    H = x.shape[1]
    F = W1.shape[2] // 2
    ws = B.alloc_workspace(B.OP_GROUPED_GEMM, R, 2 * F, H, W1.shape[0], 1, dev)
    xp = torch.empty(R, H, dtype=torch.bfloat16, device=dev)
    pd = torch.from_numpy(perm).to(dev)
    B.moe_dispatch(x.to(dev), pd, topk, xp, ws)
    h = torch.empty(R, F, dtype=torch.bfloat16, device=dev)
    B.moe_grouped_gemm(xp, W1.to(dev), torch.from_numpy(offsets).to(dev), B.EPI_SWIGLU, h, ws)
    assert B.moe_get_device_status(ws) == B.MOE_OK
    return h.cpu()


@pytest.mark.parametrize("M,H,F,E,topk,kind,pair", [(64, 128, 192, 4, 2, "skewed", "0"),
                                                     (300, 256, 384, 8, 2, "uniform", "0"),
                                                     (200, 512, 1408, 16, 4, "skewed", "0"),
                                                     (1, 64, 128, 2, 1, "uniform", "0"),
                                                     (300, 256, 384, 8, 2, "uniform", "1"),
                                                     (700, 256, 640, 2, 2, "skewed", "1")])
def test_fp8_layer_matches_oracle(cuda_dev, monkeypatch, M, H, F, E, topk, kind, pair):
    """Element by element against the oracle's FP8 stages applied to the GPU's own
    h (the rounding of h to bf16 decides E4M3 codes, so a one-ulp difference in h
    between fp32 and fp64 accumulation can move a code by a whole E4M3 step); end
    to end against the oracle's FP8 layer from x by the relative Frobenius bar; and
    within the E4M3 error bound of the exact layer."""
    monkeypatch.setenv("MOE_GEMM_PAIR", pair)
    w, x, W1, W2, ids, tw = layer_case(M, H, F, E, topk, kind, seed=M + F)
    W2q, w2s = _fp8_inputs(cuda_dev, W2)
    out = _run_fp8(cuda_dev, x, W1, W2q, w2s, ids, tw)
    counts, offsets, perm, inv, _ = oracle.plan(ids, tw, E)
    h = _gpu_h(cuda_dev, x, W1, offsets, perm, topk)
    hq, hs = oracle.quantize_rows_e4m3(h)
    wq, wsc = oracle.quantize_cols_e4m3(W2)
    y = oracle.grouped_gemm_e4m3(hq, hs, wq, wsc, offsets)
    ref_given_h = oracle.combine(y, inv, tw)
    check_close(out, ref_given_h, "FP8 layer (oracle stages on the GPU's h)")
    ref = oracle.moe_ffn_fp8(x, W1, W2, ids, tw)
    o = out.float().cpu().double().numpy()
    assert np.linalg.norm(o - ref) / np.linalg.norm(ref) < 1e-2
    exact = oracle.moe_ffn(x, W1, W2, ids, tw)
    assert np.linalg.norm(o - exact) / np.linalg.norm(exact) < 2.0 ** -4


def test_fp8_layer_equals_chain_of_calls(cuda_dev):
    """moe_ffn_fused_fp8 == plan, dispatch, GEMM1+SwiGLU, quantise rows, FP8 GEMM2
    with the weight scatter, combine -- every call separate -- bit for bit."""
    dev = cuda_dev
    M, H, F, E, topk = 333, 256, 640, 8, 3
    w, x, W1, W2, ids, tw = layer_case(M, H, F, E, topk, "skewed", seed=9)
    W2q, w2s = _fp8_inputs(dev, W2)
    fused = _run_fp8(dev, x, W1, W2q, w2s, ids, tw)
    R = M * topk
    xd, W1d = x.to(dev), W1.to(dev)
    idd, twd = torch.from_numpy(ids).to(dev), torch.from_numpy(tw).to(dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(R, dtype=torch.int32, device=dev)
    inv = torch.empty(R, dtype=torch.int32, device=dev)
    ws_ = torch.empty(R, dtype=torch.float32, device=dev)
    ws = B.alloc_workspace(B.OP_PLAN, M, H, F, E, topk, dev)
    B.moe_plan(idd, twd, E, counts, offsets, perm, inv, ws_, ws)
    xp = torch.empty(R, H, dtype=torch.bfloat16, device=dev)
    B.moe_dispatch(xd, perm, topk, xp, ws)
    h = torch.empty(R, F, dtype=torch.bfloat16, device=dev)
    B.moe_grouped_gemm(xp, W1d, offsets, B.EPI_SWIGLU, h, ws)
    hq = torch.empty(R, F, dtype=torch.uint8, device=dev)
    hs = torch.empty(R, dtype=torch.float32, device=dev)
    B.moe_quantize_rows_e4m3(h, hq, hs, ws)
    yk = torch.empty(R, H, dtype=torch.float32, device=dev)
    B.moe_grouped_gemm_e4m3(hq, hs, W2q, w2s, offsets, yk, ws, w_sorted=ws_, perm=perm)
    out = torch.empty(M, H, dtype=torch.bfloat16, device=dev)
    B.moe_combine(yk, None, None, M, topk, out, ws)
    assert B.moe_get_device_status(ws) == B.MOE_OK
    assert torch.equal(out.view(torch.int16), fused.view(torch.int16))
    # the quantised h of the chain is the oracle's quantisation of the GPU's h
    rq, rsc = oracle.quantize_rows_e4m3(h.cpu())
    assert np.array_equal(hq.cpu().numpy(), rq) and np.array_equal(hs.cpu().numpy(), rsc)


@pytest.mark.parametrize("name", ["mixtral", "phi35", "qwen2", "wide512", "wide2048"])
def test_fp8_layer_full_size_sampled(cuda_dev, name):
    """The FP8 layer at full size, in the launch configuration the benchmark times
    (CTA-pair kernels on the Mixtral and Phi-3.5 shapes): the weight quantiser bit
    for bit over all of W2, and sampled tokens against the oracle's FP8 stages on
    the GPU's own h (E4M3 decode table, fp64 dot products)."""
    from grouped_gemm_plan_b200 import workload as wl
    w = wl.WORKLOADS[name]
    dev = cuda_dev
    x = wl.make_x(w)
    W1 = torch.empty((w.E, w.H, 2 * w.F), dtype=torch.bfloat16, device=dev)
    W2 = torch.empty((w.E, w.F, w.H), dtype=torch.bfloat16, device=dev)
    wl.make_weights(w, W1, W2)
    ids, tw = wl.make_routing(w)
    W2q, w2s = _fp8_inputs(dev, W2)
    rq, rs = oracle.quantize_cols_e4m3(W2.cpu())
    assert np.array_equal(W2q.cpu().numpy(), rq) and np.array_equal(w2s.cpu().numpy(), rs)
    out = _run_fp8(dev, x, W1, W2q, w2s, ids, tw)
    counts, offsets, perm, inv, _ = oracle.plan(ids, tw, w.E)
    h = _gpu_h(dev, x, W1, offsets, perm, w.topk)
    rng = np.random.default_rng(w.seed)
    tokens = np.unique(np.concatenate([[0, w.M - 1], rng.choice(w.M, 10, replace=False)]))
    lut = oracle.e4m3_decode(np.arange(256, dtype=np.uint8))
    pairs = [(j, int(t), k) for j, t in enumerate(tokens) for k in range(w.topk)]
    y = {}
    for e in sorted({int(ids[t, k]) for _, t, k in pairs}):
        dec_w = lut[rq[e]]                                   # [H, F], decoded once per expert
        for j, t, k in pairs:
            if int(ids[t, k]) != e:
                continue
            s = int(inv[t * w.topk + k])
            hq, hs = oracle.quantize_rows_e4m3(h[s:s + 1])
            y[(j, k)] = (dec_w @ lut[hq[0]]) * float(hs[0]) * rs[e].astype(np.float64)
        del dec_w
    ref = np.zeros((len(tokens), w.H))
    for j, t, k in pairs:                                    # k ascending, as the combine
        ref[j] += float(tw[t, k]) * y[(j, k)]
    check_close(out.cpu()[torch.from_numpy(tokens)], ref, f"{name} FP8 sampled rows")
