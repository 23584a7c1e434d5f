"""GPU parity of the block-scaled (MX) E4M3 down projection with the oracle: both
quantisers bit for bit (codes and scale codes), the MX grouped GEMM within the
fp32 summation bound, the SwiGLU epilogue's in-register quantisation against
the oracle's quantiser applied to the exact h, and the MX layer element by element
against the oracle's MX stages on the GPU's quantised h (the bf16 layer's bar),
against the oracle's MX layer from x by relative Frobenius, and bit for bit against
the chain of separate calls (which reaches the scale layout of the fused layer by
another route)."""
import numpy as np
import pytest
import torch

import oracle
from grouped_gemm_plan_b200 import binding as B
from helpers import check_close, guarded_empty, layer_case

pytestmark = pytest.mark.gpu


def _np(t):
    return t.cpu().numpy()


def _bf16_cases(shape, seed, spread=3.0):
    g = torch.Generator().manual_seed(seed)
    a = torch.randn(*shape, generator=g)
    scale = torch.exp(torch.randn(*shape[:-1], 1, generator=g) * spread)
    return (a * scale).to(torch.bfloat16)


@pytest.mark.parametrize("E,K,N", [(3, 96, 80), (2, 1408, 320), (1, 32, 16)])
def test_quantize_weights_mx_matches_oracle(cuda_dev, E, K, N):
    W = _bf16_cases((E, K, N), E * K + N)
    W[0, :32, 1] = 0                                   # an all-zero block
    W[0, :32, 2] = 448.0                               # a block at exactly the format's max
    W[-1, :, -1] = 1e-40                               # blocks of fp32-subnormal values
    BqT, check_q = guarded_empty((E, N, K), torch.uint8, cuda_dev)
    sf, check_s = guarded_empty((E, N, K // 32), torch.uint8, cuda_dev)
    B.moe_quantize_weights_mx(W.to(cuda_dev), BqT, sf)
    torch.cuda.synchronize()
    check_q()
    check_s()
    rq, rsf = oracle.mx_quantize_cols(W)
    assert np.array_equal(_np(sf), rsf)
    assert np.array_equal(_np(BqT), rq)


@pytest.mark.parametrize("R,K", [(5, 32), (300, 1408), (64, 6400), (1, 14336)])
def test_quantize_rows_mx_matches_oracle(cuda_dev, R, K):
    A = _bf16_cases((R, K), R + K)
    A[R // 2, :64] = 0
    Aq, check_q = guarded_empty((R, K), torch.uint8, cuda_dev)
    sf, check_s = guarded_empty((R, K // 32), torch.uint8, cuda_dev)
    B.moe_quantize_rows_mx(A.to(cuda_dev), Aq, sf)
    torch.cuda.synchronize()
    check_q()
    check_s()
    rq, rsf = oracle.mx_quantize_rows(A)
    assert np.array_equal(_np(sf), rsf)
    assert np.array_equal(_np(Aq), rq)


def _random_codes(rng, shape):
    c = rng.integers(0, 256, shape).astype(np.uint8)
    c[(c & 0x7F) == 0x7F] ^= 0x01                      # no NaN codes
    return c


def _abs_codes(c):
    return np.where(c & 0x80, c ^ 0x80, c).astype(np.uint8)


@pytest.mark.parametrize("counts,K,N,scatter", [([100, 0, 300, 29], 192, 576, True),
                                                 ([256, 512], 1408, 256, False),
                                                 ([1, 2, 3], 128, 64, True),
                                                 ([700, 513, 0, 256], 384, 320, True),
                                                 ([5, 600], 96, 128, True),
                                                 ([i % 4 for i in range(1024)], 128, 64, True)])
def test_grouped_gemm_mx_matches_oracle(cuda_dev, counts, K, N, scatter):
    """Ragged experts (an empty one, tails of 1..255 rows), K not a multiple of the
    256-deep stage (K = 96: three MMAs in the only stage), N an odd multiple of 64
    (a half-used last column tile), and 1024 experts."""
    rng = np.random.default_rng(K + N + len(counts))
    E = len(counts)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    R = int(offsets[-1])
    Aq = _random_codes(rng, (R, K))
    Bq = _random_codes(rng, (E, N, K))
    a_sf = rng.integers(120, 135, (R, K // 32)).astype(np.uint8)
    b_sf = rng.integers(118, 133, (E, N, K // 32)).astype(np.uint8)
    perm = rng.permutation(R).astype(np.int32) if scatter else None
    w = rng.uniform(0.1, 1, R).astype(np.float32) if scatter else None
    d = lambda a: torch.from_numpy(a).to(cuda_dev) if a is not None else None
    C, check_c = guarded_empty((R, N), torch.float32, cuda_dev, fill=0x7F)
    ws = B.alloc_workspace(B.OP_GEMM_MX, R, N, K, E, 1, cuda_dev)
    B.moe_grouped_gemm_mx(d(Aq), d(a_sf), d(Bq), d(b_sf), d(offsets), C, ws, w_sorted=d(w),
                          perm=d(perm))
    assert B.moe_get_device_status(ws) == B.MOE_OK
    check_c()
    ref = oracle.grouped_gemm_mx(Aq, a_sf, Bq, b_sf, offsets)
    absref = oracle.grouped_gemm_mx(_abs_codes(Aq), a_sf, _abs_codes(Bq), b_sf, offsets)
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
    # block products of E4M3 values times powers of two are exact in fp32; the
    # K-term fp32 sum and the gate-weight scaling are within (K + 2) * 2^-24 of the
    # sum of magnitudes
    bound = (K + 2) * 2.0 ** -24 * absref + 1e-30
    assert np.isfinite(got).all()
    excess = np.abs(got - ref) / (bound + 1e-30)
    assert (np.abs(got - ref) <= bound).all(), (excess.max(), np.unravel_index(excess.argmax(), excess.shape))


def test_grouped_gemm_mx_bad_offsets(cuda_dev):
    R, K, N, E = 64, 64, 64, 2
    d = cuda_dev
    offsets = torch.tensor([0, 40, 80], dtype=torch.int32, device=d)   # past R
    ws = B.alloc_workspace(B.OP_GEMM_MX, R, N, K, E, 1, d)
    C = torch.zeros(R, N, dtype=torch.float32, device=d)
    B.moe_grouped_gemm_mx(torch.zeros(R, K, dtype=torch.uint8, device=d),
                          torch.full((R, K // 32), 127, dtype=torch.uint8, device=d),
                          torch.zeros(E, N, K, dtype=torch.uint8, device=d),
                          torch.full((E, N, K // 32), 127, dtype=torch.uint8, device=d), offsets, C, ws)
    assert B.moe_get_device_status(ws) == B.MOE_ERR_BAD_INDEX


def _e4m3_value(codes):
    return oracle.e4m3_decode(codes)


def _near_boundary(amax, rel=1e-5):
    """amax within `rel` of 448 * 2^k for some k (where fp32 and fp64 h may pick
    different exponents)."""
    with np.errstate(divide="ignore"):
        k = np.round(np.log2(np.maximum(amax, 1e-300) / 448.0))
    return np.abs(amax / (448.0 * np.exp2(k)) - 1.0) <= rel


@pytest.mark.parametrize("counts,K,F", [([300, 0, 129, 64], 256, 384),
                                         ([1000, 17], 512, 1408),
                                         ([128, 256, 5], 128, 192),
                                         ([40] * 24, 256, 128)])
def test_swiglu_mx_epilogue_matches_oracle(cuda_dev, counts, K, F):
    """GEMM1 + SwiGLU with h quantised in the epilogue (whole tiles, 128-row tails,
    N halves of the last wave, F an odd multiple of 64) against the oracle's MX
    quantiser applied to the exact (fp64) h.  The GPU computes h in fp32, so a
    scale code may differ where the block maximum sits within 1e-5 of a 448 * 2^k
    boundary and a code by one E4M3 step where h sits at a rounding midpoint; both
    are counted and bounded, and every decoded value is held to the format's
    error bound."""
    rng = np.random.default_rng(K + F)
    E = len(counts)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    R = int(offsets[-1])
    A = torch.from_numpy(rng.standard_normal((R, K)).astype(np.float32)).to(torch.bfloat16)
    W1 = torch.from_numpy((rng.standard_normal((E, K, 2 * F)) / np.sqrt(K)).astype(np.float32)).to(
        torch.bfloat16)
    d = cuda_dev
    hq, check_q = guarded_empty((R, F), torch.uint8, d)
    hsf, check_s = guarded_empty((R, F // 32), torch.uint8, d)
    ws = B.alloc_workspace(B.OP_GROUPED_GEMM, R, 2 * F, K, E, 1, d)
    B.moe_grouped_gemm_swiglu_mx(A.to(d), W1.to(d), torch.from_numpy(offsets).to(d), hq, hsf, ws)
    assert B.moe_get_device_status(ws) == B.MOE_OK
    check_q()
    check_s()
    h = oracle.swiglu(oracle.grouped_gemm(A, W1, offsets))
    rq, rsf = oracle.mx_quantize_rows(h)
    gq, gsf = _np(hq), _np(hsf)
    amax = np.abs(h).reshape(R, F // 32, 32).max(axis=2)
    sf_diff = gsf != rsf
    assert not np.any(sf_diff & ~_near_boundary(amax)), int((sf_diff & ~_near_boundary(amax)).sum())
    assert sf_diff.sum() <= max(2, 1e-3 * sf_diff.size)
    # decoded values within half an E4M3 step (2^-4 relative; 2^(e-10) absolute in
    # the subnormal range) plus the fp32 error of h
    e = gsf.astype(np.int64) - 127
    scale = np.repeat(np.exp2(e.astype(np.float64)), 32, axis=1)
    deq = _e4m3_value(gq) * scale
    err = np.abs(deq - h)
    bound = 2.0 ** -4 * np.abs(h) + 2.0 ** -10 * scale + 1e-5 * np.abs(h) + 1e-30
    assert (err <= bound).all(), float((err / bound).max())
    same_blocks = np.repeat(~sf_diff, 32, axis=1)
    code_diff = (gq != rq) & same_blocks
    assert code_diff.sum() <= max(4, 1e-3 * code_diff.size), int(code_diff.sum())
    # every differing code is a neighbour: one E4M3 step apart in value
    if code_diff.any():
        gv = _e4m3_value(gq[code_diff])
        rv = _e4m3_value(rq[code_diff])
        assert np.all(np.sign(gv) * np.sign(rv) >= 0)
        step = np.maximum(np.exp2(np.floor(np.log2(np.maximum(np.abs(rv), 2.0 ** -6))) - 3), 2.0 ** -9)
        assert np.all(np.abs(gv - rv) <= step * 1.0000001)


def _mx_weights(dev, W2):
    E, F, H = W2.shape
    W2q = torch.empty(E, H, F, dtype=torch.uint8, device=dev)
    w2sf = torch.empty(E, H, F // 32, dtype=torch.uint8, device=dev)
    B.moe_quantize_weights_mx(W2.to(dev), W2q, w2sf)
    return W2q, w2sf


def _gpu_hq(dev, x, W1, offsets, perm, topk):
    """The GPU's quantised h (dispatch + GEMM1 with the MX SwiGLU epilogue, the
    kernel of the layer), codes and scale codes on the CPU."""
    R = perm.shape[0]
    H = x.shape[1]
    F = W1.shape[2] // 2
    ws = B.alloc_workspace(B.OP_GROUPED_GEMM, R, 2 * F, H, W1.shape[0], 1, dev)
    xp = torch.empty(R, H, dtype=torch.bfloat16, device=dev)
    B.moe_dispatch(x.to(dev), torch.from_numpy(perm).to(dev), topk, xp, ws)
    hq = torch.empty(R, F, dtype=torch.uint8, device=dev)
    hsf = torch.empty(R, F // 32, dtype=torch.uint8, device=dev)
    B.moe_grouped_gemm_swiglu_mx(xp, W1 if W1.is_cuda else W1.to(dev), torch.from_numpy(offsets).to(dev),
                                 hq, hsf, ws)
    assert B.moe_get_device_status(ws) == B.MOE_OK
    return hq.cpu().numpy(), hsf.cpu().numpy()


def _run_mx(dev, x, W1, W2q, w2sf, ids, tw):
    M, H = x.shape
    E, _, F2 = W1.shape
    topk = ids.shape[1]
    R = M * topk
    out, check = guarded_empty((M, H), torch.bfloat16, dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(max(R, 1), dtype=torch.int32, device=dev)
    ws = B.alloc_workspace(B.OP_FFN_MX, M, H, F2 // 2, E, topk, dev)
    B.moe_ffn_fused_mx(x.to(dev), W1.to(dev), W2q, w2sf, torch.from_numpy(ids).to(dev),
                       torch.from_numpy(tw).to(dev), out, counts, offsets, perm, ws)
    assert B.moe_get_device_status(ws) == B.MOE_OK
    check()
    return out


@pytest.mark.parametrize("M,H,F,E,topk,kind", [(64, 128, 192, 4, 2, "skewed"),
                                                (300, 256, 384, 8, 2, "uniform"),
                                                (200, 512, 1408, 16, 4, "skewed"),
                                                (1, 64, 128, 2, 1, "uniform"),
                                                (700, 256, 640, 2, 2, "skewed"),
                                                (513, 256, 128, 1, 1, "uniform")])
def test_mx_layer_matches_oracle(cuda_dev, M, H, F, E, topk, kind):
    """Element by element against the oracle's MX stages applied to the GPU's own
    quantised h (an E4M3 code is an integer decided by h, which the GPU computes in
    fp32 and the oracle in fp64: a code at a rounding midpoint can differ by one
    step, so the decision is taken on the GPU's side, as the kernel takes it); end
    to end against the oracle's MX layer from x by relative Frobenius <= 1e-2; and
    within the E4M3 error bound of the exact layer."""
    w, x, W1, W2, ids, tw = layer_case(M, H, F, E, topk, kind, seed=M + F)
    W2q, w2sf = _mx_weights(cuda_dev, W2)
    out = _run_mx(cuda_dev, x, W1, W2q, w2sf, ids, tw)
    counts, offsets, perm, inv, _ = oracle.plan(ids, tw, E)
    hq, hsf = _gpu_hq(cuda_dev, x, W1, offsets, perm, topk)
    rq, rsf = oracle.mx_quantize_cols(W2)
    ref_given_h = oracle.combine(oracle.grouped_gemm_mx(hq, hsf, rq, rsf, offsets), inv, tw)
    check_close(out, ref_given_h, "MX layer (oracle stages on the GPU's quantised h)")
    o = out.float().cpu().double().numpy()
    ref = oracle.moe_ffn_mx(x, W1, W2, ids, tw)
    assert np.linalg.norm(o - ref) / np.linalg.norm(ref) < 1e-2
    exact = oracle.moe_ffn(x, W1, W2, ids, tw)
    assert np.linalg.norm(o - exact) / np.linalg.norm(exact) < 2.0 ** -4


def test_mx_layer_equals_chain_of_calls(cuda_dev):
    """moe_ffn_fused_mx (h's scales written by GEMM1 straight into the GEMM2 layout)
    == plan, dispatch, GEMM1 + SwiGLU + MX (row-major scales), MX GEMM2 (which
    rearranges the row-major scales itself) with the weight scatter, combine --
    bit for bit."""
    dev = cuda_dev
    M, H, F, E, topk = 333, 256, 640, 8, 3
    w, x, W1, W2, ids, tw = layer_case(M, H, F, E, topk, "skewed", seed=9)
    W2q, w2sf = _mx_weights(dev, W2)
    fused = _run_mx(dev, x, W1, W2q, w2sf, ids, tw)
    R = M * topk
    xd, W1d = x.to(dev), W1.to(dev)
    idd, twd = torch.from_numpy(ids).to(dev), torch.from_numpy(tw).to(dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(R, dtype=torch.int32, device=dev)
    inv = torch.empty(R, dtype=torch.int32, device=dev)
    w_sorted = torch.empty(R, dtype=torch.float32, device=dev)
    ws = B.alloc_workspace(B.OP_PLAN, M, H, F, E, topk, dev)
    B.moe_plan(idd, twd, E, counts, offsets, perm, inv, w_sorted, ws)
    xp = torch.empty(R, H, dtype=torch.bfloat16, device=dev)
    B.moe_dispatch(xd, perm, topk, xp, ws)
    hq = torch.empty(R, F, dtype=torch.uint8, device=dev)
    hsf = torch.empty(R, F // 32, dtype=torch.uint8, device=dev)
    B.moe_grouped_gemm_swiglu_mx(xp, W1d, offsets, hq, hsf, ws)
    yk = torch.empty(R, H, dtype=torch.float32, device=dev)
    wsg = B.alloc_workspace(B.OP_GEMM_MX, R, H, F, E, 1, dev)
    B.moe_grouped_gemm_mx(hq, hsf, W2q, w2sf, offsets, yk, wsg, w_sorted=w_sorted, perm=perm)
    out = torch.empty(M, H, dtype=torch.bfloat16, device=dev)
    B.moe_combine(yk, None, None, M, topk, out, ws)   # rows already weighted, in token order
    assert B.moe_get_device_status(ws) == B.MOE_OK
    assert B.moe_get_device_status(wsg) == B.MOE_OK
    assert torch.equal(fused.view(torch.int16), out.view(torch.int16))


def test_mx_layer_empty_batch(cuda_dev):
    x = torch.zeros(0, 128, dtype=torch.bfloat16)
    w, _, W1, W2, _, _ = layer_case(8, 128, 128, 4, 2, "uniform", seed=1)
    W2q, w2sf = _mx_weights(cuda_dev, W2)
    ids = np.zeros((0, 2), np.int32)
    tw = np.zeros((0, 2), np.float32)
    out = _run_mx(cuda_dev, x, W1, W2q, w2sf, ids, tw)
    assert out.shape == (0, 128)


@pytest.mark.parametrize("name", ["mixtral", "phi35", "qwen2", "wide2048"])
def test_mx_layer_full_size_sampled(cuda_dev, name):
    """The MX layer at full size, in the launch configuration the benchmark times:
    the weight quantiser bit for bit over all of W2; sampled tokens (every expert's
    first and last slot, both sides of the heaviest and lightest experts' m-tile
    boundaries, random ones) element by element against the oracle's MX stages on
    the GPU's quantised h, and by relative Frobenius against the oracle's MX stages
    from x (the fp64 h there can move a code at a rounding midpoint by one step)."""
    from grouped_gemm_plan_b200 import workload as wl
    from test_gpu_layer import _sample_tokens
    w = wl.WORKLOADS[name]
    dev = cuda_dev
    x = wl.make_x(w)
    W1 = torch.empty((w.E, w.H, 2 * w.F), dtype=torch.bfloat16, device=dev)
    W2 = torch.empty((w.E, w.F, w.H), dtype=torch.bfloat16, device=dev)
    wl.make_weights(w, W1, W2)
    ids, tw = wl.make_routing(w)
    W2q, w2sf = _mx_weights(dev, W2)
    rq, rsf = oracle.mx_quantize_cols(W2.cpu())
    assert np.array_equal(w2sf.cpu().numpy(), rsf) and np.array_equal(W2q.cpu().numpy(), rq)
    out = _run_mx(dev, x, W1, W2q, w2sf, ids, tw)
    counts, offsets, perm, inv, _ = oracle.plan(ids, tw, w.E)
    tokens = _sample_tokens(ids, perm, offsets, 64, w.seed)
    # the sampled (token, k) rows grouped by expert, through the oracle's stages
    rows = sorted(((int(ids[t, k]), int(t), k) for t in tokens for k in range(w.topk)))
    sub_counts = np.bincount([e for e, _, _ in rows], minlength=w.E)
    sub_off = np.concatenate([[0], np.cumsum(sub_counts)]).astype(np.int32)
    pos = {t: j for j, t in enumerate(tokens)}

    def combine_rows(y):
        ref = np.zeros((len(tokens), w.H))
        for (e, t, k), yr in sorted(zip(rows, y), key=lambda r: (r[0][1], r[0][2])):   # k ascending
            ref[pos[t]] += float(tw[t, k]) * yr
        return ref
    got = out.cpu()[torch.from_numpy(tokens)]
    # the GPU's quantised h of the sampled rows
    ghq, ghsf = _gpu_hq(dev, x, W1, offsets, perm, w.topk)
    slots = np.array([int(inv[t * w.topk + k]) for _, t, k in rows], np.int64)
    y = oracle.grouped_gemm_mx(ghq[slots], ghsf[slots], rq, rsf, sub_off)
    check_close(got, combine_rows(y), f"{name} MX sampled rows (oracle stages on the GPU's h)")
    # from x, h quantised by the oracle
    xs = x[torch.tensor([t for _, t, _ in rows])]
    h = oracle.swiglu(oracle.grouped_gemm(xs, W1.cpu(), sub_off))
    hq, hsf = oracle.mx_quantize_rows(h)
    ref = combine_rows(oracle.grouped_gemm_mx(hq, hsf, rq, rsf, sub_off))
    g = got.double().numpy()
    assert np.linalg.norm(g - ref) / np.linalg.norm(ref) < 1e-2


def test_mx_layer_bad_expert_id(cuda_dev):
    """An expert id out of range: the plan records MOE_ERR_BAD_EXPERT_ID and writes
    zero counts; the GEMMs then have no rows and the call completes."""
    w, x, W1, W2, ids, tw = layer_case(100, 128, 128, 4, 2, "uniform", seed=1)
    ids = ids.copy()
    ids[17, 0] = 4
    dev = cuda_dev
    W2q, w2sf = _mx_weights(dev, W2)
    M, H = x.shape
    out = torch.empty(M, H, dtype=torch.bfloat16, device=dev)
    counts = torch.empty(4, dtype=torch.int32, device=dev)
    offsets = torch.empty(5, dtype=torch.int32, device=dev)
    perm = torch.empty(200, dtype=torch.int32, device=dev)
    ws = B.alloc_workspace(B.OP_FFN_MX, M, H, 128, 4, 2, dev)
    B.moe_ffn_fused_mx(x.to(dev), W1.to(dev), W2q, w2sf, torch.from_numpy(ids).to(dev),
                       torch.from_numpy(tw).to(dev), out, counts, offsets, perm, ws)
    assert B.moe_get_device_status(ws) == B.MOE_ERR_BAD_EXPERT_ID
    assert counts.cpu().tolist() == [0] * 4
