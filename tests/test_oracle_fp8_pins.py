"""Pins of the oracle's FP8 (E4M3) pieces against things other than itself: the
E4M3 codes of torch.float8_e4m3fn (a library routine), brute-force nearest-value
search over the decoded grid, numpy matmul of the decoded operands, and the
quantisation error bound of the exact layer."""
import numpy as np
import pytest
import torch

import oracle
from helpers import layer_case


def _grid():
    codes = np.arange(256, dtype=np.uint8)
    vals = oracle.e4m3_decode(codes)
    return codes, vals


def test_decode_every_code_matches_torch():
    codes, vals = _grid()
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(np.isnan(vals), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(vals[ok], ref[ok])
    assert np.nanmax(vals) == 448.0 and np.nanmin(vals) == -448.0
    assert vals[1] == 2.0 ** -9 and vals[8] == 2.0 ** -6      # subnormal step, min normal


def test_encode_matches_torch_and_brute_force():
    rng = np.random.default_rng(0)
    v = (rng.standard_normal(30000) * np.exp(rng.uniform(-14, 7, 30000))).astype(np.float32)
    _, vals = _grid()
    fin = np.sort(np.unique(vals[~np.isnan(vals)]))
    mids = ((fin[1:] + fin[:-1]) / 2).astype(np.float32)        # every exact tie
    v = np.concatenate([v, mids, -mids, np.float32([0.0, -0.0, 447.9, 448.0, 463.9])])
    v = v[np.abs(v) < 464]
    got = oracle.e4m3_encode(v)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, ref)
    # brute force on a subsample: the decoded code is the nearest finite grid value;
    # at an exact tie between two grid values the chosen code has an even mantissa
    finite = np.sort(np.unique(vals[~np.isnan(vals)]))
    for x, c in zip(v[::37].astype(np.float64), got[::37]):
        d = np.abs(finite - x)
        near = finite[d == d.min()]
        dec = oracle.e4m3_decode(np.uint8(c))
        assert dec in near, (x, dec, near)
        if len(near) == 2 and near[0] != -near[1]:
            assert (int(c) & 1) == 0, (x, c)


def test_encode_saturates():
    big = np.float32([464.0, 480.0, 1e4, 3e38, -500.0])
    assert oracle.e4m3_encode(big).tolist() == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE]
    assert oracle.e4m3_encode(np.float32([np.nan]))[0] == 0x7F


def _torch_rows(a_bf16):
    af = a_bf16.float()
    amax = af.abs().amax(dim=1)
    sc = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    q = (af / sc[:, None]).to(torch.float8_e4m3fn).view(torch.uint8)
    return q.numpy(), sc.numpy()


def test_quantize_rows_matches_torch_and_bounds():
    g = torch.Generator().manual_seed(1)
    a = (torch.randn(37, 320, generator=g) * torch.rand(37, 1, generator=g) * 5).to(torch.bfloat16)
    a[3] = 0                                                    # all-zero row: scale 1, codes 0
    q, sc = oracle.quantize_rows_e4m3(a)
    rq, rsc = _torch_rows(a)
    assert np.array_equal(q, rq) and np.array_equal(sc, rsc)
    assert sc[3] == 1.0 and not q[3].any()
    dec = oracle.e4m3_decode(q) * sc[:, None].astype(np.float64)
    af = a.double().numpy()
    # the largest magnitude of every nonzero row lands on +-448
    for r in range(37):
        if r != 3:
            assert np.abs(oracle.e4m3_decode(q[r])).max() == 448.0
    # round trip within half a grid step (relative 2^-4 for normals)
    err = np.abs(dec - af)
    bound = np.maximum(np.abs(af) * 2.0 ** -4, sc[:, None] * 2.0 ** -10) * (1 + 1e-6)
    assert (err <= bound).all()


def test_quantize_cols_matches_torch():
    g = torch.Generator().manual_seed(2)
    B = (torch.randn(3, 96, 40, generator=g) / 10).to(torch.bfloat16)
    q, sc = oracle.quantize_cols_e4m3(B)
    for e in range(3):
        rq, rsc = _torch_rows(B[e].t().contiguous())
        assert np.array_equal(q[e], rq) and np.array_equal(sc[e], rsc)


def test_grouped_gemm_e4m3_matches_numpy():
    rng = np.random.default_rng(3)
    R, K, N, E = 50, 64, 24, 3
    offsets = np.array([0, 20, 20, 50], np.int32)
    Aq = rng.integers(0, 256, (R, K)).astype(np.uint8)
    Aq[(Aq & 0x7F) == 0x7F] = 0                                 # no NaN codes
    Bq = rng.integers(0, 256, (E, N, K)).astype(np.uint8)
    Bq[(Bq & 0x7F) == 0x7F] = 1
    sa = rng.uniform(0.5, 2, R).astype(np.float32)
    sb = rng.uniform(0.5, 2, (E, N)).astype(np.float32)
    got = oracle.grouped_gemm_e4m3(Aq, sa, Bq, sb, offsets)
    A = oracle.e4m3_decode(Aq)
    Bd = oracle.e4m3_decode(Bq)
    for e in range(E):
        s0, s1 = offsets[e], offsets[e + 1]
        ref = (A[s0:s1] @ Bd[e].T) * sa[s0:s1, None] * sb[e][None, :]
        np.testing.assert_allclose(got[s0:s1], ref, rtol=1e-12, atol=1e-12)


def test_fp8_layer_dense_special_case():
    """E = 1, topk = 1: the layer is h = bf16(silu(x W1g) * (x W1u)), quantised per
    row, times W2 quantised per column, computed here with torch's own conversions."""
    w, x, W1, W2, ids, tw = layer_case(40, 64, 128, 1, 1, "uniform", seed=4)
    tw = np.ones_like(tw)
    got = oracle.moe_ffn_fp8(x, W1, W2, ids, tw)
    F = W2.shape[1]
    g = x.double() @ W1[0].double()
    h = (torch.nn.functional.silu(g[:, :F]) * g[:, F:]).to(torch.bfloat16)
    hq, hs = _torch_rows(h)
    wq, ws = _torch_rows(W2[0].t().contiguous())
    hd = torch.from_numpy(hq).view(torch.float8_e4m3fn).double() * torch.from_numpy(hs).double()[:, None]
    wd = torch.from_numpy(wq).view(torch.float8_e4m3fn).double() * torch.from_numpy(ws).double()[:, None]
    ref = (hd @ wd.t()).numpy()
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert rel < 1e-6, rel


@pytest.mark.parametrize("M,E,topk", [(64, 4, 2), (33, 8, 3)])
def test_fp8_layer_within_e4m3_bound_of_exact_layer(M, E, topk):
    """FP8 error: each e4m3 value is within 2^-4 (relative) of what it encodes; over
    dot products of random signs the layer's relative Frobenius error stays well
    below 2^-4, and it is not zero (the quantisation is really applied)."""
    w, x, W1, W2, ids, tw = layer_case(M, 128, 192, E, topk, "skewed", seed=M + E)
    exact = oracle.moe_ffn(x, W1, W2, ids, tw)
    fp8 = oracle.moe_ffn_fp8(x, W1, W2, ids, tw)
    rel = np.linalg.norm(fp8 - exact) / np.linalg.norm(exact)
    assert 1e-4 < rel < 2.0 ** -4, rel
