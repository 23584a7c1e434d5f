"""Pins of the oracle's block-scaled (MX) E4M3 down projection.

The scheme (a reading: the PTO MegaMoE article, section "MegaMoE 融合算子七阶段",
only says that SwiGLU quantises what it consumes): blocks of 32 consecutive values
along the contraction dimension share a power-of-two scale 2^e, e the smallest
integer with amax <= 448 * 2^e, stored as the E8M0 code e + 127; elements are the
nearest E4M3 to v * 2^-e.  Each pin checks the oracle against something other than
itself: a brute-force search, torch's own E4M3 conversion, numpy block sums, or
the error bound of the format against the exact layer.
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import layer_case


def test_exponent_is_the_smallest_that_fits():
    rng = np.random.default_rng(0)
    vals = list(np.abs(rng.standard_normal(500)) * np.exp2(rng.integers(-30, 30, 500)))
    # the boundaries 448 * 2^k, just above and below, powers of two, 0, tiny and huge
    for k in range(-20, 21):
        b = 448.0 * 2.0 ** k
        vals += [b, np.nextafter(b, 0), np.nextafter(b, np.inf), 2.0 ** k]
    vals += [0.0, 1e-45, 3e38, 2.0 ** -140]
    for a in vals:
        e = oracle.mx_exponent(a)
        brute = next(x for x in range(-127, 128) if a <= 448.0 * 2.0 ** x) if a <= 448.0 * 2.0 ** 127 \
            else 127
        if a == 0.0:
            brute = -127
        assert e == brute, (a, e, brute)


def _e4m3_torch(v32: np.ndarray) -> np.ndarray:
    return torch.from_numpy(v32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_row_quantiser_matches_torch_e4m3():
    # bf16 inputs: v * 2^-e is exact in fp32, so torch's fp32 -> e4m3 conversion
    # (one rounding, nearest even) is an independent reference for the codes
    rng = np.random.default_rng(1)
    A = torch.from_numpy((rng.standard_normal((37, 256)) *
                          np.exp2(rng.integers(-12, 12, (37, 1)))).astype(np.float32)).to(torch.bfloat16)
    A[3, 32:64] = 0.0                              # an all-zero block
    A[5, :32] = 448.0                              # a block at exactly the format's max
    q, sf = oracle.mx_quantize_rows(A)
    a = A.double().numpy()
    assert sf[3, 1] == 0 and np.all(q[3, 32:64] == 0)
    for r in range(a.shape[0]):
        for b in range(a.shape[1] // 32):
            blk = a[r, 32 * b:32 * b + 32]
            e = int(sf[r, b]) - 127
            if not np.any(blk):
                continue
            assert e == oracle.mx_exponent(np.abs(blk).max())
            scaled = (blk * 2.0 ** -e).astype(np.float32)
            assert np.array_equal(scaled.astype(np.float64), blk * 2.0 ** -e)   # exact scaling
            assert np.array_equal(q[r, 32 * b:32 * b + 32], _e4m3_torch(scaled)), (r, b)
            # the block's largest element uses the top of the range (no saturation)
            assert 224.0 < np.abs(blk).max() * 2.0 ** -e <= 448.0


def test_column_quantiser_matches_torch_and_round_trip():
    rng = np.random.default_rng(2)
    B = torch.from_numpy(rng.standard_normal((3, 96, 40)).astype(np.float32) / 7).to(torch.bfloat16)
    qT, sf = oracle.mx_quantize_cols(B)
    b = B.double().numpy()
    dec = oracle.e4m3_decode(qT)
    for e in range(3):
        for n in range(40):
            for k0 in range(0, 96, 32):
                col = b[e, k0:k0 + 32, n]
                ex = int(sf[e, n, k0 // 32]) - 127
                assert ex == oracle.mx_exponent(np.abs(col).max())
                ref = _e4m3_torch((col * 2.0 ** -ex).astype(np.float32))
                assert np.array_equal(qT[e, n, k0:k0 + 32], ref)
                # round trip within half an E4M3 step (3 mantissa bits: 2^-4 relative)
                back = dec[e, n, k0:k0 + 32] * 2.0 ** ex
                assert np.all(np.abs(back - col) <= 2.0 ** -4 * np.abs(col) + 2.0 ** (ex - 10))


def test_mx_gemm_matches_numpy_block_sums():
    rng = np.random.default_rng(3)
    E, K, N = 3, 128, 48
    counts = [5, 0, 9]
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    R = int(off[-1])
    Aq = rng.integers(0, 256, (R, K)).astype(np.uint8)
    Aq[(Aq & 0x7F) == 0x7F] = 0                  # no NaN codes
    BqT = rng.integers(0, 256, (E, N, K)).astype(np.uint8)
    BqT[(BqT & 0x7F) == 0x7F] = 1
    a_sf = rng.integers(120, 134, (R, K // 32)).astype(np.uint8)
    b_sf = rng.integers(118, 130, (E, N, K // 32)).astype(np.uint8)
    C = oracle.grouped_gemm_mx(Aq, a_sf, BqT, b_sf, off)
    a = torch.from_numpy(Aq).view(torch.float8_e4m3fn).double().numpy()
    bq = torch.from_numpy(BqT).view(torch.float8_e4m3fn).double().numpy()
    for e in range(E):
        for s in range(off[e], off[e + 1]):
            ref = np.zeros(N)
            for blk in range(K // 32):
                sl = slice(32 * blk, 32 * blk + 32)
                part = bq[e][:, sl] @ a[s, sl]
                ref += part * np.exp2(a_sf[s, blk].astype(np.int64) - 127 +
                                      b_sf[e, :, blk].astype(np.int64) - 127)
            np.testing.assert_allclose(C[s], ref, rtol=1e-12, atol=0)


@pytest.mark.parametrize("M,H,F,E,topk", [(40, 64, 96, 4, 2), (17, 128, 64, 1, 1)])
def test_mx_layer_within_e4m3_bound_of_the_exact_layer(M, H, F, E, topk):
    w, x, W1, W2, ids, tw = layer_case(M, H, F, E, topk, "uniform", seed=M + F)
    exact = oracle.moe_ffn(x, W1, W2, ids, tw)
    mx = oracle.moe_ffn_mx(x, W1, W2, ids, tw)
    rel = np.linalg.norm(mx - exact) / np.linalg.norm(exact)
    # each of h and W2 is within 2^-4 of what it encodes (relative, half an E4M3 step);
    # errors of independent elements add in quadrature, so far below 2^-4
    assert rel < 2.0 ** -4, rel
    assert rel > 1e-4     # the quantisation is really applied


def test_mx_layer_dense_special_case():
    # E = 1, topk = 1, w = 1: the layer is the dense chain, computed here with numpy /
    # torch from the quantised parts taken from independent conversions
    w, x, W1, W2, ids, tw = layer_case(24, 64, 64, 1, 1, "uniform", seed=5)
    got = oracle.moe_ffn_mx(x, W1, W2, ids, tw)
    xd, w1, w2 = x.double().numpy(), W1[0].double().numpy(), W2[0].double().numpy()
    g = xd @ w1
    h = g[:, :64] / (1.0 + np.exp(-g[:, :64])) * g[:, 64:]
    # h quantised in blocks of 32 with torch's e4m3 conversion
    hq = np.zeros_like(h)
    for r in range(h.shape[0]):
        for b in range(2):
            blk = h[r, 32 * b:32 * b + 32]
            e = oracle.mx_exponent(np.abs(blk).max())
            hq[r, 32 * b:32 * b + 32] = torch.from_numpy(blk * 2.0 ** -e).to(
                torch.float8_e4m3fn).double().numpy() * 2.0 ** e
    wq = np.zeros_like(w2)
    for n in range(w2.shape[1]):
        for b in range(2):
            col = w2[32 * b:32 * b + 32, n]
            e = oracle.mx_exponent(np.abs(col).max())
            wq[32 * b:32 * b + 32, n] = torch.from_numpy((col * 2.0 ** -e).astype(np.float32)).to(
                torch.float8_e4m3fn).double().numpy() * 2.0 ** e
    ref = (hq @ wq) * tw[:, :1].astype(np.float64)
    np.testing.assert_allclose(got, ref, rtol=1e-9, atol=1e-12)
