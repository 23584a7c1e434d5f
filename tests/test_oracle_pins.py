"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test checks one oracle function against a textbook or library routine, a
closed form, an invariant, brute force on tiny inputs, or a worked example the
pages print (tests/golden/).  A dropped term, a wrong sign or index, a swapped
gate/up or a transposed operand in the oracle fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from grouped_gemm_plan_b200 import workload as wlmod

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_ids(rng, M, E, topk, distinct=True):
    if distinct:
        return np.stack([rng.choice(E, topk, replace=False) for _ in range(M)]).astype(np.int32) \
            if M else np.zeros((0, topk), np.int32)
    return rng.integers(0, E, size=(M, topk), dtype=np.int32)


# ----------------------------------------------------------------------------- plan

@pytest.mark.parametrize("M,E,topk,distinct", [
    (0, 4, 2, True), (1, 1, 1, True), (7, 3, 3, True), (33, 8, 2, True),
    (100, 64, 4, True), (50, 5, 3, False), (257, 16, 8, True)])
def test_plan_matches_stable_sort(M, E, topk, distinct):
    rng = np.random.default_rng(M * 131 + E)
    ids = _rand_ids(rng, M, E, topk, distinct)
    w = rng.random((M, topk)).astype(np.float32)
    counts, offsets, perm, inv, ws = oracle.plan(ids, w, E)
    flat = ids.reshape(-1)
    R = M * topk
    # an independent definition: Python's stable sort of (expert, i)
    ref_perm = sorted(range(R), key=lambda i: (int(flat[i]), i))
    assert perm.tolist() == ref_perm
    assert counts.tolist() == [int((flat == e).sum()) for e in range(E)]
    assert offsets.tolist() == [0] + list(np.cumsum([int((flat == e).sum()) for e in range(E)]))
    # invariants
    assert counts.sum() == R and offsets[-1] == R
    assert np.all(np.diff(offsets) >= 0)
    assert sorted(perm.tolist()) == list(range(R))          # bijection
    assert np.array_equal(inv[perm], np.arange(R))          # inv o perm = id
    for e in range(E):
        seg = perm[offsets[e]:offsets[e + 1]]
        assert np.all(flat[seg] == e)
        assert np.all(np.diff(seg) > 0)                       # stable
    assert np.array_equal(ws, w.reshape(-1)[perm])


def test_plan_rejects_bad_input():
    ids = np.array([[0, 1], [2, 3]], np.int32)
    with pytest.raises(oracle.OracleError):
        oracle.plan(ids, None, 3)                # id 3 >= E
    with pytest.raises(oracle.OracleError):
        oracle.plan(np.array([[0, -1]], np.int32), None, 4)
    with pytest.raises(oracle.OracleError):
        oracle.plan(np.zeros((2, 5), np.int32), None, 4)   # topk > E


def test_tiling_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "tiling_example.json")))
    offsets = np.concatenate([[0], np.cumsum(g["counts"])]).astype(np.int32)
    te, r0, r1 = oracle.tile_table(offsets, g["BM"])
    assert [list(map(int, t)) for t in zip(te, r0, r1)] == g["tiles"]


def test_tile_table_brute_force():
    rng = np.random.default_rng(5)
    for _ in range(20):
        E = int(rng.integers(1, 12))
        counts = rng.integers(0, 400, size=E)
        counts[rng.random(E) < 0.3] = 0
        offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
        BM = int(rng.choice([64, 128]))
        te, r0, r1 = oracle.tile_table(offsets, BM)
        # every row covered exactly once, by a tile of its own expert
        owner = np.full(offsets[-1], -1)
        for e, a, b in zip(te, r0, r1):
            assert 0 < b - a <= BM and offsets[e] <= a < b <= offsets[e + 1]
            assert np.all(owner[a:b] == -1)
            owner[a:b] = e
        assert np.array_equal(owner, np.repeat(np.arange(E), counts))
        assert len(te) == sum(-(-int(c) // BM) for c in counts)


def test_balanced_load_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "balanced_load.json")))
    wl = wlmod.Workload("balanced", g["M"], 64, 64, g["E"], g["topk"], "balanced", 0.0, 11)
    ids = wlmod.make_topk_ids(wl)
    counts, *_ = oracle.plan(ids, None, g["E"])
    assert counts.tolist() == [g["rows_per_expert"]] * g["E"]
    assert all(len(set(r)) == g["topk"] for r in ids.tolist())


# ----------------------------------------------------------------------------- dispatch

def test_dispatch_and_unpermute_identity():
    rng = np.random.default_rng(1)
    M, H, E, topk = 37, 24, 5, 3
    x = torch.from_numpy(rng.standard_normal((M, H), dtype=np.float32)).to(torch.bfloat16)
    ids = _rand_ids(rng, M, E, topk)
    _, _, perm, inv, _ = oracle.plan(ids, None, E)
    xp = oracle.dispatch(x, perm, topk)
    xb = wlmod.bf16_bits(x)
    assert np.array_equal(xp, xb[perm // topk])             # numpy fancy indexing
    back = oracle.unpermute_rows(xp, inv)
    assert np.array_equal(back, np.repeat(xb, topk, axis=0))  # row i holds x[i // topk]


# ----------------------------------------------------------------------------- grouped GEMM

def _bf(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def _f64(t):
    return t.to(torch.float64).numpy()


def test_grouped_gemm_matches_numpy_matmul():
    rng = np.random.default_rng(2)
    E, K, N = 4, 40, 24
    counts = np.array([5, 0, 11, 3])
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    A = _bf(rng.standard_normal((offsets[-1], K)))
    B = _bf(rng.standard_normal((E, K, N)))
    C = oracle.grouped_gemm(A, B, offsets)
    Af, Bf = _f64(A), _f64(B)
    for e in range(E):
        ref = Af[offsets[e]:offsets[e + 1]] @ Bf[e]
        np.testing.assert_allclose(C[offsets[e]:offsets[e + 1]], ref, rtol=1e-12, atol=1e-12)
    # a transposed B would not match a non-square, asymmetric operand
    assert not np.allclose(C[:5], Af[:5] @ Bf[0][::-1])


def test_swiglu_closed_form():
    G = np.array([[0.0, 1.5, 2.0, -3.0], [-1.0, 4.0, 0.5, 0.25]])
    h = oracle.swiglu(G)

    def s(v):
        return v / (1.0 + math.exp(-v))
    ref = [[s(0.0) * 2.0, s(1.5) * -3.0], [s(-1.0) * 0.5, s(4.0) * 0.25]]
    np.testing.assert_allclose(h, ref, rtol=1e-15, atol=0)


def test_combine_matches_einsum():
    rng = np.random.default_rng(3)
    M, H, E, topk = 9, 16, 4, 2
    ids = _rand_ids(rng, M, E, topk)
    w = rng.random((M, topk)).astype(np.float32)
    _, _, perm, inv, _ = oracle.plan(ids, w, E)
    yp = rng.standard_normal((M * topk, H))
    out = oracle.combine(yp, inv, w)
    y_tok = yp[inv].reshape(M, topk, H)
    np.testing.assert_allclose(out, np.einsum("tk,tkh->th", w.astype(np.float64), y_tok),
                               rtol=1e-14, atol=1e-14)


# ----------------------------------------------------------------------------- whole layer

def _case(M, H, F, E, topk, routing="uniform", seed=0):
    wl = wlmod.Workload("pin", M, H, F, E, topk, routing, 0.05, seed)
    x = wlmod.make_x(wl)
    W1, W2 = wlmod.make_weights(wl)
    ids, w = wlmod.make_routing(wl)
    return wl, x, W1, W2, ids, w


def test_dense_special_case_e1_topk1():
    # E=1, topk=1: every token goes to the one expert with weight 1 (softmax of a
    # single logit), so the layer is a dense SwiGLU FFN.
    wl, x, W1, W2, ids, w = _case(19, 32, 48, 1, 1)
    assert np.all(w == 1.0)
    out = oracle.moe_ffn(x, W1, W2, ids, w)
    X, A, B = x.double(), W1[0].double(), W2[0].double()
    F = wl.F
    ref = (torch.nn.functional.silu(X @ A[:, :F]) * (X @ A[:, F:])) @ B
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-10, atol=1e-12)


def test_scalar_closed_form_h1_f1():
    # H = F = 1: out[t] = sum_k w[t,k] * silu(x_t a_e) * (x_t b_e) * c_e with
    # W1[e] = [a_e, b_e] (gate, up) and W2[e] = [c_e].
    wl, x, W1, W2, ids, w = _case(11, 1, 1, 3, 2, seed=4)
    out = oracle.moe_ffn(x, W1, W2, ids, w)
    xs, W1s, W2s = _f64(x)[:, 0], _f64(W1), _f64(W2)
    for t in range(wl.M):
        acc = 0.0
        for k in range(wl.topk):
            e = ids[t, k]
            g, u, c = xs[t] * W1s[e, 0, 0], xs[t] * W1s[e, 0, 1], W2s[e, 0, 0]
            acc += float(w[t, k]) * (g / (1.0 + math.exp(-g))) * u * c
        assert out[t, 0] == pytest.approx(acc, rel=1e-13, abs=1e-15)


def test_identical_experts_sum_of_weights():
    # If every expert has the same weights, the top-k mixture equals FFN(x)*sum_k w.
    wl, x, W1, W2, ids, w = _case(23, 16, 32, 4, 2, seed=6)
    W1 = W1[:1].repeat(4, 1, 1).contiguous()
    W2 = W2[:1].repeat(4, 1, 1).contiguous()
    out = oracle.moe_ffn(x, W1, W2, ids, w)
    one = np.zeros_like(ids)
    dense = oracle.moe_ffn(x, W1[:1].contiguous(), W2[:1].contiguous(), one[:, :1].copy(),
                           np.ones((wl.M, 1), np.float32))
    np.testing.assert_allclose(out, dense * w.astype(np.float64).sum(1, keepdims=True),
                               rtol=1e-12, atol=1e-13)


def test_linear_in_gate_weights():
    wl, x, W1, W2, ids, w = _case(17, 16, 16, 5, 3, seed=7)
    a = oracle.moe_ffn(x, W1, W2, ids, w)
    b = oracle.moe_ffn(x, W1, W2, ids, (2 * w).astype(np.float32))
    assert np.array_equal(b, 2 * a)       # scaling by 2 is exact in binary floating point
    # one weight set to zero removes exactly that expert's contribution
    w0 = w.copy()
    w0[:, 1] = 0
    c = oracle.moe_ffn(x, W1, W2, ids, w0)
    ids1 = ids[:, [0, 2]].copy()
    d = oracle.moe_ffn(x, W1, W2, ids1, w[:, [0, 2]].copy())
    np.testing.assert_allclose(c, d, rtol=1e-13, atol=1e-14)


@pytest.mark.parametrize("routing", ["uniform", "skewed", "balanced"])
def test_bruteforce_equals_plan_path_bitwise(routing):
    wl, x, W1, W2, ids, w = _case(40, 24, 40, 6, 2, routing=routing, seed=8)
    out = oracle.moe_ffn(x, W1, W2, ids, w)
    bf = oracle.bruteforce_tokens(x, W1, W2, ids, w, np.arange(wl.M))
    assert np.array_equal(out, bf)
    sub = np.array([3, 0, 39, 17])
    assert np.array_equal(oracle.bruteforce_tokens(x, W1, W2, ids, w, sub), out[sub])


def test_layer_matches_torch_per_token_mixture():
    # The definition written out with torch float64 on a skewed routing.
    wl, x, W1, W2, ids, w = _case(29, 32, 24, 7, 3, routing="skewed", seed=9)
    out = oracle.moe_ffn(x, W1, W2, ids, w)
    X, A, B = x.double(), W1.double(), W2.double()
    F = wl.F
    ref = torch.zeros(wl.M, wl.H, dtype=torch.float64)
    for t in range(wl.M):
        for k in range(wl.topk):
            e = int(ids[t, k])
            g = X[t] @ A[e]
            ref[t] += float(w[t, k]) * ((torch.nn.functional.silu(g[:F]) * g[F:]) @ B[e])
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-10, atol=1e-12)


# ----------------------------------------------------------------------------- router

def test_route_matches_lexsort_and_softmax():
    rng = np.random.default_rng(21)
    for M, E, k in [(50, 8, 2), (20, 64, 4), (9, 16, 16), (5, 1, 1)]:
        logits = rng.standard_normal((M, E)).astype(np.float32)
        logits[0, :] = 0.5                       # all tied: lowest indices first
        ids, w = oracle.route(logits, k)
        for t in range(M):
            order = np.lexsort((np.arange(E), -logits[t].astype(np.float64)))[:k]
            assert ids[t].tolist() == order.tolist()
            chosen = logits[t, ids[t]].astype(np.float64)
            ref = np.exp(chosen - chosen.max()) / np.exp(chosen - chosen.max()).sum()
            np.testing.assert_allclose(w[t], ref, rtol=1e-14, atol=0)
        assert ids[0].tolist() == list(range(k))
        np.testing.assert_allclose(w.sum(1), 1.0, rtol=1e-14)


def test_route_closed_form_and_permutation_equivariance():
    logits = np.array([[0.0, float(np.log(3.0)), -5.0]], np.float32)
    ids, w = oracle.route(logits, 2)
    assert ids.tolist() == [[1, 0]]
    a = float(np.float32(np.log(3.0)))
    np.testing.assert_allclose(w[0], [np.exp(a) / (np.exp(a) + 1), 1 / (np.exp(a) + 1)], rtol=1e-14)
    # relabelling the experts relabels the choice and leaves the weights alone
    rng = np.random.default_rng(22)
    L = rng.standard_normal((30, 12)).astype(np.float32)   # distinct values: no ties
    p = rng.permutation(12)
    i1, w1 = oracle.route(L, 3)
    i2, w2 = oracle.route(np.ascontiguousarray(L[:, p]), 3)
    assert np.array_equal(p[i2], i1)
    np.testing.assert_allclose(w2, w1, rtol=1e-15)


def test_route_rejects_topk_above_e():
    with pytest.raises(oracle.OracleError):
        oracle.route(np.zeros((2, 3), np.float32), 4)


# ----------------------------------------------------------------------------- GemmAdd

def _gemm_add_case(seed=5):
    from helpers import layer_case
    w, x, W1, W2, ids, tw = layer_case(24, 64, 64, 4, 2, "uniform", seed=seed)
    rng = np.random.default_rng(seed)
    add = torch.from_numpy(rng.standard_normal((24, 64)).astype(np.float32)).to(torch.bfloat16)
    return x, W1, W2, ids, tw, add


def test_gemm_add_special_cases():
    """Grouped GEMM article, "Fused GemmAdd": y = alpha * acc + beta * add.  beta = 0
    is the layer itself, alpha = 0 the added tensor alone (both exact in fp64), and
    the residual form (alpha = beta = 1) minus the added tensor is the layer."""
    x, W1, W2, ids, tw, add = _gemm_add_case()
    layer = oracle.moe_ffn(x, W1, W2, ids, tw)
    add64 = add.double().numpy()
    assert np.array_equal(oracle.moe_ffn_add(x, W1, W2, ids, tw, add, 1.0, 0.0), layer)
    assert np.array_equal(oracle.moe_ffn_add(x, W1, W2, ids, tw, add, 0.0, 1.0), add64)
    assert np.array_equal(oracle.moe_ffn_add(x, W1, W2, ids, tw, add, 2.0, 0.0), 2.0 * layer)
    res = oracle.moe_ffn_add(x, W1, W2, ids, tw, add)             # alpha = beta = 1
    scale = np.abs(layer) + np.abs(add64)
    assert np.all(np.abs((res - add64) - layer) <= 4 * np.finfo(np.float64).eps * scale)
    # the residual stream as the added tensor: x + layer(x)
    resx = oracle.moe_ffn_add(x, W1, W2, ids, tw, x)
    assert np.all(np.abs(resx - x.double().numpy() - layer) <=
                  4 * np.finfo(np.float64).eps * (np.abs(layer) + np.abs(x.double().numpy())))


def test_gemm_add_linear_in_alpha_and_beta():
    x, W1, W2, ids, tw, add = _gemm_add_case(seed=6)
    layer = oracle.moe_ffn(x, W1, W2, ids, tw)
    add64 = add.double().numpy()
    for alpha, beta in [(0.5, -2.0), (-1.0, 0.25), (3.0, 3.0)]:
        y = oracle.moe_ffn_add(x, W1, W2, ids, tw, add, alpha, beta)
        ref = alpha * layer + beta * add64          # numpy on the two pinned parts
        assert np.allclose(y, ref, rtol=1e-14, atol=1e-14)
