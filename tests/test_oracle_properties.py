"""Property tests (hypothesis) of the oracle's plan and E4M3 codec over many random
shapes: the plan against Python's stable sort of (expert, i), the codec's round
trip and ordering.  Each is a fact the definition fixes, checked on inputs the
fixed-case pins do not reach."""
import numpy as np
from hypothesis import given, settings, strategies as st

import oracle


@settings(max_examples=60, deadline=None)
@given(st.integers(0, 300), st.integers(1, 40), st.integers(1, 8), st.integers(0, 2**31 - 1))
def test_plan_is_the_stable_sort(M, E, topk, seed):
    topk = min(topk, E)
    rng = np.random.default_rng(seed)
    ids = rng.integers(0, E, (M, topk)).astype(np.int32)        # duplicates allowed
    w = rng.random((M, topk)).astype(np.float32)
    counts, offsets, perm, inv, ws = oracle.plan(ids, w, E)
    flat = ids.reshape(-1)
    order = sorted(range(M * topk), key=lambda i: (flat[i], i))
    assert perm.tolist() == order
    assert counts.tolist() == np.bincount(flat, minlength=E).tolist()
    assert offsets[0] == 0 and offsets[-1] == M * topk
    assert np.array_equal(np.diff(offsets), counts)
    if M * topk:
        assert np.array_equal(inv[perm], np.arange(M * topk))
        assert np.array_equal(ws, w.reshape(-1)[perm])


@settings(max_examples=200, deadline=None)
@given(st.floats(-448.0, 448.0, allow_nan=False, width=32))
def test_e4m3_encode_is_monotone_and_round_trips(v):
    codes = np.arange(256, dtype=np.uint8)
    vals = oracle.e4m3_decode(codes)
    c = oracle.e4m3_encode(np.float32([v]))[0]
    d = oracle.e4m3_decode(np.uint8(c))
    # the decoded value is a nearest grid value and re-encodes to itself
    fin = vals[~np.isnan(vals)]
    assert abs(d - v) <= np.min(np.abs(fin - v)) + 0.0
    assert oracle.e4m3_decode(oracle.e4m3_encode(np.float32([d]))[0]) == d
    # monotone: a larger input never decodes smaller
    v2 = np.nextafter(np.float32(v), np.float32(np.inf))
    if abs(v2) <= 448.0:
        assert oracle.e4m3_decode(oracle.e4m3_encode(np.float32([v2]))[0]) >= d
