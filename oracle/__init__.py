"""CPU oracle of the MoE SwiGLU FFN layer -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and its
Python binding) never loads it and shares no code with it.

The arithmetic lives in ``oracle.c`` (plain C, fp64, loops in the pages' order);
this module only compiles it with gcc and marshals numpy arrays through ctypes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

OK, ERR_ARG, ERR_BAD_ID = 0, 1, 3

_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc, OpenMP, no FP contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                               "-fno-fast-math", "-std=c11", "-Wall", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def configure(lib):
    """Declare the C signatures on a loaded oracle library and return it."""
    P = ctypes.c_void_p
    i64, i32 = ctypes.c_int64, ctypes.c_int32
    lib.oracle_plan.argtypes = [P, P, i64, i32, i32, P, P, P, P, P]
    lib.oracle_plan.restype = ctypes.c_int
    lib.oracle_tile_table.argtypes = [P, i32, i32, P, P, P, i64]
    lib.oracle_tile_table.restype = i64
    lib.oracle_dispatch.argtypes = [P, P, i64, i64, i32, P]
    lib.oracle_unpermute_rows.argtypes = [P, P, i64, i64, P]
    lib.oracle_grouped_gemm.argtypes = [P, P, P, i32, i64, i64, P]
    lib.oracle_swiglu.argtypes = [P, i64, i64, P]
    lib.oracle_combine.argtypes = [P, P, P, i64, i64, i32, P]
    lib.oracle_moe_ffn.argtypes = [P, P, P, P, P, i64, i64, i64, i32, i32, P]
    lib.oracle_moe_ffn.restype = ctypes.c_int
    lib.oracle_bruteforce_tokens.argtypes = [P, P, P, P, P, i64, i64, i32, i32, P, i64, P]
    lib.oracle_bruteforce_tokens.restype = ctypes.c_int
    lib.oracle_num_threads.restype = ctypes.c_int
    lib.oracle_mx_exponent.argtypes = [ctypes.c_double]
    lib.oracle_mx_exponent.restype = ctypes.c_int
    lib.oracle_mx_quantize_rows.argtypes = [P, i64, i64, P, P]
    lib.oracle_mx_quantize_cols.argtypes = [P, i32, i64, i64, P, P]
    lib.oracle_grouped_gemm_mx.argtypes = [P, P, P, P, P, i32, i64, i64, P]
    lib.oracle_moe_ffn_mx.argtypes = [P, P, P, P, P, i64, i64, i64, i32, i32, P]
    lib.oracle_moe_ffn_mx.restype = ctypes.c_int
    lib.oracle_gemm_add.argtypes = [P, P, ctypes.c_double, ctypes.c_double, i64, P]
    lib.oracle_route.argtypes = [P, i64, i32, i32, P, P]
    lib.oracle_route.restype = ctypes.c_int
    lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
    lib.oracle_e4m3_decode.restype = ctypes.c_double
    lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
    lib.oracle_e4m3_encode.restype = ctypes.c_uint8
    lib.oracle_quantize_rows_e4m3.argtypes = [P, i64, i64, P, P]
    lib.oracle_quantize_cols_e4m3.argtypes = [P, i32, i64, i64, P, P]
    lib.oracle_grouped_gemm_e4m3.argtypes = [P, P, P, P, P, i32, i64, i64, P]
    lib.oracle_moe_ffn_fp8.argtypes = [P, P, P, P, P, i64, i64, i64, i32, i32, P]
    lib.oracle_moe_ffn_fp8.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = configure(ctypes.CDLL(build()))
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _u16(a) -> np.ndarray:
    """bf16 bit patterns as uint16 (accepts a CPU torch bf16 tensor or a uint16 array)."""
    if isinstance(a, np.ndarray):
        assert a.dtype == np.uint16
        return np.ascontiguousarray(a)
    import torch
    assert a.dtype == torch.bfloat16 and a.device.type == "cpu"
    return a.contiguous().view(torch.int16).numpy().view(np.uint16)


class OracleError(RuntimeError):
    pass


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def plan(ids: np.ndarray, w: np.ndarray | None, E: int):
    """counts [E], offsets [E+1], perm [R], inv [R], w_sorted [R] (or None)."""
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    M, topk = ids.shape
    R = M * topk
    counts = np.zeros(E, np.int32)
    offsets = np.zeros(E + 1, np.int32)
    perm = np.zeros(max(R, 1), np.int32)
    inv = np.zeros(max(R, 1), np.int32)
    ws = None
    if w is not None:
        w = np.ascontiguousarray(w, dtype=np.float32)
        ws = np.zeros(max(R, 1), np.float32)
    st = _load().oracle_plan(_p(ids), _p(w) if w is not None else None, M, E, topk,
                             _p(counts), _p(offsets), _p(perm), _p(inv),
                             _p(ws) if ws is not None else None)
    if st != OK:
        raise OracleError(f"oracle_plan status {st}")
    return counts, offsets, perm[:R], inv[:R], (ws[:R] if ws is not None else None)


def tile_table(offsets: np.ndarray, BM: int):
    """(expert, row0, row1) per tile, expert by expert."""
    offsets = np.ascontiguousarray(offsets, dtype=np.int32)
    E = len(offsets) - 1
    cap = int(offsets[-1]) // BM + E + 1
    te, r0, r1 = (np.zeros(cap, np.int32) for _ in range(3))
    n = _load().oracle_tile_table(_p(offsets), E, BM, _p(te), _p(r0), _p(r1), cap)
    if n < 0:
        raise OracleError("tile table overflow")
    return te[:n], r0[:n], r1[:n]


def dispatch(x, perm: np.ndarray, topk: int) -> np.ndarray:
    xb = _u16(x)
    M, H = xb.shape
    perm = np.ascontiguousarray(perm, dtype=np.int32)
    xp = np.zeros((M * topk, H), np.uint16)
    _load().oracle_dispatch(_p(xb), _p(perm), M, H, topk, _p(xp))
    return xp


def unpermute_rows(xp, inv: np.ndarray) -> np.ndarray:
    xb = _u16(xp)
    R, H = xb.shape
    inv = np.ascontiguousarray(inv, dtype=np.int32)
    back = np.zeros((R, H), np.uint16)
    _load().oracle_unpermute_rows(_p(xb), _p(inv), R, H, _p(back))
    return back


def grouped_gemm(A, B, offsets: np.ndarray) -> np.ndarray:
    """C fp64 [R, N] = per-expert A_e @ B[e]; A bf16 [R, K], B bf16 [E, K, N]."""
    Ab, Bb = _u16(A), _u16(B)
    R, K = Ab.shape
    E, K2, N = Bb.shape
    assert K2 == K
    offsets = np.ascontiguousarray(offsets, dtype=np.int32)
    C = np.zeros((R, N), np.float64)
    _load().oracle_grouped_gemm(_p(Ab), _p(Bb), _p(offsets), E, K, N, _p(C))
    return C


def swiglu(G: np.ndarray) -> np.ndarray:
    G = np.ascontiguousarray(G, dtype=np.float64)
    R, F2 = G.shape
    h = np.zeros((R, F2 // 2), np.float64)
    _load().oracle_swiglu(_p(G), R, F2 // 2, _p(h))
    return h


def combine(yp: np.ndarray, inv: np.ndarray, w: np.ndarray) -> np.ndarray:
    """out fp64 [M, H] = sum_k w[t,k] * yp[inv[t*topk+k]] (yp fp64 [R, H])."""
    yp = np.ascontiguousarray(yp, dtype=np.float64)
    w = np.ascontiguousarray(w, dtype=np.float32)
    M, topk = w.shape
    H = yp.shape[1]
    inv = np.ascontiguousarray(inv, dtype=np.int32)
    out = np.zeros((M, H), np.float64)
    _load().oracle_combine(_p(yp), _p(inv), _p(w), M, H, topk, _p(out))
    return out


def moe_ffn(x, W1, W2, ids: np.ndarray, w: np.ndarray) -> np.ndarray:
    """The whole layer through the plan; out fp64 [M, H]."""
    xb, W1b, W2b = _u16(x), _u16(W1), _u16(W2)
    M, H = xb.shape
    E, _, F2 = W1b.shape
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    w = np.ascontiguousarray(w, dtype=np.float32)
    topk = ids.shape[1]
    out = np.zeros((M, H), np.float64)
    st = _load().oracle_moe_ffn(_p(xb), _p(W1b), _p(W2b), _p(ids), _p(w), M, H, F2 // 2, E,
                                topk, _p(out))
    if st != OK:
        raise OracleError(f"oracle_moe_ffn status {st}")
    return out


def gemm_add(acc: np.ndarray, add, alpha: float, beta: float) -> np.ndarray:
    """alpha * acc + beta * add in fp64 (the Fused GemmAdd epilogue); acc fp64, add bf16."""
    a = np.ascontiguousarray(acc, dtype=np.float64)
    b = _u16(add)
    assert a.shape == b.shape
    y = np.empty_like(a)
    _load().oracle_gemm_add(_p(a), _p(b), float(alpha), float(beta), a.size, _p(y))
    return y


def moe_ffn_add(x, W1, W2, ids: np.ndarray, w: np.ndarray, add, alpha: float = 1.0,
                beta: float = 1.0) -> np.ndarray:
    """The layer with the GemmAdd epilogue: alpha * layer(x) + beta * add (fp64)."""
    return gemm_add(moe_ffn(x, W1, W2, ids, w), add, alpha, beta)


def route(logits: np.ndarray, topk: int):
    """Router: ids int32 [M, topk] (largest logits first, ties to the lower index) and
    softmax weights fp64 [M, topk] over the chosen logits."""
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    M, E = logits.shape
    ids = np.zeros((M, topk), np.int32)
    w = np.zeros((M, topk), np.float64)
    st = _load().oracle_route(_p(logits), M, E, topk, _p(ids), _p(w))
    if st != OK:
        raise OracleError(f"oracle_route status {st}")
    return ids, w


def bruteforce_tokens(x, W1, W2, ids: np.ndarray, w: np.ndarray, tokens) -> np.ndarray:
    """Rows of the layer output for the listed tokens, computed one token at a time."""
    xb, W1b, W2b = _u16(x), _u16(W1), _u16(W2)
    M, H = xb.shape
    E, _, F2 = W1b.shape
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    w = np.ascontiguousarray(w, dtype=np.float32)
    topk = ids.shape[1]
    tok = np.ascontiguousarray(tokens, dtype=np.int64)
    assert tok.size == 0 or (tok.min() >= 0 and tok.max() < M)
    out = np.zeros((tok.size, H), np.float64)
    st = _load().oracle_bruteforce_tokens(_p(xb), _p(W1b), _p(W2b), _p(ids), _p(w), H, F2 // 2, E,
                                          topk, _p(tok), tok.size, _p(out))
    if st != OK:
        raise OracleError(f"oracle_bruteforce_tokens status {st}")
    return out


# ------------------------------------------------------------------ FP8 (E4M3)

def e4m3_decode(codes) -> np.ndarray:
    """fp64 values of E4M3 codes (uint8 array)."""
    lib = _load()
    c = np.asarray(codes, dtype=np.uint8)
    return np.array([lib.oracle_e4m3_decode(int(v)) for v in c.reshape(-1)]).reshape(c.shape)


def e4m3_encode(values) -> np.ndarray:
    """E4M3 codes of float32 values (nearest, ties to even, saturating at 448)."""
    lib = _load()
    v = np.asarray(values, dtype=np.float32)
    return np.array([lib.oracle_e4m3_encode(float(x)) for x in v.reshape(-1)],
                    dtype=np.uint8).reshape(v.shape)


def quantize_rows_e4m3(A):
    """Per-row E4M3 quantisation of bf16 A [R, K] -> (codes uint8 [R, K], scale fp32 [R])."""
    a = _u16(A)
    R, K = a.shape
    q = np.empty((R, K), np.uint8)
    sc = np.empty(R, np.float32)
    _load().oracle_quantize_rows_e4m3(_p(a), R, K, _p(q), _p(sc))
    return q, sc


def quantize_cols_e4m3(B):
    """Per-output-column E4M3 quantisation of bf16 B [E, K, N] -> (codes uint8 [E, N, K]
    with K contiguous, scale fp32 [E, N])."""
    b = _u16(B)
    E, K, N = b.shape
    q = np.empty((E, N, K), np.uint8)
    sc = np.empty((E, N), np.float32)
    _load().oracle_quantize_cols_e4m3(_p(b), E, K, N, _p(q), _p(sc))
    return q, sc


def grouped_gemm_e4m3(Aq, a_scale, BqT, b_scale, offsets) -> np.ndarray:
    """fp64 C [R, N] = a_scale[s] * b_scale[e, n] * (decode(Aq[s]) . decode(BqT[e, n]))."""
    Aq = np.ascontiguousarray(Aq, np.uint8)
    BqT = np.ascontiguousarray(BqT, np.uint8)
    a_scale = np.ascontiguousarray(a_scale, np.float32)
    b_scale = np.ascontiguousarray(b_scale, np.float32)
    offsets = np.ascontiguousarray(offsets, np.int32)
    R, K = Aq.shape
    E, N, _ = BqT.shape
    C = np.zeros((R, N), np.float64)
    _load().oracle_grouped_gemm_e4m3(_p(Aq), _p(a_scale), _p(BqT), _p(b_scale), _p(offsets), E,
                                     K, N, _p(C))
    return C


def moe_ffn_fp8(x, W1, W2, ids: np.ndarray, w: np.ndarray) -> np.ndarray:
    """The layer with an E4M3 down projection (h and W2 quantised as above), fp64 [M, H]."""
    xu, w1u, w2u = _u16(x), _u16(W1), _u16(W2)
    M, H = xu.shape
    E, _, F2 = w1u.shape
    ids = np.ascontiguousarray(ids, np.int32)
    w = np.ascontiguousarray(w, np.float32)
    topk = ids.shape[1]
    out = np.zeros((M, H), np.float64)
    st = _load().oracle_moe_ffn_fp8(_p(xu), _p(w1u), _p(w2u), _p(ids), _p(w), M, H, F2 // 2, E,
                                    topk, _p(out))
    if st != OK:
        raise ValueError(f"oracle_moe_ffn_fp8 status {st}")
    return out


# ------------------------------------------------------------------ MX (block-scaled) FP8

def mx_exponent(amax: float) -> int:
    """Smallest e with amax <= 448 * 2^e (clamped to [-127, 127]; -127 for 0)."""
    return int(_load().oracle_mx_exponent(float(amax)))


def mx_quantize_rows(A) -> tuple[np.ndarray, np.ndarray]:
    """Rows of A [R, K] (fp64 values, or a bf16 tensor) in blocks of 32 along K ->
    (codes uint8 [R, K], scale exponent codes uint8 [R, K/32], value = 2^(code-127))."""
    if isinstance(A, np.ndarray) and A.dtype == np.float64:
        a = np.ascontiguousarray(A)
    else:
        import torch
        a = np.ascontiguousarray(torch.as_tensor(A).double().numpy())
    R, K = a.shape
    q = np.empty((R, K), np.uint8)
    sf = np.empty((R, K // 32), np.uint8)
    _load().oracle_mx_quantize_rows(_p(a), R, K, _p(q), _p(sf))
    return q, sf


def mx_quantize_cols(B) -> tuple[np.ndarray, np.ndarray]:
    """bf16 B [E, K, N] per output column in blocks of 32 along K -> (codes uint8
    [E, N, K] with K contiguous, scale exponent codes uint8 [E, N, K/32])."""
    b = _u16(B)
    E, K, N = b.shape
    q = np.empty((E, N, K), np.uint8)
    sf = np.empty((E, N, K // 32), np.uint8)
    _load().oracle_mx_quantize_cols(_p(b), E, K, N, _p(q), _p(sf))
    return q, sf


def grouped_gemm_mx(Aq, a_sf, BqT, b_sf, offsets) -> np.ndarray:
    """fp64 C [R, N] = sum over 32-blocks b of 2^(a_sf-127) 2^(b_sf-127) (Aq . BqT)_b."""
    Aq = np.ascontiguousarray(Aq, np.uint8)
    a_sf = np.ascontiguousarray(a_sf, np.uint8)
    BqT = np.ascontiguousarray(BqT, np.uint8)
    b_sf = np.ascontiguousarray(b_sf, np.uint8)
    offsets = np.ascontiguousarray(offsets, np.int32)
    R, K = Aq.shape
    E, N, _ = BqT.shape
    C = np.zeros((R, N), np.float64)
    _load().oracle_grouped_gemm_mx(_p(Aq), _p(a_sf), _p(BqT), _p(b_sf), _p(offsets), E, K, N,
                                   _p(C))
    return C


def moe_ffn_mx(x, W1, W2, ids: np.ndarray, w: np.ndarray) -> np.ndarray:
    """The layer with a block-scaled (MX) E4M3 down projection, fp64 [M, H]."""
    xu, w1u, w2u = _u16(x), _u16(W1), _u16(W2)
    M, H = xu.shape
    E, _, F2 = w1u.shape
    ids = np.ascontiguousarray(ids, np.int32)
    w = np.ascontiguousarray(w, np.float32)
    topk = ids.shape[1]
    out = np.zeros((M, H), np.float64)
    st = _load().oracle_moe_ffn_mx(_p(xu), _p(w1u), _p(w2u), _p(ids), _p(w), M, H, F2 // 2, E,
                                   topk, _p(out))
    if st != OK:
        raise ValueError(f"oracle_moe_ffn_mx status {st}")
    return out
