"""Thin Python binding of libmoe.so: argument marshalling only.

Every function here has the name and the meaning of the C entry point it wraps
(include/moe.h); it takes torch tensors that already live on the GPU, passes
their device pointers and the current CUDA stream, and raises MoEError on a
non-zero status.  No step of the layer runs in Python or on the CPU: if the
library is missing, importing this module's functions fails loudly.
"""
from __future__ import annotations

import ctypes
import os

import torch

from . import build as _build

MOE_OK = 0
(MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED_SHAPE, MOE_ERR_BAD_EXPERT_ID, MOE_ERR_WORKSPACE_TOO_SMALL,
 MOE_ERR_TIMEOUT, MOE_ERR_CUDA, MOE_ERR_MISALIGNED, MOE_ERR_BAD_INDEX) = range(1, 9)
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED_SHAPE",
                3: "MOE_ERR_BAD_EXPERT_ID", 4: "MOE_ERR_WORKSPACE_TOO_SMALL",
                5: "MOE_ERR_TIMEOUT", 6: "MOE_ERR_CUDA", 7: "MOE_ERR_MISALIGNED",
                8: "MOE_ERR_BAD_INDEX"}

EPI_STORE, EPI_SWIGLU, EPI_WEIGHT_SCATTER = 0, 1, 2
NOALLOC_SCRATCH_BYTES = 64 * 1024 * 1024   # MOE_NOALLOC_SCRATCH_BYTES
(OP_PLAN, OP_DISPATCH, OP_GROUPED_GEMM, OP_COMBINE, OP_FFN_FUSED, OP_ROUTE, OP_FFN_FP8,
 OP_GEMM_MX, OP_FFN_MX) = range(9)

# Every symbol include/moe.h declares.
EXPORTS = ["moe_abi_version", "moe_workspace_size", "moe_route", "moe_route_plan", "moe_plan",
           "moe_dispatch",
           "moe_grouped_gemm", "moe_combine", "moe_combine_add", "moe_ffn_fused",
           "moe_ffn_fused_add", "moe_ffn_fused_noalloc",
           "moe_get_device_status", "moe_set_wait_timeout_ns", "moe_set_fault_injection",
           "moe_set_stage_events", "moe_quantize_weights_e4m3", "moe_quantize_rows_e4m3",
           "moe_grouped_gemm_e4m3", "moe_ffn_fused_fp8", "moe_quantize_weights_mx",
           "moe_quantize_rows_mx", "moe_grouped_gemm_swiglu_mx", "moe_grouped_gemm_mx",
           "moe_ffn_fused_mx", "moe_last_error"]


class MoEError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


_lib = None


def library_path() -> str:
    return _build.LIB


def load(path: str | None = None):
    """Load libmoe.so (built in-tree by grouped_gemm_plan_b200.build). Raises if absent."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or _build.LIB
    if not os.path.exists(p):
        raise ImportError(f"{p} is missing: build it with `python -m grouped_gemm_plan_b200.build` "
                          "(there is no fallback implementation)")
    lib = ctypes.CDLL(p)
    P, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
    st = ctypes.c_int
    lib.moe_abi_version.restype = ctypes.c_int
    lib.moe_workspace_size.argtypes = [ctypes.c_int, i64, i64, i64, i32, i32]
    lib.moe_workspace_size.restype = sz
    lib.moe_route.argtypes = [P, i64, i32, i32, P, P, P, sz, P]
    lib.moe_route.restype = st
    lib.moe_route_plan.argtypes = [P, i64, i32, i32, P, P, P, P, P, P, P, P, sz, P]
    lib.moe_route_plan.restype = st
    lib.moe_plan.argtypes = [P, P, i64, i32, i32, P, P, P, P, P, P, sz, P]
    lib.moe_plan.restype = st
    lib.moe_dispatch.argtypes = [P, P, i64, i64, i32, P, P, sz, P]
    lib.moe_dispatch.restype = st
    lib.moe_grouped_gemm.argtypes = [P, P, P, i32, i64, i64, i64, ctypes.c_int, P, P, P, P, sz, P]
    lib.moe_grouped_gemm.restype = st
    lib.moe_combine.argtypes = [P, i32, P, P, i64, i64, i32, P, P, sz, P]
    lib.moe_combine.restype = st
    lib.moe_ffn_fused.argtypes = [P, P, P, P, P, i64, i64, i64, i32, i32, i32, P, P, P, P, P, sz, P]
    lib.moe_ffn_fused.restype = st
    f32 = ctypes.c_float
    lib.moe_combine_add.argtypes = [P, i32, P, P, P, f32, f32, i64, i64, i32, P, P, sz, P]
    lib.moe_combine_add.restype = st
    lib.moe_ffn_fused_add.argtypes = [P, P, P, P, P, P, f32, f32, i64, i64, i64, i32, i32, P, P,
                                      P, P, P, sz, P]
    lib.moe_ffn_fused_add.restype = st
    lib.moe_ffn_fused_noalloc.argtypes = [P, P, P, P, P, i64, i64, i64, i32, i32, P, P, P, P, P, P]
    lib.moe_ffn_fused_noalloc.restype = st
    lib.moe_get_device_status.argtypes = [P, P]
    lib.moe_get_device_status.restype = st
    lib.moe_set_wait_timeout_ns.argtypes = [ctypes.c_uint64]
    lib.moe_set_wait_timeout_ns.restype = None
    lib.moe_set_fault_injection.argtypes = [i32, i32]
    lib.moe_set_fault_injection.restype = st
    lib.moe_quantize_weights_e4m3.argtypes = [P, i32, i64, i64, P, P, P]
    lib.moe_quantize_weights_e4m3.restype = st
    lib.moe_quantize_rows_e4m3.argtypes = [P, i64, i64, P, P, P, sz, P]
    lib.moe_quantize_rows_e4m3.restype = st
    lib.moe_grouped_gemm_e4m3.argtypes = [P, P, P, P, P, i32, i64, i64, i64, P, P, P, P, sz, P]
    lib.moe_grouped_gemm_e4m3.restype = st
    lib.moe_ffn_fused_fp8.argtypes = [P, P, P, P, P, P, i64, i64, i64, i32, i32, P, P, P, P, P, sz,
                                      P]
    lib.moe_ffn_fused_fp8.restype = st
    lib.moe_quantize_weights_mx.argtypes = [P, i32, i64, i64, P, P, P]
    lib.moe_quantize_weights_mx.restype = st
    lib.moe_quantize_rows_mx.argtypes = [P, i64, i64, P, P, P]
    lib.moe_quantize_rows_mx.restype = st
    lib.moe_grouped_gemm_swiglu_mx.argtypes = [P, P, P, i32, i64, i64, i64, P, P, P, sz, P]
    lib.moe_grouped_gemm_swiglu_mx.restype = st
    lib.moe_grouped_gemm_mx.argtypes = [P, P, P, P, P, i32, i64, i64, i64, P, P, P, P, sz, P]
    lib.moe_grouped_gemm_mx.restype = st
    lib.moe_ffn_fused_mx.argtypes = [P, P, P, P, P, P, i64, i64, i64, i32, i32, P, P, P, P, P, sz,
                                     P]
    lib.moe_ffn_fused_mx.restype = st
    lib.moe_set_stage_events.argtypes = [P]
    lib.moe_set_stage_events.restype = st
    lib.moe_last_error.restype = ctypes.c_char_p
    if path is None:
        _lib = lib
    return lib


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors passed to libmoe must be on the GPU")
    if not t.is_contiguous():
        raise ValueError("tensors passed to libmoe must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(status: int):
    if status != MOE_OK:
        raise MoEError(status, load().moe_last_error().decode())


def moe_abi_version() -> int:
    return int(load().moe_abi_version())


def moe_workspace_size(op: int, M: int, H: int, F: int, E: int, topk: int) -> int:
    return int(load().moe_workspace_size(op, M, H, F, E, topk))


def alloc_workspace(op: int, M: int, H: int, F: int, E: int, topk: int, device) -> torch.Tensor:
    """A zeroed uint8 workspace of the size the op needs (torch allocations are 256-byte aligned)."""
    n = moe_workspace_size(op, M, H, F, E, topk)
    return torch.zeros(n, dtype=torch.uint8, device=device)


def moe_route(logits, topk, topk_ids, topk_w, ws, stream=None):
    M, E = logits.shape
    if logits.dtype != torch.float32:
        raise ValueError("moe_route takes fp32 logits")
    _check(load().moe_route(_ptr(logits), M, E, topk, _ptr(topk_ids), _ptr(topk_w), _ptr(ws),
                            ws.numel(), _stream(stream)))


def moe_route_plan(logits, topk, topk_ids, topk_w, counts, offsets, perm, inv_perm, w_sorted, ws,
                   stream=None):
    M, E = logits.shape
    if logits.dtype != torch.float32:
        raise ValueError("moe_route_plan takes fp32 logits")
    _check(load().moe_route_plan(_ptr(logits), M, E, topk, _ptr(topk_ids), _ptr(topk_w),
                                 _ptr(counts), _ptr(offsets), _ptr(perm), _ptr(inv_perm),
                                 _ptr(w_sorted), _ptr(ws), ws.numel(), _stream(stream)))


def moe_plan(topk_ids, topk_w, E, counts, offsets, perm, inv_perm, w_sorted, ws, stream=None):
    M, topk = topk_ids.shape
    _check(load().moe_plan(_ptr(topk_ids), _ptr(topk_w), M, E, topk, _ptr(counts), _ptr(offsets),
                           _ptr(perm), _ptr(inv_perm), _ptr(w_sorted), _ptr(ws), ws.numel(),
                           _stream(stream)))


def moe_dispatch(x, perm, topk, xp, ws, stream=None):
    M, H = x.shape
    _check(load().moe_dispatch(_ptr(x), _ptr(perm), M, H, topk, _ptr(xp), _ptr(ws), ws.numel(),
                               _stream(stream)))


def moe_grouped_gemm(A, B, offsets, epi, C, ws, w_sorted=None, perm=None, stream=None):
    R, K = A.shape
    E, K2, N = B.shape
    if K2 != K:
        raise ValueError(f"A has K={K} but B has K={K2}")
    _check(load().moe_grouped_gemm(_ptr(A), _ptr(B), _ptr(offsets), E, R, K, N, epi,
                                   _ptr(w_sorted), _ptr(perm), _ptr(C), _ptr(ws), ws.numel(),
                                   _stream(stream)))


def moe_combine(y, inv_perm, topk_w, M, topk, out, ws, stream=None):
    """y is bf16 or fp32 [R, H] (the dtype of the tensor selects the C flag)."""
    H = y.shape[1]
    if y.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("moe_combine takes bf16 or fp32 rows")
    _check(load().moe_combine(_ptr(y), 1 if y.dtype == torch.float32 else 0, _ptr(inv_perm),
                              _ptr(topk_w), M, H, topk, _ptr(out), _ptr(ws), ws.numel(),
                              _stream(stream)))


def moe_ffn_fused(x, W1, W2, topk_ids, topk_w, out, counts, offsets, perm, ws, n_c=0,
                  stream=None):
    M, H = x.shape
    E, _, F2 = W1.shape
    topk = topk_ids.shape[1]
    _check(load().moe_ffn_fused(_ptr(x), _ptr(W1), _ptr(W2), _ptr(topk_ids), _ptr(topk_w), M, H,
                                F2 // 2, E, topk, n_c, _ptr(out), _ptr(counts), _ptr(offsets),
                                _ptr(perm), _ptr(ws), ws.numel(), _stream(stream)))


def moe_combine_add(y, inv_perm, topk_w, add, alpha, beta, M, topk, out, ws, stream=None):
    """moe_combine with the GemmAdd epilogue: out = bf16(alpha * sum + beta * add)."""
    H = y.shape[1]
    if y.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("moe_combine_add takes bf16 or fp32 rows")
    _check(load().moe_combine_add(_ptr(y), 1 if y.dtype == torch.float32 else 0, _ptr(inv_perm),
                                  _ptr(topk_w), _ptr(add), float(alpha), float(beta), M, H, topk,
                                  _ptr(out), _ptr(ws), ws.numel(), _stream(stream)))


def moe_ffn_fused_add(x, W1, W2, topk_ids, topk_w, add, alpha, beta, out, counts, offsets, perm,
                      ws, stream=None):
    """The layer with the GemmAdd epilogue: out = bf16(alpha * layer(x) + beta * add)."""
    M, H = x.shape
    E, _, F2 = W1.shape
    topk = topk_ids.shape[1]
    _check(load().moe_ffn_fused_add(_ptr(x), _ptr(W1), _ptr(W2), _ptr(topk_ids), _ptr(topk_w),
                                    _ptr(add), float(alpha), float(beta), M, H, F2 // 2, E, topk,
                                    _ptr(out), _ptr(counts), _ptr(offsets), _ptr(perm), _ptr(ws),
                                    ws.numel(), _stream(stream)))


def moe_ffn_fused_noalloc(x, W1, W2, topk_ids, topk_w, out, counts, offsets, perm, status=None,
                          stream=None):
    """The layer without a workspace: intermediates in the library's own device scratch."""
    M, H = x.shape
    E, _, F2 = W1.shape
    topk = topk_ids.shape[1]
    _check(load().moe_ffn_fused_noalloc(_ptr(x), _ptr(W1), _ptr(W2), _ptr(topk_ids), _ptr(topk_w),
                                        M, H, F2 // 2, E, topk, _ptr(out), _ptr(counts),
                                        _ptr(offsets), _ptr(perm), _ptr(status), _stream(stream)))


def moe_quantize_weights_e4m3(W, Wq, scale, stream=None):
    """W bf16 [E, K, N] -> Wq uint8 [E, N, K] (E4M3 codes, K contiguous), scale fp32 [E, N]."""
    E, K, N = W.shape
    _check(load().moe_quantize_weights_e4m3(_ptr(W), E, K, N, _ptr(Wq), _ptr(scale),
                                            _stream(stream)))


def moe_quantize_rows_e4m3(A, Aq, scale, ws, stream=None):
    """A bf16 [R, K] -> Aq uint8 [R, K] (E4M3 codes), scale fp32 [R]."""
    R, K = A.shape
    _check(load().moe_quantize_rows_e4m3(_ptr(A), R, K, _ptr(Aq), _ptr(scale), _ptr(ws),
                                         ws.numel(), _stream(stream)))


def moe_grouped_gemm_e4m3(Aq, a_scale, BqT, b_scale, offsets, C, ws, w_sorted=None, perm=None,
                          stream=None):
    """C fp32 [R, N] from E4M3 Aq [R, K] and BqT [E, N, K] (see include/moe.h)."""
    R, K = Aq.shape
    E, N, K2 = BqT.shape
    if K2 != K:
        raise ValueError(f"Aq has K={K} but BqT has K={K2}")
    _check(load().moe_grouped_gemm_e4m3(_ptr(Aq), _ptr(a_scale), _ptr(BqT), _ptr(b_scale),
                                        _ptr(offsets), E, R, K, N, _ptr(w_sorted), _ptr(perm),
                                        _ptr(C), _ptr(ws), ws.numel(), _stream(stream)))


def moe_ffn_fused_fp8(x, W1, W2q, w2_scale, topk_ids, topk_w, out, counts, offsets, perm, ws,
                      stream=None):
    """The layer with the E4M3 down projection; W2q / w2_scale from moe_quantize_weights_e4m3."""
    M, H = x.shape
    E, _, F2 = W1.shape
    topk = topk_ids.shape[1]
    _check(load().moe_ffn_fused_fp8(_ptr(x), _ptr(W1), _ptr(W2q), _ptr(w2_scale), _ptr(topk_ids),
                                    _ptr(topk_w), M, H, F2 // 2, E, topk, _ptr(out), _ptr(counts),
                                    _ptr(offsets), _ptr(perm), _ptr(ws), ws.numel(),
                                    _stream(stream)))


def moe_quantize_weights_mx(W, BqT, sf, stream=None):
    """W bf16 [E, K, N] -> BqT uint8 [E, N, K] (E4M3 codes, K contiguous), sf uint8
    [E, N, K / 32] (block scale codes e + 127)."""
    E, K, N = W.shape
    _check(load().moe_quantize_weights_mx(_ptr(W), E, K, N, _ptr(BqT), _ptr(sf), _stream(stream)))


def moe_quantize_rows_mx(A, Aq, sf, stream=None):
    """A bf16 [R, K] -> Aq uint8 [R, K] (E4M3 codes), sf uint8 [R, K / 32]."""
    R, K = A.shape
    _check(load().moe_quantize_rows_mx(_ptr(A), R, K, _ptr(Aq), _ptr(sf), _stream(stream)))


def moe_grouped_gemm_swiglu_mx(A, B, offsets, hq, h_sf, ws, stream=None):
    """GEMM1 + SwiGLU with h quantised in the epilogue: hq uint8 [R, N2 / 2], h_sf
    uint8 [R, N2 / 64]."""
    R, K = A.shape
    E, K2, N2 = B.shape
    if K2 != K:
        raise ValueError(f"A has K={K} but B has K={K2}")
    _check(load().moe_grouped_gemm_swiglu_mx(_ptr(A), _ptr(B), _ptr(offsets), E, R, K, N2,
                                             _ptr(hq), _ptr(h_sf), _ptr(ws), ws.numel(),
                                             _stream(stream)))


def moe_grouped_gemm_mx(Aq, a_sf, BqT, b_sf, offsets, C, ws, w_sorted=None, perm=None,
                        stream=None):
    """C fp32 [R, N] from block-scaled E4M3 Aq [R, K] and BqT [E, N, K] (see include/moe.h)."""
    R, K = Aq.shape
    E, N, K2 = BqT.shape
    if K2 != K:
        raise ValueError(f"Aq has K={K} but BqT has K={K2}")
    _check(load().moe_grouped_gemm_mx(_ptr(Aq), _ptr(a_sf), _ptr(BqT), _ptr(b_sf), _ptr(offsets),
                                      E, R, K, N, _ptr(w_sorted), _ptr(perm), _ptr(C), _ptr(ws),
                                      ws.numel(), _stream(stream)))


def moe_ffn_fused_mx(x, W1, W2q, w2_sf, topk_ids, topk_w, out, counts, offsets, perm, ws,
                     stream=None):
    """The layer with the block-scaled E4M3 down projection; W2q / w2_sf from
    moe_quantize_weights_mx."""
    M, H = x.shape
    E, _, F2 = W1.shape
    topk = topk_ids.shape[1]
    _check(load().moe_ffn_fused_mx(_ptr(x), _ptr(W1), _ptr(W2q), _ptr(w2_sf), _ptr(topk_ids),
                                   _ptr(topk_w), M, H, F2 // 2, E, topk, _ptr(out), _ptr(counts),
                                   _ptr(offsets), _ptr(perm), _ptr(ws), ws.numel(),
                                   _stream(stream)))


def moe_get_device_status(ws, stream=None) -> int:
    """Synchronises the stream; returns the device status word and clears it."""
    return int(load().moe_get_device_status(_ptr(ws), _stream(stream)))


def moe_set_wait_timeout_ns(ns: int) -> None:
    load().moe_set_wait_timeout_ns(int(ns))


def moe_set_fault_injection(kind: int, index: int = 0) -> None:
    """Test hook (see include/moe.h): 1 = withhold one m-tile's dispatch flag, 0 = off."""
    _check(load().moe_set_fault_injection(int(kind), int(index)))


def moe_set_stage_events(events) -> None:
    """Stage timing of moe_ffn_fused (see include/moe.h): `events` is None (off) or
    six torch.cuda.Event(enable_timing=True); each is recorded once here so that its
    CUDA event exists.  The caller keeps the events alive while they are set."""
    if events is None:
        _check(load().moe_set_stage_events(None))
        return
    if len(events) != 6:
        raise ValueError("moe_set_stage_events takes six events")
    for e in events:
        if e.cuda_event == 0:
            e.record()
    arr = (ctypes.c_void_p * 6)(*[ctypes.c_void_p(e.cuda_event) for e in events])
    _check(load().moe_set_stage_events(arr))


def moe_last_error() -> str:
    return load().moe_last_error().decode()
