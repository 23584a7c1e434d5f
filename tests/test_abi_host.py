"""The C ABI on the host: the library loads, exports every symbol include/moe.h
declares, and rejects bad arguments before launching anything (no GPU needed:
validation runs before the first CUDA call)."""
import ctypes
import os
import re

import pytest

from grouped_gemm_plan_b200 import binding as B
from grouped_gemm_plan_b200 import build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return B.load()


def header_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_binding_exports():
    assert header_functions() == sorted(B.EXPORTS)


def test_every_declared_symbol_is_exported(lib):
    raw = ctypes.CDLL(B.library_path())
    for name in header_functions():
        assert hasattr(raw, name), f"{name} missing from libmoe.so"


def test_abi_version(lib):
    assert B.moe_abi_version() == 1


def test_workspace_sizes(lib):
    for op in (B.OP_DISPATCH, B.OP_GROUPED_GEMM, B.OP_COMBINE):
        assert B.moe_workspace_size(op, 4096, 4096, 14336, 8, 2) == 256
    # the plan keeps up to 256 per-chunk histograms of E + 1 counters
    assert B.moe_workspace_size(B.OP_PLAN, 4096, 0, 0, 8, 2) == 256 + 256 * 9 * 4
    assert B.moe_workspace_size(B.OP_PLAN, 4096, 0, 0, 1024, 2) == 256 + 256 * 1025 * 4
    R, H, F = 8192, 4096, 14336
    fused = B.moe_workspace_size(B.OP_FFN_FUSED, 4096, H, F, 8, 2)
    assert fused >= 256 + R * H * 2 + R * F * 2 + R * H * 4 + R * 4
    assert B.moe_workspace_size(B.OP_FFN_FUSED, 0, H, F, 8, 2) >= 256 + 256 * 9 * 4


FAKE = ctypes.c_void_p(0x10000)        # never dereferenced: validation fails first
FAKE_WS = ctypes.c_void_p(0x20000)     # 256-byte aligned


def _err(lib):
    return lib.moe_last_error().decode()


def test_plan_validation(lib):
    # topk > E
    st = lib.moe_plan(FAKE, FAKE, 4, 2, 3, FAKE, FAKE, FAKE, None, None, FAKE_WS, 256, None)
    assert st == 1 and "topk" in _err(lib)
    # E too large
    st = lib.moe_plan(FAKE, FAKE, 4, 2000, 2, FAKE, FAKE, FAKE, None, None, FAKE_WS, 256, None)
    assert st == 2
    # negative M
    assert lib.moe_plan(FAKE, FAKE, -1, 8, 2, FAKE, FAKE, FAKE, None, None, FAKE_WS, 256, None) == 1
    # null counts
    assert lib.moe_plan(FAKE, FAKE, 4, 8, 2, None, FAKE, FAKE, None, None, FAKE_WS, 256, None) == 1
    # workspace too small / misaligned / null
    assert lib.moe_plan(FAKE, FAKE, 4, 8, 2, FAKE, FAKE, FAKE, None, None, FAKE_WS, 100, None) == 4
    assert lib.moe_plan(FAKE, FAKE, 4, 8, 2, FAKE, FAKE, FAKE, None, None,
                        ctypes.c_void_p(0x20010), 256, None) == 7
    assert lib.moe_plan(FAKE, FAKE, 4, 8, 2, FAKE, FAKE, FAKE, None, None, None, 256, None) == 1
    # w_sorted without topk_w
    assert lib.moe_plan(FAKE, None, 4, 8, 2, FAKE, FAKE, FAKE, None, FAKE, FAKE_WS, 256, None) == 1


def test_route_validation(lib):
    r = lib.moe_route
    assert r(FAKE, 4, 8, 9, FAKE, FAKE, FAKE_WS, 256, None) == 1        # topk > E
    assert r(FAKE, 4, 64, 33, FAKE, FAKE, FAKE_WS, 256, None) == 2      # topk > 32
    assert r(FAKE, 4, 2000, 2, FAKE, FAKE, FAKE_WS, 256, None) == 2     # E too large
    assert r(None, 4, 8, 2, FAKE, FAKE, FAKE_WS, 256, None) == 1        # null logits
    assert r(None, 0, 8, 2, None, None, FAKE_WS, 256, None) == 0        # M = 0: no-op


def test_gemm_validation(lib):
    g = lib.moe_grouped_gemm
    ok = dict(E=8, R=256, K=256, N=512)

    def call(**kw):
        a = {**ok, **kw}
        return g(kw.get("A", FAKE), FAKE, FAKE, a["E"], a["R"], a["K"], a["N"], kw.get("epi", 0),
                 kw.get("w", None), kw.get("perm", None), FAKE, FAKE_WS, 256, None)
    assert call(K=100) == 2
    assert call(N=96) == 2
    assert call(epi=1, N=192) == 2            # N/2 = 96 not a multiple of 64
    assert call(epi=7) == 1
    assert call(E=0) == 2
    assert call(R=-1) == 1
    assert call(epi=2) == 1                    # scatter without w_sorted/perm
    assert call(A=ctypes.c_void_p(0x10008)) == 7


def test_dispatch_combine_validation(lib):
    assert lib.moe_dispatch(FAKE, FAKE, 4, 100, 2, FAKE, FAKE_WS, 256, None) == 2   # H % 8
    assert lib.moe_dispatch(FAKE, FAKE, 4, 64, 0, FAKE, FAKE_WS, 256, None) == 1    # topk
    assert lib.moe_dispatch(ctypes.c_void_p(0x10004), FAKE, 4, 64, 2, FAKE, FAKE_WS, 256, None) == 7
    assert lib.moe_dispatch(None, FAKE, 4, 64, 2, FAKE, FAKE_WS, 256, None) == 1
    assert lib.moe_combine(FAKE, 0, FAKE, FAKE, 4, 64, 2, None, FAKE_WS, 256, None) == 1
    assert lib.moe_combine(FAKE, 0, FAKE, FAKE, 4, 64, 33, FAKE, FAKE_WS, 256, None) == 1
    assert lib.moe_combine(FAKE, 2, FAKE, FAKE, 4, 64, 2, FAKE, FAKE_WS, 256, None) == 1
    # M = 0 is a no-op even with null data pointers
    assert lib.moe_dispatch(None, None, 0, 64, 2, None, FAKE_WS, 256, None) == 0
    assert lib.moe_combine(None, 0, None, None, 0, 64, 2, None, FAKE_WS, 256, None) == 0


def test_fused_validation(lib):
    f = lib.moe_ffn_fused
    need = B.moe_workspace_size(B.OP_FFN_FUSED, 16, 128, 128, 4, 2)
    args = lambda **kw: [FAKE, FAKE, FAKE, FAKE, FAKE, kw.get("M", 16), kw.get("H", 128),
                         kw.get("F", 128), kw.get("E", 4), kw.get("topk", 2), kw.get("n_c", 0),
                         FAKE, FAKE, FAKE, FAKE, FAKE_WS, kw.get("ws", need), None]
    assert f(*args(H=100)) == 2
    assert f(*args(F=96)) == 2
    assert f(*args(topk=5)) == 1
    assert f(*args(n_c=-2)) == 1
    assert lib.moe_set_fault_injection(7, 0) == 1
    assert lib.moe_set_fault_injection(0, 0) == 0
    assert f(*args(ws=need - 1)) == 4


def test_gemm_add_validation(lib):
    # moe_combine_add: beta != 0 needs the added tensor; it must be 16-byte aligned
    ca = lib.moe_combine_add
    assert ca(FAKE, 0, FAKE, FAKE, None, 1.0, 1.0, 4, 64, 2, FAKE, FAKE_WS, 256, None) == 1
    assert ca(FAKE, 0, FAKE, FAKE, ctypes.c_void_p(0x10004), 1.0, 1.0, 4, 64, 2, FAKE, FAKE_WS,
              256, None) == 7
    assert ca(FAKE, 0, FAKE, FAKE, FAKE, 1.0, 1.0, 4, 100, 2, FAKE, FAKE_WS, 256, None) == 2
    assert ca(None, 0, None, None, None, 1.0, 1.0, 0, 64, 2, None, FAKE_WS, 256, None) == 0
    # moe_ffn_fused_add: the layer's checks, then the added tensor's
    fa = lib.moe_ffn_fused_add
    need = B.moe_workspace_size(B.OP_FFN_FUSED, 16, 128, 128, 4, 2)
    args = lambda **kw: [FAKE, FAKE, FAKE, FAKE, FAKE, kw.get("add", FAKE), kw.get("alpha", 1.0),
                         kw.get("beta", 1.0), 16, kw.get("H", 128), 128, 4, 2, FAKE, FAKE, FAKE,
                         FAKE, FAKE_WS, kw.get("ws", need), None]
    assert fa(*args(H=100)) == 2
    assert fa(*args(add=None)) == 1
    assert "add is NULL" in B.moe_last_error()
    assert fa(*args(add=ctypes.c_void_p(0x10004))) == 7
    assert fa(*args(ws=need - 1)) == 4


def test_fp8_validation(lib):
    qw = lib.moe_quantize_weights_e4m3
    assert qw(FAKE, 0, 64, 64, FAKE, FAKE, None) == 2               # E
    assert qw(FAKE, 2, 40, 64, FAKE, FAKE, None) == 2               # K % 16
    assert qw(None, 2, 64, 64, FAKE, FAKE, None) == 1               # null W
    assert qw(ctypes.c_void_p(0x10008), 2, 64, 64, FAKE, FAKE, None) == 7
    qr = lib.moe_quantize_rows_e4m3
    assert qr(FAKE, 4, 96, FAKE, FAKE, FAKE_WS, 256, None) == 2     # K % 64
    assert qr(FAKE, 4, 32832, FAKE, FAKE, FAKE_WS, 256, None) == 2  # K > 32768
    assert qr(FAKE, -1, 64, FAKE, FAKE, FAKE_WS, 256, None) == 1
    assert qr(FAKE, 4, 64, FAKE, FAKE, FAKE_WS, 100, None) == 4     # workspace
    assert qr(None, 0, 64, None, None, FAKE_WS, 256, None) == 0     # R = 0: no-op
    g = lib.moe_grouped_gemm_e4m3
    args = lambda **kw: [kw.get("A", FAKE), FAKE, FAKE, FAKE, FAKE, kw.get("E", 4), kw.get("R", 64),
                         kw.get("K", 128), kw.get("N", 256), None, None, FAKE, FAKE_WS, 256, None]
    assert g(*args(K=100)) == 2
    assert g(*args(N=96)) == 2
    assert g(*args(E=0)) == 2
    assert g(*args(R=-1)) == 1
    assert g(*args(A=None)) == 1
    assert g(*args(A=ctypes.c_void_p(0x10008))) == 7
    f = lib.moe_ffn_fused_fp8
    need = B.moe_workspace_size(B.OP_FFN_FP8, 16, 128, 128, 4, 2)
    assert need >= B.moe_workspace_size(B.OP_FFN_FUSED, 16, 128, 128, 4, 2) + 32 * 128
    fa = lambda **kw: [FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, kw.get("M", 16), kw.get("H", 128),
                       kw.get("F", 128), kw.get("E", 4), kw.get("topk", 2), FAKE, FAKE, FAKE, FAKE,
                       FAKE_WS, kw.get("ws", need), None]
    assert f(*fa(H=100)) == 2
    assert f(*fa(F=32832)) == 2
    assert f(*fa(topk=5)) == 1
    assert f(*fa(ws=need - 1)) == 4


def test_mx_validation(lib):
    qw = lib.moe_quantize_weights_mx
    assert qw(FAKE, 0, 64, 64, FAKE, FAKE, None) == 2               # E
    assert qw(FAKE, 2, 48, 64, FAKE, FAKE, None) == 2               # K % 32
    assert qw(FAKE, 2, 64, 40, FAKE, FAKE, None) == 2               # N % 16
    assert qw(FAKE, 2, 64, 64, FAKE, None, None) == 1               # null sf
    assert qw(ctypes.c_void_p(0x10008), 2, 64, 64, FAKE, FAKE, None) == 7
    qr = lib.moe_quantize_rows_mx
    assert qr(FAKE, 4, 48, FAKE, FAKE, None) == 2                   # K % 32
    assert qr(FAKE, -1, 64, FAKE, FAKE, None) == 1
    assert qr(FAKE, 4, 64, None, FAKE, None) == 1
    assert qr(None, 0, 64, None, None, None) == 0                   # R = 0: no-op
    sw = lib.moe_grouped_gemm_swiglu_mx
    swa = lambda **kw: [kw.get("A", FAKE), FAKE, FAKE, kw.get("E", 4), kw.get("R", 64),
                        kw.get("K", 128), kw.get("N2", 256), FAKE, kw.get("sf", FAKE), FAKE_WS,
                        256, None]
    assert sw(*swa(N2=192)) == 2                                    # N2 % 128
    assert sw(*swa(K=96)) == 2                                      # K % 64
    assert sw(*swa(E=0)) == 2
    assert sw(*swa(A=None)) == 1
    assert sw(*swa(sf=ctypes.c_void_p(0x10001))) == 7               # 2-byte scale stores
    g = lib.moe_grouped_gemm_mx
    need = B.moe_workspace_size(B.OP_GEMM_MX, 64, 256, 128, 4, 1)
    assert need >= 256 + (64 // 256 + 4) * 2 * 1 * 512 + 4 * 1 * 1 * 2 * 512
    ga = lambda **kw: [kw.get("A", FAKE), FAKE, FAKE, FAKE, FAKE, kw.get("E", 4), kw.get("R", 64),
                       kw.get("K", 128), kw.get("N", 256), None, None, FAKE, FAKE_WS,
                       kw.get("ws", need), None]
    assert g(*ga(K=48)) == 2                                        # K % 32
    assert g(*ga(N=96)) == 2                                        # N % 64
    assert g(*ga(R=-1)) == 1
    assert g(*ga(A=None)) == 1
    assert g(*ga(ws=need - 1)) == 4
    assert g(*ga(A=ctypes.c_void_p(0x10008))) == 7
    f = lib.moe_ffn_fused_mx
    fneed = B.moe_workspace_size(B.OP_FFN_MX, 16, 128, 128, 4, 2)
    fa = lambda **kw: [FAKE, FAKE, FAKE, kw.get("sf", FAKE), FAKE, FAKE, kw.get("M", 16),
                       kw.get("H", 128), kw.get("F", 128), kw.get("E", 4), kw.get("topk", 2), FAKE,
                       FAKE, FAKE, FAKE, FAKE_WS, kw.get("ws", fneed), None]
    assert f(*fa(H=100)) == 2
    assert f(*fa(F=96)) == 2
    assert f(*fa(topk=5)) == 1
    assert f(*fa(sf=None)) == 1
    assert f(*fa(ws=fneed - 1)) == 4


def test_stage_events_switch(lib):
    # off is always accepted; no CUDA call is made until a layer runs
    assert lib.moe_set_stage_events(None) == 0
    assert lib.moe_set_stage_events(None) == 0


def test_binding_rejects_cpu_tensors(lib):
    import torch
    x = torch.zeros(4, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        B.moe_dispatch(x, torch.zeros(8, dtype=torch.int32), 2, x, torch.zeros(256, dtype=torch.uint8))


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(ImportError):
        B.load(str(tmp_path / "nope.so"))
