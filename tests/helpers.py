"""Shared test helpers: tolerances, guarded output buffers, case construction."""
from __future__ import annotations

import numpy as np
import torch

# The layer's floating-point bar: relative Frobenius error <= 1e-2 and max abs
# error <= 2e-2 * rms(reference), element by element against the fp64 oracle.
REL_FRO = 1e-2
MAX_ABS_RMS = 2e-2


def half_ulp_bf16(r: np.ndarray) -> np.ndarray:
    """Half a bf16 unit in the last place at |r|: the error of a correctly rounded
    bf16 value (bf16 keeps 8 significant bits)."""
    a = np.abs(r)
    out = np.zeros_like(a)
    nz = a >= 2.0 ** -126
    out[nz] = np.exp2(np.floor(np.log2(a[nz])) - 8)
    return out


# Elements allowed beyond the literal per-element bar 2e-2 * rms(ref) (without
# the half-ulp allowance), as a fraction of all elements: the allowance exists for
# the bf16 rounding of the largest outputs, which are rare; accumulation error
# that pushed many elements past the literal bar would show up in this count.
MAX_BEYOND_LITERAL_FRAC = 1e-4


def check_close(got, ref: np.ndarray, what: str = "", rel_fro: float = REL_FRO,
                max_abs_rms: float = MAX_ABS_RMS, ulps: float = 1.0,
                max_beyond_literal_frac: float | None = None) -> dict:
    """The layer's bar for a bf16 output against the fp64 oracle.

    relative Frobenius error <= 1e-2, and per element
        |got - ref| <= 2e-2 * rms(ref) + ulps * half_ulp_bf16(ref)
    The second term is the output's own representation error: a bf16 output can
    only be as close as the nearest bf16 value, which is up to 2^-8 |ref| away --
    more than 2e-2 * rms(ref) for the largest elements.  ulps = 2 is used when the
    reference is itself a bf16 result (two roundings).

    The count of elements beyond the literal bar 2e-2 * rms(ref) is reported
    (``beyond_literal``).  For a single bf16 rounding (ulps = 1, the layer output
    against the oracle) it is held to MAX_BEYOND_LITERAL_FRAC of all elements, so
    the half-ulp allowance cannot hide accumulation error spread over many
    elements; comparisons with more roundings only report it unless
    ``max_beyond_literal_frac`` is given.
    """
    if max_beyond_literal_frac is None:
        max_beyond_literal_frac = MAX_BEYOND_LITERAL_FRAC if ulps == 1.0 else float("inf")
    g = got.detach().to("cpu", torch.float64).numpy() if isinstance(got, torch.Tensor) else \
        np.asarray(got, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, f"{what}: shape {g.shape} vs {r.shape}"
    assert np.all(np.isfinite(g)), f"{what}: non-finite values"
    if r.size == 0:
        return {"rel_fro": 0.0, "max_abs": 0.0, "rms": 0.0}
    diff = np.abs(g - r)
    nr = np.linalg.norm(r)
    rel = np.linalg.norm(g - r) / nr if nr > 0 else np.linalg.norm(g - r)
    rms = float(np.sqrt(np.mean(r * r)))
    bound = max_abs_rms * rms + ulps * half_ulp_bf16(r)
    beyond = int((diff > max_abs_rms * rms).sum())
    stats = {"rel_fro": float(rel), "max_abs": float(diff.max()), "rms": rms,
             "max_abs_over_rms": float(diff.max() / max(rms, 1e-300)),
             "max_excess_over_bound": float((diff - bound).max()),
             "beyond_literal": beyond, "elements": int(r.size)}
    assert rel <= rel_fro, f"{what}: relative Frobenius error {rel:.3e} > {rel_fro} {stats}"
    assert bool(np.all(diff <= bound)), \
        f"{what}: {int((diff > bound).sum())} elements beyond 2e-2*rms + half-ulp {stats}"
    assert beyond <= max_beyond_literal_frac * r.size, \
        f"{what}: {beyond} of {r.size} elements beyond the literal 2e-2*rms {stats}"
    return stats


# Stage outputs that are one rounding of an fp32 accumulator (a GEMM tile, a
# SwiGLU value) are held element by element to 2^-8 |ref| (twice the largest bf16
# rounding error, 2^-9 relative) plus 2e-3 * rms(ref) for the fp32 accumulation
# error near zero; fp32 stage outputs to 1e-4 |ref| + 1e-4 * rms(ref).
STAGE_REL = {"bf16": 2.0 ** -8, "fp32": 1e-4}
STAGE_ABS = {"bf16": 2e-3, "fp32": 1e-4}


def check_stage(got, ref: np.ndarray, what: str = "", kind: str = "bf16") -> dict:
    g = got.detach().to("cpu", torch.float64).numpy()
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, f"{what}: shape {g.shape} vs {r.shape}"
    assert np.all(np.isfinite(g)), f"{what}: non-finite values"
    if r.size == 0:
        return {}
    rms = float(np.sqrt(np.mean(r * r)))
    err = np.abs(g - r)
    bound = STAGE_REL[kind] * np.abs(r) + STAGE_ABS[kind] * rms
    worst = np.unravel_index(np.argmax(err - bound), err.shape)
    rel = float(np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-300))
    stats = {"rel_fro": rel, "max_abs": float(err.max()), "rms": rms,
             "worst": (tuple(int(i) for i in worst), float(g[worst]), float(r[worst]))}
    assert rel <= REL_FRO, f"{what}: relative Frobenius error {rel:.3e} {stats}"
    assert bool(np.all(err <= bound)), f"{what}: {int((err > bound).sum())} elements out of bound {stats}"
    return stats


def guarded_empty(shape, dtype, device, pad_bytes: int = 4096, fill: int = 0x5A):
    """An output tensor with sentinel bytes before and after it.

    Returns (view, check) -- call check() after the kernel to assert that no byte
    outside the view changed.
    """
    n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
    raw = torch.full((pad_bytes + n + pad_bytes,), fill, dtype=torch.uint8, device=device)
    view = raw[pad_bytes:pad_bytes + n].view(dtype).view(*shape)

    def check():
        head = raw[:pad_bytes]
        tail = raw[pad_bytes + n:]
        assert bool((head == fill).all()), "write before the output buffer"
        assert bool((tail == fill).all()), "write after the output buffer"
    return view, check


def routing_case(M, E, topk, kind="skewed", seed=0, std=0.05):
    from grouped_gemm_plan_b200 import workload as wl
    w = wl.Workload("case", M, 64, 64, E, topk, kind, std, seed)
    return wl.make_routing(w)


def layer_case(M, H, F, E, topk, kind="skewed", seed=0, std=0.05):
    from grouped_gemm_plan_b200 import workload as wl
    w = wl.Workload("case", M, H, F, E, topk, kind, std, seed)
    x = wl.make_x(w)
    W1, W2 = wl.make_weights(w)
    ids, tw = wl.make_routing(w)
    return w, x, W1, W2, ids, tw
