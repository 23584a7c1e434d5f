"""Shared test helpers: tolerances, guarded output buffers, case construction."""
from __future__ import annotations

import numpy as np
import torch

# The layer's floating-point bar: relative Frobenius error <= 1e-2 and max abs
# error <= 2e-2 * rms(reference), element by element against the fp64 oracle.
REL_FRO = 1e-2
MAX_ABS_RMS = 2e-2


def check_close(got, ref: np.ndarray, what: str = "", rel_fro: float = REL_FRO,
                max_abs_rms: float = MAX_ABS_RMS) -> dict:
    g = got.detach().to("cpu", torch.float64).numpy() if isinstance(got, torch.Tensor) else \
        np.asarray(got, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, f"{what}: shape {g.shape} vs {r.shape}"
    assert np.all(np.isfinite(g)), f"{what}: non-finite values"
    if r.size == 0:
        return {"rel_fro": 0.0, "max_abs": 0.0, "rms": 0.0}
    diff = g - r
    nr = np.linalg.norm(r)
    rel = np.linalg.norm(diff) / nr if nr > 0 else np.linalg.norm(diff)
    rms = float(np.sqrt(np.mean(r * r)))
    mx = float(np.abs(diff).max())
    stats = {"rel_fro": float(rel), "max_abs": mx, "rms": rms}
    assert rel <= rel_fro, f"{what}: relative Frobenius error {rel:.3e} > {rel_fro} {stats}"
    assert mx <= max_abs_rms * max(rms, 1e-30), f"{what}: max abs error {mx:.3e} > {max_abs_rms}*rms {stats}"
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
