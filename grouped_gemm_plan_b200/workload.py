"""Seeded synthetic inputs for the MoE SwiGLU FFN layer.

This module holds no arithmetic of the layer itself: it only draws the inputs a
caller would hand to the layer (token activations, expert weights, routed expert
ids and gate weights).  Both the CPU oracle tests and the CUDA path read their
inputs from here, so a test compares the two on identical bytes.

Shapes follow the model table of the COMET paper review ("COMET: Fine-grained
Computation-communication Overlapping for Mixture-of-Experts", section 5.1, test
model configurations: Mixtral 8x7B, Qwen2-MoE-2.7B, Phi-3.5-MoE; its N is our
hidden size H and its K our FFN width F) and the wide top-k case of the PTO
MegaMoE article ("PTO MoE算子实战 ...", section 实测性能: K7168/N4096, topK 8, 16
experts).  Load distributions follow the COMET review, section 5.6.2 (std=0 is a
uniform load, std=0.05 a heavy skew, 0.032 the production average).

Recipe (every draw comes from its own child stream of ``SeedSequence(seed)``, so
each tensor can be regenerated alone):
  stream 0: x ~ N(0, 1), [M, H]
  stream 1+e: W1[e] ~ N(0, 1) / sqrt(H), [H, 2F]  (columns [0,F) gate, [F,2F) up)
  stream 1+E+e: W2[e] ~ N(0, 1) / sqrt(F), [F, H]
  stream 1+2E: routing (expert ids)
  stream 2+2E: gate logits ~ N(0, 1), [M, topk]; w = softmax over k (fp64, then fp32)
All floating tensors are drawn in fp32 and rounded to bf16 (round to nearest even).

Routing kinds:
  uniform   every token draws topk distinct experts, all subsets equally likely
  balanced  r = permutation(M) mod E, ids[t, k] = (r_t + k) mod E: exactly M*topk/E
            rows per expert when E divides M
  skewed    p_e = max(1e-4, 1/E + std * z_e), z ~ N(0,1)^E, renormalised; topk
            distinct experts drawn without replacement with probability
            proportional to p (Gumbel-top-k: keys log p_e + Gumbel noise, the topk
            largest keys in descending order are the draw order)
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    M: int          # tokens
    H: int          # hidden size
    F: int          # FFN width (W1 has 2F columns: gate | up)
    E: int          # experts
    topk: int       # experts per token
    routing: str    # "uniform" | "balanced" | "skewed"
    std: float      # per-expert probability std for "skewed"
    seed: int

    @property
    def R(self) -> int:
        return self.M * self.topk

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)

    def flops(self) -> int:
        """Useful FLOPs of the two contractions: GEMM1 2*R*H*2F + GEMM2 2*R*F*H."""
        return 6 * self.R * self.H * self.F


_WIDE = dict(H=7168, F=4096, E=16, topk=8, routing="skewed", std=0.032)

WORKLOADS: dict[str, Workload] = {
    "tiny": Workload("tiny", 256, 256, 512, 8, 2, "uniform", 0.0, 0),
    "mixtral": Workload("mixtral", 4096, 4096, 14336, 8, 2, "balanced", 0.0, 1),
    "qwen2": Workload("qwen2", 8192, 2048, 1408, 64, 4, "skewed", 0.032, 2),
    "phi35": Workload("phi35", 16384, 4096, 6400, 16, 2, "skewed", 0.05, 3),
    "wide16": Workload("wide16", 16, seed=16, **_WIDE),
    "wide128": Workload("wide128", 128, seed=128, **_WIDE),
    "wide512": Workload("wide512", 512, seed=512, **_WIDE),
    "wide2048": Workload("wide2048", 2048, seed=2048, **_WIDE),
    # profiling size: the Mixtral expert shape with two experts (0.7 GB of weights,
    # still far above L2), used for single-kernel hardware-counter captures
    "mixtral_prof": Workload("mixtral_prof", 2048, 4096, 14336, 2, 2, "balanced", 0.0, 101),
    # the Qwen2-MoE expert shape and load with 16 of its 64 experts (and a quarter of
    # its tokens, so experts keep their rows): 0.28 GB of weights, above L2
    "qwen2_prof": Workload("qwen2_prof", 2048, 2048, 1408, 16, 4, "skewed", 0.032, 202),
    # the Phi-3.5-MoE expert shape with 4 of its 16 experts, 4096 rows each
    # (balanced): 0.63 GB of weights; x and the dispatched rows (0.2 GB) above L2
    "phi35_prof": Workload("phi35_prof", 8192, 4096, 6400, 4, 2, "balanced", 0.0, 303),
}


def _streams(wl: Workload) -> list[np.random.SeedSequence]:
    return np.random.SeedSequence(wl.seed).spawn(3 + 2 * wl.E)


def _bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def make_x(wl: Workload) -> torch.Tensor:
    """Token activations, bf16 [M, H] on the CPU."""
    rng = np.random.default_rng(_streams(wl)[0])
    return _bf16(rng.standard_normal((wl.M, wl.H), dtype=np.float32))


def make_expert_w1(wl: Workload, e: int) -> torch.Tensor:
    rng = np.random.default_rng(_streams(wl)[1 + e])
    a = rng.standard_normal((wl.H, 2 * wl.F), dtype=np.float32)
    a *= np.float32(1.0 / np.sqrt(wl.H))
    return _bf16(a)


def make_expert_w2(wl: Workload, e: int) -> torch.Tensor:
    rng = np.random.default_rng(_streams(wl)[1 + wl.E + e])
    a = rng.standard_normal((wl.F, wl.H), dtype=np.float32)
    a *= np.float32(1.0 / np.sqrt(wl.F))
    return _bf16(a)


def make_weights(wl: Workload, out_w1: torch.Tensor | None = None,
                 out_w2: torch.Tensor | None = None,
                 threads: int = 1) -> tuple[torch.Tensor, torch.Tensor]:
    """Expert weights W1 bf16 [E, H, 2F] and W2 bf16 [E, F, H].

    ``out_w1``/``out_w2`` may be preallocated tensors (any device) that are filled
    expert by expert.  With ``threads`` > 1 the experts' matrices are drawn by a
    pool of host threads (numpy releases the GIL while it fills an array); every
    matrix has its own stream, so the values do not depend on the thread count.
    The copies into the output tensors stay on the calling thread.
    """
    W1 = out_w1 if out_w1 is not None else torch.empty((wl.E, wl.H, 2 * wl.F), dtype=torch.bfloat16)
    W2 = out_w2 if out_w2 is not None else torch.empty((wl.E, wl.F, wl.H), dtype=torch.bfloat16)
    jobs = [(make_expert_w1, W1, e) for e in range(wl.E)] + \
           [(make_expert_w2, W2, e) for e in range(wl.E)]
    if threads <= 1:
        for fn, dst, e in jobs:
            dst[e].copy_(fn(wl, e))
        return W1, W2
    from concurrent.futures import ThreadPoolExecutor
    with ThreadPoolExecutor(max_workers=threads) as ex:
        # submitted a few at a time, so that host memory holds about `threads`
        # matrices rather than all of them
        pending = []
        for fn, dst, e in jobs:
            pending.append((dst, e, ex.submit(fn, wl, e)))
            if len(pending) >= 2 * threads:
                d, i, fut = pending.pop(0)
                d[i].copy_(fut.result())
        for d, i, fut in pending:
            d[i].copy_(fut.result())
    return W1, W2


def expert_probabilities(wl: Workload) -> np.ndarray:
    """Per-expert routing probabilities of the skewed load (fp64, sums to 1)."""
    rng = np.random.default_rng(_streams(wl)[1 + 2 * wl.E])
    z = rng.standard_normal(wl.E)
    p = np.maximum(1e-4, 1.0 / wl.E + wl.std * z)
    return p / p.sum()


def make_topk_ids(wl: Workload) -> np.ndarray:
    """Routed expert ids, int32 [M, topk]; the topk ids of a token are distinct."""
    M, E, k = wl.M, wl.E, wl.topk
    if k > E:
        raise ValueError("topk must not exceed E")
    if wl.routing == "uniform":
        rng = np.random.default_rng(_streams(wl)[1 + 2 * E])
        ids = np.argsort(rng.random((M, E)), axis=1, kind="stable")[:, :k]
    elif wl.routing == "balanced":
        rng = np.random.default_rng(_streams(wl)[1 + 2 * E])
        r = rng.permutation(M) % E
        ids = (r[:, None] + np.arange(k)[None, :]) % E
    elif wl.routing == "skewed":
        p = expert_probabilities(wl)
        # the probabilities consumed the first draws of this stream; the Gumbel
        # noise continues from the same generator state
        rng = np.random.default_rng(_streams(wl)[1 + 2 * E])
        rng.standard_normal(E)
        keys = np.log(p)[None, :] + rng.gumbel(size=(M, E))
        ids = np.argsort(-keys, axis=1, kind="stable")[:, :k]
    else:
        raise ValueError(f"unknown routing {wl.routing!r}")
    return np.ascontiguousarray(ids, dtype=np.int32)


def make_topk_w(wl: Workload) -> np.ndarray:
    """Gate weights, fp32 [M, topk]: softmax over k of N(0,1) logits."""
    rng = np.random.default_rng(_streams(wl)[2 + 2 * wl.E])
    logits = rng.standard_normal((wl.M, wl.topk))
    logits -= logits.max(axis=1, keepdims=True)
    ex = np.exp(logits)
    return np.ascontiguousarray(ex / ex.sum(axis=1, keepdims=True), dtype=np.float32)


def make_routing(wl: Workload) -> tuple[np.ndarray, np.ndarray]:
    return make_topk_ids(wl), make_topk_w(wl)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """The raw bf16 bit patterns of a CPU bf16 tensor as a uint16 numpy array."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def rank_workload(wl: Workload, rank: int) -> Workload:
    """The instance a data-parallel rank processes: same shape, its own seed."""
    return wl if rank == 0 else wl.with_(seed=wl.seed + 1_000_003 * rank)
