"""Expert-parallel MoE layer across ranks (one process per GPU).

The setting of the COMET paper review (sections 3.2 and 4: layer 0 dispatches
tokens to the GPUs that hold their experts, layer 1 brings the expert outputs back
for the top-k reduction) and of the PTO MegaMoE article ("MoE dispatch/combine
为什么慢": the reorder by expert, the expert FFN and the top-k weighted
accumulation, with the dispatch and combine crossing devices): E experts are
split over G ranks in contiguous blocks of E / G, every rank holds its own tokens,
and one layer call on rank r runs

    ep_send     plan over all E experts, dispatch into expert order: the rows for
                rank d form one contiguous block (experts d*E/G .. (d+1)*E/G - 1)
    exchange    counts per (source rank, local expert), then the rows: this rank
                receives every row routed to its experts, ordered by source rank,
                then by expert
    ep_experts  plan of the received rows by local expert, gather into expert
                order, GEMM1 + SwiGLU, GEMM2 (the grouped GEMM on this rank's
                experts), gather back to the received order
    exchange    every row back to the rank of its token, in ep_send's order
    ep_finish   the top-k gate-weighted sum in token order

Every step of the arithmetic runs in the stage calls of `ops` (``CudaOps``: the
library's kernels through the C ABI); this module only moves rows between ranks
(torch.distributed all_to_all_single: NCCL on GPUs, gloo on CPU) and keeps the
index bookkeeping.  Rows cross ranks in bf16 and the expert outputs are rounded to
bf16 once before they travel back, as in the chain of separate calls on one GPU,
and every row meets the same arithmetic whatever rank computes it: with the same
stage calls the layer gives the same bits for every number of ranks.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch
import torch.distributed as dist


@dataclass(frozen=True)
class ExpertShard:
    """Contiguous blocks of E / G experts: rank r holds experts [r*El, (r+1)*El)."""
    E: int
    G: int
    rank: int

    def __post_init__(self):
        if self.G < 1 or self.E % self.G != 0:
            raise ValueError(f"E = {self.E} experts cannot be split evenly over G = {self.G} ranks")
        if not 0 <= self.rank < self.G:
            raise ValueError(f"rank {self.rank} outside [0, {self.G})")

    @property
    def local(self) -> int:
        return self.E // self.G

    @property
    def first(self) -> int:
        return self.rank * self.local


class CudaOps:
    """The stage calls on this rank's GPU: the library's kernels through the C ABI.

    Workspaces are kept per (call, sizes) and reused.  The calls are asynchronous on
    the current stream; check() synchronises once and raises if any kernel recorded
    a device error (ep_moe_ffn calls it at the end of the layer)."""

    def __init__(self, device):
        from . import binding as B
        self.B = B
        self.dev = torch.device(device)
        self._cache = {}
        B.load()

    def _ws(self, op, M, H, F, E, topk):
        key = (op, M, H, F, E, topk)
        ws = self._cache.get(key)
        if ws is None:
            ws = self._cache[key] = self.B.alloc_workspace(op, M, H, F, E, topk, self.dev)
        return ws

    def check(self):
        """Synchronise; raise MoEError if a stage call recorded a device error."""
        for key, ws in self._cache.items():
            st = self.B.moe_get_device_status(ws)
            if st != self.B.MOE_OK:
                raise self.B.MoEError(st, f"device status of stage call {key[0]}")

    def plan(self, ids, E):
        """counts [E], offsets [E+1], perm [n*k], inv [n*k] of int32 ids [n, k]."""
        B, dev = self.B, self.dev
        n, k = ids.shape
        counts = torch.empty(E, dtype=torch.int32, device=dev)
        offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
        perm = torch.empty(max(n * k, 1), dtype=torch.int32, device=dev)
        inv = torch.empty(max(n * k, 1), dtype=torch.int32, device=dev)
        ws = self._ws(B.OP_PLAN, n, 0, 0, E, k)
        B.moe_plan(ids, None, E, counts, offsets, perm[:n * k], inv[:n * k], None, ws)
        return counts, offsets, perm[:n * k], inv[:n * k]

    def gather(self, rows, idx, topk=1):
        """out[s] = rows[idx[s] // topk]."""
        B = self.B
        out = torch.empty((idx.numel(), rows.shape[1]), dtype=rows.dtype, device=self.dev)
        if idx.numel() == 0:
            return out
        ws = self._ws(B.OP_DISPATCH, rows.shape[0], rows.shape[1], 0, 1, topk)
        B.moe_dispatch(rows, idx, topk, out, ws)
        return out

    def expert_ffn(self, rows, offsets, W1, W2):
        """bf16 [n, H] expert-ordered rows -> bf16 [n, H], the SwiGLU FFN of each row's expert."""
        B = self.B
        n, H = rows.shape
        E, _, F2 = W1.shape
        y = torch.empty((n, H), dtype=torch.bfloat16, device=self.dev)
        if n == 0:
            return y
        h = torch.empty((n, F2 // 2), dtype=torch.bfloat16, device=self.dev)
        ws = self._ws(B.OP_GROUPED_GEMM, n, 0, 0, E, 1)
        B.moe_grouped_gemm(rows, W1, offsets, B.EPI_SWIGLU, h, ws)
        B.moe_grouped_gemm(h, W2, offsets, B.EPI_STORE, y, ws)
        return y

    def combine(self, y, inv, topk_w):
        """bf16 [M, H] = sum over k of topk_w[t, k] * y[inv[t*topk + k]]."""
        B = self.B
        M, k = topk_w.shape
        out = torch.empty((M, y.shape[1]), dtype=torch.bfloat16, device=self.dev)
        ws = self._ws(B.OP_COMBINE, M, y.shape[1], 0, 1, k)
        B.moe_combine(y, inv, topk_w, M, k, out, ws)
        return out


@dataclass
class Sent:
    """What one rank keeps from ep_send until ep_finish."""
    xp: torch.Tensor            # [M*topk, H] rows in global expert order
    send_counts: torch.Tensor   # int32 [G, E/G]: rows for (destination rank, its local expert)
    inv: torch.Tensor           # int32 [M*topk]: slot of (token, k) in xp

    @property
    def send_rows(self) -> list[int]:
        return [int(v) for v in self.send_counts.sum(1).tolist()]


def ep_send(x, topk_ids, shard: ExpertShard, ops) -> Sent:
    """Plan over all E experts and gather this rank's rows into expert order."""
    topk = topk_ids.shape[1]
    counts, _, perm, inv = ops.plan(topk_ids, shard.E)
    xp = ops.gather(x, perm, topk)
    return Sent(xp, counts.reshape(shard.G, shard.local), inv)


def received_local_ids(recv_counts: np.ndarray) -> np.ndarray:
    """int32 [n, 1]: the local expert of every received row.  recv_counts [G, El]
    holds the rows that source rank s sent for local expert j; the rows arrive
    source-major, expert-minor."""
    G, El = recv_counts.shape
    ids = np.repeat(np.tile(np.arange(El, dtype=np.int32), G), recv_counts.reshape(-1))
    return np.ascontiguousarray(ids.reshape(-1, 1))


def ep_experts(recv, recv_counts: np.ndarray, W1_local, W2_local, ops):
    """The expert FFN of the rows this rank received (source-major order) -> bf16
    outputs in the same order."""
    El = W1_local.shape[0]
    if recv_counts.shape[1] != El:
        raise ValueError(f"counts for {recv_counts.shape[1]} local experts, weights for {El}")
    ids = torch.from_numpy(received_local_ids(recv_counts)).to(recv.device)
    _, offsets, perm, inv = ops.plan(ids, El)
    xl = ops.gather(recv, perm)                 # expert-major, stable in the arrival order
    yl = ops.expert_ffn(xl, offsets, W1_local, W2_local)
    return ops.gather(yl, inv)                  # back to the arrival order


def ep_finish(back, sent: Sent, topk_w, ops):
    """The top-k gate-weighted sum of the returned rows (ep_send's order)."""
    return ops.combine(back, sent.inv, topk_w)


def ep_moe_ffn(x, W1_local, W2_local, topk_ids, topk_w, shard: ExpertShard, ops, group=None):
    """The MoE layer with experts sharded over the ranks of `group`.

    x bf16 [M, H] (this rank's tokens), W1_local [E/G, H, 2F] and W2_local
    [E/G, F, H] (this rank's experts), topk_ids int32 [M, topk] (global expert
    ids), topk_w fp32 [M, topk].  Returns out bf16 [M, H].  With G = 1 no
    collective is called.  Every rank of the group must call it: the exchanges are
    collective."""
    M, H = x.shape
    G, El = shard.G, shard.local
    if W1_local.shape[0] != El or W2_local.shape[0] != El:
        raise ValueError(f"rank {shard.rank} holds {El} experts, got weights for "
                         f"{W1_local.shape[0]} and {W2_local.shape[0]}")
    sent = ep_send(x, topk_ids, shard, ops)
    if G == 1:
        y = ep_experts(sent.xp, sent.send_counts.cpu().numpy(), W1_local, W2_local, ops)
        return _checked(ep_finish(y, sent, topk_w, ops), ops)

    recv_counts = torch.empty_like(sent.send_counts)
    dist.all_to_all_single(recv_counts, sent.send_counts, group=group)
    rc = recv_counts.cpu().numpy().astype(np.int64)
    send_rows, recv_rows = sent.send_rows, [int(v) for v in rc.sum(1)]
    recv = sent.xp.new_empty((sum(recv_rows), H))
    dist.all_to_all_single(recv, sent.xp, output_split_sizes=recv_rows,
                           input_split_sizes=send_rows, group=group)
    y = ep_experts(recv, rc, W1_local, W2_local, ops)
    back = y.new_empty((sent.xp.shape[0], H))
    dist.all_to_all_single(back, y, output_split_sizes=send_rows, input_split_sizes=recv_rows,
                           group=group)
    return _checked(ep_finish(back, sent, topk_w, ops), ops)


def _checked(out, ops):
    """Run the stage calls' error check, where `ops` has one."""
    check = getattr(ops, "check", None)
    if check is not None:
        check()
    return out
