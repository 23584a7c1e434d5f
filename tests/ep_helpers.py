"""Expert-parallel test helpers: stage calls computed by the oracle (on CPU
tensors), and G ranks emulated in one process by running the phases of the
expert-parallel layer rank by rank with the exchanges done as slicing."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from grouped_gemm_plan_b200 import ep


def _bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64)).to(torch.bfloat16)


class OracleOps:
    """The stage calls of the expert-parallel layer, computed by the oracle with the
    same bf16 rounding points as the library's chain of calls (expert rows, h, the
    expert outputs and the layer output are bf16)."""

    def plan(self, ids, E):
        counts, offsets, perm, inv, _ = oracle.plan(ids.numpy(), None, E)
        return tuple(torch.from_numpy(np.ascontiguousarray(a)) for a in (counts, offsets, perm, inv))

    def gather(self, rows, idx, topk=1):
        if idx.numel() == 0:
            return rows.new_empty((0, rows.shape[1]))
        return torch.from_numpy(oracle.dispatch(rows, idx.numpy(), topk)).view(torch.bfloat16)

    def expert_ffn(self, rows, offsets, W1, W2):
        if rows.shape[0] == 0:
            return rows.new_empty((0, W2.shape[2]))
        off = offsets.numpy()
        h = _bf16(oracle.swiglu(oracle.grouped_gemm(rows, W1, off)))
        return _bf16(oracle.grouped_gemm(h, W2, off))

    def combine(self, y, inv, topk_w):
        w = topk_w.numpy() if isinstance(topk_w, torch.Tensor) else topk_w
        return _bf16(oracle.combine(y.double().numpy(), inv.numpy(), w))


def emulate_ranks(xs, W1, W2, ids_list, tw_list, G, ops):
    """The layer on G emulated ranks: rank r holds xs[r], ids_list[r], tw_list[r] and
    experts [r*E/G, (r+1)*E/G).  The exchanges are done by slicing the per-rank
    tensors exactly as all_to_all_single would place them.  Returns the per-rank
    outputs."""
    E = W1.shape[0]
    El = E // G
    sents = [ep.ep_send(xs[r], ids_list[r], ep.ExpertShard(E, G, r), ops) for r in range(G)]
    counts = [s.send_counts.cpu().numpy().astype(np.int64) for s in sents]        # [G, El] each
    starts = [np.concatenate([[0], np.cumsum(c.sum(1))]) for c in counts]         # per source
    ys = []
    for d in range(G):
        recv = torch.cat([sents[s].xp[starts[s][d]:starts[s][d + 1]] for s in range(G)])
        rc = np.stack([counts[s][d] for s in range(G)])
        ys.append(ep.ep_experts(recv, rc, W1[d * El:(d + 1) * El], W2[d * El:(d + 1) * El], ops))
    outs = []
    for s in range(G):
        parts = []
        for d in range(G):
            # the rows that source s sent to d sit in ys[d] after those of sources < s
            before = sum(int(counts[q][d].sum()) for q in range(s))
            parts.append(ys[d][before:before + int(counts[s][d].sum())])
        back = torch.cat(parts)
        outs.append(ep.ep_finish(back, sents[s], tw_list[s], ops))
    return outs
