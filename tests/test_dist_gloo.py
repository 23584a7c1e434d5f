"""The multi-GPU host path on CPU: two gloo ranks run the data-parallel plumbing
that bench.py uses with NCCL (per-rank batches, barrier, max over ranks)."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from grouped_gemm_plan_b200 import dist as D
from grouped_gemm_plan_b200 import workload as W


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    try:
        assert D.init("gloo", timeout_s=60)
        r, lr, ws = D.env_rank()
        wl = D.shard(W.WORKLOADS["tiny"], r)
        ids = W.make_topk_ids(wl)
        D.barrier()
        # rank r "measured" 10 + r ms and 5 * (r + 1) ms
        mx = D.max_over_ranks([10.0 + r, 5.0 * (r + 1)])
        rate = D.whole_job_rate(wl.M, ws, mx[0] / 1e3)
        q.put((r, ws, wl.seed, ids.sum(), mx, rate))
        D.finish()
    except Exception as exc:  # surface the failure to the parent
        q.put(("error", repr(exc)))


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert all(o[0] != "error" for o in out), out
    out.sort()
    (r0, ws0, seed0, sum0, mx0, rate0), (r1, ws1, seed1, sum1, mx1, rate1) = out
    assert (r0, r1, ws0, ws1) == (0, 1, 2, 2)
    assert seed0 == W.WORKLOADS["tiny"].seed and seed1 != seed0      # own batch per rank
    assert sum0 != sum1
    assert mx0 == mx1 == [11.0, 10.0]                                  # max over ranks
    assert rate0 == rate1 == pytest.approx(2 * 256 / 0.011)           # whole-job rate


def test_single_process_is_identity(monkeypatch):
    for k in ("RANK", "LOCAL_RANK", "WORLD_SIZE"):
        monkeypatch.delenv(k, raising=False)
    assert D.env_rank() == (0, 0, 1)
    assert D.init("gloo") is False
    assert D.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]
    assert D.shard(W.WORKLOADS["mixtral"], 0) == W.WORKLOADS["mixtral"]
