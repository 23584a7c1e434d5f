"""The expert-parallel layer on CPU: its bookkeeping with oracle stage calls, G
ranks emulated in one process, and real gloo ranks exchanging rows with
all_to_all_single (the NCCL path's host logic)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from ep_helpers import OracleOps, emulate_ranks
from grouped_gemm_plan_b200 import ep
from helpers import check_close, layer_case


def _split(a, G):
    n = a.shape[0] // G
    return [a[r * n:(r + 1) * n] for r in range(G)]


def _case(M, H, F, E, topk, kind, seed):
    w, x, W1, W2, ids, tw = layer_case(M, H, F, E, topk, kind, seed=seed)
    return x, W1, W2, torch.from_numpy(ids), torch.from_numpy(tw)


def test_shard_validation():
    assert ep.ExpertShard(8, 4, 3).local == 2 and ep.ExpertShard(8, 4, 3).first == 6
    with pytest.raises(ValueError):
        ep.ExpertShard(6, 4, 0)
    with pytest.raises(ValueError):
        ep.ExpertShard(8, 2, 2)
    x, W1, W2, ids, tw = _case(8, 64, 64, 4, 2, "uniform", 0)
    with pytest.raises(ValueError):       # rank holds 2 experts, weights for 4
        ep.ep_moe_ffn(x, W1, W2, ids, tw, ep.ExpertShard(4, 2, 0), OracleOps())


def test_received_local_ids():
    rc = np.array([[2, 0, 1], [0, 0, 0], [1, 3, 0]])
    assert ep.received_local_ids(rc).ravel().tolist() == [0, 0, 2, 0, 1, 1, 1]
    assert ep.received_local_ids(np.zeros((2, 4), np.int64)).shape == (0, 1)


@pytest.mark.parametrize("M,H,F,E,topk,kind", [(48, 64, 64, 8, 2, "skewed"),
                                               (30, 128, 64, 4, 3, "uniform")])
def test_one_rank_is_the_layer(M, H, F, E, topk, kind):
    x, W1, W2, ids, tw = _case(M, H, F, E, topk, kind, M)
    out = ep.ep_moe_ffn(x, W1, W2, ids, tw, ep.ExpertShard(E, 1, 0), OracleOps())
    ref = oracle.moe_ffn(x, W1, W2, ids.numpy(), tw.numpy())
    # h, the expert outputs and the output are bf16: two roundings more than the
    # oracle's single fp64 pass, as in the library's chain of calls
    check_close(out, ref, "ep G=1", ulps=2.0)


@pytest.mark.parametrize("G", [2, 4, 8])
def test_emulated_ranks_give_the_same_bits(G):
    M, H, F, E, topk = 64, 64, 64, 8, 2
    x, W1, W2, ids, tw = _case(M * G, H, F, E, topk, "skewed", 7)
    whole = ep.ep_moe_ffn(x, W1, W2, ids, tw, ep.ExpertShard(E, 1, 0), OracleOps())
    outs = emulate_ranks(_split(x, G), W1, W2, _split(ids, G), _split(tw, G), G, OracleOps())
    assert torch.equal(torch.cat(outs).view(torch.int16), whole.view(torch.int16))


def test_emulated_ranks_with_idle_experts():
    # every token routes to experts 0 and 1 only: ranks 1..3 receive nothing and
    # rank 0 receives every row
    G, M, H, F, E = 4, 16, 64, 64, 8
    x, W1, W2, ids, tw = _case(M * G, H, F, E, 2, "uniform", 3)
    ids = torch.stack([torch.zeros(M * G, dtype=torch.int32),
                       torch.ones(M * G, dtype=torch.int32)], 1)
    whole = ep.ep_moe_ffn(x, W1, W2, ids, tw, ep.ExpertShard(E, 1, 0), OracleOps())
    outs = emulate_ranks(_split(x, G), W1, W2, _split(ids, G), _split(tw, G), G, OracleOps())
    assert torch.equal(torch.cat(outs).view(torch.int16), whole.view(torch.int16))
    check_close(whole, oracle.moe_ffn(x, W1, W2, ids.numpy(), tw.numpy()), "idle experts", ulps=2.0)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


GLOO_CASES = [
    # (M per rank, H, F, E, topk, routing, seed)
    (40, 64, 64, 8, 2, "skewed", 11),
    (17, 128, 64, 4, 4, "uniform", 12),     # topk = E: every expert gets every token
    (33, 64, 128, 12, 3, "skewed", 13),
]


def _rank_main(rank, world, port, q):
    import torch.distributed as dist
    from datetime import timedelta
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    try:
        dist.init_process_group("gloo", rank=rank, world_size=world,
                                timeout=timedelta(seconds=60))
        res = []
        for (M, H, F, E, topk, kind, seed) in GLOO_CASES:
            if E % world:
                continue
            x, W1, W2, ids, tw = _case(M * world, H, F, E, topk, kind, seed)
            El = E // world
            sl = slice(rank * M, (rank + 1) * M)
            out = ep.ep_moe_ffn(x[sl].contiguous(), W1[rank * El:(rank + 1) * El],
                                W2[rank * El:(rank + 1) * El], ids[sl].contiguous(),
                                tw[sl].contiguous(), ep.ExpertShard(E, world, rank), OracleOps())
            res.append(out.view(torch.int16).numpy().copy())
        dist.barrier()
        dist.destroy_process_group()
        q.put((rank, res))
    except Exception as exc:  # surface the failure to the parent
        q.put((rank, "error: " + repr(exc)))


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_ranks_match_one_rank(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        assert not isinstance(got[r], str), got[r]
    i = 0
    for (M, H, F, E, topk, kind, seed) in GLOO_CASES:
        if E % world:
            continue
        x, W1, W2, ids, tw = _case(M * world, H, F, E, topk, kind, seed)
        whole = ep.ep_moe_ffn(x, W1, W2, ids, tw, ep.ExpertShard(E, 1, 0), OracleOps())
        cat = np.concatenate([got[r][i] for r in range(world)])
        assert np.array_equal(cat, whole.view(torch.int16).numpy()), (world, M, E, topk)
        check_close(torch.from_numpy(cat).view(torch.bfloat16),
                    oracle.moe_ffn(x, W1, W2, ids.numpy(), tw.numpy()), "gloo ep", ulps=2.0)
        i += 1
