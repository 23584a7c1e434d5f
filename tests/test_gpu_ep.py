"""The expert-parallel layer on one GPU with the library's kernels: one rank
through ep_moe_ffn, and G ranks emulated in one process (their exchanges done by
slicing, every stage call a kernel of the library).  The multi-rank collective
path itself is covered with gloo ranks on CPU."""
import numpy as np
import pytest
import torch

import oracle
from ep_helpers import emulate_ranks
from grouped_gemm_plan_b200 import ep
from helpers import check_close, layer_case
from test_gpu_layer import run_chain

pytestmark = pytest.mark.gpu


def _split(a, G):
    n = a.shape[0] // G
    return [a[r * n:(r + 1) * n] for r in range(G)]


@pytest.mark.parametrize("M,H,F,E,topk,kind", [(256, 256, 512, 8, 2, "uniform"),
                                               (300, 512, 384, 16, 4, "skewed")])
def test_one_rank_matches_oracle_and_chain(cuda_dev, M, H, F, E, topk, kind):
    w, x, W1, W2, ids, tw = layer_case(M, H, F, E, topk, kind, seed=M + E)
    ops = ep.CudaOps(cuda_dev)
    d = cuda_dev
    out = ep.ep_moe_ffn(x.to(d), W1.to(d), W2.to(d), torch.from_numpy(ids).to(d),
                        torch.from_numpy(tw).to(d), ep.ExpertShard(E, 1, 0), ops)
    check_close(out, oracle.moe_ffn(x, W1, W2, ids, tw), "ep G=1", ulps=2.0)
    chain = run_chain(d, x, W1, W2, ids, tw)
    assert torch.equal(out.view(torch.int16), chain.view(torch.int16))


@pytest.mark.parametrize("G", [2, 4, 8])
def test_emulated_ranks_give_the_same_bits(cuda_dev, G):
    M, H, F, E, topk = 160, 256, 256, 16, 4
    w, x, W1, W2, ids, tw = layer_case(M * G, H, F, E, topk, "skewed", seed=G)
    d = cuda_dev
    ops = ep.CudaOps(d)
    xd, W1d, W2d = x.to(d), W1.to(d), W2.to(d)
    idd, twd = torch.from_numpy(ids).to(d), torch.from_numpy(tw).to(d)
    whole = ep.ep_moe_ffn(xd, W1d, W2d, idd, twd, ep.ExpertShard(E, 1, 0), ops)
    outs = emulate_ranks(_split(xd, G), W1d, W2d, _split(idd, G), _split(twd, G), G, ops)
    assert torch.equal(torch.cat(outs).view(torch.int16), whole.view(torch.int16))
    check_close(whole, oracle.moe_ffn(x, W1, W2, ids, tw), f"ep emulated G={G}", ulps=2.0)
