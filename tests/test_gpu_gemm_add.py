"""GPU parity of the Fused GemmAdd epilogue (grouped GEMM article, section "Fused
GemmAdd": Y = cast(alpha * Acc + beta * Add), the addition in fp32 before the one
cast) on the layer and on the combine, against the fp64 oracle.

The layer form moe_ffn_fused_add puts the addition into the combine, where the
top-k sum is accumulated: out = bf16(alpha * sum_k w_k y_k + beta * add).  The
bar is the layer's (helpers.check_close) against oracle.moe_ffn_add."""
import numpy as np
import pytest
import torch

import oracle
from grouped_gemm_plan_b200 import binding as B
from helpers import check_close, guarded_empty, layer_case

pytestmark = pytest.mark.gpu


def _layer_buffers(dev, M, E, R):
    return (torch.empty(E, dtype=torch.int32, device=dev),
            torch.empty(E + 1, dtype=torch.int32, device=dev),
            torch.empty(R, dtype=torch.int32, device=dev))


def _fused_add(dev, x, W1, W2, ids, tw, add, alpha, beta, out=None):
    M, H = x.shape
    E, _, F2 = W1.shape
    topk = ids.shape[1]
    counts, offsets, perm = _layer_buffers(dev, M, E, M * topk)
    check = None
    if out is None:
        out, check = guarded_empty((M, H), torch.bfloat16, dev)
    ws = B.alloc_workspace(B.OP_FFN_FUSED, M, H, F2 // 2, E, topk, dev)
    B.moe_ffn_fused_add(x, W1, W2, ids, tw, add, alpha, beta, out, counts, offsets, perm, ws)
    assert B.moe_get_device_status(ws) == B.MOE_OK
    if check is not None:
        check()
    return out


@pytest.mark.parametrize("M,H,F,E,topk,kind,alpha,beta", [
    (300, 512, 384, 8, 2, "skewed", 1.0, 1.0),      # residual: out = x + layer(x)
    (77, 256, 192, 4, 1, "uniform", 0.5, -2.0),
    (257, 1024, 256, 16, 4, "skewed", -1.25, 0.75),
])
def test_layer_gemm_add_matches_oracle(cuda_dev, M, H, F, E, topk, kind, alpha, beta):
    w, x, W1, W2, ids, tw = layer_case(M, H, F, E, topk, kind, seed=M + H)
    rng = np.random.default_rng(M)
    add = x if (alpha, beta) == (1.0, 1.0) else \
        torch.from_numpy(rng.standard_normal((M, H)).astype(np.float32)).to(torch.bfloat16)
    d = [t.to(cuda_dev) for t in (x, W1, W2)] + \
        [torch.from_numpy(ids).to(cuda_dev), torch.from_numpy(tw).to(cuda_dev)]
    add_d = d[0] if add is x else add.to(cuda_dev)
    out = _fused_add(cuda_dev, *d, add_d, alpha, beta)
    ref = oracle.moe_ffn_add(x, W1, W2, ids, tw, add, alpha, beta)
    check_close(out, ref, f"layer GemmAdd alpha={alpha} beta={beta}")


def test_layer_gemm_add_in_place_and_identity(cuda_dev):
    # out may be the added buffer itself (in-place residual update); alpha = 1,
    # beta = 0 is exactly the plain layer
    w, x, W1, W2, ids, tw = layer_case(200, 512, 256, 8, 2, "skewed", seed=3)
    d = [t.to(cuda_dev) for t in (x, W1, W2)] + \
        [torch.from_numpy(ids).to(cuda_dev), torch.from_numpy(tw).to(cuda_dev)]
    rng = np.random.default_rng(11)
    add = torch.from_numpy(rng.standard_normal((200, 512)).astype(np.float32)).to(torch.bfloat16)
    buf = add.to(cuda_dev)
    _fused_add(cuda_dev, *d, buf, 1.0, 1.0, out=buf)
    check_close(buf, oracle.moe_ffn_add(x, W1, W2, ids, tw, add, 1.0, 1.0), "in-place GemmAdd")

    plain = torch.empty(200, 512, dtype=torch.bfloat16, device=cuda_dev)
    counts, offsets, perm = _layer_buffers(cuda_dev, 200, 8, 400)
    ws = B.alloc_workspace(B.OP_FFN_FUSED, 200, 512, 256, 8, 2, cuda_dev)
    B.moe_ffn_fused(*d, plain, counts, offsets, perm, ws, n_c=0)
    ident = _fused_add(cuda_dev, *d, None, 1.0, 0.0)
    assert torch.equal(ident.view(torch.int16), plain.view(torch.int16))


def test_combine_add_matches_oracle(cuda_dev):
    # expert-ordered bf16 rows weighted in the combine, plus the added tensor
    M, H, E, topk = 333, 768, 8, 2
    w, x, W1, W2, ids, tw = layer_case(M, H, 64, E, topk, "skewed", seed=9)
    counts, offsets, perm, inv, wsorted = oracle.plan(ids, tw, E)
    rng = np.random.default_rng(9)
    yp = torch.from_numpy(rng.standard_normal((M * topk, H)).astype(np.float32)).to(torch.bfloat16)
    add = torch.from_numpy(rng.standard_normal((M, H)).astype(np.float32)).to(torch.bfloat16)
    ref = oracle.gemm_add(oracle.combine(yp.double().numpy(), inv, tw), add, 0.5, 2.0)
    out, check = guarded_empty((M, H), torch.bfloat16, cuda_dev)
    ws = B.alloc_workspace(B.OP_COMBINE, M, H, 0, 1, topk, cuda_dev)
    B.moe_combine_add(yp.to(cuda_dev), torch.from_numpy(inv).to(cuda_dev),
                      torch.from_numpy(tw).to(cuda_dev), add.to(cuda_dev), 0.5, 2.0, M, topk, out,
                      ws)
    assert B.moe_get_device_status(ws) == B.MOE_OK
    check()
    check_close(out, ref, "combine GemmAdd")


def test_gemm_add_rejects_missing_add(cuda_dev):
    w, x, W1, W2, ids, tw = layer_case(16, 256, 128, 4, 2, "uniform", seed=1)
    d = [t.to(cuda_dev) for t in (x, W1, W2)] + \
        [torch.from_numpy(ids).to(cuda_dev), torch.from_numpy(tw).to(cuda_dev)]
    with pytest.raises(B.MoEError) as ei:
        _fused_add(cuda_dev, *d, None, 1.0, 1.0)
    assert ei.value.status == B.MOE_ERR_INVALID_ARG
