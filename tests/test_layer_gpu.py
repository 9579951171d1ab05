"""GPU check of the synthetic attention layer (QKV projection, libfa
attention on strided views of the packed QKV tensor, output projection),
stage by stage: the projections against fp64 products of the bf16 tensors
the GPU produced, the attention against the fp64 oracle at the parity bar."""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_71_b200.layer import AttentionLayer, layer_flops
from tests.parity import check_fwd, check_grads, relfro, to64

GEMM_RELFRO = 5e-3     # a bf16 product output carries about 2^-9 relative rounding


@pytest.mark.gpu
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Hq,Hkv,d", [(4, 4, 64), (4, 2, 128)])
def test_layer_stage_by_stage(causal, Hq, Hkv, d):
    B, N = 2, 384
    hidden = Hq * d
    layer = AttentionLayer(hidden, Hq, Hkv, d, causal, seed=7)
    g = torch.Generator("cpu").manual_seed(8)
    x = torch.randn(B, N, hidden, generator=g).to(torch.bfloat16).cuda()
    dy = torch.randn(B, N, hidden, generator=g).to(torch.bfloat16).cuda()
    y = layer.forward(x)
    dx, dwq, dwo = layer.backward(dy)
    torch.cuda.synchronize()
    _, qkv, o, _ = layer._saved
    do, dqkv = layer._grads
    X, WQ, WO, DY = to64(x), to64(layer.w_qkv), to64(layer.w_o), to64(dy)
    QKV, O, DO, DQKV = to64(qkv), to64(o), to64(do), to64(dqkv)
    flat = lambda t: t.reshape(B * N, -1)
    # projections
    assert relfro(flat(QKV), flat(X) @ WQ) <= GEMM_RELFRO
    assert relfro(to64(y).reshape(B * N, -1), flat(O) @ WO) <= GEMM_RELFRO
    assert relfro(flat(DO), flat(DY) @ WO.T) <= GEMM_RELFRO
    assert relfro(to64(dwo), flat(O).T @ flat(DY)) <= GEMM_RELFRO
    assert relfro(to64(dwq), flat(X).T @ flat(DQKV)) <= GEMM_RELFRO
    assert relfro(to64(dx).reshape(B * N, -1), flat(DQKV) @ WQ.T) <= GEMM_RELFRO
    # attention on the packed tensors' views, against the oracle
    split = lambda t: (t[:, :, :Hq].transpose(0, 2, 1, 3), t[:, :, Hq:Hq + Hkv].transpose(0, 2, 1, 3),
                       t[:, :, Hq + Hkv:].transpose(0, 2, 1, 3))
    q, k, v = split(QKV)
    o_ref, lse_ref = oracle.attention_forward(q, k, v, causal, layer.scale)
    check_fwd(O.transpose(0, 2, 1, 3), to64(layer._saved[3]), o_ref, lse_ref)
    ref = oracle.attention_backward(q, k, v, DO.transpose(0, 2, 1, 3), causal, layer.scale)
    check_grads(split(DQKV), ref)
    assert np.isfinite(to64(dx)).all()


def test_layer_flops():
    f, b = layer_flops(2, 1024, 2048, 16, 16, 128, False)
    gemm = 2.0 * 2 * 1024 * 2048 * (3 * 2048) + 2.0 * 2 * 1024 * 2048 * 2048
    attn = 4.0 * 2 * 16 * 1024 * 1024 * 128
    assert f == gemm + attn and b == 2 * gemm + 2.5 * attn
