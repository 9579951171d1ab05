"""Strided tensors through fa_fwd_strided / fa_bwd_strided: [B, N, H, d]
storage and q, k, v as views of one packed [B, N, 3, H, d] tensor, checked
against the fp64 oracle and against the contiguous path (the forward must be
bit for bit the same: only the addressing changes)."""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_71_b200 import binding as fa
from exact_io_aware_71_b200.inputs import Workload, make_inputs
from tests.parity import check_fwd, check_grads, to64

pytestmark = pytest.mark.gpu


def bnhd(t):
    """The same [B, H, N, d] values stored as [B, N, H, d] (a permuted view)."""
    return t.permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3)


def run_both(wl, make_views):
    q, k, v, do = (t.cuda() for t in make_inputs(wl))
    o_c, l_c = fa.forward(q, k, v, wl.causal, wl.scale)
    g_c = fa.backward(q, k, v, o_c, l_c, do, wl.causal, wl.scale)
    qs, ks, vs, dos = make_views(q, k, v, do)
    assert qs.stride() != q.stride() or ks.stride() != k.stride()
    o_s = bnhd(torch.empty_like(q))
    o_s, l_s = fa.forward(qs, ks, vs, wl.causal, wl.scale, out=o_s)
    grads = (bnhd(torch.empty_like(q)), bnhd(torch.empty_like(k)), bnhd(torch.empty_like(v)))
    g_s = fa.backward(qs, ks, vs, o_s, l_s, dos, wl.causal, wl.scale, grads=grads)
    torch.cuda.synchronize()
    assert torch.equal(o_s, o_c) and torch.equal(l_s, l_c)
    for a, b in zip(g_s, g_c):
        assert (a.double() - b.double()).abs().max().item() <= 2e-2
    o_ref, lse_ref = oracle.attention_forward(to64(q), to64(k), to64(v), wl.causal, wl.scale)
    check_fwd(to64(o_s), to64(l_s), o_ref, lse_ref)
    g_ref = oracle.attention_backward(to64(q), to64(k), to64(v), to64(do), wl.causal, wl.scale)
    check_grads([to64(g) for g in g_s], g_ref)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128, 256])
def test_bnhd_layout(d, causal):
    wl = Workload(f"bnhd{d}", 2, 4, 2, 333, 333, d, causal, 51)
    run_both(wl, lambda q, k, v, do: (bnhd(q), bnhd(k), bnhd(v), bnhd(do)))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_packed_qkv_views(d, causal):
    """q, k, v sliced out of one [B, N, 3, H, d] buffer (fused QKV layout)."""
    wl = Workload(f"qkv{d}", 2, 4, 4, 300, 300, d, causal, 52)

    def views(q, k, v, do):
        B, H, N, D = q.shape
        packed = torch.empty(B, N, 3, H, D, dtype=q.dtype, device=q.device)
        for i, t in enumerate((q, k, v)):
            packed[:, :, i] = t.permute(0, 2, 1, 3)
        qv, kv, vv = (packed[:, :, i].permute(0, 2, 1, 3) for i in range(3))
        return qv, kv, vv, bnhd(do)
    run_both(wl, views)
