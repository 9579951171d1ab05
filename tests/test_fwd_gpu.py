"""GPU parity of fa_fwd against the fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_71_b200 import binding as fa
from exact_io_aware_71_b200.inputs import Workload, make_inputs, workloads
from tests.parity import check_fwd, sample_rows, to64

pytestmark = pytest.mark.gpu

DEV = "cuda"


def run(wl, scale=None, qmul=1.0):
    """Inputs of `wl` (Q optionally multiplied by qmul, exact for powers of 2)
    through fa_fwd; returns the bf16 inputs and the outputs as fp64 numpy."""
    q, k, v, _ = make_inputs(wl, with_do=False)
    if qmul != 1.0:
        q = (q.float() * qmul).to(torch.bfloat16)
    o, lse = fa.forward(q.to(DEV), k.to(DEV), v.to(DEV), wl.causal, scale or wl.scale)
    torch.cuda.synchronize()
    return (q, k, v), to64(o), to64(lse)


def full_check(wl, scale=None, qmul=1.0):
    (q, k, v), o, lse = run(wl, scale, qmul)
    o_ref, lse_ref = oracle.attention_forward(to64(q), to64(k), to64(v), wl.causal,
                                              scale or wl.scale)
    return check_fwd(o, lse, o_ref, lse_ref)


def W(B, Hq, Hkv, Nq, Nk, d, causal, seed=11):
    return Workload(f"t{B}_{Hq}_{Hkv}_{Nq}_{Nk}_{d}_{int(causal)}", B, Hq, Hkv, Nq, Nk, d,
                    causal, seed)


@pytest.mark.parametrize("name", ["tiny_b1h2n128d64_full", "tiny_b1h2n128d64_causal"])
def test_tiny_workload(name):
    full_check(workloads()[name])


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("hq,hkv", [(4, 4), (4, 2), (4, 1)])
def test_head_dims_and_gqa(d, causal, hq, hkv):
    full_check(W(2, hq, hkv, 384, 384, d, causal))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("n", [1, 17, 127, 129, 1000])
def test_ragged_lengths(n, d, causal):
    full_check(W(1, 2, 2, n, n, d, causal, seed=n))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("nq,nk", [(200, 333), (333, 200), (64, 1024), (1024, 64)])
def test_unequal_lengths(nq, nk, causal):
    full_check(W(1, 2, 1, nq, nk, 128, causal, seed=nq + nk))


@pytest.mark.parametrize("qmul", [4.0, 8.0])
@pytest.mark.parametrize("causal", [False, True])
def test_large_magnitude_scores(qmul, causal):
    """Peaky softmax: many running-max updates and lazy O rescales."""
    full_check(W(1, 2, 2, 640, 640, 64, causal, seed=5), qmul=qmul)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("qmul", [1.0, 2.0])
def test_long_rows_with_rescales(d, qmul):
    """Many key blocks per row with occasional lazy O rescales; softmax warps
    drift apart by a block and must still wait for the right P V product."""
    full_check(W(1, 2, 2, 4096, 4096, d, False, seed=5), qmul=qmul)


def test_scale_argument_is_used():
    full_check(W(1, 2, 2, 256, 256, 128, False), scale=0.3)


def test_forward_is_deterministic():
    wl = W(2, 4, 2, 777, 777, 128, True)
    q, k, v, _ = make_inputs(wl, with_do=False)
    q, k, v = q.to(DEV), k.to(DEV), v.to(DEV)
    o1, l1 = fa.forward(q, k, v, True, wl.scale)
    o2, l2 = fa.forward(q, k, v, True, wl.scale)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_guard_bands_untouched():
    """Outputs written only inside their buffers (NaN margins stay NaN)."""
    wl = W(1, 2, 2, 200, 200, 64, True)
    q, k, v, _ = make_inputs(wl, with_do=False)
    q, k, v = q.to(DEV), k.to(DEV), v.to(DEV)
    pad = 4096
    ob = torch.full((q.numel() + 2 * pad,), float("nan"), dtype=torch.bfloat16, device=DEV)
    lb = torch.full((2 * 200 + 2 * pad,), float("nan"), dtype=torch.float32, device=DEV)
    o = ob[pad:pad + q.numel()].view_as(q)
    lse = lb[pad:pad + 400].view(1, 2, 200)
    fa.forward(q, k, v, True, wl.scale, out=o, lse=lse)
    torch.cuda.synchronize()
    assert torch.isnan(ob[:pad]).all() and torch.isnan(ob[-pad:]).all()
    assert torch.isnan(lb[:pad]).all() and torch.isnan(lb[-pad:]).all()
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()
    st, _ = fa.fa_device_status(None)
    assert st == 0


# --------------------------------------------------------------- full-size workloads
FWD_WORKLOADS = [n for n, w in workloads().items() if not n.startswith("tiny")]


@pytest.mark.parametrize("name", FWD_WORKLOADS)
def test_full_size_sampled_rows(name):
    """Full-size problem on the GPU, checked on sampled rows of every head
    (rows are independent in the forward pass, so each is exact alone)."""
    wl = workloads()[name]
    (q, k, v), o, lse = run(wl)
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    q, k, v = to64(q), to64(k), to64(v)
    heads = [(b, h) for b in range(wl.B) for h in range(wl.Hq)]
    if len(heads) > 64:
        rng = np.random.default_rng(0)
        pick = sorted(rng.choice(len(heads), 64, replace=False).tolist())
        heads = [heads[i] for i in pick] + [heads[0], heads[-1]]
    got_o, got_l, ref_o, ref_l = [], [], [], []
    for (b, h) in heads:
        rows = sample_rows(wl.Nq, 64, seed=b * 1000 + h)
        ro, rl = oracle.attention_forward_rows(q, k, v, wl.causal, wl.scale, b, h, rows)
        got_o.append(o[b, h, rows]); got_l.append(lse[b, h, rows])
        ref_o.append(ro); ref_l.append(rl)
    check_fwd(np.concatenate(got_o), np.concatenate(got_l), np.concatenate(ref_o),
              np.concatenate(ref_l))
