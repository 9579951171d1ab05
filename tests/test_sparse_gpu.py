"""GPU parity of block-sparse attention (fa_fwd_block_sparse /
fa_bwd_block_sparse, through the C ABI) against the fp64 oracle with the
same block mask expanded element by element.

Rows whose mask row is all zero must come back exactly as the oracle has
them (O = 0, LSE = -inf, dQ = 0); the other rows are held to the dense
tolerances."""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_71_b200 import binding as fa
from exact_io_aware_71_b200.inputs import Workload, make_block_mask, make_inputs
from tests.parity import check_fwd, check_grads, sample_rows, to64

pytestmark = pytest.mark.gpu

DEV = "cuda"


def W(B, Hq, Hkv, Nq, Nk, d, causal, seed=71):
    return Workload(f"s{B}_{Hq}_{Hkv}_{Nq}_{Nk}_{d}_{int(causal)}", B, Hq, Hkv, Nq, Nk, d,
                    causal, seed)


def run(wl, mask, with_bwd=True):
    q, k, v, do = make_inputs(wl)
    qd, kd, vd, dod = q.to(DEV), k.to(DEV), v.to(DEV), do.to(DEV)
    md = mask.to(DEV)
    o, lse = fa.forward(qd, kd, vd, wl.causal, wl.scale, block_mask=md)
    grads = None
    if with_bwd:
        grads = fa.backward(qd, kd, vd, o, lse, dod, wl.causal, wl.scale, block_mask=md)
    torch.cuda.synchronize()
    st, where = fa.fa_device_status(None)
    assert st == 0, f"device status {st} at wait {where}"
    out = (to64(o), to64(lse)) + (tuple(to64(g) for g in grads) if grads else ())
    return (to64(q), to64(k), to64(v), to64(do)), out


def check_forward(o, lse, o_ref, lse_ref):
    empty = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse), empty), "rows that see no key differ"
    assert (o[empty] == 0).all(), "O of rows that see no key must be 0"
    if (~empty).any():
        check_fwd(o[~empty], lse[~empty], o_ref[~empty], lse_ref[~empty])


def full_check(wl, mask, with_bwd=True):
    (q, k, v, do), out = run(wl, mask, with_bwd)
    m = mask.numpy()
    o_ref, lse_ref = oracle.attention_forward(q, k, v, wl.causal, wl.scale, block_mask=m)
    check_forward(out[0], out[1], o_ref, lse_ref)
    if with_bwd:
        ref = oracle.attention_backward(q, k, v, do, wl.causal, wl.scale, block_mask=m)
        empty = np.isneginf(lse_ref)
        assert (out[2][empty] == 0).all(), "dQ of rows that see no key must be 0"
        check_grads(out[2:], ref)
    return out


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("hq,hkv", [(4, 4), (4, 1)])
def test_random_masks(d, causal, hq, hkv):
    wl = W(2, hq, hkv, 1000, 1000, d, causal, seed=d + hq + hkv)
    full_check(wl, make_block_mask(1000, 1000, 0.5, seed=d + int(causal)))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_mqa_wide_group(d, causal):
    """32 query heads on one kv head with a block mask that also empties a
    query block: the backward's exact D is recomputed by the block-sparse
    forward with the D epilogue, which leaves the empty rows' D at 0."""
    wl = W(1, 32, 1, 700, 700, d, causal, seed=50 + d)
    full_check(wl, make_block_mask(700, 700, 0.5, seed=d, empty_rows=(2,)))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("nq,nk", [(333, 700), (700, 333), (129, 1000)])
def test_unequal_lengths(nq, nk, causal):
    wl = W(1, 2, 2, nq, nk, 128, causal, seed=nq + nk)
    full_check(wl, make_block_mask(nq, nk, 0.6, seed=nq))


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("empty", [(0,), (1,), (0, 1), (2, 5), (7,)])
def test_rows_that_see_no_key(d, empty):
    """Query blocks with all-zero mask rows: the first or second tile of a
    tile pair, both, and the ragged last block."""
    wl = W(1, 2, 2, 1000, 1000, d, False, seed=5)
    full_check(wl, make_block_mask(1000, 1000, 0.7, seed=9, empty_rows=empty))


@pytest.mark.parametrize("causal", [False, True])
def test_all_zero_mask(causal):
    wl = W(1, 2, 1, 500, 500, 128, causal, seed=6)
    mask = torch.zeros(4, 4, dtype=torch.uint8)
    _, out = run(wl, mask)
    assert (out[0] == 0).all() and np.isneginf(out[1]).all()
    for g in out[2:]:
        assert (g == 0).all()


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_all_ones_mask_matches_dense_kernels(d, causal):
    """The same arithmetic as the dense path: O and LSE bit for bit; the
    gradients within the tolerance (dQ is summed with unordered atomics)."""
    wl = W(2, 4, 2, 640, 640, d, causal, seed=8)
    q, k, v, do = (t.to(DEV) for t in make_inputs(wl))
    mask = torch.ones(5, 5, dtype=torch.uint8, device=DEV)
    o1, l1 = fa.forward(q, k, v, causal, wl.scale)
    o2, l2 = fa.forward(q, k, v, causal, wl.scale, block_mask=mask)
    g1 = fa.backward(q, k, v, o1, l1, do, causal, wl.scale)
    g2 = fa.backward(q, k, v, o1, l1, do, causal, wl.scale, block_mask=mask)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    for a, b in zip(g1, g2):
        assert (a.double() - b.double()).abs().max().item() <= 2e-2


def test_long_rows_non_persistent_launch():
    """Non-causal rows longer than 4096 keys take the one-CTA-per-unit grid."""
    wl = W(1, 2, 2, 4224, 4224, 64, False, seed=12)
    full_check(wl, make_block_mask(4224, 4224, 0.3, seed=12, empty_rows=(3,)))


def test_bool_mask_and_strided_layout():
    """A bool mask and [B, N, H, d] storage go through the same entry points."""
    wl = W(2, 4, 2, 520, 520, 128, True, seed=13)
    q, k, v, do = make_inputs(wl)
    mask = make_block_mask(520, 520, 0.5, seed=13, empty_rows=(2,))
    perm = lambda t: t.permute(0, 2, 1, 3).contiguous().to(DEV).permute(0, 2, 1, 3)
    qd, kd, vd, dod = perm(q), perm(k), perm(v), perm(do)
    md = mask.bool().to(DEV)
    o, lse = fa.forward(qd, kd, vd, True, wl.scale, block_mask=md)
    g = fa.backward(qd, kd, vd, o, lse, dod, True, wl.scale, block_mask=md)
    torch.cuda.synchronize()
    m = mask.numpy()
    q64, k64, v64, do64 = to64(q), to64(k), to64(v), to64(do)
    o_ref, lse_ref = oracle.attention_forward(q64, k64, v64, True, wl.scale, block_mask=m)
    check_forward(to64(o), to64(lse), o_ref, lse_ref)
    ref = oracle.attention_backward(q64, k64, v64, do64, True, wl.scale, block_mask=m)
    check_grads([to64(x) for x in g], ref)


def test_mask_shape_is_checked():
    wl = W(1, 2, 2, 300, 300, 64, False)
    q, k, v, _ = (t.to(DEV) if t is not None else None for t in make_inputs(wl))
    with pytest.raises(ValueError):
        fa.forward(q, k, v, False, wl.scale, block_mask=torch.ones(2, 3, dtype=torch.uint8,
                                                                     device=DEV))


# --------------------------------------------------------------- larger problem
@pytest.mark.parametrize("causal", [False, True])
def test_full_size_sparse(causal):
    """B=2, H=16, N=8192, d=128 at a quarter of the blocks: sampled O / LSE
    and dQ rows of sampled heads against the oracle, full dK / dV of two
    heads."""
    wl = W(2, 16, 16, 8192, 8192, 128, causal, seed=14)
    mask = make_block_mask(8192, 8192, 0.25, seed=14, empty_rows=(5,))
    m = mask.numpy()
    (q, k, v, do), out = run(wl, mask)
    o, lse, dq, dk, dv = out
    for x in out:
        assert not np.isnan(x).any()
    rng = np.random.default_rng(3)
    heads = [(0, 0), (1, 15)] + [(int(rng.integers(2)), int(rng.integers(16))) for _ in range(4)]
    got_o, got_l, exp_o, exp_l, got_dq, exp_dq = [], [], [], [], [], []
    for (b, h) in heads:
        rows = np.concatenate([sample_rows(8192, 24, seed=b * 16 + h), np.arange(640, 648)])
        eo, el = oracle.attention_forward_rows(q, k, v, causal, wl.scale, b, h, rows,
                                               block_mask=m)
        exp_o.append(eo); exp_l.append(el)
        got_o.append(o[b, h, rows]); got_l.append(lse[b, h, rows])
        exp_dq.append(oracle.attention_backward_dq_rows(q, k, v, do, causal, wl.scale, b, h,
                                                        rows, block_mask=m))
        got_dq.append(dq[b, h, rows])
    check_forward(np.concatenate(got_o), np.concatenate(got_l), np.concatenate(exp_o),
                  np.concatenate(exp_l))
    check_grads([np.concatenate(got_dq)], [np.concatenate(exp_dq)], names=("dQ rows",))
    groups = [(0, 3), (1, 12)]
    ref = oracle.attention_backward(q, k, v, do, causal, wl.scale, heads=groups, block_mask=m)
    check_grads([np.stack([dk[b, j] for b, j in groups]), np.stack([dv[b, j] for b, j in groups])],
                [np.stack([ref[1][b, j] for b, j in groups]),
                 np.stack([ref[2][b, j] for b, j in groups])], names=("dK", "dV"))
