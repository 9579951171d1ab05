"""GPU parity of packed variable-length batches (fa_fwd_varlen /
fa_bwd_varlen, through the C ABI) against the fp64 oracle run sequence by
sequence.  Sequence ends fall inside 128-row tiles and 32-row store boxes,
so every test also checks that no sequence's outputs leak into its
neighbours' rows."""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_71_b200 import binding as fa
from exact_io_aware_71_b200.inputs import (make_inputs, make_varlen_inputs, make_varlen_lengths,
                                           Workload)
from tests.parity import check_fwd, check_grads, to64

pytestmark = pytest.mark.gpu

DEV = "cuda"


def run(lq, lk, Hq, Hkv, d, causal, seed, with_bwd=True):
    q, k, v, do, cq, ck = make_varlen_inputs(lq, lk, Hq, Hkv, d, seed)
    scale = 1.0 / np.sqrt(d)
    qd, kd, vd, dod, cqd, ckd = (t.to(DEV) for t in (q, k, v, do, cq, ck))
    mq, mk = max(max(lq), 1), max(max(lk), 1)
    o, lse = fa.forward_varlen(qd, kd, vd, cqd, ckd, mq, mk, causal, scale)
    g = fa.backward_varlen(qd, kd, vd, o, lse, dod, cqd, ckd, mq, mk, causal, scale) \
        if with_bwd else None
    torch.cuda.synchronize()
    st, where = fa.fa_device_status(None)
    assert st == 0, f"device status {st} at wait {where}"
    ins = tuple(to64(t) for t in (q, k, v, do)) + (cq.numpy(), ck.numpy(), scale)
    outs = (to64(o), to64(lse)) + (tuple(to64(t) for t in g) if g else ())
    return ins, outs


def check(lq, lk, Hq, Hkv, d, causal, seed=1, with_bwd=True):
    """Full oracle comparison, strict bar on every output."""
    (q, k, v, do, cq, ck, scale), out = run(lq, lk, Hq, Hkv, d, causal, seed, with_bwd)
    o_ref, lse_ref = oracle.attention_forward_varlen(q, k, v, cq, ck, causal, scale)
    empty = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(out[1]), empty), "rows that see no key differ"
    assert (out[0].transpose(1, 0, 2)[empty] == 0).all()
    ok = ~empty
    check_fwd(out[0].transpose(1, 0, 2)[ok], out[1][ok], o_ref.transpose(1, 0, 2)[ok],
              lse_ref[ok])
    if with_bwd:
        ref = oracle.attention_backward_varlen(q, k, v, do, cq, ck, causal, scale)
        check_grads(out[2:], ref)
    return out


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("hq,hkv", [(4, 4), (4, 1)])
def test_ragged_batches(d, causal, hq, hkv):
    lengths = [300, 1, 129, 640, 77, 256, 513]
    check(lengths, lengths, hq, hkv, d, causal, seed=d + hkv)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_mqa_wide_group_packed(d, causal):
    """32 query heads on one kv head in a packed batch: the backward's exact
    D is recomputed by the packed forward with the D epilogue, written into
    each sequence's padded workspace rows."""
    lengths = [300, 1, 129, 640, 77]
    check(lengths, lengths, 32, 1, d, causal, seed=40 + d)


@pytest.mark.parametrize("causal", [False, True])
def test_query_and_key_lengths_differ(causal):
    check([200, 33, 400, 128], [100, 257, 64, 500], 4, 2, 128, causal, seed=3)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_sequences_with_no_rows_or_no_keys(d):
    """Length-0 sequences between others, and a sequence whose queries have
    no keys (O = 0, LSE = -inf, no gradient)."""
    check([150, 0, 90, 200, 0], [150, 0, 90, 0, 60], 2, 2, d, False, seed=4)


@pytest.mark.parametrize("causal", [False, True])
def test_many_short_sequences(causal):
    lengths = make_varlen_lengths(64, 1, 300, seed=5)
    check(lengths, lengths, 4, 2, 128, causal, seed=5)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_equal_lengths_match_the_fixed_length_kernels(d, causal):
    """Equal lengths: the packed batch is the fixed-length batch in
    [B, N, H, d] storage, and the forward must agree bit for bit with the
    strided fixed-length call (same arithmetic); gradients within the
    tolerance (dQ is summed with unordered atomics)."""
    B, N, Hq, Hkv = 3, 700, 4, 2
    wl = Workload("eq", B, Hq, Hkv, N, N, d, causal, 9)
    q, k, v, do = (t.to(DEV) for t in make_inputs(wl))
    pack = lambda t: t.transpose(1, 2).contiguous()            # [B, N, H, d]
    qp, kp, vp, dop = pack(q), pack(k), pack(v), pack(do)
    cu = torch.arange(0, (B + 1) * N, N, dtype=torch.int32, device=DEV)
    o1, l1 = fa.forward_varlen(qp.view(B * N, Hq, d), kp.view(B * N, Hkv, d),
                               vp.view(B * N, Hkv, d), cu, cu, N, N, causal, wl.scale)
    view = lambda t: t.transpose(1, 2)                          # strided [B, H, N, d]
    o2, l2 = fa.forward(view(qp), view(kp), view(vp), causal, wl.scale,
                        out=torch.empty_like(qp).transpose(1, 2))
    g1 = fa.backward_varlen(qp.view(B * N, Hq, d), kp.view(B * N, Hkv, d), vp.view(B * N, Hkv, d),
                            o1, l1, dop.view(B * N, Hq, d), cu, cu, N, N, causal, wl.scale)
    g2 = fa.backward(view(qp), view(kp), view(vp), o2, l2, view(dop), causal, wl.scale)
    torch.cuda.synchronize()
    assert torch.equal(o1.view(B, N, Hq, d), o2.transpose(1, 2))
    assert torch.equal(l1.view(Hq, B, N).transpose(0, 1), l2)
    for a, b in zip(g1, g2):
        err = (a.view(B, N, -1, d).double() - b.transpose(1, 2).double()).abs().max().item()
        assert err <= 2e-2


def test_long_mixed_batch():
    """About 24k packed tokens, lengths 128..4096, 16 heads, d = 128: full
    oracle on three sequences (first, longest, last), the rest checked by
    the sums that hold at any size."""
    lengths = make_varlen_lengths(12, 128, 4096, seed=11)
    Hq = Hkv = 16
    (q, k, v, do, cq, ck, scale), out = run(lengths, lengths, Hq, Hkv, 128, True, seed=11)
    o, lse, dq, dk, dv = out
    for x in out:
        assert np.isfinite(x).all()
    pick = sorted({0, int(np.argmax(lengths)), len(lengths) - 1})
    for b in pick:
        sl = slice(int(cq[b]), int(cq[b + 1]))
        one = lambda t: t[sl]
        cu1 = np.array([0, lengths[b]])
        o_ref, lse_ref = oracle.attention_forward_varlen(one(q), one(k), one(v), cu1, cu1, True,
                                                         scale)
        check_fwd(o[sl], lse[:, sl], o_ref, lse_ref)
        ref = oracle.attention_backward_varlen(one(q), one(k), one(v), one(do), cu1, cu1, True,
                                               scale)
        check_grads((dq[sl], dk[sl], dv[sl]), ref)
    # rows of dS sum to zero: per sequence and head, dK sums to zero over keys
    for b in range(len(lengths)):
        sl = slice(int(cq[b]), int(cq[b + 1]))
        s = np.abs(dk[sl].sum(axis=0)).max()
        assert s <= 2e-3 * max(1.0, np.abs(dk[sl]).sum(axis=0).max())
