"""Pins for the fp64 oracle, against facts that do not come from the oracle.

Each test checks the oracle against something fixed by the pages or by the
mathematics: hand-derived closed forms (tests/golden/closed_form.json),
brute force in pure Python, special cases with a known answer, invariants,
a library logsumexp, and central finite differences for the gradients.
The mutation tests at the end plant plausible mistakes in copies of the
oracle's outputs and check that some pin catches each one.
"""
import json
import math
import os
import random

import numpy as np
import pytest
import scipy.special

import oracle
from oracle import attention as oa

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "closed_form.json")


def rnd(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


# ---------------------------------------------------------------- closed forms
@pytest.mark.parametrize("case", json.load(open(GOLDEN))["cases"], ids=lambda c: c["name"])
def test_closed_form_golden(case):
    q, k, v = (np.array(case[x]) for x in ("q", "k", "v"))
    o, lse = oracle.attention_forward(q, k, v, case["causal"], case["scale"])
    np.testing.assert_allclose(o, np.array(case["o"]), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, np.array(case["lse"]), rtol=0, atol=1e-12)
    if "dq" in case:
        do = np.array(case["do"])
        dq, dk, dv = oracle.attention_backward(q, k, v, do, case["causal"], case["scale"])
        np.testing.assert_allclose(dq, np.array(case["dq"]), atol=1e-12)
        np.testing.assert_allclose(dk, np.array(case["dk"]), atol=1e-12)
        np.testing.assert_allclose(dv, np.array(case["dv"]), atol=1e-12)


def test_two_keys_is_a_sigmoid():
    """With two keys softmax is a logistic function of the score gap."""
    rng = np.random.default_rng(7)
    for _ in range(20):
        d = 3
        q = rng.standard_normal((1, 1, 1, d))
        k = rng.standard_normal((1, 1, 2, d))
        v = rng.standard_normal((1, 1, 2, d))
        sc = 0.7
        gap = sc * float(q[0, 0, 0] @ (k[0, 0, 0] - k[0, 0, 1]))
        w0 = 1.0 / (1.0 + math.exp(-gap))
        o, _ = oracle.attention_forward(q, k, v, False, sc)
        np.testing.assert_allclose(o[0, 0, 0], w0 * v[0, 0, 0] + (1 - w0) * v[0, 0, 1],
                                   atol=1e-13)


# ------------------------------------------------------------ brute force
def brute_force(q, k, v, causal, scale):
    """Pure-Python loops (no NumPy), softmax without any max shift."""
    B, Hq, Nq, d = len(q), len(q[0]), len(q[0][0]), len(q[0][0][0])
    Hkv, Nk = len(k[0]), len(k[0][0])
    g = Hq // Hkv
    O = [[[[0.0] * d for _ in range(Nq)] for _ in range(Hq)] for _ in range(B)]
    L = [[[0.0] * Nq for _ in range(Hq)] for _ in range(B)]
    for b in range(B):
        for h in range(Hq):
            kh = h // g
            for i in range(Nq):
                w = []
                for j in range(Nk):
                    if causal and j > i:
                        w.append(0.0)
                        continue
                    dot = sum(q[b][h][i][c] * k[b][kh][j][c] for c in range(d))
                    w.append(math.exp(scale * dot))
                z = sum(w)
                L[b][h][i] = math.log(z)
                for c in range(d):
                    O[b][h][i][c] = sum(w[j] * v[b][kh][j][c] for j in range(Nk)) / z
    return O, L


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("hq,hkv", [(2, 2), (4, 2), (3, 1)])
@pytest.mark.parametrize("nq,nk,d", [(5, 5, 4), (8, 8, 8), (3, 7, 2), (7, 3, 5)])
def test_brute_force(causal, hq, hkv, nq, nk, d):
    q = rnd((2, hq, nq, d), 1)
    k = rnd((2, hkv, nk, d), 2)
    v = rnd((2, hkv, nk, d), 3)
    sc = 1 / math.sqrt(d)
    o, lse = oracle.attention_forward(q, k, v, causal, sc)
    ob, lb = brute_force(q.tolist(), k.tolist(), v.tolist(), causal, sc)
    np.testing.assert_allclose(o, np.array(ob), atol=1e-12)
    np.testing.assert_allclose(lse, np.array(lb), atol=1e-12)


# ------------------------------------------------------------ special cases
@pytest.mark.parametrize("causal", [False, True])
def test_identity_values_give_probabilities(causal):
    """With V = I (Nk = d) the output rows are the rows of P: they are
    non-negative, sum to 1, and vanish above the diagonal when causal."""
    n = 16
    q = rnd((1, 2, n, n), 4)
    k = rnd((1, 2, n, n), 5)
    v = np.broadcast_to(np.eye(n), (1, 2, n, n)).copy()
    p, _ = oracle.attention_forward(q, k, v, causal, 0.5)
    assert (p >= 0).all()
    np.testing.assert_allclose(p.sum(-1), 1.0, atol=1e-14)
    if causal:
        assert np.all(np.triu(p[0, 0], 1) == 0)
        assert np.all(np.triu(p[0, 1], 1) == 0)


@pytest.mark.parametrize("causal", [False, True])
def test_zero_query_averages_values(causal):
    n, d = 33, 8
    q = np.zeros((1, 1, n, d))
    k = rnd((1, 1, n, d), 6)
    v = rnd((1, 1, n, d), 7)
    o, lse = oracle.attention_forward(q, k, v, causal, 0.3)
    for i in range(n):
        hi = i + 1 if causal else n
        np.testing.assert_allclose(o[0, 0, i], v[0, 0, :hi].mean(0), atol=1e-13)
        assert abs(lse[0, 0, i] - math.log(hi)) < 1e-13


def test_causal_row_zero_is_first_value():
    q = rnd((2, 3, 9, 4), 8)
    k = rnd((2, 3, 9, 4), 9)
    v = rnd((2, 3, 9, 4), 10)
    o, lse = oracle.attention_forward(q, k, v, True, 0.25)
    np.testing.assert_allclose(o[:, :, 0], v[:, :, 0], atol=1e-15)
    np.testing.assert_allclose(lse[:, :, 0],
                               0.25 * np.einsum("bhc,bhc->bh", q[:, :, 0], k[:, :, 0]),
                               atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_constant_values_give_constant_output(causal):
    q = rnd((1, 2, 12, 6), 11)
    k = rnd((1, 2, 12, 6), 12)
    v = np.tile(rnd((1, 2, 1, 6), 13), (1, 1, 12, 1))
    o, _ = oracle.attention_forward(q, k, v, causal, 1.0)
    np.testing.assert_allclose(o, v, atol=1e-13)


def test_large_scale_tends_to_hard_attention():
    """As the scale grows, softmax tends to the argmax row of V."""
    q = rnd((1, 1, 6, 4), 14)
    k = rnd((1, 1, 10, 4), 15)
    v = rnd((1, 1, 10, 4), 16)
    o, _ = oracle.attention_forward(q, k, v, False, 1e4)
    am = (q[0, 0] @ k[0, 0].T).argmax(1)
    np.testing.assert_allclose(o[0, 0], v[0, 0, am], atol=1e-9)


def test_lse_matches_library_logsumexp():
    q = rnd((2, 2, 20, 8), 17, 3.0)
    k = rnd((2, 2, 25, 8), 18, 3.0)
    v = rnd((2, 2, 25, 8), 19)
    for causal in (False, True):
        _, lse = oracle.attention_forward(q, k, v, causal, 0.35)
        s = 0.35 * np.einsum("bhid,bhjd->bhij", q, k)
        if causal:
            s = np.where(np.tril(np.ones((20, 25), bool)), s, -np.inf)
        np.testing.assert_allclose(lse, scipy.special.logsumexp(s, axis=-1), atol=1e-12)


def test_key_shift_invariance():
    """Adding c to every key adds scale*q.c to each score row: O is
    unchanged and LSE moves by scale*q.c."""
    q = rnd((1, 2, 10, 5), 20)
    k = rnd((1, 2, 14, 5), 21)
    v = rnd((1, 2, 14, 5), 22)
    c = rnd((5,), 23)
    for causal in (False, True):
        o1, l1 = oracle.attention_forward(q, k, v, causal, 0.5)
        o2, l2 = oracle.attention_forward(q, k + c, v, causal, 0.5)
        np.testing.assert_allclose(o1, o2, atol=1e-12)
        np.testing.assert_allclose(l2 - l1, 0.5 * (q @ c), atol=1e-12)


def test_permutation_equivariance():
    q = rnd((1, 1, 7, 4), 24)
    k = rnd((1, 1, 11, 4), 25)
    v = rnd((1, 1, 11, 4), 26)
    pk = np.random.default_rng(0).permutation(11)
    pq = np.random.default_rng(1).permutation(7)
    o1, l1 = oracle.attention_forward(q, k, v, False, 0.5)
    o2, l2 = oracle.attention_forward(q[:, :, pq], k[:, :, pk], v[:, :, pk], False, 0.5)
    np.testing.assert_allclose(o2, o1[:, :, pq], atol=1e-13)
    np.testing.assert_allclose(l2, l1[:, :, pq], atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_gqa_equals_repeated_kv(causal):
    hq, hkv = 6, 2
    q = rnd((2, hq, 9, 4), 27)
    k = rnd((2, hkv, 9, 4), 28)
    v = rnd((2, hkv, 9, 4), 29)
    do = rnd((2, hq, 9, 4), 30)
    kr, vr = np.repeat(k, hq // hkv, axis=1), np.repeat(v, hq // hkv, axis=1)
    o1, l1 = oracle.attention_forward(q, k, v, causal, 0.5)
    o2, l2 = oracle.attention_forward(q, kr, vr, causal, 0.5)
    np.testing.assert_allclose(o1, o2, atol=1e-14)
    np.testing.assert_allclose(l1, l2, atol=1e-14)
    dq1, dk1, dv1 = oracle.attention_backward(q, k, v, do, causal, 0.5)
    dq2, dk2, dv2 = oracle.attention_backward(q, kr, vr, do, causal, 0.5)
    np.testing.assert_allclose(dq1, dq2, atol=1e-13)
    g = hq // hkv
    np.testing.assert_allclose(dk1, dk2.reshape(2, hkv, g, 9, 4).sum(2), atol=1e-13)
    np.testing.assert_allclose(dv1, dv2.reshape(2, hkv, g, 9, 4).sum(2), atol=1e-13)


def test_kv_head_mapping_is_contiguous_groups():
    assert [oracle.kv_head(h, 8, 2) for h in range(8)] == [0, 0, 0, 0, 1, 1, 1, 1]
    assert [oracle.kv_head(h, 4, 1) for h in range(4)] == [0] * 4
    with pytest.raises(ValueError):
        oracle.kv_head(0, 6, 4)


def test_rows_and_chunking_are_exact(monkeypatch):
    q = rnd((1, 4, 40, 8), 31)
    k = rnd((1, 2, 40, 8), 32)
    v = rnd((1, 2, 40, 8), 33)
    do = rnd((1, 4, 40, 8), 34)
    for causal in (False, True):
        o, lse = oracle.attention_forward(q, k, v, causal, 0.4)
        rows = [0, 3, 17, 39]
        orow, lrow = oracle.attention_forward_rows(q, k, v, causal, 0.4, 0, 3, rows)
        np.testing.assert_allclose(orow, o[0, 3, rows], atol=1e-14)
        np.testing.assert_allclose(lrow, lse[0, 3, rows], atol=1e-14)
        g_full = oracle.attention_backward(q, k, v, do, causal, 0.4)
        monkeypatch.setattr(oa, "_MAX_CHUNK_ELEMS", 3 * 40)
        o2, l2 = oracle.attention_forward(q, k, v, causal, 0.4)
        g_chunk = oracle.attention_backward(q, k, v, do, causal, 0.4)
        monkeypatch.undo()
        np.testing.assert_allclose(o2, o, atol=1e-14)
        np.testing.assert_allclose(l2, lse, atol=1e-14)
        for a, b in zip(g_full, g_chunk):
            np.testing.assert_allclose(a, b, atol=1e-13)


# ------------------------------------------------------------ gradients
def finite_difference_grads(q, k, v, do, causal, scale, h=1e-6):
    """Central differences of L = <O, dO> through the forward oracle."""
    def loss(q_, k_, v_):
        o, _ = oracle.attention_forward(q_, k_, v_, causal, scale)
        return float((o * do).sum())
    grads = []
    for which in range(3):
        xs = [q.copy(), k.copy(), v.copy()]
        g = np.zeros_like(xs[which])
        it = np.nditer(xs[which], flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp = [x.copy() for x in xs]
            xm = [x.copy() for x in xs]
            xp[which][idx] += h
            xm[which][idx] -= h
            g[idx] = (loss(*xp) - loss(*xm)) / (2 * h)
        grads.append(g)
    return grads


def rel_err(a, b):
    return float(np.abs(a - b).max() / max(1e-30, np.abs(b).max()))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("hq,hkv,nq,nk,d", [(2, 2, 6, 6, 4), (4, 2, 5, 7, 3), (3, 1, 8, 8, 8)])
def test_gradients_match_finite_differences(causal, hq, hkv, nq, nk, d):
    q = rnd((1, hq, nq, d), 35)
    k = rnd((1, hkv, nk, d), 36)
    v = rnd((1, hkv, nk, d), 37)
    do = rnd((1, hq, nq, d), 38)
    sc = 1 / math.sqrt(d)
    got = oracle.attention_backward(q, k, v, do, causal, sc)
    ref = finite_difference_grads(q, k, v, do, causal, sc)
    for g, r in zip(got, ref):
        assert rel_err(g, r) < 1e-6


@pytest.mark.parametrize("causal", [False, True])
def test_gradient_invariants(causal):
    """Rows of dS sum to zero, so keys' gradients sum to zero; rows of P sum
    to one, so the value gradients sum to the output gradients; and D from
    P*dP equals rowsum(dO*O)."""
    q = rnd((2, 4, 30, 8), 39)
    k = rnd((2, 2, 30, 8), 40)
    v = rnd((2, 2, 30, 8), 41)
    do = rnd((2, 4, 30, 8), 42)
    dq, dk, dv, (o, lse, dd) = oracle.attention_backward(q, k, v, do, causal, 0.3,
                                                         return_aux=True)
    np.testing.assert_allclose(dk.sum(2), 0.0, atol=1e-12)
    np.testing.assert_allclose(dv.sum(2), do.reshape(2, 2, 2, 30, 8).sum((2, 3)), atol=1e-12)
    np.testing.assert_allclose(dd, (do * o).sum(-1), atol=1e-12)
    o2, l2 = oracle.attention_forward(q, k, v, causal, 0.3)
    np.testing.assert_allclose(o, o2, atol=1e-14)
    np.testing.assert_allclose(lse, l2, atol=1e-14)


def test_dq_rows_match_full_backward():
    q = rnd((2, 4, 21, 8), 60)
    k = rnd((2, 2, 21, 8), 61)
    v = rnd((2, 2, 21, 8), 62)
    do = rnd((2, 4, 21, 8), 63)
    for causal in (False, True):
        dq = oracle.attention_backward(q, k, v, do, causal, 0.4)[0]
        rows = [0, 1, 7, 20]
        got = oracle.attention_backward_dq_rows(q, k, v, do, causal, 0.4, 1, 3, rows)
        np.testing.assert_allclose(got, dq[1, 3, rows], atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("hq,hkv,nq,nk", [(4, 2, 21, 21), (4, 1, 30, 17), (4, 4, 13, 29),
                                          (8, 1, 40, 40)])
def test_kv_rows_match_full_backward(monkeypatch, causal, hq, hkv, nq, nk):
    """dK / dV of sampled key rows equal the full backward's rows; small row
    chunks make the per-chunk causal key horizon cut across the rows."""
    import oracle.attention as oa
    monkeypatch.setattr(oa, "_MAX_CHUNK_ELEMS", 7 * nk)
    q = rnd((2, hq, nq, 8), 70)
    k = rnd((2, hkv, nk, 8), 71)
    v = rnd((2, hkv, nk, 8), 72)
    do = rnd((2, hq, nq, 8), 73)
    _, dk, dv = oracle.attention_backward(q, k, v, do, causal, 0.4)
    keys = [0, 1, nk // 2, nk - 1]
    for kvh in range(hkv):
        gk, gv = oracle.attention_backward_kv_rows(q, k, v, do, causal, 0.4, 1, kvh, keys)
        np.testing.assert_allclose(gk, dk[1, kvh, keys], atol=1e-13)
        np.testing.assert_allclose(gv, dv[1, kvh, keys], atol=1e-13)
    # a subset of the group's heads gives that subset's share; the shares add up
    g = hq // hkv
    parts = [oracle.attention_backward_kv_rows(q, k, v, do, causal, 0.4, 0, 0, keys, heads=[h])
             for h in range(g)]
    np.testing.assert_allclose(sum(p_[0] for p_ in parts), dk[0, 0, keys], atol=1e-13)
    np.testing.assert_allclose(sum(p_[1] for p_ in parts), dv[0, 0, keys], atol=1e-13)
    if hkv > 1:                      # a head of another group is refused
        with pytest.raises(ValueError):
            oracle.attention_backward_kv_rows(q, k, v, do, causal, 0.4, 0, 0, keys,
                                              heads=[hq - 1])


def test_kv_rows_with_block_mask_and_empty_rows():
    q = rnd((1, 2, 300, 8), 74)
    k = rnd((1, 1, 260, 8), 75)
    v = rnd((1, 1, 260, 8), 76)
    do = rnd((1, 2, 300, 8), 77)
    mask = np.array([[1, 0, 1], [0, 0, 0], [1, 1, 0]], np.uint8)   # query block 1 sees nothing
    for causal in (False, True):
        _, dk, dv = oracle.attention_backward(q, k, v, do, causal, 0.3, block_mask=mask)
        keys = [0, 127, 128, 200, 259]
        gk, gv = oracle.attention_backward_kv_rows(q, k, v, do, causal, 0.3, 0, 0, keys,
                                                   block_mask=mask)
        np.testing.assert_allclose(gk, dk[0, 0, keys], atol=1e-13)
        np.testing.assert_allclose(gv, dv[0, 0, keys], atol=1e-13)


def test_backward_group_subset():
    q = rnd((2, 4, 10, 4), 43)
    k = rnd((2, 2, 10, 4), 44)
    v = rnd((2, 2, 10, 4), 45)
    do = rnd((2, 4, 10, 4), 46)
    full = oracle.attention_backward(q, k, v, do, True, 0.5)
    part = oracle.attention_backward(q, k, v, do, True, 0.5, heads=[(1, 0)])
    np.testing.assert_allclose(part[0][1, 0:2], full[0][1, 0:2], atol=1e-14)
    np.testing.assert_allclose(part[1][1, 0], full[1][1, 0], atol=1e-14)
    assert np.isnan(part[1][0, 0]).all()


# ------------------------------------------------------------ planted mistakes
def _grad_pins_pass(dq, dk, dv, q, k, v, do, causal, sc):
    ref = finite_difference_grads(q, k, v, do, causal, sc)
    return all(rel_err(g, r) < 1e-6 for g, r in zip((dq, dk, dv), ref))


def test_pins_catch_planted_gradient_mistakes():
    """Each plausible slip (a dropped scale, a wrong sign, a transposed
    operand, a missing D term) makes the finite-difference pin fail."""
    q = rnd((1, 2, 5, 3), 47)
    k = rnd((1, 2, 5, 3), 48)
    v = rnd((1, 2, 5, 3), 49)
    do = rnd((1, 2, 5, 3), 50)
    sc = 0.6
    dq, dk, dv = oracle.attention_backward(q, k, v, do, True, sc)
    assert _grad_pins_pass(dq, dk, dv, q, k, v, do, True, sc)
    assert not _grad_pins_pass(dq, dk / sc, dv, q, k, v, do, True, sc)      # dropped scale
    assert not _grad_pins_pass(-dq, dk, dv, q, k, v, do, True, sc)          # sign
    assert not _grad_pins_pass(dq, dk, dv[:, :, ::-1], q, k, v, do, True, sc)  # index order
    # dS without the D term: P * dP
    o, lse = oracle.attention_forward(q, k, v, True, sc)
    s = sc * np.einsum("bhid,bhjd->bhij", q, k)
    s = np.where(np.tril(np.ones((5, 5), bool)), s, -np.inf)
    p = np.exp(s - lse[..., None])
    dp = np.einsum("bhid,bhjd->bhij", do, v)
    dq_bad = sc * np.einsum("bhij,bhjd->bhid", p * dp, k)
    assert not _grad_pins_pass(dq_bad, dk, dv, q, k, v, do, True, sc)


def test_pins_catch_planted_forward_mistakes():
    """A transposed score matrix, a mask on the wrong side and a missing scale
    each break a forward pin."""
    n, d = 6, 4
    q = rnd((1, 1, n, d), 51)
    k = rnd((1, 1, n, d), 52)
    v = rnd((1, 1, n, d), 53)
    ob, lb = brute_force(q.tolist(), k.tolist(), v.tolist(), True, 0.5)
    ob = np.array(ob)
    s = 0.5 * q[0, 0] @ k[0, 0].T

    def fwd(s_):
        p = np.exp(s_ - scipy.special.logsumexp(s_, axis=1, keepdims=True))
        return p @ v[0, 0]
    tril = np.tril(np.ones((n, n), bool))
    assert np.allclose(fwd(np.where(tril, s, -np.inf)), ob[0, 0])
    assert not np.allclose(fwd(np.where(tril, s.T, -np.inf)), ob[0, 0])
    assert not np.allclose(fwd(np.where(tril.T, s, -np.inf)), ob[0, 0])
    assert not np.allclose(fwd(np.where(tril, s / 0.5, -np.inf)), ob[0, 0])
