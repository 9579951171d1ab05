"""Pins for the oracle's block-sparse attention (QbitAI FA1 article, results
section: block-sparse FlashAttention), against facts that do not come from
the oracle's masking code:

  * an all-ones mask is the (already pinned) dense attention, and a
    block-lower-triangular mask under the causal mask is plain causal
    attention;
  * a mask that sends every query block to exactly one key block equals the
    dense oracle run on that (query block, key block) sub-problem, which
    fixes the mask's orientation (rows = query blocks) and its indexing;
  * pure-Python brute force with the block mask expanded element by element;
  * rows whose mask row is all zero give O = 0, LSE = -inf and no gradient,
    and removing them does not change dK, dV;
  * central finite differences of <O, dO> through the masked forward.
"""
import math

import numpy as np
import pytest

import oracle

BLK = oracle.BLOCK


def rnd(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def nblocks(n):
    return (n + BLK - 1) // BLK


def test_block_is_128():
    assert BLK == 128


@pytest.mark.parametrize("causal", [False, True])
def test_all_ones_mask_is_dense(causal):
    q, k, v, do = rnd((1, 2, 200, 4), 1), rnd((1, 1, 300, 4), 2), rnd((1, 1, 300, 4), 3), \
        rnd((1, 2, 200, 4), 4)
    m = np.ones((nblocks(200), nblocks(300)), np.uint8)
    o, lse = oracle.attention_forward(q, k, v, causal, 0.5)
    om, lm = oracle.attention_forward(q, k, v, causal, 0.5, block_mask=m)
    assert np.array_equal(o, om) and np.array_equal(lse, lm)
    g = oracle.attention_backward(q, k, v, do, causal, 0.5)
    gm = oracle.attention_backward(q, k, v, do, causal, 0.5, block_mask=m)
    for a, b in zip(g, gm):
        assert np.array_equal(a, b)


def test_block_lower_triangular_mask_with_causal_is_causal():
    n = 300
    q, k, v = rnd((1, 1, n, 4), 5), rnd((1, 1, n, 4), 6), rnd((1, 1, n, 4), 7)
    m = np.tril(np.ones((nblocks(n), nblocks(n)), np.uint8))
    o, lse = oracle.attention_forward(q, k, v, True, 0.5)
    om, lm = oracle.attention_forward(q, k, v, True, 0.5, block_mask=m)
    np.testing.assert_array_equal(o, om)
    np.testing.assert_array_equal(lse, lm)


def _one_block_per_row_case(nq, nk, shift, seed=11):
    nbq, nbk = nblocks(nq), nblocks(nk)
    m = np.zeros((nbq, nbk), np.uint8)
    target = [(i + shift) % nbk for i in range(nbq)]
    for i, j in enumerate(target):
        m[i, j] = 1
    q, k, v, do = (rnd((1, 2, nq, 4), seed), rnd((1, 2, nk, 4), seed + 1),
                   rnd((1, 2, nk, 4), seed + 2), rnd((1, 2, nq, 4), seed + 3))
    return m, target, q, k, v, do


@pytest.mark.parametrize("nq,nk,shift", [(300, 300, 1), (300, 300, 2), (260, 400, 1)])
def test_one_key_block_per_query_block_is_the_sub_problem(nq, nk, shift):
    """Query block I sees only key block J(I): its rows equal dense attention
    of Q_I on (K_J, V_J), and dK_J, dV_J sum the sub-problems that use J."""
    m, target, q, k, v, do = _one_block_per_row_case(nq, nk, shift)
    o, lse = oracle.attention_forward(q, k, v, False, 0.4, block_mask=m)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, False, 0.4, block_mask=m)
    dk_exp, dv_exp = np.zeros_like(dk), np.zeros_like(dv)
    for i, j in enumerate(target):
        r = slice(i * BLK, min(nq, (i + 1) * BLK))
        c = slice(j * BLK, min(nk, (j + 1) * BLK))
        o_s, l_s = oracle.attention_forward(q[:, :, r], k[:, :, c], v[:, :, c], False, 0.4)
        np.testing.assert_allclose(o[:, :, r], o_s, atol=1e-13)
        np.testing.assert_allclose(lse[:, :, r], l_s, atol=1e-13)
        g = oracle.attention_backward(q[:, :, r], k[:, :, c], v[:, :, c], do[:, :, r], False, 0.4)
        np.testing.assert_allclose(dq[:, :, r], g[0], atol=1e-12)
        dk_exp[:, :, c] += g[1]
        dv_exp[:, :, c] += g[2]
    np.testing.assert_allclose(dk, dk_exp, atol=1e-12)
    np.testing.assert_allclose(dv, dv_exp, atol=1e-12)


def test_transposed_mask_is_caught():
    """Planted mistake: applying the mask with rows and columns swapped
    breaks the sub-problem pin."""
    m, target, q, k, v, _ = _one_block_per_row_case(300, 300, 1)
    o_bad, _ = oracle.attention_forward(q, k, v, False, 0.4, block_mask=m.T.copy())
    r, c = slice(0, BLK), slice(target[0] * BLK, (target[0] + 1) * BLK)
    o_s, _ = oracle.attention_forward(q[:, :, r], k[:, :, c], v[:, :, c], False, 0.4)
    assert not np.allclose(o_bad[:, :, r], o_s, atol=1e-6)


def brute_force_masked(q, k, v, causal, scale, mask):
    """Pure-Python loops (no NumPy), the block mask looked up per element;
    returns O and LSE (None for rows that see no key)."""
    Nq, d = len(q), len(q[0])
    Nk = len(k)
    O, L = [], []
    for i in range(Nq):
        w = []
        for j in range(Nk):
            if (causal and j > i) or not mask[i // BLK][j // BLK]:
                w.append(0.0)
                continue
            w.append(math.exp(scale * sum(q[i][c] * k[j][c] for c in range(d))))
        z = sum(w)
        if z == 0.0:
            O.append([0.0] * d)
            L.append(None)
            continue
        O.append([sum(w[j] * v[j][c] for j in range(Nk)) / z for c in range(d)])
        L.append(math.log(z))
    return O, L


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("nq,nk", [(300, 300), (260, 140), (140, 390)])
def test_brute_force_random_mask(causal, nq, nk):
    rng = np.random.default_rng(nq * 7 + nk + int(causal))
    m = (rng.random((nblocks(nq), nblocks(nk))) < 0.6).astype(np.uint8)
    m[0, 0] = 1
    q, k, v = rnd((1, 1, nq, 2), 21), rnd((1, 1, nk, 2), 22), rnd((1, 1, nk, 2), 23)
    o, lse = oracle.attention_forward(q, k, v, causal, 0.9, block_mask=m)
    ob, lb = brute_force_masked(q[0, 0].tolist(), k[0, 0].tolist(), v[0, 0].tolist(), causal,
                                0.9, m.tolist())
    np.testing.assert_allclose(o[0, 0], np.array(ob), atol=1e-12)
    for i, l_ in enumerate(lb):
        if l_ is None:
            assert lse[0, 0, i] == -np.inf
        else:
            assert abs(lse[0, 0, i] - l_) < 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_rows_that_see_nothing(causal):
    """Query block 1 has an all-zero mask row: O = 0, LSE = -inf, dQ = 0,
    and dK, dV equal the backward without those query rows at all."""
    nq = nk = 300
    m = np.ones((3, 3), np.uint8)
    m[1, :] = 0
    q, k, v, do = (rnd((1, 2, nq, 4), 31), rnd((1, 1, nk, 4), 32), rnd((1, 1, nk, 4), 33),
                   rnd((1, 2, nq, 4), 34))
    o, lse = oracle.attention_forward(q, k, v, causal, 0.5, block_mask=m)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, causal, 0.5, block_mask=m)
    rows = slice(128, 256)
    assert (o[:, :, rows] == 0).all() and (lse[:, :, rows] == -np.inf).all()
    assert (dq[:, :, rows] == 0).all()
    assert np.isfinite(dq).all() and np.isfinite(dk).all() and np.isfinite(dv).all()
    if not causal:
        keep = np.r_[0:128, 256:300]
        g = oracle.attention_backward(q[:, :, keep], k, v, do[:, :, keep], False, 0.5)
        np.testing.assert_allclose(dk, g[1], atol=1e-12)
        np.testing.assert_allclose(dv, g[2], atol=1e-12)
    # the other rows are untouched by the empty block row
    o_d, _ = oracle.attention_forward(q, k, v, causal, 0.5)
    np.testing.assert_allclose(o[:, :, :128], o_d[:, :, :128], atol=1e-14)


def _fd_grads(q, k, v, do, causal, scale, mask, h=1e-6):
    def loss(q_, k_, v_):
        o, _ = oracle.attention_forward(q_, k_, v_, causal, scale, block_mask=mask)
        return float((o * do).sum())
    out = []
    for which in range(3):
        xs = [q.copy(), k.copy(), v.copy()]
        g = np.zeros_like(xs[which])
        for idx in np.ndindex(*xs[which].shape):
            xp = [x.copy() for x in xs]
            xm = [x.copy() for x in xs]
            xp[which][idx] += h
            xm[which][idx] -= h
            g[idx] = (loss(*xp) - loss(*xm)) / (2 * h)
        out.append(g)
    return out


@pytest.mark.parametrize("causal,mask", [(False, [[1, 0], [1, 1]]), (False, [[0, 1], [1, 0]]),
                                         (True, [[1, 0], [0, 1]]), (True, [[0, 0], [1, 1]])])
def test_masked_gradients_match_finite_differences(causal, mask):
    n, d = 136, 2
    m = np.array(mask, np.uint8)
    q, k, v, do = rnd((1, 1, n, d), 41), rnd((1, 1, n, d), 42), rnd((1, 1, n, d), 43), \
        rnd((1, 1, n, d), 44)
    got = oracle.attention_backward(q, k, v, do, causal, 0.8, block_mask=m)
    ref = _fd_grads(q, k, v, do, causal, 0.8, m)
    for g, r in zip(got, ref):
        assert np.abs(g - r).max() <= 1e-6 * max(1.0, np.abs(r).max())


def test_dq_rows_with_mask_match_full_backward():
    m = np.array([[1, 0, 1], [0, 1, 1], [1, 1, 0]], np.uint8)
    q, k, v, do = rnd((1, 2, 300, 4), 51), rnd((1, 2, 300, 4), 52), rnd((1, 2, 300, 4), 53), \
        rnd((1, 2, 300, 4), 54)
    dq = oracle.attention_backward(q, k, v, do, False, 0.5, block_mask=m)[0]
    rows = [0, 127, 128, 200, 299]
    got = oracle.attention_backward_dq_rows(q, k, v, do, False, 0.5, 0, 1, rows, block_mask=m)
    np.testing.assert_allclose(got, dq[0, 1, rows], atol=1e-14)
    o, lse = oracle.attention_forward(q, k, v, False, 0.5, block_mask=m)
    o_r, l_r = oracle.attention_forward_rows(q, k, v, False, 0.5, 0, 1, rows, block_mask=m)
    np.testing.assert_allclose(o_r, o[0, 1, rows], atol=1e-14)
    np.testing.assert_allclose(l_r, lse[0, 1, rows], atol=1e-14)
