"""Pins for the oracle's variable-length batches (packed sequences with
cumulative offsets), against facts that do not come from its own packing:

  * equal lengths are the (already pinned) batched dense attention of the
    same tensors viewed as [B, H, N, d];
  * pure-Python brute force per sequence, lengths 0 and 1 included;
  * sequences do not see each other: changing one sequence's inputs leaves
    every other sequence's outputs and gradients unchanged;
  * a sequence with queries but no keys gives O = 0 and LSE = -inf;
  * central finite differences of <O, dO> through the packed forward.
"""
import math

import numpy as np
import pytest

import oracle


def rnd(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def cum(lengths):
    return np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)


@pytest.mark.parametrize("causal", [False, True])
def test_equal_lengths_are_the_batched_dense_attention(causal):
    B, H, Hkv, N, d = 3, 4, 2, 37, 8
    q, k, v, do = rnd((B * N, H, d), 1), rnd((B * N, Hkv, d), 2), rnd((B * N, Hkv, d), 3), \
        rnd((B * N, H, d), 4)
    cu = cum([N] * B)
    o, lse = oracle.attention_forward_varlen(q, k, v, cu, cu, causal, 0.3)
    bat = lambda x: x.reshape(B, N, x.shape[1], d).transpose(0, 2, 1, 3)
    o_ref, lse_ref = oracle.attention_forward(bat(q), bat(k), bat(v), causal, 0.3)
    np.testing.assert_allclose(bat(o), o_ref, atol=1e-14)
    np.testing.assert_allclose(lse.reshape(H, B, N).transpose(1, 0, 2), lse_ref, atol=1e-14)
    g = oracle.attention_backward_varlen(q, k, v, do, cu, cu, causal, 0.3)
    g_ref = oracle.attention_backward(bat(q), bat(k), bat(v), bat(do), causal, 0.3)
    for a, r in zip(g, g_ref):
        np.testing.assert_allclose(bat(a), r, atol=1e-13)


def brute(q, k, v, causal, scale):
    """One sequence, one head, pure Python: (O rows, LSE list or None rows)."""
    O, L = [], []
    for i in range(len(q)):
        w = [0.0 if (causal and j > i) else
             math.exp(scale * sum(a * b for a, b in zip(q[i], k[j]))) for j in range(len(k))]
        z = sum(w)
        if z == 0.0:
            O.append([0.0] * len(q[i]))
            L.append(None)
            continue
        O.append([sum(w[j] * v[j][c] for j in range(len(k))) / z for c in range(len(q[i]))])
        L.append(math.log(z))
    return O, L


@pytest.mark.parametrize("causal", [False, True])
def test_brute_force_ragged(causal):
    lq, lk = [5, 0, 1, 9, 3, 4], [5, 2, 1, 9, 6, 0]
    H, Hkv, d = 2, 1, 3
    cq, ck = cum(lq), cum(lk)
    q, k, v = rnd((cq[-1], H, d), 5), rnd((ck[-1], Hkv, d), 6), rnd((ck[-1], Hkv, d), 7)
    o, lse = oracle.attention_forward_varlen(q, k, v, cq, ck, causal, 0.7)
    for b in range(len(lq)):
        for h in range(H):
            qs = q[cq[b]:cq[b + 1], h].tolist()
            ks = k[ck[b]:ck[b + 1], h // (H // Hkv)].tolist()
            vs = v[ck[b]:ck[b + 1], h // (H // Hkv)].tolist()
            ob, lb = brute(qs, ks, vs, causal, 0.7)
            for i in range(lq[b]):
                np.testing.assert_allclose(o[cq[b] + i, h], ob[i], atol=1e-12)
                if lb[i] is None:
                    assert lse[h, cq[b] + i] == -np.inf
                else:
                    assert abs(lse[h, cq[b] + i] - lb[i]) < 1e-12
    # the last sequence has queries but no keys
    assert (o[cq[5]:cq[6]] == 0).all() and np.isneginf(lse[:, cq[5]:cq[6]]).all()


def test_sequences_do_not_see_each_other():
    lq = lk = [7, 12, 5]
    cu = cum(lq)
    H, d = 2, 4
    q, k, v, do = rnd((24, H, d), 8), rnd((24, H, d), 9), rnd((24, H, d), 10), rnd((24, H, d), 11)
    o1, _ = oracle.attention_forward_varlen(q, k, v, cu, cu, False, 0.5)
    g1 = oracle.attention_backward_varlen(q, k, v, do, cu, cu, False, 0.5)
    k2, v2, q2 = k.copy(), v.copy(), q.copy()
    k2[7:19] += 1.0
    v2[7:19] -= 2.0
    q2[7:19] *= 3.0
    o2, _ = oracle.attention_forward_varlen(q2, k2, v2, cu, cu, False, 0.5)
    g2 = oracle.attention_backward_varlen(q2, k2, v2, do, cu, cu, False, 0.5)
    other = np.r_[0:7, 19:24]
    np.testing.assert_array_equal(o1[other], o2[other])
    for a, b in zip(g1, g2):
        np.testing.assert_array_equal(a[other], b[other])
    assert not np.allclose(o1[7:19], o2[7:19])


def test_packing_mistake_is_caught():
    """Planted mistake: attending across the whole packed batch (one long
    sequence) differs from the per-sequence result."""
    cu = cum([6, 6])
    q, k, v = rnd((12, 1, 4), 12), rnd((12, 1, 4), 13), rnd((12, 1, 4), 14)
    o, _ = oracle.attention_forward_varlen(q, k, v, cu, cu, False, 0.5)
    o_bad, _ = oracle.attention_forward_varlen(q, k, v, [0, 12], [0, 12], False, 0.5)
    assert not np.allclose(o, o_bad, atol=1e-6)


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_gradients_match_finite_differences(causal):
    lq, lk = [3, 5], [4, 2]
    cq, ck = cum(lq), cum(lk)
    q, k, v, do = rnd((8, 2, 2), 15), rnd((6, 1, 2), 16), rnd((6, 1, 2), 17), rnd((8, 2, 2), 18)
    got = oracle.attention_backward_varlen(q, k, v, do, cq, ck, causal, 0.9)

    def loss(q_, k_, v_):
        o, _ = oracle.attention_forward_varlen(q_, k_, v_, cq, ck, causal, 0.9)
        return float((o * do).sum())
    h = 1e-6
    for which, g in enumerate(got):
        xs = [q, k, v]
        for idx in np.ndindex(*xs[which].shape):
            xp = [x.copy() for x in xs]
            xm = [x.copy() for x in xs]
            xp[which][idx] += h
            xm[which][idx] -= h
            fd = (loss(*xp) - loss(*xm)) / (2 * h)
            assert abs(g[idx] - fd) <= 1e-6 * max(1.0, abs(fd))
