"""GPU parity of fa_bwd (with fa_fwd's O and LSE) against the fp64 oracle,
through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_71_b200 import binding as fa
from exact_io_aware_71_b200.inputs import Workload, make_inputs, workloads
from tests.parity import check_grads, sample_rows, to64

pytestmark = pytest.mark.gpu

DEV = "cuda"


def run(wl, qmul=1.0, residual=False):
    """fa.forward + fa.backward on the GPU; with ``residual`` through
    fa_fwd_residual / fa_bwd_residual (the output's rounding residual kept)."""
    q, k, v, do = make_inputs(wl)
    if qmul != 1.0:
        q = (q.float() * qmul).to(torch.bfloat16)
    qd, kd, vd, dod = q.to(DEV), k.to(DEV), v.to(DEV), do.to(DEV)
    o_res = torch.empty_like(qd) if residual else None
    o, lse = fa.forward(qd, kd, vd, wl.causal, wl.scale, o_res=o_res)
    dq, dk, dv = fa.backward(qd, kd, vd, o, lse, dod, wl.causal, wl.scale, o_res=o_res)
    torch.cuda.synchronize()
    st, where = fa.fa_device_status(None)
    assert st == 0, f"device status {st} at wait {where}"
    return (q, k, v, do), (to64(dq), to64(dk), to64(dv))


def full_check(wl, qmul=1.0, frobenius_only=(), residual=False):
    (q, k, v, do), got = run(wl, qmul, residual)
    ref = oracle.attention_backward(to64(q), to64(k), to64(v), to64(do), wl.causal, wl.scale)
    return check_grads(got, ref, frobenius_only=frobenius_only)


def W(B, Hq, Hkv, Nq, Nk, d, causal, seed=21):
    return Workload(f"b{B}_{Hq}_{Hkv}_{Nq}_{Nk}_{d}_{int(causal)}", B, Hq, Hkv, Nq, Nk, d,
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
    """Includes key blocks no query can see (causal, Nk > Nq): dK = dV = 0."""
    full_check(W(1, 2, 1, nq, nk, 128, causal, seed=nq + nk))


@pytest.mark.parametrize("b,hq,hkv,n", [(1, 9, 9, 2048), (3, 6, 3, 1500)])
def test_causal_longest_first_head_groups(b, hq, hkv, n):
    """The causal d = 128 backward orders its CTAs longest walk first inside
    groups of kv heads whose Q, dO and fp32 dQ rows take at most 16 MiB.
    Nine heads at N = 2048 (2 MiB each) form groups of 8 and 1; nine kv
    heads of two query heads at N = 1500 (3 MiB each) form groups of 5 and
    4.  Both end on a short group, the decode's edge case."""
    full_check(W(b, hq, hkv, n, n, 128, True, seed=b * 100 + n))


@pytest.mark.parametrize("residual", [False, True])
@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_mqa_wide_group(causal, d, residual):
    """32 query heads on one kv head (N=1024): the per-CTA loop over the
    group.  Wide groups take an exact D (from the forward's residual output,
    or recomputed by a forward pass) and dS rounded to fp16, with every
    product on fp16 operands.  Strict bar on all three gradients
    (tests/test_precision_model.py shows why both are needed)."""
    full_check(W(1, 32, 1, 1024, 1024, d, causal, seed=3), residual=residual)


@pytest.mark.parametrize("hkv,residual", [(8, False), (1, False), (1, True), (2, False)])
def test_long_gqa_shape_full_oracle(hkv, residual):
    """The long-sequence GQA/MQA workload's head structure (Hq=32, Hkv=8, 2
    or 1, d=128, causal) at N=4096, where the complete fp64 backward is
    affordable for every head.  Strict bar on all three gradients."""
    full_check(W(1, 32, hkv, 4096, 4096, 128, True, seed=4), residual=residual)


@pytest.mark.parametrize("qmul", [2.0, 4.0])
def test_large_magnitude_scores(qmul):
    """Peaky softmax (stress inputs Q x 2 and Q x 4, outside the named
    workloads); dK held to the Frobenius bar.  With one query head per kv
    head the backward takes D from the bf16 output and dS as bf16 (the
    exact D and the fp16 dS are for wide groups); the exact-arithmetic model
    in tests/test_precision_model.py shows dK above the per-element bound
    there, mostly from D, and within it once D is exact."""
    full_check(W(1, 2, 2, 512, 512, 64, True, seed=9), qmul=qmul, frobenius_only=("dK",))


@pytest.mark.parametrize("hkv", [4, 2])
def test_backward_repeatable_within_tolerance(hkv):
    """dQ is accumulated with unordered fp32 atomics, so runs may differ in
    the last bits.  With one kv head per query head, dK and dV are
    accumulated in a fixed order and repeat bit for bit; when a GQA group's
    query heads are split over CTAs (as here, few key blocks), dK and dV are
    fp32 atomic sums too."""
    wl = W(1, 4, hkv, 640, 640, 128, True)
    _, g1 = run(wl)
    _, g2 = run(wl)
    if hkv == 4:
        assert np.array_equal(g1[1], g2[1]) and np.array_equal(g1[2], g2[2])
    for a, b in zip(g1, g2):
        assert np.abs(a - b).max() <= 2e-2


# --------------------------------------------------------------- full-size workloads
BWD_WORKLOADS = [n for n, w in workloads().items()
                 if "bwd" in w.directions and not n.startswith("tiny")]


@pytest.mark.parametrize("name", BWD_WORKLOADS)
def test_full_size(name):
    """Full-size backward on the GPU.  The oracle runs the complete backward
    on sampled (batch, kv head) groups whose query group is at most 4 heads
    (dK/dV need every query row of the group), dQ on sampled rows of
    sampled heads for every workload (each dQ row is exact on its own), and
    for GQA / MQA workloads dK / dV on sampled key rows (the first 8, the
    last 8 and 256 random) of every kv head."""
    wl = workloads()[name]
    (q, k, v, do), (dq, dk, dv) = run(wl)
    for g in (dq, dk, dv):
        assert np.isfinite(g).all()
    q, k, v, do = to64(q), to64(k), to64(v), to64(do)
    g = wl.Hq // wl.Hkv
    rng = np.random.default_rng(1)
    if g <= 4:
        groups = sorted({(0, 0), (wl.B - 1, wl.Hkv - 1),
                         (int(rng.integers(wl.B)), int(rng.integers(wl.Hkv)))})[:2]
        ref = oracle.attention_backward(q, k, v, do, wl.causal, wl.scale, heads=groups)
        sel_q = [(b, h) for (b, j) in groups for h in range(j * g, (j + 1) * g)]
        got = (np.stack([dq[b, h] for b, h in sel_q]), np.stack([dk[b, j] for b, j in groups]),
               np.stack([dv[b, j] for b, j in groups]))
        exp = (np.stack([ref[0][b, h] for b, h in sel_q]),
               np.stack([ref[1][b, j] for b, j in groups]),
               np.stack([ref[2][b, j] for b, j in groups]))
        check_grads(got, exp)
    heads = [(int(rng.integers(wl.B)), int(rng.integers(wl.Hq))) for _ in range(6)]
    heads += [(0, 0), (wl.B - 1, wl.Hq - 1)]
    got, exp = [], []
    for (b, h) in heads:
        rows = sample_rows(wl.Nq, 32, seed=7 * b + h)
        exp.append(oracle.attention_backward_dq_rows(q, k, v, do, wl.causal, wl.scale, b, h,
                                                     rows))
        got.append(dq[b, h, rows])
    check_grads([np.concatenate(got)], [np.concatenate(exp)], names=("dQ rows",))
    if g > 1:
        # GQA / MQA: dK and dV of sampled key rows of every kv head, each
        # summed over all query rows of the group's heads (the oracle's
        # per-head shares run in parallel threads; numpy releases the GIL).
        keys = sample_rows(wl.Nk, 256, seed=11)
        got_k, got_v, ref_k, ref_v = kv_rows_parallel(wl, q, k, v, do, dk, dv, keys)
        check_grads((got_k, got_v), (ref_k, ref_v), names=("dK rows", "dV rows"))


def kv_rows_parallel(wl, q, k, v, do, dk, dv, keys):
    """GPU and oracle dK / dV rows ``keys`` of every (batch, kv head)."""
    from concurrent.futures import ThreadPoolExecutor
    import os
    from threadpoolctl import threadpool_limits
    g = wl.Hq // wl.Hkv
    jobs = [(b, j, h) for b in range(wl.B) for j in range(wl.Hkv) for h in range(j * g, (j + 1) * g)]
    with threadpool_limits(limits=1), ThreadPoolExecutor(len(os.sched_getaffinity(0))) as ex:
        parts = list(ex.map(lambda a: oracle.attention_backward_kv_rows(
            q, k, v, do, wl.causal, wl.scale, a[0], a[1], keys, heads=[a[2]]), jobs))
    ref_k = np.zeros((wl.B, wl.Hkv, len(keys), wl.d))
    ref_v = np.zeros_like(ref_k)
    for (b, j, _), (pk, pv) in zip(jobs, parts):
        ref_k[b, j] += pk
        ref_v[b, j] += pv
    return dk[:, :, keys], dv[:, :, keys], ref_k, ref_v


def _grads_with_do_scaled(wl, k):
    """fa.forward + fa.backward with dO multiplied by 2^k (exact in bf16)."""
    q, kk, v, do = (t.to(DEV) for t in make_inputs(wl))
    do = (do.float() * 2.0 ** k).to(torch.bfloat16)
    o, lse = fa.forward(q, kk, v, wl.causal, wl.scale)
    grads = fa.backward(q, kk, v, o, lse, do, wl.causal, wl.scale)
    torch.cuda.synchronize()
    st, where = fa.fa_device_status(None)
    assert st == 0, f"device status {st} at wait {where}"
    return [g.float().cpu().double().numpy() for g in grads]


@pytest.mark.parametrize("wl", [W(1, 8, 2, 640, 640, 128, True),     # GQA: fp16 dP, dV
                                W(1, 16, 1, 512, 512, 128, False),    # MQA: every product fp16
                                W(1, 2, 2, 384, 384, 256, False)],    # d = 256: fp16 dP, dV
                         ids=lambda w: w.name)
@pytest.mark.parametrize("k", [-24, 16])
def test_fp16_operand_scales_follow_a_power_of_two(wl, k):
    """The fp16 operands carry scales chosen from the largest |dO|, |V| (and
    |Q|, |K|, and the bound on |dS| for wide groups).  Multiplying dO by 2^k
    must multiply every gradient by exactly 2^k: the kernels' powers of two
    absorb k (including max |dO| near 2^18, beyond fp16's range, for
    k = 16).  The only difference allowed is the order of the fp32
    reduce-adds of dQ and of split dK / dV (atomics, in no fixed order):
    one bf16 ulp, plus fp32 rounding noise on elements whose partial sums
    cancel (2^-16 of the largest gradient; a wrong power of two would be a
    factor of 2).  With the parity tests at k = 0 this covers dO at any
    scale."""
    base = _grads_with_do_scaled(wl, 0)
    scaled = _grads_with_do_scaled(wl, k)
    for name, g0, gk in zip(("dQ", "dK", "dV"), base, scaled):
        assert np.isfinite(gk).all(), name
        back = gk * 2.0 ** -k
        ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(g0), 1e-300))) - 7)
        tol = ulp + 2.0 ** -16 * np.abs(g0).max()
        diff = np.abs(back - g0)
        assert (diff <= tol).all(), (
            f"{name}: worst {float((diff / tol).max()):.2f} x the allowance, "
            f"max |diff| {float(diff.max()):.3e}, max |g| {float(np.abs(g0).max()):.3e}")
