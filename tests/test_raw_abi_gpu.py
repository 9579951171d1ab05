"""GPU parity of the plain C entry points on raw device pointers: fa_fwd,
fa_bwd, and fa_bwd_stage called stage by stage (preprocess, main, dQ
convert), the calls bench.py times, against the fp64 oracle.  The other GPU
tests reach the kernels through the strided entry points of the torch-level
binding; these go through the contiguous ones, which build their own
strides."""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_71_b200 import binding as fa
from exact_io_aware_71_b200.inputs import Workload, make_inputs, workloads
from tests.parity import check_fwd, check_grads, sample_rows, to64

pytestmark = pytest.mark.gpu


def _raw_step(wl, staged: bool):
    """The bench step on raw pointers: fa_fwd, then fa_bwd (staged=False) or
    fa_bwd_stage(PRE), (MAIN), (DQ) on one stream."""
    q, k, v, do = (t.cuda() for t in make_inputs(wl))
    o = torch.empty_like(q)
    lse = torch.empty(wl.B, wl.Hq, wl.Nq, dtype=torch.float32, device="cuda")
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    # NaN-filled outputs: an element the kernels never write shows up
    for t in (o, lse, dq, dk, dv):
        t.fill_(float("nan"))
    wsb = fa.fa_bwd_workspace_size(wl.B, wl.Hq, wl.Hkv, wl.Nq, wl.Nk, wl.d, wl.causal)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    sh = torch.cuda.current_stream().cuda_stream
    dims = (wl.B, wl.Hq, wl.Hkv, wl.Nq, wl.Nk, wl.d, int(wl.causal), wl.scale)
    st = fa.fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                   *dims, sh)
    assert st == 0, fa.STATUS_NAMES.get(st, st)
    ptrs = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
            do.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr())
    if staged:
        for stage in (fa.FA_BWD_PRE, fa.FA_BWD_MAIN, fa.FA_BWD_DQ):
            st = fa.fa_bwd_stage(stage, *ptrs, *dims, ws.data_ptr(), wsb, sh)
            assert st == 0, fa.STATUS_NAMES.get(st, st)
    else:
        st = fa.fa_bwd(*ptrs, *dims, ws.data_ptr(), wsb, sh)
        assert st == 0, fa.STATUS_NAMES.get(st, st)
    torch.cuda.synchronize()
    s, where = fa.fa_device_status(None)
    assert s == 0, f"device status {s} at wait {where}"
    return tuple(to64(t) for t in (q, k, v, do)), tuple(to64(t) for t in (o, lse, dq, dk, dv))


def W(B, Hq, Hkv, N, d, causal, seed=81):
    return Workload(f"raw{B}_{Hq}_{Hkv}_{N}_{d}_{int(causal)}", B, Hq, Hkv, N, N, d, causal, seed)


@pytest.mark.parametrize("staged", [False, True])
@pytest.mark.parametrize("wl", [workloads()["tiny_b1h2n128d64_full"],
                                workloads()["tiny_b1h2n128d64_causal"],
                                W(2, 4, 2, 333, 128, True), W(1, 4, 1, 200, 256, False),
                                W(1, 32, 1, 384, 128, True)],
                         ids=lambda w: w.name)
def test_plain_entry_points_match_the_oracle(wl, staged):
    (q, k, v, do), (o, lse, dq, dk, dv) = _raw_step(wl, staged)
    o_ref, lse_ref = oracle.attention_forward(q, k, v, wl.causal, wl.scale)
    check_fwd(o, lse, o_ref, lse_ref)
    check_grads((dq, dk, dv), oracle.attention_backward(q, k, v, do, wl.causal, wl.scale))


def test_bench_step_at_full_size():
    """bench.py's default workload through exactly its timed calls: forward
    rows, dQ rows and dK / dV rows of sampled keys against the oracle."""
    import bench
    from tests.test_bwd_gpu import kv_rows_parallel
    wl = workloads()[bench.DEFAULT_WORKLOAD]
    (q, k, v, do), (o, lse, dq, dk, dv) = _raw_step(wl, staged=True)
    for t in (o, lse, dq, dk, dv):
        assert np.isfinite(t).all()
    rng = np.random.default_rng(5)
    heads = [(0, 0), (wl.B - 1, wl.Hq - 1)] + [(int(rng.integers(wl.B)), int(rng.integers(wl.Hq)))
                                               for _ in range(2)]
    for (b, h) in heads:
        rows = sample_rows(wl.Nq, 64, seed=b * 131 + h)
        o_ref, lse_ref = oracle.attention_forward_rows(q, k, v, wl.causal, wl.scale, b, h, rows)
        check_fwd(o[b, h, rows], lse[b, h, rows], o_ref, lse_ref)
        dq_ref = oracle.attention_backward_dq_rows(q, k, v, do, wl.causal, wl.scale, b, h, rows)
        check_grads([dq[b, h, rows]], [dq_ref], names=("dQ rows",))
    keys = sample_rows(wl.Nk, 64, seed=3)
    got_k, got_v, ref_k, ref_v = kv_rows_parallel(wl, q, k, v, do, dk, dv, keys)
    check_grads((got_k, got_v), (ref_k, ref_v), names=("dK rows", "dV rows"))
