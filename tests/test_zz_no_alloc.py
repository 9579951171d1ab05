"""fa_bwd_noalloc: the backward pass for callers that cannot allocate device
memory (for instance a plug-in whose host application owns every device
allocation, or a latency-critical path where cudaMalloc, which may
synchronise the device, is not allowed).  Its scratch is the library's
built-in device array instead of a caller workspace.

The test calls it several times in a row through the C ABI, on different
problems, and checks each result against fa_bwd's on the same inputs, within
the gradient tolerance the parity tests use (2e-2 max-abs).  Each call finds
the previous call's data still in the shared array, so it also shows that
each call re-initialises what it reads: a GQA problem whose dK / dV partial
sums live in the array follows an MHA one of another shape, and a wide
group (32 query heads on one kv head, whose exact D is recomputed into the
array) follows both.  The file is named to be collected last, and it passes
alone in a fresh process as well as after the others.
"""
import numpy as np
import pytest
import torch

from exact_io_aware_71_b200 import binding as fa
from exact_io_aware_71_b200.inputs import Workload, make_inputs

TOL = 2e-2


def _problem(B, Hq, Hkv, N, d, causal, seed):
    wl = Workload(f"noalloc{seed}", B, Hq, Hkv, N, N, d, causal, seed)
    q, k, v, do = (t.cuda() for t in make_inputs(wl))
    o, lse = fa.forward(q, k, v, causal, wl.scale)
    return wl, q, k, v, do, o, lse


def _noalloc(wl, q, k, v, do, o, lse):
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    st = fa.fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                           lse.data_ptr(), do.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                           dv.data_ptr(), wl.B, wl.Hq, wl.Hkv, wl.Nq, wl.Nk, wl.d, wl.causal,
                           wl.scale, torch.cuda.current_stream().cuda_stream)
    assert st == 0, fa.STATUS_NAMES.get(st, st)
    return dq, dk, dv


@pytest.mark.gpu
def test_noalloc_matches_fa_bwd_on_calls_in_a_row():
    problems = [(2, 8, 2, 1024, 128, True, 31), (1, 4, 4, 640, 64, False, 32),
                (1, 8, 2, 384, 64, False, 33), (1, 32, 1, 512, 128, True, 34)]
    for args in problems:
        wl, q, k, v, do, o, lse = _problem(*args)
        ref = fa.backward(q, k, v, o, lse, do, wl.causal, wl.scale)
        got = _noalloc(wl, q, k, v, do, o, lse)
        torch.cuda.synchronize()
        assert fa.fa_device_status(None)[0] == 0
        for name, g, r in zip(("dq", "dk", "dv"), got, ref):
            err = (g.double() - r.double()).abs().max().item()
            assert err <= TOL, f"{args}: {name} differs from fa_bwd by {err:.3e}"
            assert torch.isfinite(g).all()


def test_noalloc_rejects_problems_beyond_its_scratch():
    """Checked before any launch, so this runs without a GPU."""
    a = 0x7F0000000000
    need = fa.fa_bwd_workspace_size(8, 16, 16, 2048, 2048, 128, 0)
    assert need > fa.NOALLOC_SCRATCH_BYTES
    st = fa.fa_bwd_noalloc(a, a, a, a, a, a, a, a, a, 8, 16, 16, 2048, 2048, 128, 0, 0.088, None)
    assert st == 7 and fa.fa_status_string(st) == "FA_ERR_TOO_LARGE"
    assert fa.fa_bwd_noalloc(None, a, a, a, a, a, a, a, a, 1, 2, 2, 64, 64, 64, 0, 0.1, None) == 1
