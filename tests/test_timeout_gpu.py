"""The bounded-wait path on the GPU, without faulting or hanging it.

fa_debug_inject makes the forward producers withhold their K/V tiles and
shortens the pipeline-wait limit to 0.2 s: every CTA's wait then expires,
the kernel records FA_ERR_DEVICE_TIMEOUT with the code of the wait, frees its
TMEM and returns.  A normal call afterwards must succeed with correct
results (the context stays usable)."""
import time

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_71_b200 import binding as fa
from exact_io_aware_71_b200.inputs import Workload, make_inputs
from tests.parity import check_fwd, to64

W_KV_FULL, W_S_FULL = 3, 4


def test_debug_inject_rejects_bad_arguments():
    assert fa.fa_debug_inject(2, 0.0) == 1
    assert fa.fa_debug_inject(0, -1.0) == 1
    assert fa.fa_debug_inject(0, 120.0) == 1


@pytest.mark.gpu
@pytest.mark.parametrize("d", [64, 256])
def test_stalled_pipeline_times_out_and_recovers(d):
    wl = Workload(f"timeout{d}", 1, 2, 2, 256, 256, d, False, 40)
    q, k, v, _ = (t.cuda() if t is not None else None for t in make_inputs(wl, with_do=False))
    assert fa.fa_device_status(None)[0] == 0
    assert fa.fa_debug_inject(1, 0.2) == 0
    try:
        t0 = time.time()
        fa.forward(q, k, v, False, wl.scale)
        st, where = fa.fa_device_status(None)
        elapsed = time.time() - t0
    finally:
        assert fa.fa_debug_inject(0, 0.0) == 0
    assert st == 6 and fa.fa_status_string(st) == "FA_ERR_DEVICE_TIMEOUT"
    assert where in (W_KV_FULL, W_S_FULL), where
    assert elapsed < 30.0
    # the same context, normal operation
    o, lse = fa.forward(q, k, v, False, wl.scale)
    torch.cuda.synchronize()
    assert fa.fa_device_status(None)[0] == 0
    o_ref, lse_ref = oracle.attention_forward(to64(q), to64(k), to64(v), False, wl.scale)
    check_fwd(to64(o), to64(lse), o_ref, lse_ref)
