"""The seeded input recipe: deterministic, bf16, the documented draw order and
the Q*2 range widening on the first half of the heads."""
import torch

from exact_io_aware_71_b200.inputs import make_inputs, workloads


def test_workload_table():
    w = workloads()
    assert len([n for n in w if n.startswith("sweep_")]) == 24
    t = w["train_b8h16n2048d128_full"]
    assert (t.B, t.Hq, t.Hkv, t.Nq, t.d, t.causal) == (8, 16, 16, 2048, 128, False)
    assert t.fwd_flops() == 4 * 8 * 16 * 2048 * 2048 * 128
    assert w["train_b8h16n2048d128_causal"].fwd_flops() == t.fwd_flops() / 2
    assert t.bwd_flops() == 2.5 * t.fwd_flops()
    for n, x in w.items():
        if n.startswith("sweep_"):
            assert x.B * x.Nq == 16384 and x.Hq * x.d == 2048
    g = w["long_gqa_hkv1_n16384_d128_causal"]
    assert (g.Hq, g.Hkv) == (32, 1)


def test_inputs_are_seeded_bf16_normal():
    wl = workloads()["tiny_b1h2n128d64_causal"]
    a = make_inputs(wl)
    b = make_inputs(wl)
    for x, y in zip(a, b):
        assert x.dtype == torch.bfloat16
        assert torch.equal(x, y)
    q = a[0].float()
    assert abs(q.mean().item()) < 0.1 and abs(q.std().item() - 1) < 0.1
    # draw order q, k, v, dO from one generator
    g = torch.Generator("cpu").manual_seed(wl.seed)
    q_ref = torch.randn(1, 2, 128, 64, generator=g).to(torch.bfloat16)
    k_ref = torch.randn(1, 2, 128, 64, generator=g).to(torch.bfloat16)
    assert torch.equal(a[0], q_ref) and torch.equal(a[1], k_ref)


def test_q_scaled_on_first_half_of_heads():
    wl = workloads()["tiny_b1h2n128d64_full"].with_(q_scale_half_heads=True, Hq=4, Hkv=4)
    q2 = make_inputs(wl)[0]
    q1 = make_inputs(wl.with_(q_scale_half_heads=False))[0]
    assert torch.equal(q2[:, :2], q1[:, :2] * 2)
    assert torch.equal(q2[:, 2:], q1[:, 2:])
