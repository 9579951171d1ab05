"""Host logic of bench.py on the CPU: whole-job aggregation over ranks
(gloo, world size 2), clock-sample parsing, and the traffic record gate."""
import json
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, times, out):
    import torch
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        def reduce_max(x):
            t = torch.tensor([x], dtype=torch.float64)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            return float(t.item())
        t, rate = bench.aggregate(times[rank], 1e12, world, reduce_max)
        out[rank] = (t, rate)
    finally:
        dist.destroy_process_group()


def test_aggregate_takes_the_slowest_rank_over_gloo():
    times = [100.0, 250.0]
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(2, _free_port(), times, out), nprocs=2, join=True)
        res = dict(out)
    for r in (0, 1):
        t, rate = res[r]
        assert t == 250.0
        assert rate == pytest.approx(2 * 1e12 / 0.25)


def test_aggregate_single_rank():
    t, rate = bench.aggregate(50.0, 3e12, 1)
    assert t == 50.0 and rate == pytest.approx(6e13)


def test_parse_clock_samples():
    text = ("0, 1965, 1965, 400.1, 0x0, Not Active, Not Active, Not Active, Not Active\n"
            "0, 1800, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active\n"
            "0, 1965, 1965, 500.0, 0x0, Not Active, Not Active, Not Active, Not Active\n")
    c = bench.parse_clock_samples(text)
    assert c["sm_mhz"] == 1965 and c["sm_max_mhz"] == 1965
    assert c["reasons"] == ["sw_power_cap"] and c["samples"] == 3
    assert bench.parse_clock_samples("")["sm_mhz"] is None


def test_nvml_samples_outside_the_timed_window_are_dropped():
    """Only samples between start() and stop() count: idle samples before
    and after the timed region (at max clock, no reason) must not move the
    median or hide a reason seen under load."""
    cap, hw = bench.NVML_REASON_BITS["sw_power_cap"], bench.NVML_REASON_BITS["hw_slowdown"]
    samples = [(0.0, 1965.0, 90.0, 0), (0.9, 1965.0, 95.0, hw),          # before the window
               (1.0, 1800.0, 900.0, cap), (1.1, 1820.0, 950.0, cap), (1.2, 1850.0, 980.0, 0),
               (2.5, 1965.0, 100.0, 0)]                                  # after it
    c = bench.summarise_clock_samples(samples, 1.0, 1.2, 1965.0)
    assert c["samples"] == 3 and c["sm_mhz"] == 1820.0 and c["sm_max_mhz"] == 1965.0
    assert c["reasons"] == ["sw_power_cap"] and c["power_w_max"] == 980.0
    assert bench.summarise_clock_samples(samples, 3.0, 4.0, 1965.0)["reasons"] == ["no samples"]
    # a region shorter than the polling interval takes the nearest sample (within 10 ms)
    c = bench.summarise_clock_samples(samples, 1.203, 1.204, 1965.0)
    assert c["samples"] == 1 and c["sm_mhz"] == 1850.0 and "nearest" in c["source"]


def test_edge_samples_stand_in_only_when_polling_left_none():
    """The samples the timing thread takes itself at the region's start and
    end are used only when the polling thread took none in or near it."""
    cap = bench.NVML_REASON_BITS["sw_power_cap"]
    polled = [(0.0, 1965.0, 90.0, 0), (1.1, 1800.0, 900.0, cap), (5.0, 1965.0, 95.0, 0)]
    edges = [(1.0, 1700.0, 800.0, 0), (2.0, 1750.0, 850.0, cap)]
    c = bench.summarise_clock_samples(polled, 1.0, 2.0, 1965.0, edges)
    assert c["samples"] == 1 and c["sm_mhz"] == 1800.0 and "edge" not in c["source"]
    c = bench.summarise_clock_samples(polled, 2.5, 3.5, 1965.0, [(2.5, 1700.0, 800.0, 0),
                                                                (3.5, 1750.0, 850.0, cap)])
    assert c["samples"] == 2 and c["sm_mhz"] == 1725.0 and c["reasons"] == ["sw_power_cap"]
    assert "start and end" in c["source"]
    assert bench.summarise_clock_samples(polled, 2.5, 3.5, 1965.0, [])["reasons"] == ["no samples"]


def test_traffic_is_reported_only_for_current_sources(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    for rel in bench.KERNEL_SOURCES:
        p = tmp_path / rel
        p.parent.mkdir(parents=True, exist_ok=True)
        p.write_text("kernel " + rel)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    sha = bench.kernel_source_hash()
    rec = {"entries": [{"kernel": "k", "workload": "w", "src_sha": sha,
                        "dram_bytes_per_launch": 123}]}
    (prof / "traffic.json").write_text(json.dumps(rec))
    assert bench.recorded_traffic("k", "w") == 123
    assert bench.recorded_traffic("k", "other") is None
    # a comment-only edit keeps the record; a code edit drops it
    (tmp_path / bench.KERNEL_SOURCES[0]).write_text("kernel  " + bench.KERNEL_SOURCES[0] +
                                                    "  // note\n/* block */")
    assert bench.recorded_traffic("k", "w") == 123
    (tmp_path / bench.KERNEL_SOURCES[0]).write_text("changed")
    assert bench.recorded_traffic("k", "w") is None


def test_forward_traffic_survives_backward_edits(tmp_path, monkeypatch):
    """A forward kernel's record is keyed on the forward's own sources: an
    edit of a backward source keeps it and drops the backward's record; an
    edit of a shared header drops both."""
    prof = tmp_path / "profiles"
    prof.mkdir()
    for rel in bench.KERNEL_SOURCES:
        p = tmp_path / rel
        p.parent.mkdir(parents=True, exist_ok=True)
        p.write_text("kernel " + rel)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert set(bench.FWD_KERNEL_SOURCES) < set(bench.KERNEL_SOURCES)
    assert not any("fa_bwd" in r for r in bench.FWD_KERNEL_SOURCES)
    rec = {"entries": [
        {"kernel": "fa_fwd_kernel", "workload": "w", "dram_bytes_per_launch": 1,
         "src_sha": bench.kernel_source_hash("fa_fwd_kernel")},
        {"kernel": "fa_bwd_main_kernel", "workload": "w", "dram_bytes_per_launch": 2,
         "src_sha": bench.kernel_source_hash("fa_bwd_main_kernel")}]}
    (prof / "traffic.json").write_text(json.dumps(rec))
    assert bench.recorded_traffic("fa_fwd_kernel", "w") == 1
    assert bench.recorded_traffic("fa_bwd_main_kernel", "w") == 2
    bwd = next(r for r in bench.KERNEL_SOURCES if r.endswith("fa_bwd128.cuh"))
    (tmp_path / bwd).write_text("changed")
    assert bench.recorded_traffic("fa_fwd_kernel", "w") == 1
    assert bench.recorded_traffic("fa_bwd_main_kernel", "w") is None
    shared = next(r for r in bench.KERNEL_SOURCES if r.endswith("sm100.cuh"))
    (tmp_path / shared).write_text("changed")
    assert bench.recorded_traffic("fa_fwd_kernel", "w") is None


def test_peaks_fallback(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    pk, src = bench.load_peaks()
    assert src == "fallback" and pk["bf16_tflops"] == 1590.0


def test_kept_fraction_of_block_masks():
    """The FLOP scale of block-sparse steps: visible (query, key) pairs over
    those of the dense problem, counted per element on small cases."""
    import numpy as np
    from exact_io_aware_71_b200.inputs import Workload
    for causal in (False, True):
        for nq, nk in ((300, 300), (260, 400), (400, 130)):
            wl = Workload("t", 1, 1, 1, nq, nk, 64, causal, 0)
            rng = np.random.default_rng(nq + nk)
            m = rng.random(((nq + 127) // 128, (nk + 127) // 128)) < 0.5
            i = np.arange(nq)[:, None]
            j = np.arange(nk)[None, :]
            vis = m[i // 128, j // 128]
            base = (j <= i) if causal else np.ones((nq, nk), bool)
            assert bench.kept_fraction(wl, m) == pytest.approx((vis & base).sum() / base.sum())
            assert bench.kept_fraction(wl, None) == 1.0
            assert bench.kept_fraction(wl, np.ones_like(m)) == pytest.approx(1.0)


def test_launches_per_step():
    from exact_io_aware_71_b200.inputs import workloads
    w = workloads()
    assert bench.launches_per_step(w["train_b8h16n2048d128_full"], 148) == 4
    # d = 256: the fp16 copy of dO and V
    assert bench.launches_per_step(w["large_b4h8n4096d256_full"], 148) == 5
    # 32 query heads on one kv head, 128 key blocks: the fp16 copies (dO, V;
    # Q, K), the split and its dK/dV convert, and the forward pass that
    # recomputes D
    assert bench.launches_per_step(w["long_gqa_hkv1_n16384_d128_causal"], 148) == 8
    # 8 kv heads x 128 key blocks = 1024 CTAs: no split; the fp16 copy
    assert bench.launches_per_step(w["long_gqa_hkv8_n16384_d128_causal"], 148) == 5


def test_roofline_picks_the_bound_by_arithmetic_intensity():
    from exact_io_aware_71_b200.inputs import workloads
    peaks = {"hbm_gbs": 6529.4, "bf16_tflops": 1674.6, "bf16_tflops_sustained": 1388.6}
    w = workloads()
    for name, bound in (("long_gqa_hkv8_n16384_d128_causal", "tensor"),
                        ("sweep_n512_d64_full", "hbm")):
        wl = w[name]
        fb, bb = bench.algorithmic_bytes(wl)
        # forward bytes: Q, K, V, O in bf16 plus the fp32 LSE
        q = wl.B * wl.Hq * wl.Nq * wl.d
        kv = wl.B * wl.Hkv * wl.Nk * wl.d
        assert fb == 2 * (2 * q + 2 * kv) + 4 * wl.B * wl.Hq * wl.Nq
        r = bench.roofline("k", wl.fwd_flops(), fb, 1.0, peaks, "measured")
        assert r["bound"] == bound
        assert r["tensor"]["tflops"] == pytest.approx(wl.fwd_flops() / 1e-3 / 1e12, rel=1e-3)
        assert r["hbm"]["gbs"] == pytest.approx(fb / 1e-3 / 1e9, rel=1e-3)
        assert r["frac"] == (r["hbm"]["frac"] if bound == "hbm" else r["tensor"]["frac"])


def test_peak_clock_lookup(tmp_path):
    """The clock the measured peak was taken at is found in the peaks file
    whatever its nesting; a clock recorded with the GEMM is preferred."""
    import json
    f = tmp_path / "peaks.json"
    f.write_text(json.dumps({"bf16_tflops": 1674.6, "clocks": {"median_sm_mhz": 1327,
                                                               "max_sm_mhz": 1965}}))
    assert bench.peak_clock_mhz(str(f)) == 1327
    f.write_text(json.dumps({"hbm": {"sm_clock_mhz": 1800}, "bf16": {"sm_clock_mhz": 1330}}))
    assert bench.peak_clock_mhz(str(f)) == 1330
    f.write_text(json.dumps({"bf16_tflops": 1674.6}))
    assert bench.peak_clock_mhz(str(f)) is None
    assert bench.peak_clock_mhz(str(tmp_path / "absent.json")) is None


def test_varlen_lengths_and_flops():
    from exact_io_aware_71_b200.inputs import workloads
    wl = workloads()["train_b8h16n2048d128_causal"]
    L = bench.varlen_lengths(wl, "100:300")
    assert len(L) == wl.B and all(100 <= n <= 300 for n in L)
    assert L == bench.varlen_lengths(wl, "100:300")          # seeded
    assert bench.varlen_fwd_flops(wl, [wl.Nq] * wl.B) == pytest.approx(wl.fwd_flops())
    with pytest.raises(ValueError):
        bench.varlen_lengths(wl, "0:10")


def test_reference_arm_varlen_runs_on_cpu():
    out = bench.run_reference(bench.parse_args(["--impl", "reference", "--workload",
                                                "tiny_b1h2n128d64_full", "--varlen", "20:60",
                                                "--steps", "1", "--warmup", "1"]))
    assert out["impl"] == "reference" and out["value"] > 0
    assert out["config"]["workload"].endswith("_varlen20:60")


@pytest.mark.parametrize("extra", [[], ["--block-density", "0.5"]])
def test_reference_arm_line_keeps_the_contract(extra):
    """The oracle arm's JSON line carries every key of the bench contract,
    with its e2e and cpu_baseline describing the same CPU run."""
    out = bench.run_reference(bench.parse_args(["--impl", "reference", "--workload",
                                                "tiny_b1h2n128d64_full", "--steps", "1",
                                                "--warmup", "1"] + extra))
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in out, key
    assert out["impl"] == "reference" and out["higher_is_better"] is True
    assert out["value"] > 0 and out["unit"] == "TFLOP/s" and out["n_gpus"] == 1
    assert out["vs_baseline"] is None
    cb = out["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == out["value"]
    e2e = out["e2e"]
    assert e2e["value"] == out["value"] and e2e["unit"] == out["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
    assert out["config"]["workload"].startswith("tiny_b1h2n128d64_full")
