#!/usr/bin/env python
"""Throughput of exact attention forward + backward on B200 through libfa.

One *step* is one pass of the whole hot path on one batch: fa_fwd (tiled
forward, O and LSE) followed by the three backward stages (preprocess, main,
dQ convert).  The default workload is the long-sequence GQA shape B=1,
Hq=32, Hkv=8, N=16384, d=128, causal (bf16 inputs iid N(0, 1) from a fixed
seed), the largest d = 128, N >= 4k configuration; ``--workload`` selects any
other named workload (e.g. the training shape train_b8h16n2048d128_full or
the short sequences sweep_n512_d64_full).

Prints ONE JSON line (rank 0).  ``value`` is whole-job attention TFLOP/s over
all ranks, with the nominal FLOP count 3.5 * 4*B*Hq*N^2*d per step, halved
when causal (forward 4*B*Hq*N^2*d, backward 2.5x that).  Timing: W untimed
warm-up steps, then K steps between a barrier + synchronize on both sides,
CUDA events on the launching stream, max over ranks.  Every named workload's
inputs exceed the 126 MB L2 except where the line's ``l2`` note says
otherwise.

``--block-density P`` measures block-sparse attention instead (QbitAI FA1
article, results section): a seeded block mask keeps each 128 x 128 (query,
key) block with probability P (diagonal blocks always), the step is
fa_fwd_block_sparse + fa_bwd_block_sparse, and FLOPs count only the kept
(query, key) pairs.

``--varlen LO:HI`` measures a packed variable-length batch instead: the
workload's B sequences get seeded lengths uniform in [LO, HI], the step is
fa_fwd_varlen + fa_bwd_varlen, and FLOPs are summed per sequence.

``--impl reference`` times the fp64 CPU oracle instead (the only other place
this script runs it), on a bounded sample of the same workload.
Multi-GPU (torchrun): every rank runs an independent batch of the same shape
(weak scaling, no collective on the data path).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

DEFAULT_WORKLOAD = "long_gqa_hkv8_n16384_d128_causal"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_SOURCES = ["exact_io_aware_71_b200/csrc/sm100.cuh", "exact_io_aware_71_b200/csrc/fa_fwd.cuh",
                  "exact_io_aware_71_b200/csrc/fa_bwd.cuh", "exact_io_aware_71_b200/csrc/fa_mask.cuh",
                  "exact_io_aware_71_b200/csrc/fa_bwd128.cuh", "exact_io_aware_71_b200/csrc/fa_rows.cuh"]
# The forward kernels are built from these alone (fa_fwd.cuh includes no
# backward source); the backward's traffic is keyed on all of them.
FWD_KERNEL_SOURCES = [r for r in KERNEL_SOURCES if "fa_bwd" not in r]
METRIC = "attention fwd / fwd+bwd TFLOP/s (bf16, 1×B200) and % of dense BF16 peak"


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU work for the oracle baseline sample")
    ap.add_argument("--block-density", type=float, default=None,
                    help="block-sparse attention with this fraction of 128x128 blocks kept")
    ap.add_argument("--layer", action="store_true",
                    help="time the synthetic attention layer (QKV projection, attention, output "
                         "projection; hidden = Hq * d) and report model TFLOP/s and MFU")
    ap.add_argument("--varlen", default=None, metavar="LO:HI",
                    help="packed variable-length batch: the workload's B sequences get seeded "
                         "lengths uniform in [LO, HI] (its H, d and causal flag)")
    return ap.parse_args(argv)


# ----------------------------------------------------------------- host logic
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return {k: float(pk[k]) for k in FALLBACK_PEAKS}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash(kernel: str = ""):
    """Hash of the code of the sources a kernel is built from (the forward
    kernels' own for names starting with fa_fwd, else all): comments and
    whitespace are dropped first, so an edit that only touches comments keeps
    a traffic record, and so does a backward edit for a forward record."""
    import re
    h = hashlib.sha256()
    for rel in (FWD_KERNEL_SOURCES if kernel.startswith("fa_fwd") else KERNEL_SOURCES):
        with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel sources; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    for r in rec.get("entries", []):
        if (r.get("kernel") == kernel and r.get("workload") == workload
                and r.get("src_sha") == kernel_source_hash(kernel)):
            return r.get("dram_bytes_per_launch")
    return None


def aggregate(local_ms: float, local_units: float, world: int, reduce_max=None):
    """Whole-job throughput: units processed by all ranks over the slowest
    rank's time.  ``reduce_max`` maps a local float to the max over ranks."""
    t = reduce_max(local_ms) if reduce_max else local_ms
    return t, local_units * world / (t / 1e3)


# NVML clock-event reason bits (nvmlClocksEventReason*) reported in `clocks`
NVML_REASON_BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
                    "hw_thermal_slowdown": 0x40}


def summarise_clock_samples(samples, t0: float, t1: float, max_mhz, edges=()):
    """Clock summary of the samples taken inside the timed window [t0, t1]
    (host perf_counter seconds).  samples: (t, sm_mhz, power_w, reason_bits).
    A reason counts if any window sample has it.  edges: samples taken by
    the timing thread itself at t0 and t1, used only when the polling thread
    left none in or within 10 ms of the window."""
    win = [x for x in samples if t0 <= x[0] <= t1]
    source = "nvml, 5 ms polling inside the timed region"
    if not win:
        # a region shorter than the polling interval: the sample nearest to it,
        # if one was taken within 10 ms
        near = sorted(samples, key=lambda x: max(t0 - x[0], x[0] - t1))[:1]
        win = [x for x in near if max(t0 - x[0], x[0] - t1) <= 0.010]
        source = "nvml, nearest sample to a timed region shorter than the 5 ms polling"
    if not win and edges:
        win = list(edges)
        source = "nvml, samples at the timed region's start and end (none polled inside it)"
    if not win:
        return {"sm_mhz": None, "sm_max_mhz": max_mhz, "reasons": ["no samples"]}
    reasons = sorted(n for n, bit in NVML_REASON_BITS.items() if any(x[3] & bit for x in win))
    return {"sm_mhz": statistics.median(x[1] for x in win), "sm_max_mhz": max_mhz,
            "reasons": reasons, "samples": len(win), "power_w_max": max(x[2] for x in win),
            "source": source}


class ClockSampler:
    """SM clock, power and clock-event reasons during the timed region.
    NVML is polled from a thread every 5 ms and only the samples between
    start() and stop() (called right around the synchronised timed region)
    are kept; without NVML, nvidia-smi samples at 100 ms instead.  Reads
    only: no setting of the GPU is changed."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None
        self.nvml = None
        self.handle = None
        self.samples = []
        self.edges = []
        self.running = False
        self.thread = None
        self.t0 = self.t1 = 0.0

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(self.index).uuid)
            return pynvml, pynvml.nvmlDeviceGetHandleByUUID("GPU-" + uuid)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.index)

    def _sample(self):
        nv, h = self.nvml, self.handle
        return (time.perf_counter(), float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)),
                nv.nvmlDeviceGetPowerUsage(h) / 1000.0,
                int(nv.nvmlDeviceGetCurrentClocksEventReasons(h)))

    def _edge(self):
        try:
            self.edges.append(self._sample())
        except Exception:
            pass

    def _poll(self):
        while self.running:
            try:
                self.samples.append(self._sample())
            except Exception:
                pass
            time.sleep(0.005)

    def start(self):
        try:
            import threading
            self.nvml, self.handle = self._nvml_handle()
            self.running = True
            self.thread = threading.Thread(target=self._poll, daemon=True)
            self.thread.start()
            time.sleep(0.02)
            self._edge()
            self.t0 = time.perf_counter()
            return
        except Exception:
            self.nvml = None
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except OSError:
            self.proc = None

    def stop(self):
        if self.nvml is not None:
            self.t1 = time.perf_counter()
            self._edge()
            self.running = False
            self.thread.join()
            try:
                mx = float(self.nvml.nvmlDeviceGetMaxClockInfo(self.handle, self.nvml.NVML_CLOCK_SM))
            except Exception:
                mx = None
            return summarise_clock_samples(self.samples, self.t0, self.t1, mx, self.edges)
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        self.proc.wait()
        return parse_clock_samples(open(self.path).read())


def parse_clock_samples(text: str):
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    sm, mx, reasons, power = [], [], set(), []
    for line in text.strip().splitlines():
        parts = [p.strip() for p in line.split(",")]
        if len(parts) < 9:
            continue
        try:
            sm.append(float(parts[1]))
            mx.append(float(parts[2]))
            power.append(float(parts[3]))
        except ValueError:
            continue
        for n, v in zip(names, parts[5:9]):
            if v.lower().startswith("active"):
                reasons.add(n)
    if not sm:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
    return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
            "samples": len(sm), "power_w_max": max(power)}


# ----------------------------------------------------------------- oracle timing
_INPUT_CACHE = {}


# Query heads per kv head from which the backward recomputes D with one more
# forward pass (the library's wide-group rule, include/fa.h, fa_bwd; at
# d = 256 every GQA / MQA group).
EXACT_GROUP = 16
DATASHEET_BF16_TFLOPS = 2250.0   # NVIDIA B200 dense BF16 (the sparse figure halved)


def launches_per_step(wl, sms: int) -> int:
    """Kernels one step launches: the forward kernel, the backward's
    preprocess, main and dQ-convert kernels; the fp16 copy of dO and V when
    dP and dV take fp16 operands (GQA / MQA groups and d = 256, the library's
    rule); the dK/dV convert kernel when a GQA group's query heads are split
    over CTAs (the library splits when one CTA per (batch, kv head, key
    block) would give fewer than two CTAs per SM); and for groups of 16 or
    more (any GQA group at d = 256) the fp16 copy of Q and K and the
    D-recomputing forward pass."""
    g = wl.Hq // wl.Hkv
    f16 = g > 1 or wl.d == 256
    if g == 1:
        return 4 + (1 if f16 else 0)
    base = ((wl.Nk + 127) // 128) * wl.B * wl.Hkv * (2 if wl.d == 256 else 1)
    gsplit = next((s_ for s_ in range(1, g + 1) if g % s_ == 0 and base * s_ >= 2 * sms), g)
    exact = g >= EXACT_GROUP or (wl.d == 256 and g > 1)
    # exact: also the fp16 copy of Q and K, and the D-recomputing forward pass
    return 4 + 1 + (1 if gsplit > 1 else 0) + (2 if exact else 0)


def algorithmic_bytes(wl, frac: float = 1.0):
    """Minimum HBM bytes of the forward and of the backward's main kernel for
    one step.  Forward: read Q, K, V, write O (bf16) and the fp32 LSE.
    Backward main: read Q, K, V, dO (bf16) and the fp32 LSE and D rows,
    write dK, dV (bf16), and read-modify-write the fp32 dQ accumulator once.
    Block-sparse steps scale the per-block traffic (K, V reads) by the kept
    fraction of pairs; the rest is per row."""
    q = wl.B * wl.Hq * wl.Nq * wl.d
    kv = wl.B * wl.Hkv * wl.Nk * wl.d
    rows = wl.B * wl.Hq * wl.Nq
    fwd = 2 * (q + 2 * kv * frac + q) + 4 * rows
    bwd = 2 * (2 * q + 2 * kv * frac) + 8 * rows + 2 * 2 * kv + 2 * 4 * q
    return fwd, bwd


def peak_clock_mhz(path=None):
    """Median SM clock of the measured bf16 peak, if the peaks file
    (MEASURED_PEAKS.json by default) records one (else None)."""
    try:
        with open(path or os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            pk = json.load(f)
    except (OSError, ValueError):
        return None

    def walk(x, path=""):
        if isinstance(x, dict):
            for k, v in x.items():
                yield from walk(v, f"{path}.{k}".lower())
        elif isinstance(x, (int, float)) and not isinstance(x, bool):
            yield path, float(x)
    cands = [(p, v) for p, v in walk(pk) if ("mhz" in p or "clock" in p) and "max" not in p
             and 300 < v < 3000]
    # prefer a clock recorded with the GEMM (bf16) measurement, then any SM clock
    cands.sort(key=lambda c: (not any(t in c[0] for t in ("bf16", "gemm", "tflops")),
                              "sm" not in c[0]))
    return cands[0][1] if cands else None


def roofline(name, flops, nbytes, ms, peaks, peak_src, traffic=None):
    """Roofline object of one kernel: bound by its arithmetic intensity
    against the ridge of the measured peaks; both fractions reported."""
    s = ms / 1e3
    tf = flops / s / 1e12
    gbs = nbytes / s / 1e9
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    hbm = flops / nbytes < ridge
    src = (f"{peak_src} (MEASURED_PEAKS.json)" if peak_src == "measured"
           else "fallback 1.59 PFLOP/s / 6.65 TB/s")
    out = {"bound": "hbm" if hbm else "tensor", "kernel": name,
           "achieved": round(gbs if hbm else tf, 2), "peak": peaks["hbm_gbs" if hbm
                                                              else "bf16_tflops"],
           "unit": "GB/s" if hbm else "TFLOP/s",
           "frac": round((gbs / peaks["hbm_gbs"]) if hbm else (tf / peaks["bf16_tflops"]), 4),
           "traffic": traffic, "peak_source": src,
           "tensor": {"tflops": round(tf, 2), "frac": round(tf / peaks["bf16_tflops"], 4)},
           "hbm": {"algorithmic_bytes": int(nbytes), "gbs": round(gbs, 1),
                   "frac": round(gbs / peaks["hbm_gbs"], 4)},
           "arithmetic_intensity": round(flops / nbytes, 1), "ridge": round(ridge, 1)}
    return out


def block_mask_for(wl, density):
    """Seeded block mask of the block-sparse measurement (None: dense)."""
    if density is None:
        return None
    from exact_io_aware_71_b200.inputs import make_block_mask
    return make_block_mask(wl.Nq, wl.Nk, density, seed=wl.seed)


def kept_fraction(wl, mask) -> float:
    """Visible (query, key) pairs under the block mask (and the causal mask)
    over those of the dense problem: the FLOP scale of block-sparse steps."""
    import numpy as np
    if mask is None:
        return 1.0
    m = np.asarray(mask, dtype=bool)
    rows = np.minimum(wl.Nq, (np.arange(m.shape[0]) + 1) * 128) - np.arange(m.shape[0]) * 128
    cols = np.minimum(wl.Nk, (np.arange(m.shape[1]) + 1) * 128) - np.arange(m.shape[1]) * 128
    if not wl.causal:
        return float((m * np.outer(rows, cols)).sum() / (wl.Nq * wl.Nk))
    # causal: pairs (i, j) with j <= i inside each block
    kept = dense = 0.0
    for bi in range(m.shape[0]):
        i = np.arange(bi * 128, bi * 128 + rows[bi])
        for bj in range(m.shape[1]):
            j0, j1 = bj * 128, bj * 128 + cols[bj]
            n = np.clip(np.minimum(i + 1, j1) - j0, 0, None).sum()
            dense += n
            kept += n if m[bi, bj] else 0
    return float(kept / dense)


ORACLE_ROWS = 2048      # query rows per oracle timing sample


def oracle_samples(wl):
    """Timing samples of the fp64 oracle for a workload: blocks of up to
    ORACLE_ROWS query rows of one (batch, query head), each against all of
    that head's keys, in an order that spreads over batches, heads and rows
    (last rows first).  Returns a list of (b, h, r0, r1)."""
    rows = min(wl.Nq, ORACLE_ROWS)
    blocks = [(r0, min(wl.Nq, r0 + rows)) for r0 in range(0, wl.Nq, rows)][::-1]
    heads = [(b, h) for b in range(wl.B) for h in range(wl.Hq)]
    order = []
    for i in range(len(heads) * len(blocks)):
        b, h = heads[(i * 7919) % len(heads)] if len(heads) > 1 else heads[0]
        order.append((b, h) + blocks[(i // len(heads)) % len(blocks)])
    return order


def time_oracle(wl, seconds: float, max_samples=None, mask=None):
    """fp64 oracle forward + backward on samples of the workload (see
    oracle_samples), as many as fit in about `seconds`; returns (TFLOP/s,
    cores, sample description, seconds, FLOPs).  The oracle forms every
    query row's full row of scores (masked entries included), so its work
    per row is the same for every row of a head: the time for the whole
    workload is exactly the number of rows over the sampled rows times the
    sampled time, and the rate is the workload's nominal FLOPs over that."""
    from threadpoolctl import threadpool_limits

    import oracle
    from exact_io_aware_71_b200.inputs import make_inputs

    cores = len(os.sched_getaffinity(0))
    if wl.name not in _INPUT_CACHE:
        _INPUT_CACHE.clear()
        _INPUT_CACHE[wl.name] = make_inputs(wl)
    q, k, v, do = _INPUT_CACHE[wl.name]
    g = wl.Hq // wl.Hkv
    total_rows = wl.B * wl.Hq * wl.Nq
    nominal = 3.5 * wl.fwd_flops() * kept_fraction(wl, mask)
    done_rows, t_total, n = 0, 0.0, 0
    with threadpool_limits(limits=cores):
        for (b, h, r0, r1) in oracle_samples(wl):
            if max_samples is not None and n >= max_samples:
                break
            j = h // g
            qs = q[b:b + 1, h:h + 1, r0:r1].double().numpy()
            dos = do[b:b + 1, h:h + 1, r0:r1].double().numpy()
            ks = k[b:b + 1, j:j + 1].double().numpy()
            vs = v[b:b + 1, j:j + 1].double().numpy()
            m = None if mask is None else mask.numpy()[r0 // 128:(r1 + 127) // 128]
            t0 = time.perf_counter()
            oracle.attention_backward(qs, ks, vs, dos, wl.causal, wl.scale, return_aux=True,
                                      block_mask=m)
            t_total += time.perf_counter() - t0
            done_rows += r1 - r0
            n += 1
            if max_samples is None and t_total >= seconds and n >= 2:
                break
    flops = nominal * done_rows / total_rows
    tflops = flops / t_total / 1e12
    sample = (f"fp64 NumPy oracle fwd+bwd on {n} sample(s) of up to {ORACLE_ROWS} query rows of one "
              f"(batch, query head) against all its keys, {done_rows} of {total_rows} query rows "
              f"of {wl.name}{'' if mask is None else ' with the same block mask'}; "
              f"{t_total:.1f} s of CPU work; rate scaled by rows (the oracle's work per row is "
              f"uniform)")
    return tflops, cores, sample, t_total, flops


# ----------------------------------------------------------------- packed batches
def varlen_lengths(wl, spec, rank=0):
    """Seeded sequence lengths of the --varlen measurement."""
    from exact_io_aware_71_b200.inputs import make_varlen_lengths
    lo, hi = (int(x) for x in spec.split(":"))
    if not 1 <= lo <= hi:
        raise ValueError("--varlen wants LO:HI with 1 <= LO <= HI")
    return make_varlen_lengths(wl.B, lo, hi, seed=wl.seed + 1000 * rank)


def varlen_fwd_flops(wl, lengths) -> float:
    """Nominal forward FLOPs of a packed batch: 4*Hq*n^2*d per sequence,
    halved when causal."""
    f = sum(4.0 * wl.Hq * n * n * wl.d for n in lengths)
    return f / 2 if wl.causal else f


def time_oracle_varlen(wl, lengths, seconds: float, max_seqs=None):
    """fp64 oracle forward + backward on whole sequences of the packed batch,
    as many as fit in about `seconds` (shortest first, so a bounded sample
    covers several); returns (TFLOP/s, cores, sample, seconds, FLOPs)."""
    from threadpoolctl import threadpool_limits

    import numpy as np

    import oracle
    from exact_io_aware_71_b200.inputs import make_varlen_inputs

    cores = len(os.sched_getaffinity(0))
    q, k, v, do, cq, ck = make_varlen_inputs(lengths, lengths, wl.Hq, wl.Hkv, wl.d, wl.seed)
    order = sorted(range(len(lengths)), key=lambda b: lengths[b])
    done, t_total, flops = 0, 0.0, 0.0
    with threadpool_limits(limits=cores):
        for b in order:
            if max_seqs is not None and done >= max_seqs:
                break
            sl = slice(int(cq[b]), int(cq[b + 1]))
            cu = np.array([0, lengths[b]])
            args = [t[sl].double().numpy() for t in (q, k, v, do)]
            t0 = time.perf_counter()
            oracle.attention_backward_varlen(*args, cu, cu, wl.causal, wl.scale)
            t_total += time.perf_counter() - t0
            flops += 3.5 * varlen_fwd_flops(wl, [lengths[b]])
            done += 1
            if max_seqs is None and t_total >= seconds and done >= 2:
                break
    sample = (f"fp64 NumPy oracle fwd+bwd on {done} of {len(lengths)} sequences (shortest "
              f"first) of the packed batch; {t_total:.1f} s of CPU work; rate scaled by FLOPs")
    return flops / t_total / 1e12, cores, sample, t_total, flops


def run_ours_varlen(args, rank, world, local_rank):
    """The --varlen step: fa_fwd_varlen + fa_bwd_varlen on packed inputs."""
    import torch

    from exact_io_aware_71_b200 import binding as fa
    from exact_io_aware_71_b200.inputs import make_varlen_inputs, workloads

    wl = workloads()[args.workload]
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    fa.load()
    lengths = varlen_lengths(wl, args.varlen, rank if world > 1 else 0)
    q, k, v, do, cq, ck = (t.to(dev) for t in make_varlen_inputs(
        lengths, lengths, wl.Hq, wl.Hkv, wl.d, wl.seed + (1000 * rank if world > 1 else 0)))
    B, tq, mx = len(lengths), q.shape[0], max(lengths)
    o = torch.empty_like(q)
    lse = torch.empty(wl.Hq, tq, dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    wsb = fa.fa_bwd_varlen_workspace_size(B, tq, tq, wl.Hq, wl.Hkv, wl.d)
    ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream
    geo = (cq.data_ptr(), ck.data_ptr(), B, mx, mx, tq, tq, wl.Hq, wl.Hkv, wl.d, int(wl.causal),
           wl.scale)

    def step(evs=None):
        if evs:
            evs[0].record(stream)
        st = fa.fa_fwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                              lse.data_ptr(), *geo, sh)
        if st:
            raise fa.FaError(st, "fa_fwd_varlen")
        if evs:
            evs[1].record(stream)
        st = fa.fa_bwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                              lse.data_ptr(), do.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                              dv.data_ptr(), *geo, ws.data_ptr(), wsb, sh)
        if st:
            raise fa.FaError(st, "fa_bwd_varlen")
        if evs:
            evs[2].record(stream)

    dist = torch.distributed if world > 1 else None

    def reduce_max(x):
        if dist is None:
            return x
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    st, where = fa.fa_device_status(sh)
    if st:
        raise RuntimeError(f"device status {st} at wait {where} during warm-up")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local_rank)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    e0.record(stream)
    for s_ in range(args.steps):
        step(evs[s_])
    e1.record(stream)
    torch.cuda.synchronize(dev)
    if dist is not None:
        dist.barrier()
    clk = clocks.stop()
    per_ms = [sum(evs[s_][i].elapsed_time(evs[s_][i + 1]) for s_ in range(args.steps))
              / args.steps for i in range(2)]
    st, where = fa.fa_device_status(sh)
    if st:
        raise RuntimeError(f"device status {st} at wait {where} in the timed region")
    fwd_flops = varlen_fwd_flops(wl, lengths)
    bwd_flops = 2.5 * fwd_flops
    t_ms, fps = aggregate(e0.elapsed_time(e1), args.steps * (fwd_flops + bwd_flops), world,
                          reduce_max)
    peaks, peak_src = load_peaks()
    names = ["fa_fwd_pair_kernel (packed)", "fa_bwd (pre, main, dq; packed)"]
    dom = 0 if per_ms[0] >= per_ms[1] else 1
    achieved = (fwd_flops, bwd_flops)[dom] / (per_ms[dom] / 1e3) / 1e12
    roof = {"bound": "tensor", "kernel": names[dom], "achieved": round(achieved, 2),
            "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
            "frac": round(achieved / peaks["bf16_tflops"], 4),
            "peak_source": f"{peak_src} bf16 cuBLAS burst (MEASURED_PEAKS.json)"
            if peak_src == "measured" else "fallback 1.59 PFLOP/s", "traffic": None}

    # end to end: pinned host inputs in, outputs back, through the torch-level binding
    host_in = [t.cpu().pin_memory() for t in (q, k, v, do)]

    def alloc_out():
        return [torch.empty_like(q), torch.empty(wl.Hq, tq, dtype=torch.float32, device=dev),
                torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)]

    def compute(din, dout):
        fa.forward_varlen(din[0], din[1], din[2], cq, ck, mx, mx, wl.causal, wl.scale,
                          out=dout[0], lse=dout[1])
        fa.backward_varlen(din[0], din[1], din[2], dout[0], dout[1], din[3], cq, ck, mx, mx,
                           wl.causal, wl.scale, workspace=ws, grads=(dout[2], dout[3], dout[4]))

    e_ms_raw, bi, bo = pipelined_e2e(dev, host_in, alloc_out, compute, args.e2e_steps)
    e_ms, e_fps = aggregate(e_ms_raw, args.e2e_steps * 3.5 * fwd_flops, world, reduce_max)
    e2e = {"value": round(e_fps / 1e12, 2), "unit": "TFLOP/s",
           "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo,
           "steps": args.e2e_steps, "ms_per_step": round(e_ms / args.e2e_steps, 3),
           "pipeline": "upload, kernels and download on three streams, double-buffered"}
    fwd_tf = fwd_flops / (per_ms[0] / 1e3) / 1e12
    bwd_tf = bwd_flops / (per_ms[1] / 1e3) / 1e12
    return {
        "metric": METRIC, "value": round(fps / 1e12, 2), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(3, args.warmup),
        "ms_per_step": round(t_ms / args.steps, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded iid N(0,1), bf16)",
        "config": {"workload": f"{wl.name}_varlen{args.varlen}", "B": B, "Hq": wl.Hq,
                   "Hkv": wl.Hkv, "d": wl.d, "causal": wl.causal, "total_tokens": tq,
                   "max_seqlen": mx, "lengths_seed": wl.seed,
                   "step": "fa_fwd_varlen + fa_bwd_varlen (packed [total, H, d])",
                   "parallelism": f"{world} independent replica(s), no collective",
                   "l2": "inputs larger than L2, no flush" if 4 * q.numel() * 2 > 126e6
                   else "inputs smaller than L2: re-read from L2 between steps",
                   "flops": "sum over sequences of 4*Hq*n^2*d (x1/2 causal), x3.5 per step"},
        "fwd_tflops": round(fwd_tf, 2), "bwd_tflops": round(bwd_tf, 2),
        "fwd_frac_of_peak": round(fwd_tf / peaks["bf16_tflops"], 4),
        "bwd_frac_of_peak": round(bwd_tf / peaks["bf16_tflops"], 4),
        "per_kernel_ms": {n: round(t, 4) for n, t in zip(names, per_ms)},
        "roofline": roof, "e2e": e2e, "clocks": clk,
        "gpu_launches": launches_per_step(wl, torch.cuda.get_device_properties(dev)
                                          .multi_processor_count) * args.steps,
    }


# ----------------------------------------------------------------- attention layer
def run_layer(args, rank, world, local_rank):
    """The --layer measurement: forward + backward of the synthetic attention
    layer (exact_io_aware_71_b200.layer) on the workload's B, N, Hq, Hkv, d
    with hidden = Hq * d.  Model FLOPs count the projection GEMMs (cuBLAS)
    and the attention's nominal FLOPs; MFU divides by the measured bf16
    peak."""
    import torch

    from exact_io_aware_71_b200.inputs import workloads
    from exact_io_aware_71_b200.layer import AttentionLayer, layer_flops

    wl = workloads()[args.workload]
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    hidden = wl.Hq * wl.d
    layer = AttentionLayer(hidden, wl.Hq, wl.Hkv, wl.d, wl.causal, device=dev, seed=wl.seed)
    g = torch.Generator("cpu").manual_seed(wl.seed + 1000 * rank)
    x = torch.randn(wl.B, wl.Nq, hidden, generator=g).to(torch.bfloat16).to(dev)
    dy = torch.randn(wl.B, wl.Nq, hidden, generator=g).to(torch.bfloat16).to(dev)
    stream = torch.cuda.current_stream(dev)

    def step(evs=None):
        if evs:
            evs[0].record(stream)
        layer.forward(x)
        if evs:
            evs[1].record(stream)
        layer.backward(dy)
        if evs:
            evs[2].record(stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local_rank)
    torch.cuda.synchronize(dev)
    clocks.start()
    e0.record(stream)
    for s_ in range(args.steps):
        step(evs[s_])
    e1.record(stream)
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    ff, fb = layer_flops(wl.B, wl.Nq, hidden, wl.Hq, wl.Hkv, wl.d, wl.causal)
    ms = e0.elapsed_time(e1) / args.steps
    fwd_ms = sum(e[0].elapsed_time(e[1]) for e in evs) / args.steps
    bwd_ms = sum(e[1].elapsed_time(e[2]) for e in evs) / args.steps
    peaks, peak_src = load_peaks()
    tf = (ff + fb) / (ms / 1e3) / 1e12
    return {
        "metric": "attention layer (QKV projection + exact attention + output projection) "
                  "fwd+bwd model TFLOP/s and model-FLOP utilisation",
        "value": round(tf, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": round(ms, 4), "higher_is_better": True,
        "dtype": "bf16", "data": "synthetic (seeded iid N(0,1) activations, seeded weights)",
        "config": {"workload": wl.name + "_layer", "B": wl.B, "N": wl.Nq, "hidden": hidden,
                   "Hq": wl.Hq, "Hkv": wl.Hkv, "d": wl.d, "causal": wl.causal,
                   "step": "layer forward + backward: 4 cuBLAS GEMMs fwd, 4 bwd (dW, dx "
                           "for both projections), fa_fwd_strided + fa_bwd_strided on "
                           "views of the packed QKV tensor"},
        "mfu": round(tf / peaks["bf16_tflops"], 4),
        "mfu_peak": {"tflops": peaks["bf16_tflops"], "source": peak_src},
        "fwd_ms": round(fwd_ms, 4), "bwd_ms": round(bwd_ms, 4),
        "model_gflop_per_step": {"fwd": round(ff / 1e9, 1), "bwd": round(fb / 1e9, 1)},
        "clocks": clk,
    }


# ----------------------------------------------------------------- our arm
def run_ours(args, rank, world, local_rank):
    import torch

    from exact_io_aware_71_b200 import binding as fa
    from exact_io_aware_71_b200.inputs import make_inputs, workloads

    wl = workloads()[args.workload]
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    fa.load()
    seed_wl = wl.with_(seed=wl.seed + 1000 * rank) if world > 1 else wl
    q, k, v, do = (t.to(dev) for t in make_inputs(seed_wl))
    o = torch.empty_like(q)
    lse = torch.empty(wl.B, wl.Hq, wl.Nq, dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    wsb = fa.fa_bwd_workspace_size(wl.B, wl.Hq, wl.Hkv, wl.Nq, wl.Nk, wl.d, wl.causal)
    ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream
    dims = (wl.B, wl.Hq, wl.Hkv, wl.Nq, wl.Nk, wl.d, int(wl.causal), wl.scale)
    bwd_args = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                do.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr()) + dims

    mask = block_mask_for(wl, args.block_density)
    frac = kept_fraction(wl, mask)
    sparse = mask is not None
    if sparse:
        mask_d = mask.to(dev)
        # one event pair per call: the backward's three kernels are timed together
        names = ["fa_fwd_kernel", "fa_bwd (pre, main, dq)"]
    else:
        names = ["fa_fwd_kernel", "fa_bwd_pre_kernel", "fa_bwd_main_kernel", "fa_bwd_dq_kernel"]
    nk = len(names)

    def step(evs=None):
        if evs:
            evs[0].record(stream)
        if sparse:
            st = fa.fa_fwd_block_sparse(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                        lse.data_ptr(), None, mask_d.data_ptr(), *dims, sh)
            if st:
                raise fa.FaError(st, "fa_fwd_block_sparse")
            if evs:
                evs[1].record(stream)
            st = fa.fa_bwd_block_sparse(*bwd_args[:9], None, mask_d.data_ptr(), *dims,
                                        ws.data_ptr(), wsb, sh)
            if st:
                raise fa.FaError(st, "fa_bwd_block_sparse")
            if evs:
                evs[2].record(stream)
            return
        st = fa.fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                       *dims, sh)
        if st:
            raise fa.FaError(st, "fa_fwd")
        for i, stage in enumerate((fa.FA_BWD_PRE, fa.FA_BWD_MAIN, fa.FA_BWD_DQ)):
            if evs:
                evs[i + 1].record(stream)
            st = fa.fa_bwd_stage(stage, *bwd_args, ws.data_ptr(), wsb, sh)
            if st:
                raise fa.FaError(st, "fa_bwd_stage")
        if evs:
            evs[4].record(stream)

    dist = None
    if world > 1:
        import torch.distributed as dist

    def barrier():
        if dist is not None:
            dist.barrier()

    def reduce_max(x):
        if dist is None:
            return x
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    st, where = fa.fa_device_status(sh)
    if st:
        raise RuntimeError(f"device status {st} at wait {where} during warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nk + 1)]
           for _ in range(args.steps)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local_rank)
    barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    e0.record(stream)
    for s in range(args.steps):
        step(evs[s])
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    clk = clocks.stop()
    local_ms = e0.elapsed_time(e1)
    per_kernel_ms = [sum(evs[s][i].elapsed_time(evs[s][i + 1]) for s in range(args.steps))
                     / args.steps for i in range(nk)]
    st, where = fa.fa_device_status(sh)
    if st:
        raise RuntimeError(f"device status {st} at wait {where} in the timed region")

    fwd_flops, bwd_flops = wl.fwd_flops() * frac, wl.bwd_flops() * frac
    flops_step = fwd_flops + bwd_flops
    t_ms, flops_per_s = aggregate(local_ms, args.steps * flops_step, world, reduce_max)
    value = flops_per_s / 1e12

    # ---- roofline of the dominant kernel (largest share of the step), and of
    # the forward and the backward main kernel each
    peaks, peak_src = load_peaks()
    fwd_bytes, bwd_bytes = algorithmic_bytes(wl, frac)
    main = 1 if sparse else 2
    kern_roof = {
        names[0]: roofline(names[0], fwd_flops, fwd_bytes, per_kernel_ms[0], peaks, peak_src,
                           recorded_traffic(names[0], wl.name)),
        names[main]: roofline(names[main], bwd_flops, bwd_bytes, per_kernel_ms[main], peaks,
                              peak_src, recorded_traffic(names[main], wl.name)),
    }
    dom = max((0, main), key=lambda i: per_kernel_ms[i])
    roof = kern_roof[names[dom]]
    fwd_tflops = fwd_flops / (per_kernel_ms[0] / 1e3) / 1e12
    bwd_ms = sum(per_kernel_ms[1:])
    bwd_tflops = bwd_flops / (bwd_ms / 1e3) / 1e12

    # ---- end to end through the public API with host buffers
    e2e = run_e2e(args, wl, dev, stream, fa, q, k, v, do, reduce_max, world,
                  mask_d if sparse else None, frac)

    out = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": round(t_ms / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded iid N(0,1), bf16)",
        "config": {"workload": wl.name + (f"_blocksparse{args.block_density:g}" if sparse else ""),
                   "B": wl.B, "Hq": wl.Hq, "Hkv": wl.Hkv, "Nq": wl.Nq,
                   "Nk": wl.Nk, "d": wl.d, "causal": wl.causal,
                   "step": ("fa_fwd_block_sparse + fa_bwd_block_sparse" if sparse
                            else "fa_fwd + fa_bwd (pre, main, dq)"),
                   "parallelism": f"{world} independent replica(s), no collective",
                   "l2": l2_note(q, k, v, do)},
        "fwd_tflops": round(fwd_tflops, 2), "bwd_tflops": round(bwd_tflops, 2),
        "fwd_frac_of_peak": round(fwd_tflops / peaks["bf16_tflops"], 4),
        "bwd_frac_of_peak": round(bwd_tflops / peaks["bf16_tflops"], 4),
        "frac_of_datasheet": {"fwd": round(fwd_tflops / DATASHEET_BF16_TFLOPS, 4),
                              "bwd": round(bwd_tflops / DATASHEET_BF16_TFLOPS, 4),
                              "peak": DATASHEET_BF16_TFLOPS},
        "clock_normalised": clock_normalised(fwd_tflops, bwd_tflops, clk, peaks),
        "per_kernel_ms": {n: round(t, 4) for n, t in zip(names, per_kernel_ms)},
        "roofline": roof, "kernel_roofline": kern_roof, "e2e": e2e, "clocks": clk,
        "gpu_launches": launches_per_step(wl, torch.cuda.get_device_properties(dev)
                                          .multi_processor_count) * args.steps,
    }
    if sparse:
        out["config"]["block_mask"] = {
            "block": 128, "density": args.block_density, "seed": wl.seed,
            "kept_pair_fraction": round(frac, 4),
            "flops": "nominal dense FLOPs x kept (query, key) pair fraction"}
    return out


def l2_note(*ts):
    nbytes = sum(t.numel() * t.element_size() for t in ts)
    if nbytes > 126e6:
        return f"inputs larger than L2 ({nbytes / 2**20:.0f} MiB read per step), no flush"
    return f"inputs ({nbytes / 2**20:.0f} MiB) fit in L2: re-read from L2 between steps"


def clock_normalised(fwd_tflops, bwd_tflops, clk, peaks):
    """Fractions of peak per SM clock cycle: the run's TFLOP/s at its median
    sampled SM clock against the measured peak at the clock it was measured
    at (None when either clock is unknown)."""
    pmhz = peak_clock_mhz()
    mhz = clk.get("sm_mhz") if isinstance(clk, dict) else None
    if not pmhz or not mhz:
        return {"fwd": None, "bwd": None, "run_sm_mhz": mhz, "peak_sm_mhz": pmhz}
    per = peaks["bf16_tflops"] / pmhz
    return {"fwd": round(fwd_tflops / mhz / per, 4), "bwd": round(bwd_tflops / mhz / per, 4),
            "run_sm_mhz": mhz, "peak_sm_mhz": pmhz}


def pipelined_e2e(dev, host_in, alloc_out, compute, steps, warmup=2):
    """End-to-end steps through the public API with host buffers.  Every step
    copies its inputs from pinned host memory, computes, and copies all its
    outputs back to pinned host memory; the three run on separate streams
    with double-buffered device tensors, so step i+1's upload and step
    i-1's download overlap step i's kernels (both PCIe directions at once).
    Returns the device time of `steps` steps in ms (first upload to last
    download, CUDA events)."""
    import torch

    s_in, s_cmp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    dev_in = [[torch.empty(t.shape, dtype=t.dtype, device=dev) for t in host_in]
              for _ in range(2)]
    dev_out = [alloc_out() for _ in range(2)]
    host_out = [[torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in dev_out[0]]
                for _ in range(2)]
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_cmp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    used = [False, False]

    def one(i):
        b = i % 2
        with torch.cuda.stream(s_in):
            if used[b]:
                s_in.wait_event(ev_cmp[b])          # step i-2 done with these inputs
            for d, h in zip(dev_in[b], host_in):
                d.copy_(h, non_blocking=True)
            ev_in[b].record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(ev_in[b])
            if used[b]:
                s_cmp.wait_event(ev_out[b])         # step i-2's outputs copied out
            compute(dev_in[b], dev_out[b])
            ev_cmp[b].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_cmp[b])
            for h, d in zip(host_out[b], dev_out[b]):
                h.copy_(d, non_blocking=True)
            ev_out[b].record(s_out)
        used[b] = True

    for i in range(warmup):
        one(i)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(steps):
        one(warmup + i)
    e1.record(s_out)
    torch.cuda.synchronize(dev)
    bi = sum(t.numel() * t.element_size() for t in host_in)
    bo = sum(t.numel() * t.element_size() for t in host_out[0])
    return e0.elapsed_time(e1), bi, bo


def run_e2e(args, wl, dev, stream, fa, q, k, v, do, reduce_max, world, mask=None, frac=1.0):
    """Same metric through the public torch-level binding with host buffers:
    each step copies q, k, v, dO from pinned host memory, runs fa.forward and
    fa.backward, and reads o, lse, dq, dk, dv back to pinned host memory
    (pipelined over three streams, see pipelined_e2e)."""
    import torch

    host_in = [t.cpu().pin_memory() for t in (q, k, v, do)]
    wsb = fa.fa_bwd_workspace_size(wl.B, wl.Hq, wl.Hkv, wl.Nq, wl.Nk, wl.d, wl.causal)
    ws = torch.empty(wsb, dtype=torch.uint8, device=dev)

    def alloc_out():
        return [torch.empty_like(q), torch.empty(wl.B, wl.Hq, wl.Nq, dtype=torch.float32,
                                                 device=dev),
                torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)]

    def compute(din, dout):
        fa.forward(din[0], din[1], din[2], wl.causal, wl.scale, out=dout[0], lse=dout[1],
                   block_mask=mask)
        fa.backward(din[0], din[1], din[2], dout[0], dout[1], din[3], wl.causal, wl.scale,
                    workspace=ws, grads=(dout[2], dout[3], dout[4]), block_mask=mask)

    ms, bi, bo = pipelined_e2e(dev, host_in, alloc_out, compute, args.e2e_steps)
    t_ms, fps = aggregate(ms, args.e2e_steps * 3.5 * wl.fwd_flops() * frac, world, reduce_max)
    return {"value": round(fps / 1e12, 2), "unit": "TFLOP/s", "h2d_bytes_per_step": bi,
            "d2h_bytes_per_step": bo, "steps": args.e2e_steps,
            "ms_per_step": round(t_ms / args.e2e_steps, 3),
            "pipeline": "upload, kernels and download on three streams, double-buffered"}


# ----------------------------------------------------------------- reference arm
def run_reference(args):
    from exact_io_aware_71_b200.inputs import workloads
    wl = workloads()[args.workload]
    mask = block_mask_for(wl, args.block_density)
    lengths = varlen_lengths(wl, args.varlen) if args.varlen else None

    def sample_step():
        if lengths is not None:
            return time_oracle_varlen(wl, lengths, 0.0, max_seqs=1)
        return time_oracle(wl, 0.0, max_samples=1, mask=mask)
    for _ in range(args.warmup):
        sample_step()
    t_all, f_all = 0.0, 0.0
    cores = len(os.sched_getaffinity(0))
    for _ in range(args.steps):
        _, cores, sample, t, f = sample_step()
        t_all += t
        f_all += f
    value = f_all / t_all / 1e12
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * t_all / args.steps, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded iid N(0,1), bf16 inputs upcast to fp64)",
        "config": {"workload": wl.name + ("" if mask is None
                                          else f"_blocksparse{args.block_density:g}")
                   + (f"_varlen{args.varlen}" if lengths is not None else ""),
                   "B": wl.B, "Hq": wl.Hq, "Hkv": wl.Hkv, "Nq": wl.Nq,
                   "Nk": wl.Nk, "d": wl.d, "causal": wl.causal,
                   "step": "oracle fwd+bwd on one sample of the workload (up to 2048 query "
                           "rows of one head against all its keys)"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    args = parse_args(argv)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args)), flush=True)
        return 0

    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        if args.layer:
            out = run_layer(args, rank, world, local_rank)
            if rank == 0:
                print(json.dumps(out), flush=True)
            return 0
        out = (run_ours_varlen if args.varlen else run_ours)(args, rank, world, local_rank)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            from exact_io_aware_71_b200.inputs import workloads
            wl = workloads()[args.workload]
            if args.varlen:
                tf, cores, sample, _, _ = time_oracle_varlen(wl, varlen_lengths(wl, args.varlen),
                                                             args.cpu_seconds)
            else:
                tf, cores, sample, _, _ = time_oracle(wl, args.cpu_seconds,
                                                      mask=block_mask_for(wl, args.block_density))
            out["cpu_baseline"] = {"value": round(tf, 6), "unit": "TFLOP/s", "cores": cores,
                                   "kind": "oracle", "sample": sample}
        if rank == 0:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
