"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle.

This module only draws random numbers and names workload shapes; it holds
none of the attention arithmetic.  Inputs are iid N(0, 1) in fp32 drawn from
``torch.Generator('cpu').manual_seed(seed)`` in the order q, k, v, dO and
then rounded to bf16 (round-to-nearest-even).  Workloads that widen the
softmax dynamic range multiply Q by 2 on the first half of the query heads
(exact in bf16, so scaling before or after the cast is the same tensor).

Shapes follow the attention workloads on the FlashAttention pages: sequence
lengths 512..16k at hidden size 2048 with head dim 64 or 128, causal on and
off (FA2 post on t.iss.one, section "Результаты"), head dims up to 256 and
MQA/GQA (QbitAI FA2 article, section "具体实现"), and 64k context (QbitAI FA1
article, results section).
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    """One attention problem: sizes, masking and the input recipe."""
    name: str
    B: int
    Hq: int
    Hkv: int
    Nq: int
    Nk: int
    d: int
    causal: bool
    seed: int
    q_scale_half_heads: bool = False
    directions: tuple = ("fwd", "bwd")

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def fwd_flops(self) -> float:
        """Nominal forward FLOPs 4*B*Hq*Nq*Nk*d, halved when causal."""
        f = 4.0 * self.B * self.Hq * self.Nq * self.Nk * self.d
        return f / 2 if self.causal else f

    def bwd_flops(self) -> float:
        """Nominal backward FLOPs: 2.5x the forward."""
        return 2.5 * self.fwd_flops()

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def _w(name, B, H, N, d, causal, seed, Hkv=None, q2=False, dirs=("fwd", "bwd")):
    return Workload(name, B, H, Hkv or H, N, N, d, causal, seed, q2, dirs)


def workloads() -> dict:
    """All named workloads (the tiny case, the training shape, the
    sequence-length sweep, long-context GQA/MQA and the large-head / 64k
    cases)."""
    w = {}
    for c in (False, True):
        tag = "causal" if c else "full"
        w[f"tiny_b1h2n128d64_{tag}"] = _w(f"tiny_b1h2n128d64_{tag}", 1, 2, 128, 64, c, 1)
        w[f"train_b8h16n2048d128_{tag}"] = _w(f"train_b8h16n2048d128_{tag}", 8, 16, 2048, 128, c, 2)
        for d, h in ((64, 32), (128, 16)):
            for n in (512, 1024, 2048, 4096, 8192, 16384):
                nm = f"sweep_n{n}_d{d}_{tag}"
                w[nm] = _w(nm, 16384 // n, h, n, d, c, 3)
    for hkv in (8, 1):
        nm = f"long_gqa_hkv{hkv}_n16384_d128_causal"
        w[nm] = _w(nm, 1, 32, 16384, 128, True, 4, Hkv=hkv)
    w["large_b4h8n4096d256_full"] = _w("large_b4h8n4096d256_full", 4, 8, 4096, 256,
                                       False, 5, q2=True)
    w["long_b1h8n65536d64_causal"] = _w("long_b1h8n65536d64_causal", 1, 8, 65536, 64,
                                        True, 6, q2=True, dirs=("fwd",))
    return w


MASK_BLOCK = 128


def make_block_mask(Nq: int, Nk: int, density: float, seed: int, keep_diagonal: bool = True,
                    empty_rows=()):
    """Seeded block mask for block-sparse attention, uint8
    [ceil(Nq/128), ceil(Nk/128)] on the CPU.  Each (query block, key block)
    entry is kept with probability ``density`` (uniform draws from
    ``torch.Generator('cpu').manual_seed(seed)``); with ``keep_diagonal``
    the blocks (I, I) are always kept, so every query row sees some key;
    query blocks listed in ``empty_rows`` are cleared entirely."""
    nbq = (Nq + MASK_BLOCK - 1) // MASK_BLOCK
    nbk = (Nk + MASK_BLOCK - 1) // MASK_BLOCK
    g = torch.Generator("cpu").manual_seed(seed)
    m = (torch.rand(nbq, nbk, generator=g) < density).to(torch.uint8)
    if keep_diagonal:
        i = torch.arange(min(nbq, nbk))
        m[i, i] = 1
    for r in empty_rows:
        m[r] = 0
    return m


def make_inputs(wl: Workload, device="cpu", with_do: bool = True):
    """Return bf16 (q, k, v, dO) for a workload, drawn on the CPU.

    Layout is contiguous [B, H, N, d] (H = Hq for q and dO, Hkv for k, v)."""
    g = torch.Generator("cpu").manual_seed(wl.seed)
    q = torch.randn(wl.B, wl.Hq, wl.Nq, wl.d, generator=g)
    k = torch.randn(wl.B, wl.Hkv, wl.Nk, wl.d, generator=g)
    v = torch.randn(wl.B, wl.Hkv, wl.Nk, wl.d, generator=g)
    do = torch.randn(wl.B, wl.Hq, wl.Nq, wl.d, generator=g) if with_do else None
    if wl.q_scale_half_heads:
        q[:, : wl.Hq // 2] *= 2.0
    out = [q, k, v] + ([do] if with_do else [])
    out = [t.to(torch.bfloat16).to(device) for t in out]
    if not with_do:
        out.append(None)
    return tuple(out)


def make_varlen_lengths(B: int, lo: int, hi: int, seed: int):
    """Seeded sequence lengths, uniform integers in [lo, hi]."""
    g = torch.Generator("cpu").manual_seed(seed)
    return torch.randint(lo, hi + 1, (B,), generator=g).tolist()


def cu_seqlens(lengths):
    """Cumulative offsets [0, l0, l0 + l1, ...] as int32 (CPU)."""
    out = [0]
    for n in lengths:
        out.append(out[-1] + int(n))
    return torch.tensor(out, dtype=torch.int32)


def make_varlen_inputs(lengths_q, lengths_k, Hq: int, Hkv: int, d: int, seed: int):
    """Packed bf16 q [total_q, Hq, d], k, v [total_k, Hkv, d], dO like q,
    iid N(0, 1) drawn in that order from ``manual_seed(seed)``, plus the
    int32 cumulative offsets of both sides (all on the CPU)."""
    g = torch.Generator("cpu").manual_seed(seed)
    tq, tk = int(sum(lengths_q)), int(sum(lengths_k))
    q = torch.randn(tq, Hq, d, generator=g)
    k = torch.randn(tk, Hkv, d, generator=g)
    v = torch.randn(tk, Hkv, d, generator=g)
    do = torch.randn(tq, Hq, d, generator=g)
    q, k, v, do = (t.to(torch.bfloat16) for t in (q, k, v, do))
    return q, k, v, do, cu_seqlens(lengths_q), cu_seqlens(lengths_k)
