"""A synthetic attention layer, for an end-to-end model-FLOP utilisation
check of the attention kernels inside a transformer block.

The FA2 pages report FlashAttention-2 inside whole GPT-style training runs
(QbitAI FA2 article, section "实验评估": 225 TFLOP/s, 72 % model-FLOP
utilisation end to end).  Without models or data, this layer is the part of
such a block that the attention kernels sit in:

    qkv = x W_qkv          x [B, N, hidden], W_qkv [hidden, (Hq + 2 Hkv) d]
    q, k, v                strided [B, H, N, d] views of the packed qkv
    o = attention(q, k, v) libfa, written as [B, N, Hq, d]
    y = o W_o              W_o [Hq d, hidden]

and its backward pass.  The two projections are plain library GEMMs
(torch.matmul, i.e. cuBLAS); the attention runs the library's strided entry
points on views of the packed tensors, so no transpose or copy is
materialised on either side.  Weights are seeded random (std 1/sqrt(fan-in))
in bf16.  The argument marshalling here is thin: every step of the
attention is in the CUDA kernels.
"""
from __future__ import annotations

import math

from . import binding as fa


def layer_flops(B, N, hidden, Hq, Hkv, d, causal):
    """(forward, backward) model FLOPs of one layer step: the projection
    GEMMs (2 FLOPs per multiply-add; backward twice the forward) and the
    attention's nominal 4*B*Hq*N^2*d (halved when causal; backward 2.5x)."""
    gemm = 2.0 * B * N * hidden * (Hq + 2 * Hkv) * d + 2.0 * B * N * Hq * d * hidden
    attn = 4.0 * B * Hq * N * N * d * (0.5 if causal else 1.0)
    return gemm + attn, 2.0 * gemm + 2.5 * attn


class AttentionLayer:
    """QKV projection, exact attention (libfa), output projection."""

    def __init__(self, hidden, Hq, Hkv, d, causal, device="cuda", seed=0):
        import torch
        if Hq % Hkv:
            raise ValueError("Hq must be a multiple of Hkv")
        self.hidden, self.Hq, self.Hkv, self.d, self.causal = hidden, Hq, Hkv, d, bool(causal)
        self.scale = 1.0 / math.sqrt(d)
        g = torch.Generator("cpu").manual_seed(seed)
        nqkv = (Hq + 2 * Hkv) * d
        self.w_qkv = (torch.randn(hidden, nqkv, generator=g) / math.sqrt(hidden)).to(
            torch.bfloat16).to(device)
        self.w_o = (torch.randn(Hq * d, hidden, generator=g) / math.sqrt(Hq * d)).to(
            torch.bfloat16).to(device)
        self._ws = None
        self._saved = None
        self._grads = None

    def _split(self, t):
        """q, k, v views [B, H, N, d] of a packed [B, N, Hq + 2 Hkv, d] tensor."""
        Hq, Hkv = self.Hq, self.Hkv
        return (t[:, :, :Hq].transpose(1, 2), t[:, :, Hq:Hq + Hkv].transpose(1, 2),
                t[:, :, Hq + Hkv:].transpose(1, 2))

    def forward(self, x):
        """y [B, N, hidden] for x [B, N, hidden] (bf16, CUDA); keeps what the
        backward pass needs."""
        import torch
        B, N, _ = x.shape
        qkv = torch.matmul(x, self.w_qkv).view(B, N, self.Hq + 2 * self.Hkv, self.d)
        q, k, v = self._split(qkv)
        o = torch.empty(B, N, self.Hq, self.d, dtype=x.dtype, device=x.device)
        lse = torch.empty(B, self.Hq, N, dtype=torch.float32, device=x.device)
        fa.forward(q, k, v, self.causal, self.scale, out=o.transpose(1, 2), lse=lse)
        y = torch.matmul(o.view(B, N, self.Hq * self.d), self.w_o)
        self._saved = (x, qkv, o, lse)
        return y

    def backward(self, dy):
        """(dx, dW_qkv, dW_o) for the output gradient dy [B, N, hidden]."""
        import torch
        x, qkv, o, lse = self._saved
        B, N, _ = x.shape
        o2 = o.view(B * N, self.Hq * self.d)
        dy2 = dy.reshape(B * N, self.hidden)
        dw_o = torch.matmul(o2.t(), dy2)
        do = torch.matmul(dy2, self.w_o.t()).view(B, N, self.Hq, self.d)
        dqkv = torch.empty_like(qkv)
        q, k, v = self._split(qkv)
        need = fa.fa_bwd_workspace_size(B, self.Hq, self.Hkv, N, N, self.d, self.causal)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(need, dtype=torch.uint8, device=x.device)
        fa.backward(q, k, v, o.transpose(1, 2), lse, do.transpose(1, 2), self.causal,
                    self.scale, workspace=self._ws, grads=self._split(dqkv))
        self._grads = (do, dqkv)         # the attention's inputs / outputs, for inspection
        dq2 = dqkv.view(B * N, -1)
        dw_qkv = torch.matmul(x.reshape(B * N, self.hidden).t(), dq2)
        dx = torch.matmul(dq2, self.w_qkv.t()).view(B, N, self.hidden)
        return dx, dw_qkv, dw_o
