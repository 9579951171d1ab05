// Where the backward pass keeps its fp32 row vectors (D = rowsum(dO o O) and
// LSE * log2 e) in the caller's workspace.  Both the backward kernels and the
// forward kernel's D epilogue (which recomputes D from the fp32 output for
// wide GQA / MQA groups) address them through these helpers.
//
// Fixed-length batches: row n of (batch, query head) bh is entry
// bh * Nq_pad + n, with Nq_pad = ceil(Nq / 128) * 128.
// Packed variable-length batches: row n of sequence b at query head h is
// entry h * ld + varlen_pad_start(cu_q[b], b) + n, where ld covers every
// sequence's rows padded to a multiple of 128 (16-byte aligned starts).
#pragma once

namespace fa {

__host__ __device__ __forceinline__ long long varlen_pad_start(int off, int b) {
  return (long long)((off + 3) & ~3) + 256LL * b;
}

}  // namespace fa
