// Helpers shared by the forward and backward kernels.
//
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

// Power-of-two scale 2^e of an fp16 copy of a bf16 tensor whose largest
// magnitude m has the float bits amax_bits: m * 2^e in [2^14, 2^15), below
// fp16's largest finite value, so the copy is exact for every element
// within 2^24 of m.  0 for zero, inf or NaN; clamped to [-60, 60].
__host__ __device__ __forceinline__ int f16_exp(unsigned amax_bits) {
  const int ex = int((amax_bits >> 23) & 0xFFu);   // biased exponent of m (m >= 0)
  if (ex == 255 || amax_bits == 0u) return 0;      // inf / NaN, or all zero: no scaling
  if (ex == 0) return 60;                          // m below the normal range
  const int k = ex - 126;                          // m = f * 2^k with f in [0.5, 1)
  const int e = 15 - k;
  return e < -60 ? -60 : (e > 60 ? 60 : e);
}

}  // namespace fa
