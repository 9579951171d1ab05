// Backward pass of exact tiled attention on sm_100a.
//
// The backward pass recomputes the probabilities block by block from Q, K
// and the saved log-sum-exp instead of storing them (QbitAI FA1 article,
// section "FlashAttention": recalculation in the backward pass), and it is
// parallel over key blocks, whose gradients are independent (FA2 post,
// section "Параллелизм": in the backward pass the columns are independent).
//
// Three kernels:
//   fa_bwd_pre      D_i = sum_c dO_ic * O_ic and LSE_i * log2(e) into padded
//                   fp32 rows, and dQacc <- 0            (HBM-bound)
//   fa_bwd_main     one CTA per (batch, kv head, 128-key block[, d half]):
//                   K_j, V_j stay in shared memory; for every query head of
//                   the kv group and every 64-row query block i at or below
//                   the diagonal ("step" t):
//                     S^T  = K_j Q_i^T           (TMEM, lanes = keys)
//                     P^T  = exp2(S^T * scale*log2e - LSE_i*log2e)
//                     dV_j += P^T dO_i           (P^T from TMEM; fp16 P and dO for GQA, d=256)
//                     dP^T = V_j dO_i^T          (fp16 V and dO with them)
//                     dS^T = P^T o (dP^T - D_i)
//                     dK_j += dS^T Q_i           (dS^T read from TMEM; fp16 dS and Q, and
//                                                 fp16 S^T and dQ^T, for wide groups)
//                     dQ_i^T = K_j^T dS^T  -> fp32 reduce-add into dQacc
//                   then dK_j * scale and dV_j are written as bf16
//   fa_bwd_dq       dq = bf16(scale * dQacc)              (HBM-bound)
//
// fa_bwd_main roles (512 threads): warpgroups 0 and 1 are compute warps
// (TMEM lane = key row); warpgroup w owns query columns [32w, 32w+32) of
// every step, and writes its P^T (hi, lo) and dS^T only over its own S^T /
// dP^T columns, so neither group can overwrite scores the other has not yet
// read.  Warp 8 issues the TMA loads, warp 9 the MMAs (10, 11 idle), and
// warpgroup 3 reads dQ^T out of TMEM and reduce-adds it into the fp32
// accumulator, so those global reductions overlap the compute warps' work.
// TMEM (512 columns): S^T x2 | dP^T | dQ^T | dK | dV.  S^T is double-buffered
// so S^T of step t+1 is computed while step t's dS is formed; per step the
// MMA order is dV_t, S_{t+1}, dK_t, dQ_t, dP_{t+1}.  For d = 256 the dK / dV
// accumulators alone would fill TMEM, so two CTAs share a key block, each
// owning one 128-wide half of d for dK, dV and dQ (both recompute S and dP).
#pragma once
#include "sm100.cuh"
#include "fa_mask.cuh"
#include "fa_rows.cuh"

#include <type_traits>

namespace fa {

template <int D>
struct BwdCfg {
  static constexpr int BC = 128;                        // keys per CTA (TMEM lanes)
  static constexpr int BR = 64;                         // query rows per step
  static constexpr int DH = (D == 256) ? 128 : D;       // d columns owned by a CTA
  static constexpr int NSPLIT = D / DH;                 // CTAs per key block
  static constexpr int KCH = D / 64;
  static constexpr int QS = (D == 256) ? 1 : 3;         // Q/dO pipeline stages
  static constexpr int K_BYTES = BC * D * 2;
  static constexpr int QT_BYTES = BR * D * 2;           // one Q or dO tile
  static constexpr int STAGE_BYTES = 2 * QT_BYTES + 2 * BR * 4;
  static constexpr int STAGE_STRIDE = (STAGE_BYTES + 1023) / 1024 * 1024;
  static constexpr int DS_BYTES = BC * BR * 2;          // dS^T: [BC keys][BR queries] bf16
  static constexpr int TM_S = 0;                        // two S^T buffers of BR columns
  static constexpr int TM_DP = 2 * BR;
  static constexpr int TM_DQ = 3 * BR;
  static constexpr int TM_DK = 4 * BR;
  static constexpr int TM_DV = 4 * BR + DH;
  static constexpr int TMEM_COLS = 512;
  static constexpr int NTHREADS = 512;
  // setmaxnreg split of the 512 threads' registers: compute warpgroups 0-1,
  // producer / MMA warpgroup 2, dQ read-out warpgroup 3.
  static constexpr int REGS_COMPUTE = 168;
  static constexpr int REGS_OTHER = 88;
  static constexpr int REGS_READ = 80;
  static constexpr int REGS_NEEDED = 256 * REGS_COMPUTE + 128 * REGS_OTHER + 128 * REGS_READ;
  static_assert(REGS_NEEDED <= 65536, "register split");
  static constexpr int SMEM_BYTES = 2 * K_BYTES + QS * STAGE_STRIDE + DS_BYTES + 1024 + 1024;
  static_assert(TM_DV + DH <= TMEM_COLS, "TMEM budget");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
  static_assert(QS * STAGE_STRIDE >= 2 * BC * DH * 2, "dK/dV staging fits in the Q/dO stages");
};

inline int round_up(int x, int m) { return (x + m - 1) / m * m; }

// Groups whose dK the backward computes from dS rounded to fp16 (every
// product then takes fp16 operands: op_scales) and from an exact D (the
// forward's residual output, or D recomputed by a forward pass with the D
// epilogue): the errors of a bf16 dS and of D from the bf16 O add up over
// every query row of the group.  From 16 query heads per kv head
// on at d <= 128; at d = 256, whose dK carries more of that error (measured
// 2.1e-2 on a packed batch with 4 query heads per kv head), for every GQA /
// MQA group.
constexpr int kExactGroup = 16;
inline bool exact_dk(int group, int d) { return group >= kExactGroup || (d == 256 && group > 1); }

// Problems whose dP^T and dV products take fp16 operands (scaled copies of
// dO and V, and P as fp16): where a bf16 P rounds too coarsely for dV.  A
// GQA / MQA group adds that rounding up over every query head of the group,
// and at d = 256 |dV| is large enough that the output rounding leaves no
// room.  MHA at d <= 128 keeps bf16 operands and skips the fp16 copies.
inline bool bwd_f16(int Hq, int Hkv, int d) { return Hq > Hkv || d == 256; }

// Workspace: dQacc fp32 [B*Hq, Nq, d] | Dpad fp32 [B*Hq, Nq_pad] |
// Lpad fp32 [B*Hq, Nq_pad] | (GQA/MQA only) dKacc, dVacc fp32 [B*Hkv, Nk, d]
// for the partial sums of a kv group split across CTAs | (bwd_f16 only)
// dO16 fp16 [B*Hq, Nq, d] and V16 fp16 [B*Hkv, Nk, d]: dO and V scaled by
// powers of two (the operands of the dP^T and dV products) | (exact_dk
// only) Q16, K16 likewise | amax: four words, the largest |dO|, |V|, |Q|,
// |K| (float bits) that choose those powers.
struct BwdWorkspace {
  size_t dq_off, d_off, l_off, kv_off, kv_elems, do16_off, v16_off, q16_off, k16_off, amax_off,
      total;
};
// The fp16 copies: dO and V (bwd_f16), and Q and K as well (exact_dk, where
// dS and every product that reads it are fp16 too); sizes in elements.
inline void bwd_workspace_tail(BwdWorkspace& w, size_t do_elems, size_t v_elems, size_t q_elems,
                               size_t k_elems) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  w.do16_off = w.kv_off + up(2 * w.kv_elems * 4);
  w.v16_off = w.do16_off + up(do_elems * 2);
  w.q16_off = w.v16_off + up(v_elems * 2);
  w.k16_off = w.q16_off + up(q_elems * 2);
  w.amax_off = w.k16_off + up(k_elems * 2);
  w.total = w.amax_off + 256;
}
inline BwdWorkspace bwd_workspace_layout(int B, int Hq, int Hkv, int Nq, int Nk, int d) {
  const size_t bh = size_t(B) * Hq;
  const size_t nq_pad = size_t(round_up(Nq, 128));
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  BwdWorkspace w;
  w.dq_off = 0;
  w.d_off = up(bh * Nq * d * 4);
  w.l_off = w.d_off + up(bh * nq_pad * 4);
  w.kv_off = w.l_off + up(bh * nq_pad * 4);
  w.kv_elems = (Hq > Hkv) ? size_t(B) * Hkv * Nk * d : 0;   // per tensor
  const bool f16 = bwd_f16(Hq, Hkv, d), all16 = exact_dk(Hq / Hkv, d);
  bwd_workspace_tail(w, f16 ? bh * Nq * d : 0, f16 ? size_t(B) * Hkv * Nk * d : 0,
                     all16 ? bh * Nq * d : 0, all16 ? size_t(B) * Hkv * Nk * d : 0);
  return w;
}
inline size_t bwd_workspace_bytes(int B, int Hq, int Hkv, int Nq, int Nk, int d) {
  return bwd_workspace_layout(B, Hq, Hkv, Nq, Nk, d).total;
}

// Packed variable-length batch of B sequences: dQacc fp32 [Hq, total_q, d] |
// Dpad, Lpad fp32 [Hq, ld] with ld = round_up(total_q, 4) + 256 (B + 1),
// each sequence's rows starting at varlen_pad_start | (GQA/MQA only)
// dKacc, dVacc fp32 [Hkv, total_k, d] | dO16 fp16 [Hq, total_q, d] |
// V16 fp16 [Hkv, total_k, d] | Q16, K16 | amax.
inline long long varlen_lpad_ld(int B, int total_q) {
  return (long long)((total_q + 3) & ~3) + 256LL * (B + 1);
}
inline BwdWorkspace bwd_workspace_layout_varlen(int B, int Hq, int Hkv, int total_q, int total_k,
                                                int d) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  const size_t ld = size_t(varlen_lpad_ld(B, total_q));
  BwdWorkspace w;
  w.dq_off = 0;
  w.d_off = up(size_t(Hq) * total_q * d * 4);
  w.l_off = w.d_off + up(size_t(Hq) * ld * 4);
  w.kv_off = w.l_off + up(size_t(Hq) * ld * 4);
  w.kv_elems = (Hq > Hkv) ? size_t(Hkv) * total_k * d : 0;
  const bool f16 = bwd_f16(Hq, Hkv, d), all16 = exact_dk(Hq / Hkv, d);
  bwd_workspace_tail(w, f16 ? size_t(Hq) * total_q * d : 0, f16 ? size_t(Hkv) * total_k * d : 0,
                     all16 ? size_t(Hq) * total_q * d : 0, all16 ? size_t(Hkv) * total_k * d : 0);
  return w;
}

// ------------------------------------------------------------------ pre
// One group of D/8 threads per row; each thread handles 8 consecutive
// elements (16 bytes) of O and dO and zeroes 8 floats of dQacc.
// Element strides (batch, head, row) of a [B, H, N, d] view; d contiguous.
struct Strides {
  long long b, h, n;
};

// Packed-batch helper: sequence b's rows clamped to [0, total] (its padded
// fp32 row vectors start at varlen_pad_start, fa_rows.cuh: 16-byte aligned,
// with room for ceil(n / 128) * 128 entries before the next sequence).
__device__ __forceinline__ void varlen_rows(const int* cu, int b, int total, int& off, int& n) {
  const int a = min(max(__ldg(cu + b), 0), total);
  n = min(max(__ldg(cu + b + 1), a), total) - a;
  off = a;
}

// ores (optional, at o's strides): the forward's residual bf16(O - bf16(O));
// D then uses o + ores, the fp32 output to 16 bits.
// ---- fp16 operands of the dP^T and dV products.  dO and V are copied once
// into fp16, each scaled by a power of two 2^e chosen from its largest
// magnitude m (m * 2^e in [2^14, 2^15), below fp16's largest finite value),
// so the copies are exact for every element within 2^24 of m (smaller ones
// keep an absolute error below m * 2^-25).  P then goes into dV as fp16
// (relative rounding 2^-11 instead of bf16's 2^-8), which keeps dV within
// the parity bound without a second (lo) product; the kernels multiply
// dP^T by 2^-(e_dO + e_V) and dV by 2^-e_dO, exactly.
// (f16_exp, the exponent rule, is in fa_rows.cuh.)

// Largest |x| over one thread's 8 bf16 elements.
__device__ __forceinline__ float absmax8(uint4 v) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
  }
  return m;
}

// Block-wide max of m (256 threads; NaN is ignored by fmaxf) merged into
// *dst as float bits, which order like the values for m >= 0.
__device__ __forceinline__ void block_max_to(float m, unsigned* dst) {
  __shared__ float red[8];
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float r = red[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) r = fmaxf(r, red[i]);
    if (r > 0.f) atomicMax(dst, __float_as_uint(r));
  }
  __syncthreads();
}

// Largest |x| of a [batch, heads, rows, D] view (element strides sv),
// merged into *dst.
template <int D>
__device__ __forceinline__ void absmax_scan(const __nv_bfloat16* __restrict__ v, Strides sv,
                                            int batch, int heads, int rows, unsigned* dst) {
  constexpr int PR = D / 8;                        // 8-element pieces per row
  const long long n = (long long)batch * heads * rows * PR;
  float m = 0.f;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const long long row = i / PR;
    const int sb = int(i - row * PR);
    const long long r = row % rows, bh = row / rows, hh = bh % heads, bb = bh / heads;
    m = fmaxf(m, absmax8(*reinterpret_cast<const uint4*>(v + bb * sv.b + hh * sv.h + r * sv.n +
                                                        sb * 8)));
  }
  block_max_to(m, dst);
}

// Two fp16 copies in one launch: A16 = fp16(A * 2^e_A) for a query-side
// tensor A (dO, or Q) and B16 = fp16(B * 2^e_B) for a key-side tensor B (V,
// or K), contiguous [batch * heads, rows, D] (packed batches: batch 1, rows
// = the total), after the preprocess kernel has left their largest
// magnitudes in amax_a, amax_b.
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_f16_kernel(
    const __nv_bfloat16* __restrict__ dO, Strides sdo, int bq, int Hq, int rows_q,
    const __nv_bfloat16* __restrict__ v, Strides sv, int bk, int Hkv, int rows_k,
    __half* __restrict__ do16, __half* __restrict__ v16, const unsigned* __restrict__ amax_a,
    const unsigned* __restrict__ amax_b) {
  constexpr int PR = D / 8;
  const float s_do = ldexpf(1.f, f16_exp(*amax_a)), s_v = ldexpf(1.f, f16_exp(*amax_b));
  const long long n_do = (long long)bq * Hq * rows_q * PR;
  const long long n_all = n_do + (long long)bk * Hkv * rows_k * PR;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n_all;
       i += (long long)gridDim.x * blockDim.x) {
    const bool isv = i >= n_do;
    const long long j = isv ? i - n_do : i;
    const int heads = isv ? Hkv : Hq, rows = isv ? rows_k : rows_q;
    const Strides st = isv ? sv : sdo;
    const float sc = isv ? s_v : s_do;
    const long long row = j / PR;
    const int sb = int(j - row * PR);
    const long long r = row % rows, bh = row / rows, hh = bh % heads, bb = bh / heads;
    const uint4 x = *reinterpret_cast<const uint4*>((isv ? v : dO) + bb * st.b + hh * st.h +
                                                    r * st.n + sb * 8);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&x);
    uint4 y;
    uint32_t* yw = reinterpret_cast<uint32_t*>(&y);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __bfloat1622float2(h[k]);
      yw[k] = pack_f16(f.x * sc, f.y * sc);
    }
    *reinterpret_cast<uint4*>((isv ? v16 : do16) + row * D + sb * 8) = y;
  }
}

template <int D>
__global__ void __launch_bounds__(256) fa_bwd_pre_kernel(
    const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ ores,
    const __nv_bfloat16* __restrict__ dO,
    const float* __restrict__ lse, float* __restrict__ dqacc, float* __restrict__ Dpad,
    float* __restrict__ Lpad, int rows_bh, int Hq, int Nq, int Nq_pad, Strides so, Strides sdo,
    float* __restrict__ kvacc, long long kv_n4, const __nv_bfloat16* __restrict__ v, Strides sv,
    int B, int Hkv, int Nk, unsigned* __restrict__ amax, const __nv_bfloat16* __restrict__ qin,
    Strides sq, const __nv_bfloat16* __restrict__ kin, Strides sk) {
  constexpr int TPR = D / 8;                       // threads per row
  constexpr int RPB = 256 / TPR;                   // rows per block pass
  const int sub = threadIdx.x % TPR;
  const int rlocal = threadIdx.x / TPR;
  const long long total = (long long)rows_bh * Nq_pad;
  float mdo = 0.f;                                 // largest |dO| seen by this thread
  for (long long r = (long long)blockIdx.x * RPB + rlocal; r < total;
       r += (long long)gridDim.x * RPB) {
    const long long bh = r / Nq_pad;
    const int q = int(r - bh * Nq_pad);
    float acc = 0.f;
    const bool valid = q < Nq;
    if (valid) {
      const size_t e = (size_t(bh) * Nq + q) * D + sub * 8;
      const long long bb = bh / Hq, hh = bh - bb * Hq;
      const long long oi = bb * so.b + hh * so.h + q * so.n + sub * 8;
      const uint4 ov = *reinterpret_cast<const uint4*>(o + oi);
      const uint4 rv = ores ? *reinterpret_cast<const uint4*>(ores + oi) : make_uint4(0u, 0u, 0u, 0u);
      const uint4 dv = *reinterpret_cast<const uint4*>(dO + bb * sdo.b + hh * sdo.h +
                                                       q * sdo.n + sub * 8);
      const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&ov);
      const __nv_bfloat162* r2 = reinterpret_cast<const __nv_bfloat162*>(&rv);
      const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&dv);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 a = __bfloat1622float2(o2[i]);
        const float2 r = __bfloat1622float2(r2[i]);
        const float2 b = __bfloat1622float2(d2[i]);
        acc = fmaf(a.x + r.x, b.x, acc);
        acc = fmaf(a.y + r.y, b.y, acc);
        mdo = fmaxf(mdo, fmaxf(fabsf(b.x), fabsf(b.y)));
      }
      float4* z = reinterpret_cast<float4*>(dqacc + e);
      z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
      z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int off = TPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (sub == 0) {
      const size_t pi = size_t(bh) * Nq_pad + q;
      Dpad[pi] = valid ? acc : 0.f;
      Lpad[pi] = valid ? lse[size_t(bh) * Nq + q] * 1.4426950408889634f : INFINITY;
    }
  }
  // dK/dV partial-sum accumulators (only when a kv group is split across CTAs)
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < kv_n4;
       i += (long long)gridDim.x * blockDim.x)
    reinterpret_cast<float4*>(kvacc)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  if (amax) {                                      // the fp16 operand scales (bwd_f16)
    block_max_to(mdo, amax);
    absmax_scan<D>(v, sv, B, Hkv, Nk, amax + 1);
    if (qin) {                                     // and Q, K (exact_dk)
      absmax_scan<D>(qin, sq, B, Hq, Nq, amax + 2);
      absmax_scan<D>(kin, sk, B, Hkv, Nk, amax + 3);
    }
  }
}

// The same for a packed variable-length batch: o and dO are [total_q, Hq, d]
// at strides so / sdo (batch stride unused), lse is [Hq, total_q], dQacc is
// [Hq, total_q, d].  Row n of the packed tensors belongs to the sequence b
// with cu_q[b] <= n < cu_q[b+1] (found by bisection); its D and LSE*log2(e)
// go to h * ld + varlen_pad_start(cu_q[b], b) + (n - cu_q[b]).  Afterwards
// the entries from each sequence's length up to the next multiple of 128
// are padding: D = 0, LSE = +inf, so the main kernel's P is 0 there.
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_pre_varlen_kernel(
    const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dO,
    const float* __restrict__ lse, float* __restrict__ dqacc, float* __restrict__ Dpad,
    float* __restrict__ Lpad, const int* __restrict__ cu_q, int B, int Hq, int total_q,
    long long ld, Strides so, Strides sdo, float* __restrict__ kvacc, long long kv_n4,
    const __nv_bfloat16* __restrict__ v, Strides sv, int Hkv, int total_k,
    unsigned* __restrict__ amax, const __nv_bfloat16* __restrict__ qin, Strides sq,
    const __nv_bfloat16* __restrict__ kin, Strides sk) {
  constexpr int TPR = D / 8;
  constexpr int RPB = 256 / TPR;
  const int sub = threadIdx.x % TPR;
  const int rlocal = threadIdx.x / TPR;
  auto start = [&](int bb) { return min(max(__ldg(cu_q + bb), 0), total_q); };
  // The loop bound is a multiple of RPB so that every warp runs its
  // shuffles with all lanes; rows past the end only do nothing.
  const long long total = (long long)Hq * total_q;
  const long long total_pad = (total + RPB - 1) / RPB * RPB;
  float mdo = 0.f;                                 // largest |dO| seen by this thread
  for (long long r = (long long)blockIdx.x * RPB + rlocal; r < total_pad;
       r += (long long)gridDim.x * RPB) {
    const bool valid = r < total;
    const int h = valid ? int(r / total_q) : 0;
    const int n = valid ? int(r - (long long)h * total_q) : 0;
    int lo = 0, hi = B - 1;                        // last sequence starting at or before n
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (start(mid) <= n) lo = mid; else hi = mid - 1;
    }
    const int off = start(lo);
    const int len = min(max(__ldg(cu_q + lo + 1), off), total_q) - off;
    const bool in_seq = valid && n >= off && n < off + len;
    float acc = 0.f;
    if (valid) {
      const uint4 ov = *reinterpret_cast<const uint4*>(o + h * so.h + (long long)n * so.n +
                                                       sub * 8);
      const uint4 dv = *reinterpret_cast<const uint4*>(dO + h * sdo.h + (long long)n * sdo.n +
                                                       sub * 8);
      const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&ov);
      const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&dv);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 a = __bfloat1622float2(o2[i]);
        const float2 b2 = __bfloat1622float2(d2[i]);
        acc = fmaf(a.x, b2.x, acc);
        acc = fmaf(a.y, b2.y, acc);
        mdo = fmaxf(mdo, fmaxf(fabsf(b2.x), fabsf(b2.y)));
      }
      float4* z = reinterpret_cast<float4*>(dqacc + ((size_t)h * total_q + n) * D + sub * 8);
      z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
      z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int s = TPR / 2; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
    if (sub == 0 && in_seq) {
      const long long pi = h * ld + varlen_pad_start(off, lo) + (n - off);
      Dpad[pi] = acc;
      Lpad[pi] = lse[(size_t)h * total_q + n] * 1.4426950408889634f;
    }
  }
  // padding entries of every (head, sequence)
  const long long npad = (long long)Hq * B * 128;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < npad;
       i += (long long)gridDim.x * blockDim.x) {
    const int e = int(i % 128);
    const int bb = int((i / 128) % B);
    const int h = int(i / (128LL * B));
    const int off = start(bb);
    const int len = min(max(__ldg(cu_q + bb + 1), off), total_q) - off;
    if (len + e < ((len + 127) & ~127)) {
      const long long pi = h * ld + varlen_pad_start(off, bb) + len + e;
      Dpad[pi] = 0.f;
      Lpad[pi] = INFINITY;
    }
  }
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < kv_n4;
       i += (long long)gridDim.x * blockDim.x)
    reinterpret_cast<float4*>(kvacc)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  if (amax) {                                      // the fp16 operand scales (bwd_f16)
    block_max_to(mdo, amax);
    absmax_scan<D>(v, sv, 1, Hkv, total_k, amax + 1);
    if (qin) {                                     // and Q, K (exact_dk)
      absmax_scan<D>(qin, sq, 1, Hq, total_q, amax + 2);
      absmax_scan<D>(kin, sk, 1, Hkv, total_k, amax + 3);
    }
  }
}

// dk, dv = bf16 of the fp32 partial-sum accumulators (dK already scaled).
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_kv_kernel(const float* __restrict__ kvacc,
                                                        __nv_bfloat16* __restrict__ dk,
                                                        __nv_bfloat16* __restrict__ dv,
                                                        long long n8, int Hkv, int Nk,
                                                        Strides sdk, Strides sdv) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < 2 * n8;
       i += (long long)gridDim.x * blockDim.x) {
    const long long j = i < n8 ? i : i - n8;       // 8-element chunk of [B*Hkv, Nk, D]
    const long long row = j / (D / 8), c8 = j - row * (D / 8);
    const long long bh = row / Nk, n = row - bh * Nk;
    const long long bb = bh / Hkv, hh = bh - bb * Hkv;
    const Strides& so = i < n8 ? sdk : sdv;
    const long long dst = bb * so.b + hh * so.h + n * so.n + c8 * 8;
    const float4 a = reinterpret_cast<const float4*>(kvacc)[2 * i];
    const float4 b = reinterpret_cast<const float4*>(kvacc)[2 * i + 1];
    uint4 out;
    out.x = pack_bf16(a.x, a.y);
    out.y = pack_bf16(a.z, a.w);
    out.z = pack_bf16(b.x, b.y);
    out.w = pack_bf16(b.z, b.w);
    *reinterpret_cast<uint4*>((i < n8 ? dk : dv) + dst) = out;
  }
}

// ------------------------------------------------------------------ dq convert
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_dq_kernel(const float* __restrict__ dqacc,
                                                        __nv_bfloat16* __restrict__ dq,
                                                        long long n8, float scale, int Hq, int Nq,
                                                        Strides sdq) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n8;
       i += (long long)gridDim.x * blockDim.x) {
    const long long row = i / (D / 8), c8 = i - row * (D / 8);
    const long long bh = row / Nq, n = row - bh * Nq;
    const long long bb = bh / Hq, hh = bh - bb * Hq;
    const float4 a = reinterpret_cast<const float4*>(dqacc)[2 * i];
    const float4 b = reinterpret_cast<const float4*>(dqacc)[2 * i + 1];
    uint4 out;
    out.x = pack_bf16(a.x * scale, a.y * scale);
    out.y = pack_bf16(a.z * scale, a.w * scale);
    out.z = pack_bf16(b.x * scale, b.y * scale);
    out.w = pack_bf16(b.z * scale, b.w * scale);
    *reinterpret_cast<uint4*>(dq + bb * sdq.b + hh * sdq.h + n * sdq.n + c8 * 8) = out;
  }
}

// ------------------------------------------------------------------ main
struct BwdParams {
  int B, Hq, Hkv, Nq, Nk, Nq_pad;
  int group;          // Hq / Hkv
  int n_kblocks;      // ceil(Nk / 128)
  int n_qblocks;      // ceil(Nq / BR)
  float scale;
  float scale_log2;
  const float* Dpad;
  const float* Lpad;
  float* dqacc;
  const unsigned* amax;  // workspace words: largest |dO|, |V| (their fp16 scales, f16_exp)
  int gsplit;         // CTAs sharing one kv group's query heads (1 = none)
  int hps;            // query heads per CTA: group / gsplit
  int hg;             // > 0: kv heads per group of the longest-first CTA order (bwd_cta)
  float* dkacc;       // fp32 dK / dV partial sums when gsplit > 1
  float* dvacc;
  DevStatus* status;
  const uint8_t* mask;  // block-sparse only: [ceil(Nq/128)][mask_ld] block mask
  int mask_ld;          // ceil(Nk / 128)
  // Variable-length batches only: B packed sequences (cu_q / cu_k offsets,
  // clamped to the totals on the device); Nq / Nk are the longest lengths.
  // The workspace's D / LSE rows of sequence b at head h start at
  // h * lpad_ld + varlen_pad_start(b); dK / dV rows that a TMA box would
  // overrun into the next sequence are stored directly through dk / dv.
  const int* cu_q;
  const int* cu_k;
  int total_q, total_k;
  long long lpad_ld;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  Strides sdk, sdv;
};

// CTA order of the dense causal d = 128 kernel.  By default (and in every
// other instance, which decode it inline) the group share varies
// fastest, then the key block, then the (batch, kv head): the CTAs running
// at once work on one or two heads, whose Q, dO and fp32 dQ rows stay in L2.
// Under the causal mask a key block's walk shrinks as the block moves right,
// so in that order the last head's longest CTAs start at the end of the grid
// and run on while the other SMs idle.  With hg > 0 the kv heads go in
// groups of hg (sized on the host so that a group's rows fit in L2) and,
// inside a group, key block by key block across the group's heads: the
// longest walks first, the shortest last.
__device__ __forceinline__ void bwd_cta(const BwdParams& p, int rest, int& gs, int& kb, int& bkv) {
  gs = rest % p.gsplit;
  rest /= p.gsplit;
  if (p.hg > 0) {
    const int per = p.hg * p.n_kblocks;              // CTAs of a full group
    const int grp = rest / per;
    const int r = rest - grp * per;
    const int hgt = min(p.hg, p.B * p.Hkv - grp * p.hg);   // the last group may be short
    kb = r / hgt;
    bkv = grp * p.hg + (r - kb * hgt);
  } else {
    kb = rest % p.n_kblocks;
    bkv = rest / p.n_kblocks;
  }
}

enum : int { BMODE_DENSE = 0, BMODE_SPARSE = 1, BMODE_VARLEN = 2 };


enum : unsigned { WB_KV = 16, WB_QEMPTY, WB_QFULL, WB_S, WB_DP, WB_P, WB_DS, WB_DQFULL,
                  WB_DQEMPTY, WB_FINAL, WB_DRAIN };

__device__ __forceinline__ void bulk_load_1d(void* dst, const void* src, uint32_t bytes,
                                             uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Scale factors of the fp16 operands (f16_exp), per launch.
//  F16 (bwd_f16): dP^T = 2^(e_dO + e_V) dP and dV_acc = 2^e_dO dV.
//  ALL16 (exact_dk): also S^T = 2^(e_Q + e_K) S from the fp16 copies of Q
//  and K, and dS goes in as fp16(dS * 2^e_dS), with 2^e_dS chosen from the
//  bound |dS| <= |dP - D| <= 2 max|dP| <= 2 d max|dO| max|V| (P <= 1, D a
//  P-weighted mean of the row's dP), so dK_acc = 2^(e_dS + e_Q) dK and the
//  dQ^T product gives 2^(e_dS + e_K) dQ.  Every factor is a power of two.
struct OpScales {
  float sl2;      // multiplies S^T (scale * log2 e, unscaled)
  float inv_vd;   // multiplies dP^T
  float s_ds;     // multiplies dS before fp16 rounding
  float mul_dk;   // multiplies the dK accumulator (includes the softmax scale)
  float mul_dv;   // multiplies the dV accumulator
  float mul_dq;   // multiplies dQ^T before its fp32 reduce-adds
};
template <int D, bool F16, bool ALL16>
__device__ __forceinline__ OpScales op_scales(const unsigned* amax, float scale, float scale_log2) {
  OpScales o{scale_log2, 1.f, 1.f, scale, 1.f, 1.f};
  if constexpr (F16) {
    const int e_do = f16_exp(__ldg(amax)), e_v = f16_exp(__ldg(amax + 1));
    o.inv_vd = ldexpf(1.f, -e_do - e_v);
    o.mul_dv = ldexpf(1.f, -e_do);
    if constexpr (ALL16) {
      const int e_q = f16_exp(__ldg(amax + 2)), e_k = f16_exp(__ldg(amax + 3));
      const float bound = 2.f * float(D) * __uint_as_float(__ldg(amax)) *
                          __uint_as_float(__ldg(amax + 1));
      const int e_ds = f16_exp(__float_as_uint(bound));
      o.sl2 = scale_log2 * ldexpf(1.f, -e_q - e_k);
      o.s_ds = ldexpf(1.f, e_ds);
      o.mul_dk = scale * ldexpf(1.f, -e_ds - e_q);
      o.mul_dq = ldexpf(1.f, -e_ds - e_k);
    }
  }
  return o;
}

// Block-sparse (SPARSE): a key block visits only the query blocks whose mask
// entry for it is set, in the same cyclic order for every role.
template <int D, bool CAUSAL, int MODE, bool ALL16, bool F16>
__global__ void __launch_bounds__(BwdCfg<D>::NTHREADS, 1)
    fa_bwd_main_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV,
                       const __grid_constant__ CUtensorMap tmdO,
                       const __grid_constant__ CUtensorMap tmdK,
                       const __grid_constant__ CUtensorMap tmdV, const BwdParams p) {
  using C = BwdCfg<D>;
  constexpr int BR = C::BR, BC = C::BC, DH = C::DH, QS = C::QS;
  constexpr bool SPARSE = MODE == BMODE_SPARSE, VARLEN = MODE == BMODE_VARLEN;
  static_assert(BC == MASK_BLOCK, "a CTA's key block is one block-mask column");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sK = smem;                                   // [KCH][BC][128B]
  uint8_t* sV = sK + C::K_BYTES;
  uint8_t* sStage = sV + C::K_BYTES;                    // QS x {Q | dO | L | D}
  uint8_t* sdS = sStage + QS * C::STAGE_STRIDE;         // [BC][128B] dS^T, 64 queries per row
  uint64_t* bars = reinterpret_cast<uint64_t*>(sdS + C::DS_BYTES);
  uint64_t* bar_kv = bars + 0;
  uint64_t* bar_qfull = bars + 1;                       // [QS]
  uint64_t* bar_qempty = bars + 1 + QS;                 // [QS]
  uint64_t* bar_s = bars + 1 + 2 * QS;                  // [2] per S^T buffer
  uint64_t* bar_dp = bars + 3 + 2 * QS;
  uint64_t* bar_p = bars + 4 + 2 * QS;
  uint64_t* bar_ds = bars + 5 + 2 * QS;
  uint64_t* bar_dqfull = bars + 6 + 2 * QS;
  uint64_t* bar_dqempty = bars + 7 + 2 * QS;
  uint64_t* bar_final = bars + 8 + 2 * QS;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 9 + 2 * QS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  int* sparse_ni = reinterpret_cast<int*>(tmem_holder + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Work unit: (batch, kv head, key block, d half), key block fastest after
  // the d half and the group share (the longest-first order of bwd_cta is
  // for d = 128 only).  With a large GQA/MQA group and few key blocks, the
  // group's query heads are split over `gsplit` CTAs that add fp32 partial
  // dK / dV.
  const int split = blockIdx.x % C::NSPLIT;
  int rest = blockIdx.x / C::NSPLIT;
  const int gs = rest % p.gsplit;
  rest /= p.gsplit;
  const int kb = rest % p.n_kblocks;
  const int bkv = rest / p.n_kblocks;
  const int b = bkv / p.Hkv;
  const int hkv = bkv - b * p.Hkv;
  const int key0 = kb * BC;
  // Sequence geometry: lengths, first packed rows and TMA "bh" coordinates
  // (variable-length batches address packed tensors with one batch entry).
  int nq = p.Nq, nk = p.Nk, qoff = 0, koff = 0;
  if constexpr (VARLEN) {
    varlen_rows(p.cu_q, b, p.total_q, qoff, nq);
    varlen_rows(p.cu_k, b, p.total_k, koff, nk);
    if (key0 >= nk) return;                             // past this sequence's keys
  }
  const int tkv = VARLEN ? hkv : bkv;
  const int n_qblocks = VARLEN ? (nq + BR - 1) / BR : p.n_qblocks;
  const int i0 = CAUSAL ? (key0 / BR) : 0;              // first query block that sees key0
  const int span = max(0, n_qblocks - i0);
  int n_i = span;                                       // query blocks visited per head
  const int dcol0 = split * DH;                         // first d column owned here
  const int head0 = hkv * p.group + gs * p.hps;         // first query head (within batch b)
  // Without the causal mask every key block visits every query block; key
  // blocks start at different query blocks so that their fp32 dQ reduce-adds
  // do not all land on the same rows at once.
  const int rot = CAUSAL ? 0 : int((long long)kb * span / p.n_kblocks);
  auto step_q = [&](int t, int& hh, int& qi) {
    hh = t / n_i;
    int li = t - hh * n_i + rot;
    if (li >= n_i) li -= n_i;
    qi = i0 + li;
  };
  // Block-sparse: query block i (BR rows) is visited iff its mask entry for
  // this key block is set; the visited blocks are taken cyclically from
  // i0 + rot, head after head.
  auto qvis = [&](int i) -> bool {
    return __ldg(p.mask + size_t(i * BR / MASK_BLOCK) * p.mask_ld + kb) != 0;
  };
  auto qnext = [&](int i) -> int {        // next visited block at or after i, cyclically
    for (int k = 0; k < span; ++k, ++i) {
      if (i >= n_qblocks) i = i0;
      if (qvis(i)) return i;
    }
    return i0;                            // not reached while n_i > 0
  };
  struct Seq { int hh, qi, c; };
  auto seq_begin = [&](Seq& q) { q.hh = 0; q.c = 0; q.qi = qnext(i0 + rot); };
  auto seq_next = [&](Seq& q) {
    if (++q.c == n_i) { q.c = 0; ++q.hh; q.qi = qnext(i0 + rot); }
    else q.qi = qnext(q.qi + 1);
  };

  if (threadIdx.x == 0) {
    mbar_init(bar_kv, 1);
    for (int i = 0; i < QS; ++i) {
      mbar_init(bar_qfull + i, 1);
      mbar_init(bar_qempty + i, 1);
    }
    mbar_init(bar_s + 0, 1);
    mbar_init(bar_s + 1, 1);
    mbar_init(bar_dp, 1);
    mbar_init(bar_p, 256);
    mbar_init(bar_ds, 256);
    mbar_init(bar_dqfull, 1);
    mbar_init(bar_dqempty, 128);
    mbar_init(bar_final, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_holder, C::TMEM_COLS);
    tmem_relinquish();
  }
  if constexpr (SPARSE) {
    if (warp == 10) {                     // count the visited query blocks once
      int c = 0;
      for (int i = i0 + lane; i < n_qblocks; i += 32) c += qvis(i) ? 1 : 0;
      c = __reduce_add_sync(0xffffffffu, c);
      if (lane == 0) *sparse_ni = c;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  if constexpr (SPARSE) n_i = *sparse_ni;
  const int n_steps = p.hps * n_i;

  if (warp >= 8 && warp < 12) {
    regs_dec<C::REGS_OTHER>();
  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && n_steps > 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmdO);
      mbar_arrive_expect_tx(bar_kv, 2 * C::K_BYTES);
      for (int c = 0; c < C::KCH; ++c) {
        tma_load_bh(sK + c * BC * 128, &tmK, bar_kv, c * 64, koff + key0, tkv, p.Hkv);
        tma_load_bh(sV + c * BC * 128, &tmV, bar_kv, c * 64, koff + key0, tkv, p.Hkv);
      }
      int issued = 0;
      Seq sq;
      if constexpr (SPARSE) seq_begin(sq);
      for (int t = 0; t < n_steps; ++t) {
        int hh, qi;
        if constexpr (SPARSE) {
          hh = sq.hh;
          qi = sq.qi;
          seq_next(sq);
        } else {
          step_q(t, hh, qi);
        }
        const int bh = b * p.Hq + head0 + hh;
        const int tq = VARLEN ? head0 + hh : bh;
        const int st = t % QS;
        if (!mbar_wait(bar_qempty + st, ((t / QS) & 1) ^ 1, abort_flag, p.status, WB_QEMPTY))
          break;
        uint8_t* sq = sStage + st * C::STAGE_STRIDE;
        uint8_t* sdo = sq + C::QT_BYTES;
        float* sl = reinterpret_cast<float*>(sdo + C::QT_BYTES);
        float* sd = sl + BR;
        mbar_arrive_expect_tx(bar_qfull + st, C::STAGE_BYTES);
        for (int c = 0; c < C::KCH; ++c) {
          tma_load_bh(sq + c * BR * 128, &tmQ, bar_qfull + st, c * 64, qoff + qi * BR, tq, p.Hq);
          tma_load_bh(sdo + c * BR * 128, &tmdO, bar_qfull + st, c * 64, qoff + qi * BR, tq,
                      p.Hq);
        }
        const size_t ro = VARLEN ? size_t((head0 + hh) * p.lpad_ld + varlen_pad_start(qoff, b) +
                                          qi * BR)
                                 : size_t(bh) * p.Nq_pad + size_t(qi) * BR;
        bulk_load_1d(sl, p.Lpad + ro, BR * 4, bar_qfull + st);
        bulk_load_1d(sd, p.Dpad + ro, BR * 4, bar_qfull + st);
        ++issued;
      }
      if (issued < n_steps) {
        for (int t = issued - 1; t >= 0 && t >= issued - QS; --t) {
          volatile int no_abort = 0;
          mbar_wait(bar_qfull + (t % QS), (t / QS) & 1, &no_abort, nullptr, WB_DRAIN);
        }
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && n_steps > 0) {
      constexpr uint32_t ID_S = ALL16 ? idesc_f16_f32(128, BR, 0, 0)   // S^T: K-major both
                                      : idesc_bf16_f32(128, BR, 0, 0);
      constexpr uint32_t ID_DP = F16 ? idesc_f16_f32(128, BR, 0, 0)   // dP^T: fp16 V, dO
                                        : idesc_bf16_f32(128, BR, 0, 0);
      constexpr uint32_t ID_KV = ALL16 ? idesc_f16_f32(128, DH, 0, 1)  // dK: B MN-major
                                       : idesc_bf16_f32(128, DH, 0, 1);
      constexpr uint32_t ID_V = F16 ? idesc_f16_f32(128, DH, 0, 1)    // dV: fp16 P, dO
                                       : idesc_bf16_f32(128, DH, 0, 1);
      constexpr uint32_t ID_DQ = ALL16 ? idesc_f16_f32(128, BR, 1, 1)  // dQ^T: A, B MN-major
                                       : idesc_bf16_f32(128, BR, 1, 1);
      // Descriptor low words: K-major (S^T, dP^T operands) and MN-major (the
      // B operands of dV, dK and both operands of dQ^T).
      const uint32_t kK = sdesc_sw128_lo(smem_u32(sK), 16);
      const uint32_t mK = sdesc_sw128_lo(smem_u32(sK), BC * 128);
      const uint32_t kV = sdesc_sw128_lo(smem_u32(sV), 16);
      const uint32_t kS0 = sdesc_sw128_lo(smem_u32(sStage), 16);
      const uint32_t mS0 = sdesc_sw128_lo(smem_u32(sStage), BR * 128);
      const uint32_t mdS = sdesc_sw128_lo(smem_u32(sdS), BC * 128);
      constexpr uint32_t STG = C::STAGE_STRIDE >> 4, QT = C::QT_BYTES >> 4;
      // A-operand column (within a P^T / dS^T buffer) of k-step kk: compute
      // group kk/2 wrote queries [32(kk/2), +32) packed into its own columns.
      auto pcol = [](int kk) { return uint32_t((kk >> 1) * 32 + (kk & 1) * 8); };
      auto mma_sdp = [&](uint32_t d_tm, uint32_t a_lo, uint32_t b_lo, uint32_t idesc) {
#pragma unroll (D == 256 ? 4 : D / 16)
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ko = ((kk >> 2) * BC * 128 + (kk & 3) * 32) >> 4;
          const uint32_t qo = ((kk >> 2) * BR * 128 + (kk & 3) * 32) >> 4;
          umma_ss_lo(d_tm, a_lo + ko, b_lo + qo, idesc, kk > 0);
        }
      };
      auto kst = [&](int t) { return kS0 + uint32_t(t % QS) * STG; };   // Q of step t, K-major
      auto mst = [&](int t) { return mS0 + uint32_t(t % QS) * STG; };   // Q of step t, MN-major
      // S^T of step t into buffer t mod 2
      auto mma_s = [&](int t) { mma_sdp(tmem + C::TM_S + (t & 1) * BR, kK, kst(t), ID_S); };
      // start of this CTA's share of d (DH columns, whole 64-column chunks) in
      // the MN-major operands
      const uint32_t dq_off = uint32_t((dcol0 / 64) * BR * 128) >> 4;
      const uint32_t dk_off = uint32_t((dcol0 / 64) * BC * 128) >> 4;
      bool ok = mbar_wait(bar_kv, 0, abort_flag, p.status, WB_KV) &&
                mbar_wait(bar_qfull + 0, 0, abort_flag, p.status, WB_QFULL);
      tc_fence_after();
      if (ok) {
        mma_s(0);
        umma_commit(bar_s + 0);
        mma_sdp(tmem + C::TM_DP, kV, kst(0) + QT, ID_DP);
        umma_commit(bar_dp);
      }
      for (int t = 0; t < n_steps && ok; ++t) {
        const int st = t % QS;
        const uint32_t mQ = mst(t) + dq_off, mdO = mQ + QT;
        const uint32_t tS = tmem + C::TM_S + (t & 1) * BR;
        // dV += P^T dO  (fp16 P and dO)
        if (!(ok = mbar_wait(bar_p, t & 1, abort_flag, p.status, WB_P))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BR / 16; ++kk)
          umma_ts_lo(tmem + C::TM_DV, tS + pcol(kk), mdO + kk * 128, ID_V,
                     (t > 0 || kk > 0) ? 1u : 0u);
        // S^T of the next step into the other buffer.  With one Q/dO stage
        // the next Q only arrives after this step's dK releases the stage,
        // so S^T_{t+1} then waits until after dQ_t (below).
        auto next_s = [&]() -> bool {
          if (t + 1 >= n_steps) return true;
          if (!mbar_wait(bar_qfull + (t + 1) % QS, ((t + 1) / QS) & 1, abort_flag, p.status,
                         WB_QFULL))
            return false;
          tc_fence_after();
          mma_s(t + 1);
          umma_commit(bar_s + ((t + 1) & 1));
          return true;
        };
        if (QS > 1 && !(ok = next_s())) break;
        // dK += dS^T Q
        if (!(ok = mbar_wait(bar_ds, t & 1, abort_flag, p.status, WB_DS))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BR / 16; ++kk)
          umma_ts_lo(tmem + C::TM_DK, tmem + C::TM_DP + pcol(kk), mQ + kk * 128, ID_KV,
                     (t > 0 || kk > 0) ? 1u : 0u);
        umma_commit(bar_qempty + st);
        // dQ^T = K^T dS^T  (M = 128 rows of d, N = BR queries, K = 128 keys).
        if (t > 0 && !(ok = mbar_wait(bar_dqempty, (t - 1) & 1, abort_flag, p.status, WB_DQEMPTY)))
          break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BC / 16; ++kk)
          umma_ss_lo(tmem + C::TM_DQ, mK + dk_off + kk * 128, mdS + kk * 128, ID_DQ, kk > 0);
        umma_commit(bar_dqfull);
        if (QS == 1 && !(ok = next_s())) break;
        // dP^T of the next step (overwrites dS^T_t, read by dK_t above)
        if (t + 1 < n_steps) {
          mma_sdp(tmem + C::TM_DP, kV, kst(t + 1) + QT, ID_DP);
          umma_commit(bar_dp);
        }
      }
      umma_commit(bar_final);
      volatile int no_abort = 0;
      mbar_wait(bar_final, 0, &no_abort, nullptr, WB_DRAIN);
    }
  }
    // warps 10 and 11 have no role
  } else if (warp >= 12) {
    regs_dec<C::REGS_READ>();
    // ------------------------------------------------------------ dQ read-out
    // Warp 12 + w reads TMEM lane quarter w of dQ^T (lanes = d rows, all 64
    // query columns of the step) and reduce-adds it into the fp32
    // accumulator, coalesced over d, while the compute warps form the next
    // step's P and dS.
    const int w = warp - 12;
    const int r = w * 32 + lane;                   // d row
    const uint32_t tl = tmem + (uint32_t(w * 32) << 16);
    // ALL16: dQ^T came from fp16 K and dS, scaled by 2^(e_dS + e_K)
    const float mul_dq = op_scales<D, F16, ALL16>(p.amax, p.scale, p.scale_log2).mul_dq;
    auto dqv = [&](uint32_t x) { return ALL16 ? __uint_as_float(x) * mul_dq : __uint_as_float(x); };
    Seq sq;
    if constexpr (SPARSE) seq_begin(sq);
    for (int u = 0; u < n_steps; ++u) {
      int hh, qi;
      if constexpr (SPARSE) {
        hh = sq.hh;
        qi = sq.qi;
        seq_next(sq);
      } else {
        step_q(u, hh, qi);
      }
      const bool okk = mbar_wait(bar_dqfull, u & 1, abort_flag, p.status, WB_DQFULL);
      if (!__all_sync(0xffffffffu, okk)) break;
      tc_fence_after();
      if (r < DH) {
        uint32_t v[64];
        FA_TMEM_LD32(tl + C::TM_DQ, v);
        FA_TMEM_LD32(tl + C::TM_DQ + 32, (v + 32));
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(bar_dqempty);
        const int q0 = qi * BR;
        const int bh = b * p.Hq + head0 + hh;
        float* dst = p.dqacc + (VARLEN ? (size_t(head0 + hh) * p.total_q + qoff + q0) * D
                                       : (size_t(bh) * p.Nq + q0) * D) + dcol0 + r;
        if (q0 + BR <= nq) {
#pragma unroll
          for (int i = 0; i < BR; ++i) atomicAdd(dst + i * D, dqv(v[i]));
        } else {
          const int nvalid = nq - q0;
#pragma unroll
          for (int i = 0; i < BR; ++i)
            if (i < nvalid) atomicAdd(dst + i * D, dqv(v[i]));
        }
      } else {
        tc_fence_before();
        mbar_arrive(bar_dqempty);
      }
    }
  } else {
    regs_inc<C::REGS_COMPUTE>();
    // ------------------------------------------------------------ compute warps
    const int g = warp >> 2;                       // compute group: query columns [32g, 32g+32)
    const int w = warp & 3;                        // TMEM lane quarter
    const int r = w * 32 + lane;                   // key row == TMEM lane (also d row for dQ^T)
    const uint32_t tl = tmem + (uint32_t(w * 32) << 16);
    const int key = key0 + r;
    // fp16 operands (F16, ALL16) come scaled by powers of two (op_scales)
    const OpScales os = op_scales<D, F16, ALL16>(p.amax, p.scale, p.scale_log2);
    const float sl2 = os.sl2;
    const float2 inv_vd2 = make_float2(os.inv_vd, os.inv_vd);
    const float2 s_ds2 = make_float2(os.s_ds, os.s_ds);
    bool ok = true;

    Seq sq;
    if constexpr (SPARSE) seq_begin(sq);
    for (int t = 0; t < n_steps && ok; ++t) {
      int hh, qi;
      if constexpr (SPARSE) {
        hh = sq.hh;
        qi = sq.qi;
        seq_next(sq);
      } else {
        step_q(t, hh, qi);
      }
      const int st = t % QS;
      const float* sl = reinterpret_cast<const float*>(sStage + st * C::STAGE_STRIDE +
                                                       2 * C::QT_BYTES) + g * 32;
      const float* sd = sl + BR;
      const int qg = qi * BR + g * 32;              // first query of this group's columns
      // Columns c < cstart are masked: causal (query < key) or padding key.
      const bool need_mask = (CAUSAL && key0 + BC - 1 > qg) || (key0 + BC > nk);
      const int cstart = key >= nk ? 32 : (CAUSAL ? key - qg : 0);
      const uint32_t tS = tl + C::TM_S + (t & 1) * BR + g * 32;
      const uint32_t tDP = tl + C::TM_DP + g * 32;

      ok = mbar_wait(bar_qfull + st, (t / QS) & 1, abort_flag, p.status, WB_QFULL) &&
           mbar_wait(bar_s + (t & 1), (t >> 1) & 1, abort_flag, p.status, WB_S);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      // ---- P^T for this key row and the group's 32 queries: fp16 P over
      // columns [0,16) of the group's S^T columns, the A operand of dV (fp16
      // rounding keeps dV within the bound over the query rows of a whole
      // GQA group, where bf16 would not).
      float P[32];
      {
        uint32_t u[32];
        FA_TMEM_LD32(tS, u);
        float lse2[32];
#pragma unroll
        for (int i = 0; i < 32; i += 4) *reinterpret_cast<float4*>(lse2 + i) =
            *reinterpret_cast<const float4*>(sl + i);
        tmem_wait_ld();
        const float2 sl22 = make_float2(sl2, sl2);
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const float2 x = ffma2(make_float2(__uint_as_float(u[i]), __uint_as_float(u[i + 1])),
                                 sl22, make_float2(-lse2[i], -lse2[i + 1]));
          P[i] = ex2(x.x);
          P[i + 1] = ex2(x.y);
        }
        if (need_mask) {
#pragma unroll
          for (int i = 0; i < 32; ++i) P[i] = (i < cstart) ? 0.f : P[i];
        }
        uint32_t ph[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          ph[i] = F16 ? pack_f16(P[2 * i], P[2 * i + 1]) : pack_bf16(P[2 * i], P[2 * i + 1]);
        FA_TMEM_ST16(tS, ph);
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(bar_p);

      // ---- dS^T = P^T o (dP^T - D)
      ok = mbar_wait(bar_dp, t & 1, abort_flag, p.status, WB_DP);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      {
        uint32_t u[32];
        FA_TMEM_LD32(tDP, u);
        float dd[32];
#pragma unroll
        for (int i = 0; i < 32; i += 4) *reinterpret_cast<float4*>(dd + i) =
            *reinterpret_cast<const float4*>(sd + i);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          // dP^T came from the scaled fp16 operands: dP = dP^T_scaled * 2^-(e_dO + e_V)
          const float2 dp2 = make_float2(__uint_as_float(u[2 * i]), __uint_as_float(u[2 * i + 1]));
          const float2 nd = make_float2(-dd[2 * i], -dd[2 * i + 1]);
          const float2 x = F16 ? ffma2(dp2, inv_vd2, nd) : fadd2(dp2, nd);
          const float2 y = fmul2(make_float2(P[2 * i], P[2 * i + 1]), x);
          if constexpr (ALL16) {                 // fp16(dS * 2^e_dS)
            const float2 z = fmul2(y, s_ds2);
            pk[i] = pack_f16(z.x, z.y);
          } else {
            pk[i] = pack_bf16(y.x, y.y);
          }
        }
        FA_TMEM_ST16(tDP, pk);
        // dS^T row r, queries 32g..32g+31: half of a 128-byte swizzled row
        uint8_t* row = sdS + r * 128;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const int unit = g * 4 + q4;
          *reinterpret_cast<uint4*>(row + ((unit ^ (r & 7)) * 16)) =
              make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
        }
        tmem_wait_st();
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar_ds);
    }

    // ---- epilogue: group 0 writes dK = scale * dK_acc, group 1 writes dV,
    // bf16 through the (now free) Q/dO stages, one 4 KiB box per warp and
    // 64 columns.
    if (ok && n_steps > 0) {
      ok = mbar_wait(bar_final, 0, abort_flag, p.status, WB_FINAL);
      ok = __all_sync(0xffffffffu, ok);
      if (ok) tc_fence_after();
    }
    if (ok && p.gsplit > 1) {
      // Partial sums of this CTA's query heads: fp32 reduce-adds, row by row
      // (all lanes load from TMEM together; rows past Nk add nothing).
      if (n_steps > 0) {
        const int tcol = g == 0 ? C::TM_DK : C::TM_DV;
        const float mul = g == 0 ? os.mul_dk : os.mul_dv;
        float* dst = (g == 0 ? p.dkacc : p.dvacc) +
                     (VARLEN ? size_t(hkv) * p.total_k + koff + key : size_t(bkv) * p.Nk + key) *
                         D + dcol0;
        const bool row_ok = key < nk;
#pragma unroll
        for (int c = 0; c < DH / 32; ++c) {
          uint32_t u[32];
          FA_TMEM_LD32(tl + tcol + c * 32, u);
          tmem_wait_ld();
          if (row_ok) {
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst + c * 32 + i),
                           "f"(__uint_as_float(u[i]) * mul), "f"(__uint_as_float(u[i + 1]) * mul),
                           "f"(__uint_as_float(u[i + 2]) * mul),
                           "f"(__uint_as_float(u[i + 3]) * mul)
                           : "memory");
          }
        }
      }
    } else if (ok) {
      const int tcol = g == 0 ? C::TM_DK : C::TM_DV;
      const float mul = g == 0 ? os.mul_dk : os.mul_dv;
      uint8_t* stage = sStage + g * (BC * DH * 2);
      // Packed batches: a warp whose 32 key rows run past the sequence's
      // end stores its rows directly (a TMA box would reach the next one).
      const bool direct = VARLEN && (key0 + w * 32 + 32 > nk);
#pragma unroll
      for (int c = 0; c < DH / 32; ++c) {
        uint32_t u[32];
        if (n_steps > 0) {
          FA_TMEM_LD32(tl + tcol + c * 32, u);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) u[i] = 0u;
        }
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack_bf16(__uint_as_float(u[2 * i]) * mul, __uint_as_float(u[2 * i + 1]) * mul);
        if (direct) {
          if (key < nk) {
            const Strides& so = g == 0 ? p.sdk : p.sdv;
            uint4* dst = reinterpret_cast<uint4*>((g == 0 ? p.dk : p.dv) + hkv * so.h +
                                                  (long long)(koff + key) * so.n + dcol0 + c * 32);
#pragma unroll
            for (int u4 = 0; u4 < 4; ++u4)
              dst[u4] = make_uint4(pk[4 * u4], pk[4 * u4 + 1], pk[4 * u4 + 2], pk[4 * u4 + 3]);
          }
          continue;
        }
        uint8_t* box = stage + ((c >> 1) * 4 + w) * 4096 + lane * 128;
#pragma unroll
        for (int u4 = 0; u4 < 4; ++u4) {
          const int unit = (c & 1) * 4 + u4;
          *reinterpret_cast<uint4*>(box + ((unit ^ (lane & 7)) * 16)) =
              make_uint4(pk[4 * u4], pk[4 * u4 + 1], pk[4 * u4 + 2], pk[4 * u4 + 3]);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0 && !direct && key0 + w * 32 < nk) {
        const CUtensorMap* tm = g == 0 ? &tmdK : &tmdV;
        for (int c = 0; c < DH / 64; ++c)
          tma_store_bh(tm, stage + (c * 4 + w) * 4096, dcol0 + c * 64, koff + key0 + w * 32, tkv,
                       p.Hkv);
        bulk_commit();
        bulk_wait0();
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace fa

#include "fa_bwd128.cuh"

namespace fa {

// ------------------------------------------------------------------ launch
bool make_map_bf16(CUtensorMap* m, const void* base, int d, int rows, int heads, int batch,
                   const Strides& st, int box_rows);

// A packed variable-length batch: B sequences with cumulative offsets
// cu_q / cu_k (device int32 [B + 1]) into [total_q, Hq, d] / [total_k, Hkv, d]
// tensors.  Nq / Nk passed alongside are the longest lengths.
struct Varlen {
  const int* cu_q;
  const int* cu_k;
  int total_q, total_k;
};

template <int D, bool CAUSAL>
int launch_bwd_t(int stages, const void* q, const void* k, const void* v, const void* o,
                 const void* ores, const float* lse, const void* dO, void* dq, void* dk, void* dv,
                 const Strides* st, int B, int Hq, int Hkv, int Nq, int Nk, float scale,
                 const uint8_t* mask, const Varlen* vl, void* workspace, DevStatus* status,
                 cudaStream_t stream) {
  using C = BwdCfg<D>;
  const BwdWorkspace w = vl ? bwd_workspace_layout_varlen(B, Hq, Hkv, vl->total_q, vl->total_k, D)
                            : bwd_workspace_layout(B, Hq, Hkv, Nq, Nk, D);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* dqacc = reinterpret_cast<float*>(ws + w.dq_off);
  float* Dpad = reinterpret_cast<float*>(ws + w.d_off);
  float* Lpad = reinterpret_cast<float*>(ws + w.l_off);
  float* kvacc = reinterpret_cast<float*>(ws + w.kv_off);
  __half* do16 = reinterpret_cast<__half*>(ws + w.do16_off);
  __half* v16 = reinterpret_cast<__half*>(ws + w.v16_off);
  __half* q16 = reinterpret_cast<__half*>(ws + w.q16_off);
  __half* k16 = reinterpret_cast<__half*>(ws + w.k16_off);
  unsigned* amax = reinterpret_cast<unsigned*>(ws + w.amax_off);
  const int Nq_pad = round_up(Nq, 128);
  const int bhq = B * Hq;
  const int group = Hq / Hkv;
  const int n_kblocks = (Nk + C::BC - 1) / C::BC;
  // Rows and batch entries the tensor maps and the convert kernels see:
  // packed batches are one batch entry of total_q / total_k rows.
  const int rows_q = vl ? vl->total_q : Nq, rows_k = vl ? vl->total_k : Nk;
  const int map_b = vl ? 1 : B;
  // Split a kv group's query heads over several CTAs when the key blocks
  // alone would leave SMs idle: the smallest divisor of the group that
  // gives at least two CTAs per SM (same choice in every stage call).
  int gsplit = 1;
  if (group > 1) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long base = (long long)n_kblocks * B * Hkv * C::NSPLIT;
    gsplit = group;
    for (int s = 1; s <= group; ++s)
      if (group % s == 0 && base * s >= 2LL * sms) { gsplit = s; break; }
  }

  CUtensorMap mq, mk, mv, mdo, mdk, mdv;
  // strides: q, k, v, o, dO, dq, dk, dv
  // d <= 128 runs the 128-query-step kernel (fa_bwd128.cuh); d = 256 the
  // general one with 64-query steps.
  constexpr bool STEP128 = D <= 128;
  constexpr int BRK = STEP128 ? 128 : C::BR;
  // V and dO reach the main kernel as the preprocess stage's contiguous
  // fp16 copies (TMA moves the 16-bit elements unchanged; the map's element
  // type only matters for a NaN out-of-bounds fill, which is not used).
  const bool f16 = bwd_f16(Hq, Hkv, D);
  // exact_dk: dS, and with it S^T, dK and dQ^T, take fp16 operands as well
  const bool all16 = exact_dk(group, D);
  const Strides s_v16{(long long)Hkv * rows_k * D, (long long)rows_k * D, D};
  const Strides s_do16{(long long)Hq * rows_q * D, (long long)rows_q * D, D};
  if ((stages & 2) &&
      (!make_map_bf16(&mq, all16 ? q16 : q, D, rows_q, Hq, map_b, all16 ? s_do16 : st[0], BRK) ||
       !make_map_bf16(&mk, all16 ? k16 : k, D, rows_k, Hkv, map_b, all16 ? s_v16 : st[1], C::BC) ||
      !make_map_bf16(&mv, f16 ? v16 : v, D, rows_k, Hkv, map_b, f16 ? s_v16 : st[2], C::BC) ||
      !make_map_bf16(&mdo, f16 ? do16 : dO, D, rows_q, Hq, map_b, f16 ? s_do16 : st[4], BRK) ||
      !make_map_bf16(&mdk, dk, D, rows_k, Hkv, map_b, st[6], 32) ||
      !make_map_bf16(&mdv, dv, D, rows_k, Hkv, map_b, st[7], 32)))
    return 5;
  const long long kv_n4 = gsplit > 1 ? (long long)(2 * w.kv_elems / 4) : 0LL;

  if (stages & 1) {
    constexpr int RPB = 256 / (D / 8);
    if (f16 && cudaMemsetAsync(amax, 0, 4 * sizeof(unsigned), stream) != cudaSuccess) return 5;
    if (vl) {
      const long long rows = (long long)Hq * vl->total_q;
      const long long blocks = std::max<long long>(
          1, std::min<long long>((rows + RPB - 1) / RPB, 148LL * 16));
      fa_bwd_pre_varlen_kernel<D><<<unsigned(blocks), 256, 0, stream>>>(
          static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dO), lse, dqacc,
          Dpad, Lpad, vl->cu_q, B, Hq, vl->total_q, varlen_lpad_ld(B, vl->total_q), st[3], st[4],
          kvacc, kv_n4, static_cast<const __nv_bfloat16*>(v), st[2], Hkv, vl->total_k,
          f16 ? amax : nullptr, all16 ? static_cast<const __nv_bfloat16*>(q) : nullptr, st[0],
          static_cast<const __nv_bfloat16*>(k), st[1]);
    } else {
      const long long rows = (long long)bhq * Nq_pad;
      const long long blocks = std::min<long long>((rows + RPB - 1) / RPB, 148LL * 16);
      fa_bwd_pre_kernel<D><<<unsigned(blocks), 256, 0, stream>>>(
          static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(ores),
          static_cast<const __nv_bfloat16*>(dO), lse, dqacc,
          Dpad, Lpad, bhq, Hq, Nq, Nq_pad, st[3], st[4], kvacc, kv_n4,
          static_cast<const __nv_bfloat16*>(v), st[2], B, Hkv, Nk, f16 ? amax : nullptr,
          all16 ? static_cast<const __nv_bfloat16*>(q) : nullptr, st[0],
          static_cast<const __nv_bfloat16*>(k), st[1]);
    }
    if (f16) {
      const long long pieces = ((long long)map_b * Hq * rows_q + (long long)map_b * Hkv * rows_k) *
                               (D / 8);
      const long long blocks = std::max<long long>(1, std::min<long long>((pieces + 255) / 256,
                                                                          148LL * 16));
      fa_bwd_f16_kernel<D><<<unsigned(blocks), 256, 0, stream>>>(
          static_cast<const __nv_bfloat16*>(dO), st[4], map_b, Hq, rows_q,
          static_cast<const __nv_bfloat16*>(v), st[2], map_b, Hkv, rows_k, do16, v16, amax,
          amax + 1);
      if (all16)
        fa_bwd_f16_kernel<D><<<unsigned(blocks), 256, 0, stream>>>(
            static_cast<const __nv_bfloat16*>(q), st[0], map_b, Hq, rows_q,
            static_cast<const __nv_bfloat16*>(k), st[1], map_b, Hkv, rows_k, q16, k16, amax + 2,
            amax + 3);
    }
    if (cudaGetLastError() != cudaSuccess) return 5;
  }
  if (stages & 2) {
    using C2 = typename std::conditional<STEP128, Bwd128Cfg<(D <= 128 ? D : 128)>, C>::type;
    // dK sums dS^T Q over every query row of the kv group: for wide groups
    // rounding dS to bf16 alone moves dK by about 2e-2 (causal, N = 4096),
    // so dS goes in as fp16 there (exact_dk: all16).
    // instances: (fp16 dP / dV, fp16 dS) = (no, no) for MHA at d <= 128,
    // (yes, exact_dk) otherwise; d = 256 is always fp16 (bwd_f16)
    auto pick = [&](auto split_tag, auto f16_tag) {
      constexpr bool S = decltype(split_tag)::value, F = decltype(f16_tag)::value;
      if constexpr (STEP128)
        return vl ? fa_bwd_main128_kernel<D, CAUSAL, BMODE_VARLEN, S, F>
               : mask ? fa_bwd_main128_kernel<D, CAUSAL, BMODE_SPARSE, S, F>
                      : fa_bwd_main128_kernel<D, CAUSAL, BMODE_DENSE, S, F>;
      else
        return static_cast<void>(F),   // d = 256 always takes fp16 operands
               vl ? fa_bwd_main_kernel<D, CAUSAL, BMODE_VARLEN, S, true>
               : mask ? fa_bwd_main_kernel<D, CAUSAL, BMODE_SPARSE, S, true>
                      : fa_bwd_main_kernel<D, CAUSAL, BMODE_DENSE, S, true>;
    };
    auto kern = !f16    ? pick(std::false_type{}, std::false_type{})
                : all16 ? pick(std::true_type{}, std::true_type{})
                        : pick(std::false_type{}, std::true_type{});
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C2::SMEM_BYTES) !=
        cudaSuccess)
      return 5;
    // The warpgroups' setmaxnreg split must fit in the registers the block
    // is launched with, or a setmaxnreg.inc would wait forever: refuse.
    cudaFuncAttributes fattr;
    if (cudaFuncGetAttributes(&fattr, kern) != cudaSuccess) return 5;
    if (fattr.numRegs * C2::NTHREADS < C2::REGS_NEEDED) return 2;
    BwdParams p;
    p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.Nq = Nq; p.Nk = Nk; p.Nq_pad = Nq_pad;
    p.group = group;
    p.n_kblocks = n_kblocks;
    p.amax = f16 ? amax : nullptr;
    p.gsplit = gsplit;
    p.hps = group / gsplit;
    // Longest-first CTA order for the dense causal backward at d = 128, in
    // groups of kv heads whose Q and dO (2 bytes an element each) and fp32
    // dQ rows (4 bytes) take at most 16 MiB of L2.  Measured against the
    // key-block-fastest order: causal N = 4096 +4 %, N = 2048 +4 % (16 MiB
    // beat 48 and 96); at d = 64 every budget was 1-2 % slower.
    p.hg = 0;
    if (CAUSAL && D == 128 && !vl && !mask) {
      const long long per_head = (long long)group * Nq_pad * D * 8;
      p.hg = int(std::max<long long>(1, std::min<long long>((16LL << 20) / per_head,
                                                            (long long)B * Hkv)));
    }
    p.dkacc = kvacc;
    p.dvacc = kvacc + w.kv_elems;
    p.n_qblocks = (Nq + BRK - 1) / BRK;
    p.scale = scale;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.Dpad = Dpad;
    p.Lpad = Lpad;
    p.dqacc = dqacc;
    p.status = status;
    p.mask = mask;
    p.mask_ld = (Nk + MASK_BLOCK - 1) / MASK_BLOCK;
    p.cu_q = vl ? vl->cu_q : nullptr;
    p.cu_k = vl ? vl->cu_k : nullptr;
    p.total_q = rows_q;
    p.total_k = rows_k;
    p.lpad_ld = vl ? varlen_lpad_ld(B, vl->total_q) : 0;
    p.dk = static_cast<__nv_bfloat16*>(dk);
    p.dv = static_cast<__nv_bfloat16*>(dv);
    p.sdk = st[6];
    p.sdv = st[7];
    const unsigned grid = unsigned(p.n_kblocks) * unsigned(B * Hkv) * C::NSPLIT * gsplit;
    kern<<<grid, C2::NTHREADS, C2::SMEM_BYTES, stream>>>(mq, mk, mv, mdo, mdk, mdv, p);
    if (cudaGetLastError() != cudaSuccess) return 5;
  }
  if (stages & 4) {
    const long long n8 = (long long)Hq * map_b * rows_q * D / 8;
    const long long blocks = std::max<long long>(1, std::min<long long>((n8 + 255) / 256,
                                                                        148LL * 16));
    fa_bwd_dq_kernel<D><<<unsigned(blocks), 256, 0, stream>>>(
        dqacc, static_cast<__nv_bfloat16*>(dq), n8, scale, Hq, rows_q, st[5]);
    if (cudaGetLastError() != cudaSuccess) return 5;
    if (gsplit > 1) {
      const long long kv8 = (long long)w.kv_elems / 8;
      const long long kblocks = std::min<long long>((2 * kv8 + 255) / 256, 148LL * 16);
      fa_bwd_kv_kernel<D><<<unsigned(kblocks), 256, 0, stream>>>(
          kvacc, static_cast<__nv_bfloat16*>(dk), static_cast<__nv_bfloat16*>(dv), kv8, Hkv,
          rows_k, st[6], st[7]);
      if (cudaGetLastError() != cudaSuccess) return 5;
    }
  }
  return 0;
}

// stages: bit 0 = preprocess, bit 1 = main, bit 2 = dq convert.  mask: the
// block mask of block-sparse attention, or null; vl: a packed
// variable-length batch, or null.
// ores: the forward's residual output (o's strides), or null.
inline int launch_bwd(int stages, const void* q, const void* k, const void* v, const void* o,
                      const void* ores, const float* lse, const void* dO, void* dq, void* dk,
                      void* dv, const Strides* st, int B, int Hq, int Hkv, int Nq, int Nk, int d,
                      int causal, float scale, const uint8_t* mask, const Varlen* vl,
                      void* workspace, DevStatus* status, cudaStream_t stream) {
#define FA_BWD_CASE(DD)                                                                          \
  if (d == DD)                                                                                   \
    return causal ? launch_bwd_t<DD, true>(stages, q, k, v, o, ores, lse, dO, dq, dk, dv, st, B, \
                                           Hq, Hkv, Nq, Nk, scale, mask, vl, workspace, status,  \
                                           stream)                                               \
                  : launch_bwd_t<DD, false>(stages, q, k, v, o, ores, lse, dO, dq, dk, dv, st,   \
                                            B, Hq, Hkv, Nq, Nk, scale, mask, vl, workspace,      \
                                            status, stream);
  FA_BWD_CASE(64)
  FA_BWD_CASE(128)
  FA_BWD_CASE(256)
#undef FA_BWD_CASE
  return 2;
}

}  // namespace fa
