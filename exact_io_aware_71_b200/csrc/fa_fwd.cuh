// Forward pass of exact tiled attention on sm_100a.
//
// The score matrix stays on chip: only O and the log-sum-exp reach HBM
// (QbitAI FA2 article, section "具体实现"; FA1 article, section
// "FlashAttention").  Per key block j the tensor cores compute S_j = Q K_j^T
// into TMEM and O += P_j V_j with P_j read straight from TMEM.  The online
// softmax keeps a running max and sum and defers the division by the sum to
// the end (FA2 article, section "具体实现", first improvement: fewer
// rescaling operations without changing the output); O is rescaled only when
// a row's max grows by more than 2^8, which is exact because O and the sums
// always carry the same (possibly stale) max.  Causal key blocks wholly above
// the diagonal are never loaded or computed (FA2 post, section "Алгоритм
// вычисления").  Forward rows are independent (FA2 post, section
// "Параллелизм"), so the grid runs over (batch, head, query tile).
//
// Thread t of a softmax warpgroup owns query row t of its tile (TMEM lane t):
// the row max and sums never leave the thread.
//
// Two kernels:
//  * fa_fwd_pair_kernel (d = 64, 128): a CTA owns two 128-row query tiles of
//    one head and streams K/V once for both.  Warps 0-3 and 4-7 are the two
//    tiles' softmax warpgroups; in the third warpgroup warp 8 is the TMA
//    producer, warp 9 the MMA issuer (10, 11 idle).  TMEM holds S and O of
//    each tile (2 x (128 + d) columns, + 16 at d = 64 where the P V product
//    also sums the rounded P); while one warpgroup exponentiates its
//    S, the tensor pipe works on the other tile, and two softmax warps share
//    each SM sub-partition.  The softmax warpgroups take 208 registers per
//    thread from the third warpgroup's share (setmaxnreg, 208 / 88).
//  * fa_fwd_kernel (d = 256): one 128-row tile per CTA with two S buffers
//    (O alone takes 256 TMEM columns), warps 0-3 softmax, 4 producer, 5 MMA.
#pragma once
#include "sm100.cuh"
#include "fa_mask.cuh"
#include "fa_rows.cuh"

// A row's O and sums are rescaled only when its running max (log2 units)
// grows by more than this; in between, probabilities reach at most 2^threshold.
#ifndef FA_RESCALE_LOG2_THRESHOLD
#define FA_RESCALE_LOG2_THRESHOLD 8.0f
#endif

namespace fa {

struct FwdParams {
  int B, Hq, Hkv, Nq, Nk;
  int group;          // Hq / Hkv
  int n_qblocks;      // ceil(Nq / 128)
  int n_units;        // query units per head: tiles (one-tile kernel) or tile pairs
  int causal;
  float scale_log2;   // scale * log2(e)
  float* lse;         // [B, Hq, Nq]
  DevStatus* status;
  // Block-sparse attention only (null / unused otherwise): the block mask
  // [ceil(Nq/128)][mask_ld] of 128 x 128 (query, key) blocks, shared by all
  // batches and heads, and the output tensor itself, for the rows of query
  // tiles that see no key (O = 0 there, written without the TMA epilogue).
  const uint8_t* mask;
  int mask_ld;        // ceil(Nk / 128)
  __nv_bfloat16* o;
  long long o_sb, o_sh, o_sn;
  // Variable-length batches only: B sequences packed back to back, q / o as
  // [total_q, Hq, d], k / v as [total_k, Hkv, d], lse as [Hq, total_q];
  // sequence b is rows cu_q[b] .. cu_q[b+1] (cu_k for keys).  Nq and Nk are
  // then the longest lengths, which size the grid.
  const int* cu_q;
  const int* cu_k;
  int total_q, total_k;
  // Optional residual output (null: none): o_res = bf16(O - bf16(O)) at o's
  // strides, the part of the fp32 output that rounding O to bf16 dropped.
  // The backward pass forms D = rowsum(dO o (o + o_res)) from it.
  __nv_bfloat16* o_res;
  // D epilogue (null: the normal output).  The kernel then writes neither O
  // nor the LSE: each row's epilogue dots its fp32 output with the row of
  // dO and stores D = sum_c dO_c O_c into the backward workspace's row
  // vector (fa_rows.cuh: entry bh * d_ld + row, or for packed batches
  // h * d_ld + varlen_pad_start(cu_q[b], b) + row).
  float* d_out;
  long long d_ld;
  const __nv_bfloat16* dO;
  long long do_sb, do_sh, do_sn;
  // D epilogue of the tile-pair kernel: V is the backward workspace's fp16
  // copy, scaled by 2^f16_exp(*v_amax) (the largest |V|), and P V is one
  // fp16 product.  Null elsewhere.
  const unsigned* v_amax = nullptr;
};

// Kernel variants: fixed-length batch, block-sparse, variable-length batch.
enum : int { MODE_DENSE = 0, MODE_SPARSE = 1, MODE_VARLEN = 2 };
// Epilogues: O and the LSE; the same plus the residual output; D only (the
// backward's exact D for wide groups).  A compile-time choice, so the plain
// output path carries none of the others' registers.
enum : int { EPI_O = 0, EPI_RES = 1, EPI_D = 2 };

// Where one (batch, head)'s rows live.  Fixed-length batches: rows [0, Nq)
// of the (b, h) slice of the 4-D tensor maps.  Variable-length batches: rows
// [qoff, qoff + nq) of the packed tensors, whose maps have a single batch
// entry; the offsets are clamped to the packed totals, so no access leaves
// the tensors whatever the offsets hold.
struct SeqGeo {
  int nq, nk;          // sequence lengths
  int qoff, koff;      // first packed row (0 for fixed-length batches)
  int tq, tkv;         // TMA "bh" coordinates of q / o and of k / v
  float* lse;          // LSE of the sequence's row 0 at this head
  __nv_bfloat16* o;    // O of row 0 at this head (direct row stores)
  __nv_bfloat16* ores; // residual output of row 0 (null: none)
  float* dpad;         // D epilogue: D of row 0 (null: normal output)
  const __nv_bfloat16* dO;   // D epilogue: dO of row 0
};

template <bool VARLEN, int EPI>
__device__ __forceinline__ SeqGeo seq_geo(const FwdParams& p, int bh) {
  const int b = bh / p.Hq, h = bh - b * p.Hq;
  SeqGeo g;
  if constexpr (VARLEN) {
    const int q0 = min(max(__ldg(p.cu_q + b), 0), p.total_q);
    const int q1 = min(max(__ldg(p.cu_q + b + 1), q0), p.total_q);
    const int k0 = min(max(__ldg(p.cu_k + b), 0), p.total_k);
    const int k1 = min(max(__ldg(p.cu_k + b + 1), k0), p.total_k);
    g.nq = q1 - q0;
    g.nk = k1 - k0;
    g.qoff = q0;
    g.koff = k0;
    g.tq = h;
    g.tkv = h / p.group;
    g.lse = p.lse + size_t(h) * p.total_q + q0;
    g.o = p.o + h * p.o_sh + (long long)q0 * p.o_sn;
    g.ores = EPI == EPI_RES ? p.o_res + h * p.o_sh + (long long)q0 * p.o_sn : nullptr;
    g.dpad = EPI == EPI_D ? p.d_out + h * p.d_ld + varlen_pad_start(q0, b) : nullptr;
    g.dO = EPI == EPI_D ? p.dO + h * p.do_sh + (long long)q0 * p.do_sn : nullptr;
  } else {
    g.nq = p.Nq;
    g.nk = p.Nk;
    g.qoff = g.koff = 0;
    g.tq = bh;
    g.tkv = b * p.Hkv + h / p.group;
    g.lse = p.lse + size_t(bh) * p.Nq;
    g.o = p.o + b * p.o_sb + h * p.o_sh;
    g.ores = EPI == EPI_RES ? p.o_res + b * p.o_sb + h * p.o_sh : nullptr;
    g.dpad = EPI == EPI_D ? p.d_out + size_t(bh) * p.d_ld : nullptr;
    g.dO = EPI == EPI_D ? p.dO + b * p.do_sb + h * p.do_sh : nullptr;
  }
  return g;
}

// A query row that sees no key at all (every block of its mask row is
// zero, or its sequence has no keys): O = 0 and LSE = -inf, the limits of
// an empty softmax.
// In the D epilogue nothing is written: the backward's preprocess already
// set D = rowsum(dO o 0) = 0 for such a row.
template <int D, int EPI>
__device__ __forceinline__ void write_empty_row(const FwdParams& p, const SeqGeo& g, int grow) {
  if (EPI == EPI_D || grow >= g.nq) return;
  uint4* dst = reinterpret_cast<uint4*>(g.o + (long long)grow * p.o_sn);
#pragma unroll
  for (int c = 0; c < D / 8; ++c) dst[c] = make_uint4(0u, 0u, 0u, 0u);
  if (EPI == EPI_RES) {
    uint4* dr = reinterpret_cast<uint4*>(g.ores + (long long)grow * p.o_sn);
#pragma unroll
    for (int c = 0; c < D / 8; ++c) dr[c] = make_uint4(0u, 0u, 0u, 0u);
  }
  g.lse[grow] = -INFINITY;
}

// Wait codes recorded on a timeout.
enum : unsigned { W_Q = 1, W_KV_EMPTY, W_KV_FULL, W_S_FULL, W_P_FULL, W_O_DONE, W_DRAIN };

// ------------------------------------------------------------------ softmax
// Running state of one query row, held by the thread that owns the row.
// l: fp32 sum of the probabilities (for the log-sum-exp); lr: the same
// probabilities after rounding to bf16, i.e. the weights that actually
// multiply V, so that O = sum(p~ v) / sum(p~) stays a convex combination
// even when one key dominates a row.  At d = 64 (plain output) the tensor
// core forms that sum instead, in O's TMEM column d (LR_TC).
struct RowState {
  float m, l, lr;
};

// One key block of the online softmax for this thread's row.
//   tS     TMEM address (this warp's lanes) of the block's BC fp32 scores;
//          P is written back over them as packed bf16 (BC/2 columns)
//   tO     the row's O accumulator (D fp32 columns)
//   j      key block index; key0 = j * BC
//   first  this is the first block the row sees (initialises the max)
//   gj     running block index of this TMEM tile across the CTA's work
//          (phases of the barriers); equals j when a CTA has one tile and
//          the blocks are not sparse
//   q_tile first query row of the tile, grow this thread's query row
//   o_done the two barriers that complete after P V of even / odd blocks
// The caller has waited for S; the function waits for P_{j-1} V_{j-1} only
// if it has to rescale O.  Returns false if that wait gave up.
// SPLIT_P (the residual and D epilogues): P also goes to TMEM as
// lo = bf16(P - hi) over the block's last BC/2 columns (all of S has been
// read by then), and the MMA issuer adds P_lo V, so the fp32 output that
// the backward's D is formed from carries no bf16 rounding of P.
// HALVES: once the first half of the block's keys has its P in TMEM, the
// thread arrives on p_half (the MMA issuer starts that half's P V); the
// caller arrives on the block's P-full barrier after the function returns.
// LR_TC: the tensor core forms the sum of the rounded P (the P V product has a
// column of ones beyond V's d columns, so O's TMEM column D holds it); the
// thread neither adds it up nor keeps it, but rescales that column with O.
template <int BC, int D, bool CAUSAL, bool SPLIT_P = false, bool HALVES = false,
          bool F16P = false, bool LR_TC = false>
__device__ __forceinline__ bool softmax_block(RowState& st, uint32_t tS, uint32_t tO, int j,
                                              bool first, int gj, int q_tile, int grow, int Nk,
                                              float sl2,
                                              uint64_t* o_done, volatile int* abort,
                                              DevStatus* status, uint64_t* p_half = nullptr) {
  float s[BC];
  {
    uint32_t* r = reinterpret_cast<uint32_t*>(s);
#pragma unroll
    for (int c = 0; c < BC / 32; ++c) FA_TMEM_LD32(tS + c * 32, (r + c * 32));
    tmem_wait_ld();
  }
  const int key0 = j * BC;
  if ((key0 + BC > Nk) || (CAUSAL && key0 + BC - 1 > q_tile)) {
    const int lim = CAUSAL ? min(Nk - key0, grow - key0 + 1) : (Nk - key0);
#pragma unroll
    for (int c = 0; c < BC; ++c)
      if (c >= lim) s[c] = -INFINITY;
  }
  // Row max as four independent three-input max chains.
  float mx;
  {
    float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
    for (int c = 0; c < BC; c += 8) {
#pragma unroll
      for (int q = 0; q < 4; ++q) m4[q] = fmax3(m4[q], s[c + 2 * q], s[c + 2 * q + 1]);
    }
    mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
  }
  const float mc = mx * sl2;
  if (first) {
    st.m = mc;
  } else {
    const bool need = mc > st.m + FA_RESCALE_LOG2_THRESHOLD;
    if (__any_sync(0xffffffffu, need)) {
      const float mn = need ? mc : st.m;
      const float alpha = ex2(st.m - mn);
      // O must hold every block up to j-1 before it is rescaled.  The
      // barriers alternate by block parity: warps of a warpgroup may be one
      // block apart, and one barrier would let a warp at block j+1 take
      // P_{j-1}V_{j-1}'s completion (same parity) for P_j V_j's.
      bool ok = mbar_wait(o_done + ((gj - 1) & 1), ((gj - 1) >> 1) & 1, abort, status, W_O_DONE);
      if (!__all_sync(0xffffffffu, ok)) return false;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        FA_TMEM_LD32(tO + c * 32, r);
        tmem_wait_ld();
        float2* r2 = reinterpret_cast<float2*>(r);
#pragma unroll
        for (int i = 0; i < 16; ++i) r2[i] = fmul2(r2[i], make_float2(alpha, alpha));
        FA_TMEM_ST32(tO + c * 32, r);
      }
      if constexpr (LR_TC) {
        uint32_t r;
        FA_TMEM_LD1(tO + D, r);
        tmem_wait_ld();
        r = __float_as_uint(__uint_as_float(r) * alpha);
        FA_TMEM_ST1(tO + D, r);
      }
      tmem_wait_st();
      st.l *= alpha;
      st.lr *= alpha;
      st.m = mn;
    }
  }
  const float neg = (st.m == -INFINITY) ? 0.f : -st.m;
  // p = 2^(s*scale*log2e - m): packed FMA, MUFU ex2, both sums in four packed
  // accumulator pairs; P is stored to TMEM 32 columns at a time.
  float2 al[4], ar[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) al[q] = ar[q] = make_float2(0.f, 0.f);
  const float2 sl22 = make_float2(sl2, sl2), neg2 = make_float2(neg, neg);
#pragma unroll
  for (int c = 0; c < BC / 32; ++c) {
    uint32_t pk[16], lo[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int e = c * 32 + 2 * i;
      const float2 t = ffma2(make_float2(s[e], s[e + 1]), sl22, neg2);
      const float2 pp = make_float2(ex2(t.x), ex2(t.y));
      al[i & 3] = fadd2(al[i & 3], pp);
      if constexpr (F16P) {                        // fp16 P (the D epilogue; normalised by l)
        pk[i] = pack_f16(pp.x, pp.y);
        continue;
      }
      const uint32_t pr = pack_bf16(pp.x, pp.y);
      if constexpr (LR_TC) {
        pk[i] = pr;
        continue;
      }
      ar[i & 3] = make_float2(add_bf16_lo(pr, ar[i & 3].x), add_bf16_hi(pr, ar[i & 3].y));
      pk[i] = pr;
      if constexpr (SPLIT_P)
        lo[i] = pack_bf16(pp.x - __uint_as_float(pr << 16), pp.y - __uint_as_float(pr & 0xFFFF0000u));
    }
    FA_TMEM_ST16(tS + c * 16, pk);
    if constexpr (SPLIT_P) FA_TMEM_ST16(tS + BC / 2 + c * 16, lo);
    if constexpr (HALVES) {
      if (c == BC / 64 - 1) {                      // keys [0, BC/2) are in TMEM
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(p_half);
      }
    }
  }
  const float2 la = fadd2(fadd2(al[0], al[1]), fadd2(al[2], al[3]));
  const float2 lb = fadd2(fadd2(ar[0], ar[1]), fadd2(ar[2], ar[3]));
  st.l += la.x + la.y;
  st.lr += lb.x + lb.y;
  tmem_wait_st();
  tc_fence_before();
  return true;
}

// After the tile's last P V: O / lr to bf16, staged in `stage` (the tile's
// free Q buffer) in the 128-byte swizzled layout, one 4 KiB box per warp and
// 64 columns, TMA-stored by lane 0 of each warp; then the log-sum-exp.  In
// a packed variable-length batch a warp whose 32 rows run past its
// sequence's end stores its rows directly instead (a TMA box would spill
// into the next sequence).  With a residual output the row's residual
// bf16(O - bf16(O)) is stored directly as well.  In the D epilogue
// (g.dpad set) the row's fp32 output is only dotted with its row of dO and
// D is written; O and the LSE are left alone.
template <int D, bool VARLEN, int EPI, bool LR_TC = false>
__device__ __forceinline__ void softmax_finish(const RowState& st, uint32_t tO, uint8_t* stage,
                                               int w, int lane, const CUtensorMap* tmO,
                                               int q_tile, const SeqGeo& g, long long o_sn,
                                               long long do_sn, int H, int grow,
                                               float o_mul = 1.f) {
  // The residual and D epilogues' P V used P as hi + lo (or as fp16): normalise
  // by the fp32 sum of P.  o_mul undoes the scale of an fp16 copy of V.
  float lr = st.lr;
  if constexpr (LR_TC) {
    uint32_t r;
    FA_TMEM_LD1(tO + D, r);
    tmem_wait_ld();
    lr = __uint_as_float(r);
  }
  const float inv = o_mul / (EPI != EPI_O ? st.l : lr);
  if constexpr (EPI == EPI_D) {
    const bool row_ok = grow < g.nq;
    const uint4* dor = reinterpret_cast<const uint4*>(g.dO + (long long)(row_ok ? grow : 0) * do_sn);
    float2 acc = make_float2(0.f, 0.f);
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t r[32];
      FA_TMEM_LD32(tO + c * 32, r);
      uint4 dv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) dv[u] = row_ok ? dor[c * 4 + u] : make_uint4(0u, 0u, 0u, 0u);
      tmem_wait_ld();
      const uint32_t* dw = reinterpret_cast<const uint32_t*>(dv);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float2 x = fmul2(make_float2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1])),
                               make_float2(inv, inv));
        acc = ffma2(x, make_float2(__uint_as_float(dw[i] << 16), __uint_as_float(dw[i] & 0xFFFF0000u)),
                    acc);
      }
    }
    if (row_ok) g.dpad[grow] = acc.x + acc.y;
    return;
  }
  const bool direct = VARLEN && (q_tile + w * 32 + 32 > g.nq);   // warp-uniform
#pragma unroll
  for (int c = 0; c < D / 32; ++c) {
    uint32_t r[32];
    FA_TMEM_LD32(tO + c * 32, r);
    tmem_wait_ld();
    uint32_t pk2[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
      pk2[i] = pack_bf16(__uint_as_float(r[2 * i]) * inv, __uint_as_float(r[2 * i + 1]) * inv);
    if constexpr (EPI == EPI_RES) {
      if (grow < g.nq) {
        uint32_t rs[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          rs[i] = pack_bf16(__uint_as_float(r[2 * i]) * inv - __uint_as_float(pk2[i] << 16),
                            __uint_as_float(r[2 * i + 1]) * inv -
                                __uint_as_float(pk2[i] & 0xFFFF0000u));
        uint4* dst = reinterpret_cast<uint4*>(g.ores + (long long)grow * o_sn + c * 32);
#pragma unroll
        for (int u = 0; u < 4; ++u)
          dst[u] = make_uint4(rs[4 * u], rs[4 * u + 1], rs[4 * u + 2], rs[4 * u + 3]);
      }
    }
    if (direct) {
      if (grow < g.nq) {
        uint4* dst = reinterpret_cast<uint4*>(g.o + (long long)grow * o_sn + c * 32);
#pragma unroll
        for (int u = 0; u < 4; ++u)
          dst[u] = make_uint4(pk2[4 * u], pk2[4 * u + 1], pk2[4 * u + 2], pk2[4 * u + 3]);
      }
      continue;
    }
    uint8_t* box = stage + ((c >> 1) * 4 + w) * 4096 + lane * 128;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int unit = (c & 1) * 4 + u;
      *reinterpret_cast<uint4*>(box + ((unit ^ (lane & 7)) * 16)) =
          make_uint4(pk2[4 * u], pk2[4 * u + 1], pk2[4 * u + 2], pk2[4 * u + 3]);
    }
  }
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0 && !direct && q_tile + w * 32 < g.nq) {
    for (int c = 0; c < D / 64; ++c)
      tma_store_bh(tmO, stage + (c * 4 + w) * 4096, c * 64, g.qoff + q_tile + w * 32, g.tq, H);
    bulk_commit();
    bulk_wait0();
  }
  if (grow < g.nq) g.lse[grow] = (st.m + __log2f(st.l)) * 0.69314718055994531f;
}

// ------------------------------------------------------------------ tile pairs (d = 64, 128)
template <int D>
struct FwdPairCfg {
  static constexpr int BR = 128;                    // query rows per tile (two tiles per CTA)
  static constexpr int BC = 128;                    // keys per block
  static constexpr int KCH = D / 64;                // 128-byte chunks along d
  static constexpr int Q_BYTES = BR * D * 2;        // one tile
  static constexpr int KV_BYTES = BC * D * 2;
  static constexpr int NS = (D == 64) ? 8 : 5;      // K/V ring slots
  // P handed to the MMA issuer in two halves of 64 keys (P V of the first
  // half runs while the second half is exponentiated): measured 1-2% faster
  // at d = 64 and 4-5% slower at d = 128, where the extra handshake costs
  // more than the overlap gains.
  static constexpr bool P_HALVES = D == 64;
  static constexpr int TM_TILE = 256;               // tile t: S at t*256, O at t*256 + 128
  static constexpr int TMEM_COLS = 512;
  static constexpr int NTHREADS = 384;
  static constexpr int REGS_SOFTMAX = 208;          // per thread, warpgroups 0 and 1
  static constexpr int REGS_OTHER = 88;             // per thread, warpgroup 2
  static constexpr int REGS_NEEDED = 256 * REGS_SOFTMAX + 128 * REGS_OTHER;
  // d = 64: a 128 x 64 bf16 chunk of ones after the K/V ring, the P V
  // product's extra B columns (its N = d + 16), so that O's column d sums
  // the rounded P on the tensor core.
  static constexpr bool LR_TC = D == 64;
  static constexpr int ONES_BYTES = LR_TC ? BC * 128 : 0;
  static constexpr int SMEM_BYTES = 2 * Q_BYTES + NS * KV_BYTES + ONES_BYTES + 1024 + 1024;
  static_assert(128 + D + (LR_TC ? 16 : 0) <= TM_TILE, "TMEM budget");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

enum : uint32_t { KV_T0 = 1, KV_T1 = 2, KV_LAST = 4, KV_EMPTY = 8, KV_ACT0 = 16, KV_ACT1 = 32 };

// The CTAs are persistent: grid = min(#units, #SMs) and CTA c takes units
// c, c + grid, ...  A unit is (batch, head, tile pair); the list is
// head-major so that concurrently running units share K/V in L2, and under
// the causal mask each head's longest pair comes first.  All roles walk the
// same list; barrier phases run on across units.  Between units of a tile,
// "Q free" (the epilogue's TMA store has read the staging buffer, the tile's
// Q buffer) gates the next Q load and "O free" (the epilogue has read O from
// TMEM) gates the next unit's first P V, while the tensor pipe already
// computes the next unit's first S.
//
// Block-sparse (SPARSE): a unit's K/V stream is the union of the key blocks
// its two tiles see; a tile takes part in the blocks its own mask row keeps,
// and a tile that sees none is written out as empty rows.
template <int D, bool CAUSAL, int MODE, int EPI>
__global__ void __launch_bounds__(FwdPairCfg<D>::NTHREADS, 1)
    fa_fwd_pair_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV,
                       const __grid_constant__ CUtensorMap tmO, const FwdParams p) {
  using C = FwdPairCfg<D>;
  constexpr int BR = C::BR, BC = C::BC, NS = C::NS;
  constexpr bool SPARSE = MODE == MODE_SPARSE, VARLEN = MODE == MODE_VARLEN;
  // The D epilogue reads V as the backward workspace's scaled fp16 copy and
  // multiplies it by P as fp16 (one product; p.v_amax gives the scale).
  constexpr bool PV16 = EPI == EPI_D;
  // The tensor core sums the rounded P (plain output with one bf16 P only).
  constexpr bool LR_TC = C::LR_TC && EPI == EPI_O;
  constexpr int NO = D + (LR_TC ? 16 : 0);       // P V product's N

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem;                          // 2 tiles of [KCH][BR][128B]; O staging later
  uint8_t* sKV = smem + 2 * C::Q_BYTES;        // NS slots of [KCH][BC][128B]
  uint8_t* sOnes = sKV + NS * C::KV_BYTES;     // [BC][128B] bf16 ones (d = 64)
  uint64_t* bars = reinterpret_cast<uint64_t*>(sOnes + C::ONES_BYTES);
  uint64_t* bar_q = bars + 0;                  // [2] Q tile loaded
  uint64_t* bar_kv_full = bars + 2;            // [NS]
  uint64_t* bar_kv_empty = bars + 2 + NS;      // [NS]
  uint64_t* bar_s_full = bars + 2 + 2 * NS;    // [2] per tile
  uint64_t* bar_p_full = bars + 4 + 2 * NS;    // [2] per tile
  uint64_t* bar_o_done = bars + 6 + 2 * NS;    // [2 tiles][2 parities]
  uint64_t* bar_q_free = bars + 10 + 2 * NS;   // [2] Q/staging buffer free (4 warps)
  uint64_t* bar_o_free = bars + 12 + 2 * NS;   // [2] O read out of TMEM (128 threads)
  uint64_t* bar_drain = bars + 14 + 2 * NS;
  uint64_t* bar_p_half = bars + 16 + 2 * NS;   // [2] per tile (P halves only): first 64 keys' P
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + (C::P_HALVES ? 18 : 16) + 2 * NS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  // Block-sparse: the producer tags each K ring item with the tiles that
  // take its block (KV_T0, KV_T1), the unit's last block (KV_LAST) and, on
  // a unit's first item, the tiles that take any block (KV_ACT0, KV_ACT1);
  // a unit that takes no block at all gets one KV_EMPTY item with no copy.
  uint8_t* kv_meta = reinterpret_cast<uint8_t*>(tmem_holder + 2);   // [NS]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int bhq = p.B * p.Hq;
  const int total_units = p.n_units * bhq;

  // Unit u -> (bh, q0) and the number of key blocks of each tile.
  // Non-causal units are equal: head-major order, so concurrent units share
  // K/V in L2.  Causal units shrink with the pair index: pair-major from the
  // longest pair down, and the k-th round of units is dealt to the CTAs in
  // alternating direction (CTA c gets slot c, then grid-1-c, ...), which
  // evens out the total work per CTA.
  auto unit = [&](int u, int& bh, int& q0, int* nt, SeqGeo& sg) {
    int pu;
    if (CAUSAL) {
      const int g = gridDim.x;
      const int round = u / g, c = u - round * g;
      // snake order; a partial last round keeps its order (a bijection)
      const int v = ((round & 1) && (round + 1) * g <= total_units) ? round * g + (g - 1 - c) : u;
      pu = p.n_units - 1 - v / bhq;
      bh = v - (p.n_units - 1 - pu) * bhq;
    } else {
      bh = u / p.n_units;
      pu = u - bh * p.n_units;
    }
    q0 = pu * 2 * BR;
    sg = seq_geo<VARLEN, EPI>(p, bh);
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int qt = q0 + t * BR;
      const int kv_end = CAUSAL ? min(sg.nk, qt + BR) : sg.nk;
      nt[t] = (qt < sg.nq) ? (kv_end + BC - 1) / BC : 0;   // tile 1 may lie past Nq
    }
  };
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_q + i, 1);
      mbar_init(bar_s_full + i, 1);
      mbar_init(bar_p_full + i, BR);
      if (C::P_HALVES) mbar_init(bar_p_half + i, BR);
      mbar_init(bar_q_free + i, 4);
      mbar_init(bar_o_free + i, BR);
    }
    for (int i = 0; i < NS; ++i) {
      mbar_init(bar_kv_full + i, 1);
      mbar_init(bar_kv_empty + i, 1);
    }
    for (int i = 0; i < 4; ++i) mbar_init(bar_o_done + i, 1);
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_holder, C::TMEM_COLS);
    tmem_relinquish();
  }
  if constexpr (C::ONES_BYTES > 0) {
    uint4* o4 = reinterpret_cast<uint4*>(sOnes);
    for (int i = threadIdx.x; i < C::ONES_BYTES / 16; i += C::NTHREADS)
      o4[i] = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
    fence_proxy_async_smem();                  // the tensor core reads it
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp >= 8) {
    regs_dec<C::REGS_OTHER>();
  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      int cnt = 0;                                 // K/V ring position
      int uses[2] = {0, 0};                        // units in which each tile was active
      bool ok = !p.status->stall_kv;   // test control: withhold K/V (see fa_debug_inject)
      for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x) {
        int bh, q0, nt[2];
        SeqGeo sg;
        unit(u, bh, q0, nt, sg);
        // Ring order = MMA consumption order: K0, V0, K1, V1, ... over the
        // unit's (union of) key blocks.  The first ring items of a unit go
        // out before its Q loads, which wait for the previous unit's
        // epilogue to release the Q/staging buffers.
        int cnt_t[2] = {nt[0], nt[1]}, nu = max(nt[0], nt[1]);
        PairWalk pw;
        uint32_t act = 0;
        if constexpr (SPARSE) {
          const uint8_t* row0 = p.mask + size_t(q0 / MASK_BLOCK) * p.mask_ld;
          pw.init(row0, p.mask_ld, nt[0], nt[1]);
          nu = pw.counts(cnt_t[0], cnt_t[1]);
          act = (cnt_t[0] ? KV_ACT0 : 0u) | (cnt_t[1] ? KV_ACT1 : 0u);
          if (nu == 0) {                             // one tagged item, no copy
            const int slot = cnt % NS;
            if (!(ok = mbar_wait(bar_kv_empty + slot, ((cnt / NS) & 1) ^ 1, abort_flag,
                                 p.status, W_KV_EMPTY)))
              break;
            kv_meta[slot] = uint8_t(KV_EMPTY);
            mbar_arrive(bar_kv_full + slot);
            ++cnt;
            continue;
          }
        }
        const int items = 2 * nu;
        int jc = -1;                               // key block of the latest K item
        auto ring = [&](int item) -> bool {
          uint32_t meta = 0;
          if constexpr (SPARSE) {
            if (!(item & 1)) {
              bool f0, f1;
              jc = pw.next(jc + 1, f0, f1);
              meta = (f0 ? KV_T0 : 0u) | (f1 ? KV_T1 : 0u) | (item + 2 == items ? KV_LAST : 0u) |
                     (item == 0 ? act : 0u);
            }
          } else {
            jc = item >> 1;
          }
          const int slot = cnt % NS;
          if (!mbar_wait(bar_kv_empty + slot, ((cnt / NS) & 1) ^ 1, abort_flag, p.status,
                         W_KV_EMPTY))
            return false;
          if (SPARSE && !(item & 1)) kv_meta[slot] = uint8_t(meta);
          mbar_arrive_expect_tx(bar_kv_full + slot, C::KV_BYTES);
          uint8_t* dst = sKV + slot * C::KV_BYTES;
          const CUtensorMap* tm = (item & 1) ? &tmV : &tmK;
          for (int c = 0; c < C::KCH; ++c)
            tma_load_bh(dst + c * BC * 128, tm, bar_kv_full + slot, c * 64, sg.koff + jc * BC,
                        sg.tkv, p.Hkv);
          ++cnt;
          return true;
        };
        const int early = min(items, NS);
        for (int it = 0; it < early && ok; ++it) ok = ring(it);
        for (int t = 0; t < 2 && ok; ++t) {
          if (cnt_t[t] == 0) continue;
          if (uses[t] > 0 &&
              !(ok = mbar_wait(bar_q_free + t, (uses[t] - 1) & 1, abort_flag, p.status, W_Q)))
            break;
          mbar_arrive_expect_tx(bar_q + t, C::Q_BYTES);
          for (int c = 0; c < C::KCH; ++c)
            tma_load_bh(sQ + t * C::Q_BYTES + c * BR * 128, &tmQ, bar_q + t, c * 64,
                        sg.qoff + q0 + t * BR, sg.tq, p.Hq);
          ++uses[t];
        }
        for (int it = early; it < items && ok; ++it) ok = ring(it);
      }
      if (!ok) {
        // Let the copies already issued land before the CTA exits.
        for (int i = cnt - 1; i >= 0 && i >= cnt - NS; --i) {
          volatile int no_abort = 0;
          mbar_wait(bar_kv_full + (i % NS), (i / NS) & 1, &no_abort, nullptr, W_DRAIN);
        }
        for (int t = 0; t < 2; ++t) {
          volatile int no_abort = 0;
          if (uses[t] > 0) mbar_wait(bar_q + t, (uses[t] - 1) & 1, &no_abort, nullptr, W_DRAIN);
        }
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_bf16_f32(BR, BC, 0, 0);
      constexpr uint32_t IDESC_O =
          PV16 ? idesc_f16_f32(BR, NO, 0, 1) : idesc_bf16_f32(BR, NO, 0, 1);
      const uint32_t sQ_addr = smem_u32(sQ);
      const uint32_t sKV_addr = smem_u32(sKV);
      int cnt = 0;                                 // K/V ring position
      int uses[2] = {0, 0};                        // units in which each tile was active
      int gb[2] = {0, 0};                          // running block count per tile
      bool ok = true;
      auto acquire = [&](int& slot) -> bool {
        slot = cnt % NS;
        if (!mbar_wait(bar_kv_full + slot, (cnt / NS) & 1, abort_flag, p.status, W_KV_FULL))
          return false;
        tc_fence_after();
        ++cnt;
        return true;
      };
      // Descriptor low words of the Q tiles and the first K/V slot (K-major;
      // V MN-major); a k-step adds its byte offset / 16.
      const uint32_t qlo = sdesc_sw128_lo(sQ_addr, 16);
      const uint32_t klo = sdesc_sw128_lo(sKV_addr, 16);
      const uint32_t vlo = sdesc_sw128_lo(sKV_addr, BC * 128);
      // V of ring slot `slot` as the P V product's B operand.  With LR_TC its
      // 64-column chunks step by the leading byte offset to the ones chunk,
      // which holds the product's columns d .. d + 15.
      const uint32_t ones_addr = smem_u32(sOnes);
      auto vdesc = [&](int slot) -> uint32_t {
        if constexpr (LR_TC) {
          const uint32_t a = sKV_addr + uint32_t(slot * C::KV_BYTES);
          return sdesc_sw128_lo(a, ones_addr - a);
        } else {
          return vlo + uint32_t(slot * (C::KV_BYTES >> 4));
        }
      };
      // At d = 128 the descriptors are built per k-step from the byte
      // address instead: measured about 2% faster there (and 3% slower at
      // d = 64) than adding offsets to precomputed low words.
      constexpr bool LEAN = D != 128;
      static_assert(LEAN || !LR_TC, "the ones chunk is addressed through the low-word descriptors");
      auto mma_s = [&](int t, int slot) {
        if constexpr (LEAN) {
          const uint32_t a0 = qlo + uint32_t(t * (C::Q_BYTES >> 4));
          const uint32_t b0 = klo + uint32_t(slot * (C::KV_BYTES >> 4));
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            umma_ss_lo(tmem + t * C::TM_TILE, a0 + (((kk >> 2) * BR * 128 + (kk & 3) * 32) >> 4),
                       b0 + (((kk >> 2) * BC * 128 + (kk & 3) * 32) >> 4), IDESC_S, kk > 0);
        } else {
          const uint32_t qbase = sQ_addr + t * C::Q_BYTES;
          const uint32_t kbase = sKV_addr + slot * C::KV_BYTES;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            umma_ss(tmem + t * C::TM_TILE,
                    sdesc_sw128(qbase + (kk >> 2) * BR * 128 + (kk & 3) * 32, 16, 1024),
                    sdesc_sw128(kbase + (kk >> 2) * BC * 128 + (kk & 3) * 32, 16, 1024), IDESC_S,
                    kk > 0);
        }
        umma_commit(bar_s_full + t);
      };
      // P_t V_j of the tile's block j (running index gj).  Its first block
      // in a unit overwrites O, so it waits until the tile's previous
      // epilogue has read O out of TMEM.
      auto mma_pv = [&](int t, int j, int gj, int slot) -> bool {
        if (j == 0 && uses[t] > 1 &&
            !mbar_wait(bar_o_free + t, (uses[t] - 2) & 1, abort_flag, p.status, W_O_DONE))
          return false;
        // the residual and D epilogues also add P_lo V (P_lo in the block's
        // last BC/2 columns)
        constexpr int NPH = (EPI != EPI_O && !PV16) ? 2 : 1;
        constexpr int NH = C::P_HALVES ? 2 : 1;         // P handed over in NH parts
        constexpr int KH = BC / 16 / NH;                // k-steps per part
        if constexpr (NPH == 1 && NH == 1) {
          if (!mbar_wait(bar_p_full + t, gj & 1, abort_flag, p.status, W_P_FULL)) return false;
          tc_fence_after();
          const uint32_t tt = tmem + t * C::TM_TILE;
          if constexpr (LEAN) {
            const uint32_t b0 = vdesc(slot);
#pragma unroll
            for (int kk = 0; kk < BC / 16; ++kk)
              umma_ts_lo(tt + 128, tt + kk * 8, b0 + kk * 128, IDESC_O,
                         (j > 0 || kk > 0) ? 1u : 0u);
          } else {
            const uint32_t vbase = sKV_addr + slot * C::KV_BYTES;
#pragma unroll
            for (int kk = 0; kk < BC / 16; ++kk)
              umma_ts(tt + 128, tt + kk * 8, sdesc_sw128(vbase + kk * 16 * 128, BC * 128, 1024),
                      IDESC_O, (j > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(bar_o_done + t * 2 + (gj & 1));
          return true;
        }
        const uint32_t tt = tmem + t * C::TM_TILE;
#pragma unroll
        for (int hf = 0; hf < NH; ++hf) {
          uint64_t* pb = (hf + 1 < NH) ? bar_p_half + t : bar_p_full + t;
          if (!mbar_wait(pb, gj & 1, abort_flag, p.status, W_P_FULL)) return false;
          tc_fence_after();
          if constexpr (LEAN) {
            const uint32_t b0 = vdesc(slot);
#pragma unroll
            for (int ph = 0; ph < NPH; ++ph)
#pragma unroll
              for (int kk = hf * KH; kk < (hf + 1) * KH; ++kk)
                umma_ts_lo(tt + 128, tt + ph * (BC / 2) + kk * 8, b0 + kk * 128, IDESC_O,
                           (j > 0 || kk > 0 || ph > 0) ? 1u : 0u);
          } else {
            const uint32_t vbase = sKV_addr + slot * C::KV_BYTES;
#pragma unroll
            for (int ph = 0; ph < NPH; ++ph)
#pragma unroll
              for (int kk = hf * KH; kk < (hf + 1) * KH; ++kk)
                umma_ts(tt + 128, tt + ph * (BC / 2) + kk * 8,
                        sdesc_sw128(vbase + kk * 16 * 128, BC * 128, 1024), IDESC_O,
                        (j > 0 || kk > 0 || ph > 0) ? 1u : 0u);
          }
        }
        umma_commit(bar_o_done + t * 2 + (gj & 1));
        return true;
      };
      for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x) {
        int bh, q0, nt[2];
        SeqGeo sg;
        unit(u, bh, q0, nt, sg);
        int sK = 0, sV = 0;
        if constexpr (!SPARSE) {
          const int nmax = max(nt[0], nt[1]);
          if (VARLEN && nmax == 0) continue;         // past its sequence, or no keys
          if (!(ok = acquire(sK))) break;
          for (int t = 0; t < 2 && ok; ++t) {
            if (nt[t] == 0) continue;
            if (!(ok = mbar_wait(bar_q + t, uses[t] & 1, abort_flag, p.status, W_Q))) break;
            tc_fence_after();
            ++uses[t];
            mma_s(t, sK);
          }
          if (!ok) break;
          umma_commit(bar_kv_empty + sK);
          // Per block j: P0 V_j, then S0_{j+1} (it overwrites P0_j in TMEM,
          // so it must follow P0_j V_j; tcgen05 MMAs run in issue order),
          // then the same for tile 1.  Each K/V slot is released after its
          // last reader.
          for (int j = 0; j < nmax && ok; ++j) {
            if (!(ok = acquire(sV))) break;
            if (j < nt[0] && !(ok = mma_pv(0, j, gb[0] + j, sV))) break;
            const bool next = j + 1 < nmax;
            if (next) {
              if (!(ok = acquire(sK))) break;
              if (j + 1 < nt[0]) mma_s(0, sK);
            }
            if (j < nt[1] && !(ok = mma_pv(1, j, gb[1] + j, sV))) break;
            umma_commit(bar_kv_empty + sV);
            if (next) {
              if (j + 1 < nt[1]) mma_s(1, sK);
              umma_commit(bar_kv_empty + sK);
            }
          }
          gb[0] += nt[0];
          gb[1] += nt[1];
        } else {
          // The same order over the union of the tiles' key blocks, read
          // from the K items' tags: a tile's S of its next block follows
          // its own last P V, and l[t] counts the blocks tile t has taken.
          if (!(ok = acquire(sK))) break;
          uint32_t m = kv_meta[sK];
          if (m & KV_EMPTY) {                        // the unit takes no block
            umma_commit(bar_kv_empty + sK);
            continue;
          }
          for (int t = 0; t < 2 && ok; ++t) {
            if (!(m & (KV_ACT0 << t))) continue;
            if (!(ok = mbar_wait(bar_q + t, uses[t] & 1, abort_flag, p.status, W_Q))) break;
            tc_fence_after();
            ++uses[t];
            if (m & (KV_T0 << t)) mma_s(t, sK);
          }
          if (!ok) break;
          umma_commit(bar_kv_empty + sK);
          int l[2] = {0, 0};
          for (;;) {
            const bool last = m & KV_LAST;
            uint32_t mn = 0;
            if (!(ok = acquire(sV))) break;
            if (m & KV_T0) {
              if (!(ok = mma_pv(0, l[0], gb[0] + l[0], sV))) break;
              ++l[0];
            }
            if (!last) {
              if (!(ok = acquire(sK))) break;
              mn = kv_meta[sK];
              if (mn & KV_T0) mma_s(0, sK);
            }
            if (m & KV_T1) {
              if (!(ok = mma_pv(1, l[1], gb[1] + l[1], sV))) break;
              ++l[1];
            }
            umma_commit(bar_kv_empty + sV);
            if (last) break;
            if (mn & KV_T1) mma_s(1, sK);
            umma_commit(bar_kv_empty + sK);
            m = mn;
          }
          gb[0] += l[0];
          gb[1] += l[1];
        }
      }
      umma_commit(bar_drain);
      volatile int no_abort = 0;
      mbar_wait(bar_drain, 0, &no_abort, nullptr, W_DRAIN);
    }
  }
    // warps 10 and 11 have no role
  } else {
    regs_inc<C::REGS_SOFTMAX>();
    // ------------------------------------------------------------ softmax (tile = warp / 4)
    const int t = warp >> 2;                        // 0 or 1 (warps 0..7)
    const int w = warp & 3;                         // TMEM lane quarter
    const int row = w * 32 + lane;
    const uint32_t tl = tmem + t * C::TM_TILE + (uint32_t(w * 32) << 16);
    uint64_t* o_done = bar_o_done + t * 2;
    float o_mul = 1.f;                              // undoes the fp16 copy's scale of V
    if constexpr (PV16) o_mul = ldexpf(1.f, -f16_exp(__ldg(p.v_amax)));
    int gb = 0;                                     // running block count of this tile
    bool ok = true;
    for (int u = blockIdx.x; u < total_units && ok; u += gridDim.x) {
      int bh, q0, nt[2];
      SeqGeo sg;
      unit(u, bh, q0, nt, sg);
      if (nt[t] == 0) {
        // tile past its sequence's end, or (packed batches) a sequence with
        // queries but no keys
        if (VARLEN && q0 + t * BR < sg.nq) write_empty_row<D, EPI>(p, sg, q0 + t * BR + row);
        continue;
      }
      int n = nt[t];
      bool last_kept = true;
      if constexpr (SPARSE) {
        const uint8_t* row = p.mask + size_t(q0 / MASK_BLOCK + t) * p.mask_ld;
        n = mask_count(row, nt[t]);
        last_kept = __ldg(row + nt[t] - 1) != 0;
      }
      const int q_tile = q0 + t * BR;
      const int grow = q_tile + row;
      if constexpr (SPARSE) {
        if (n == 0) {                               // sees no key
          write_empty_row<D, EPI>(p, sg, grow);
          continue;
        }
      }
      RowState st{-INFINITY, 0.f, 0.f};
      if constexpr (!SPARSE) {
        for (int j = 0; j < n && ok; ++j) {
          ok = mbar_wait(bar_s_full + t, (gb + j) & 1, abort_flag, p.status, W_S_FULL);
          if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
          tc_fence_after();
          ok = softmax_block<BC, D, CAUSAL, EPI != EPI_O && !PV16, C::P_HALVES, PV16, LR_TC>(
              st, tl, tl + 128, j, j == 0, gb + j, q_tile, grow, sg.nk, p.scale_log2, o_done,
              abort_flag, p.status, bar_p_half + t);
          if (!ok) break;
          mbar_arrive(bar_p_full + t);
        }
      } else {
        // l: blocks taken so far (barrier phases).  Of the tile's blocks
        // in range only the last one (nt - 1) can need the causal or
        // key-length mask; every other kept block is passed as block 0,
        // which needs neither when the tile has more than one block in
        // range.
        for (int l = 0; l < n && ok; ++l) {
          const int j = (l == n - 1 && last_kept) ? nt[t] - 1 : 0;
          ok = mbar_wait(bar_s_full + t, (gb + l) & 1, abort_flag, p.status, W_S_FULL);
          if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
          tc_fence_after();
          ok = softmax_block<BC, D, CAUSAL, EPI != EPI_O && !PV16, C::P_HALVES, PV16, LR_TC>(
              st, tl, tl + 128, j, l == 0, gb + l, q_tile, grow, sg.nk, p.scale_log2, o_done,
              abort_flag, p.status, bar_p_half + t);
          if (!ok) break;
          mbar_arrive(bar_p_full + t);
        }
      }
      if (!ok) break;
      const int jl = gb + n - 1;
      ok = mbar_wait(o_done + (jl & 1), (jl >> 1) & 1, abort_flag, p.status, W_O_DONE);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      softmax_finish<D, VARLEN, EPI, LR_TC>(st, tl + 128, sQ + t * C::Q_BYTES, w, lane, &tmO,
                                            q_tile, sg, p.o_sn, p.do_sn, p.Hq, grow, o_mul);
      tc_fence_before();
      mbar_arrive(bar_o_free + t);                  // O has been read out of TMEM
      if (lane == 0) mbar_arrive(bar_q_free + t);   // this warp's staging boxes were read
      gb += n;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ one tile (d = 256)
template <int D>
struct FwdCfg {
  static constexpr int BR = 128;                       // query rows per tile
  static constexpr int BC = (D == 256) ? 64 : 128;     // keys per block
  static constexpr int KCH = D / 64;                   // 128-byte chunks along d
  static constexpr int Q_BYTES = BR * D * 2;
  static constexpr int KV_BYTES = BC * D * 2;
  static constexpr int NS = (D == 64) ? 8 : (D == 128 ? 5 : 4);  // ring slots
  static constexpr int TM_S = 0;                       // S buffer b at TM_S + b*BC
  static constexpr int TM_O = 2 * BC;                  // O accumulator (D columns)
  static constexpr int TMEM_COLS = 512;
  static constexpr int NTHREADS = 192;
  static constexpr int SMEM_BYTES = Q_BYTES + NS * KV_BYTES + 1024 /*barriers*/ + 1024 /*align*/;
  static_assert(TM_O + D <= TMEM_COLS, "TMEM budget");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

// Block-sparse (SPARSE): the tile walks only the key blocks its mask row
// keeps (two 64-key blocks per mask block); the MMA issuer sees just the
// sequence, the producer and softmax map it back to key blocks.
template <int D, bool CAUSAL, int MODE, int EPI>
__global__ void __launch_bounds__(FwdCfg<D>::NTHREADS, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                  const FwdParams p) {
  using C = FwdCfg<D>;
  constexpr int BR = C::BR, BC = C::BC, NS = C::NS;
  constexpr bool SPARSE = MODE == MODE_SPARSE, VARLEN = MODE == MODE_VARLEN;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem;                       // [KCH][BR][128B], swizzled; reused for O staging
  uint8_t* sKV = smem + C::Q_BYTES;         // NS slots of [KCH][BC][128B]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sKV + NS * C::KV_BYTES);
  uint64_t* bar_q = bars + 0;
  uint64_t* bar_kv_full = bars + 1;
  uint64_t* bar_kv_empty = bars + 1 + NS;
  uint64_t* bar_s_full = bars + 1 + 2 * NS;      // [2]
  uint64_t* bar_p_full = bars + 3 + 2 * NS;      // [2]
  uint64_t* bar_o_done = bars + 5 + 2 * NS;      // [2] by block parity
  uint64_t* bar_drain = bars + 7 + 2 * NS;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 8 + 2 * NS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int bh = blockIdx.x / p.n_units;
  int qb = blockIdx.x - bh * p.n_units;
  if (CAUSAL) qb = p.n_units - 1 - qb;
  const SeqGeo sg = seq_geo<VARLEN, EPI>(p, bh);
  const int q_row0 = qb * BR;
  // A tile past its (packed) sequence's end has nothing to do.
  if (VARLEN && q_row0 >= sg.nq) return;
  const int kv_end = CAUSAL ? min(sg.nk, q_row0 + BR) : sg.nk;
  const int n_kv = (kv_end + BC - 1) / BC;             // key blocks in range
  constexpr int SUB = MASK_BLOCK / BC;                 // key blocks per mask block
  // Block-sparse: walks over the kept key blocks (one mask entry covers SUB
  // of them); next_vis(rm, j) is the first kept block >= j, n_kv if none.
  auto mask_row = [&](RowWalk& rm) {
    rm.init(p.mask + size_t(qb) * p.mask_ld, (n_kv + SUB - 1) / SUB);
  };
  auto next_vis = [&](RowWalk& rm, int j) -> int {
    if constexpr (!SPARSE) return min(j, n_kv);
    if (j >= n_kv) return n_kv;
    const int c = rm.next(j / SUB);
    return c == MASK_NONE ? n_kv : max(j, c * SUB);
  };
  int n_blocks = n_kv;                                 // blocks the tile takes
  if constexpr (SPARSE) {
    RowWalk rm;
    mask_row(rm);
    n_blocks = 0;
    for (int j = next_vis(rm, 0); j < n_kv; j = next_vis(rm, j + 1)) ++n_blocks;
  }

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int i = 0; i < NS; ++i) {
      mbar_init(bar_kv_full + i, 1);
      mbar_init(bar_kv_empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_s_full + i, 1);
      mbar_init(bar_p_full + i, BR);
      mbar_init(bar_o_done + i, 1);
    }
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_holder, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && n_blocks > 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      mbar_arrive_expect_tx(bar_q, C::Q_BYTES);
      for (int c = 0; c < C::KCH; ++c)
        tma_load_bh(sQ + c * BR * 128, &tmQ, bar_q, c * 64, sg.qoff + q_row0, sg.tq, p.Hq);
      int cnt = 0;
      bool ok = !p.status->stall_kv;   // test control: withhold K/V (see fa_debug_inject)
      auto load = [&](const CUtensorMap* tm, int j) {
        const int slot = cnt % NS;
        const uint32_t ph = (cnt / NS) & 1;
        if (!mbar_wait(bar_kv_empty + slot, ph ^ 1, abort_flag, p.status, W_KV_EMPTY)) {
          ok = false;
          return;
        }
        mbar_arrive_expect_tx(bar_kv_full + slot, C::KV_BYTES);
        uint8_t* dst = sKV + slot * C::KV_BYTES;
        for (int c = 0; c < C::KCH; ++c)
          tma_load_bh(dst + c * BC * 128, tm, bar_kv_full + slot, c * 64, sg.koff + j * BC,
                      sg.tkv, p.Hkv);
        ++cnt;
      };
      // Ring order = MMA consumption order: K0, K1, V0, K2, V1, ... over the
      // blocks the tile takes (jk: block of the latest K, jv: of the next V).
      RowWalk rk, rv;
      if constexpr (SPARSE) {
        mask_row(rk);
        mask_row(rv);
      }
      int jk = next_vis(rk, 0), jv = jk;
      if (ok) load(&tmK, jk);
      for (int i = 1; i < n_blocks && ok; ++i) {
        jk = next_vis(rk, jk + 1);
        load(&tmK, jk);
        if (ok) load(&tmV, jv);
        jv = next_vis(rv, jv + 1);
      }
      if (ok) load(&tmV, jv);
      if (!ok) {
        // Let the copies already issued land before the CTA exits.
        for (int i = cnt - 1; i >= 0 && i >= cnt - NS; --i) {
          volatile int no_abort = 0;
          mbar_wait(bar_kv_full + (i % NS), (i / NS) & 1, &no_abort, nullptr, W_DRAIN);
        }
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && n_blocks > 0) {
      constexpr uint32_t IDESC_S = idesc_bf16_f32(BR, BC, 0, 0);
      constexpr uint32_t IDESC_O = idesc_bf16_f32(BR, D, 0, 1);
      const uint32_t sQ_addr = smem_u32(sQ);
      const uint32_t sKV_addr = smem_u32(sKV);
      bool ok = mbar_wait(bar_q, 0, abort_flag, p.status, W_Q);
      tc_fence_after();
      int cnt = 0;
      auto acquire = [&](int& slot) -> bool {
        slot = cnt % NS;
        if (!mbar_wait(bar_kv_full + slot, (cnt / NS) & 1, abort_flag, p.status, W_KV_FULL))
          return false;
        tc_fence_after();
        return true;
      };
      auto release = [&](int slot) {
        umma_commit(bar_kv_empty + slot);
        ++cnt;
      };
      const uint32_t qlo = sdesc_sw128_lo(sQ_addr, 16);
      const uint32_t klo = sdesc_sw128_lo(sKV_addr, 16);
      const uint32_t vlo = sdesc_sw128_lo(sKV_addr, BC * 128);
      auto mma_s = [&](int j) {
        int slot;
        if (!acquire(slot)) { ok = false; return; }
        const uint32_t d_tm = tmem + C::TM_S + (j & 1) * BC;
        const uint32_t b0 = klo + uint32_t(slot * (C::KV_BYTES >> 4));
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_ss_lo(d_tm, qlo + (((kk >> 2) * BR * 128 + (kk & 3) * 32) >> 4),
                     b0 + (((kk >> 2) * BC * 128 + (kk & 3) * 32) >> 4), IDESC_S, kk > 0);
        umma_commit(bar_s_full + (j & 1));
        release(slot);
      };
      auto mma_pv = [&](int j) {
        if (!mbar_wait(bar_p_full + (j & 1), (j >> 1) & 1, abort_flag, p.status, W_P_FULL)) {
          ok = false;
          return;
        }
        tc_fence_after();
        int slot;
        if (!acquire(slot)) { ok = false; return; }
        const uint32_t a_tm = tmem + C::TM_S + (j & 1) * BC;   // P_j (bf16 pairs)
        const uint32_t b0 = vlo + uint32_t(slot * (C::KV_BYTES >> 4));
        constexpr int NPH = EPI != EPI_O ? 2 : 1;   // residual / D epilogues add P_lo V
#pragma unroll
        for (int ph = 0; ph < NPH; ++ph)
#pragma unroll
          for (int kk = 0; kk < BC / 16; ++kk)
            umma_ts_lo(tmem + C::TM_O, a_tm + ph * (BC / 2) + kk * 8, b0 + kk * 128, IDESC_O,
                       (j > 0 || kk > 0 || ph > 0) ? 1u : 0u);
        umma_commit(bar_o_done + (j & 1));
        release(slot);
      };
      // S_{j+1} is issued before P_j V_j so that softmax on block j+1 can
      // start as soon as P_j is handed over (two S buffers).
      if (ok) mma_s(0);
      for (int j = 1; j < n_blocks && ok; ++j) {
        mma_s(j);
        if (ok) mma_pv(j - 1);
      }
      if (ok) mma_pv(n_blocks - 1);
      // All MMAs must finish before TMEM is released.
      umma_commit(bar_drain);
      volatile int no_abort = 0;
      mbar_wait(bar_drain, 0, &no_abort, nullptr, W_DRAIN);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int row = threadIdx.x;                       // 0..127 == TMEM lane
    const uint32_t tl = tmem + (uint32_t(warp * 32) << 16);
    const int grow = q_row0 + row;
    RowState st{-INFINITY, 0.f, 0.f};
    bool ok = true;
    if (n_blocks == 0) {                                 // sees no key (sparse)
      write_empty_row<D, EPI>(p, sg, grow);
      ok = false;
    }
    RowWalk rm;
    if constexpr (SPARSE) mask_row(rm);
    for (int j = 0, jb = next_vis(rm, 0); j < n_blocks && ok; ++j, jb = next_vis(rm, jb + 1)) {
      ok = mbar_wait(bar_s_full + (j & 1), (j >> 1) & 1, abort_flag, p.status, W_S_FULL);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      ok = softmax_block<BC, D, CAUSAL, EPI != EPI_O>(st, tl + C::TM_S + (j & 1) * BC,
                                                     tl + C::TM_O, jb, j == 0, j, q_row0, grow,
                                                     sg.nk, p.scale_log2, bar_o_done,
                                                     abort_flag, p.status);
      if (!ok) break;
      mbar_arrive(bar_p_full + (j & 1));
    }
    if (ok) {
      const int jl = n_blocks - 1;
      ok = mbar_wait(bar_o_done + (jl & 1), (jl >> 1) & 1, abort_flag, p.status, W_O_DONE);
      if (__all_sync(0xffffffffu, ok)) {
        tc_fence_after();
        softmax_finish<D, VARLEN, EPI>(st, tl + C::TM_O, sQ, warp, lane, &tmO, q_row0, sg, p.o_sn,
                                  p.do_sn, p.Hq, grow);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace fa
