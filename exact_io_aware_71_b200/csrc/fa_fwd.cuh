// Forward pass of exact tiled attention on sm_100a.
//
// One CTA computes one tile: 128 query rows of one (batch, query head).
// Warp roles (192 threads):
//   warps 0-3  softmax: thread t owns query row t of the tile, reads its row of
//              S from TMEM, keeps the running max m and running sum l, writes
//              P (bf16) back into TMEM, rescales O lazily, and finally writes
//              O / l and the log-sum-exp;
//   warp 4     TMA producer: Q once, then K_j / V_j through an NS-slot ring;
//   warp 5     MMA issuer (one thread) and TMEM owner.
// Per key block j the tensor cores compute S_j = Q K_j^T into one of two TMEM
// S buffers and O += P_j V_j with P_j read straight from TMEM, so softmax on
// block j overlaps S_{j+1} and P_{j-1} V_{j-1}.  The score matrix stays on
// chip; only O and the log-sum-exp reach HBM (QbitAI FA2 article, section
// "具体实现"; FA1 article, section "FlashAttention").  The online softmax
// keeps a running max and sum and defers the division by l to the end
// (FA2 article, section "具体实现", first improvement: fewer rescaling
// operations without changing the output); O is rescaled only when a row's
// max grows by more than 2^8, which is exact because O and l always carry the
// same (possibly stale) max.  Causal key blocks wholly above the diagonal
// are never loaded or computed (FA2 post, section "Алгоритм вычисления").
#pragma once
#include "sm100.cuh"

// A row's O and l are rescaled only when its running max (log2 units) grows
// by more than this; in between, probabilities reach at most 2^threshold.
#ifndef FA_RESCALE_LOG2_THRESHOLD
#define FA_RESCALE_LOG2_THRESHOLD 8.0f
#endif

namespace fa {

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

struct FwdParams {
  int B, Hq, Hkv, Nq, Nk;
  int group;          // Hq / Hkv
  int n_qblocks;      // ceil(Nq / 128)
  int causal;
  float scale_log2;   // scale * log2(e)
  float* lse;         // [B, Hq, Nq]
  DevStatus* status;
};

// Wait codes recorded on a timeout.
enum : unsigned { W_Q = 1, W_KV_EMPTY, W_KV_FULL, W_S_FULL, W_P_FULL, W_O_DONE, W_DRAIN };

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(FwdCfg<D>::NTHREADS, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                  const FwdParams p) {
  using C = FwdCfg<D>;
  constexpr int BR = C::BR, BC = C::BC, NS = C::NS;

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
  // O-done barriers alternate by key-block parity: softmax warps may drift one
  // block apart, and with a single barrier a warp already at block j+1 could
  // mistake the completion of P_{j-1} V_{j-1} (same parity) for P_j V_j.
  uint64_t* bar_o_done = bars + 5 + 2 * NS;      // [2]
  uint64_t* bar_drain = bars + 7 + 2 * NS;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 8 + 2 * NS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Tile coordinates: consecutive CTAs share a (batch, head) so that its K/V
  // stay hot in L2; within a head causal tiles run longest first.
  const int bh = blockIdx.x / p.n_qblocks;
  int qb = blockIdx.x - bh * p.n_qblocks;
  if (CAUSAL) qb = p.n_qblocks - 1 - qb;
  const int b = bh / p.Hq;
  const int h = bh - b * p.Hq;
  const int bkv = b * p.Hkv + h / p.group;
  const int q_row0 = qb * BR;
  const int kv_end = CAUSAL ? min(p.Nk, q_row0 + BR) : p.Nk;
  const int n_blocks = (kv_end + BC - 1) / BC;

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int i = 0; i < NS; ++i) {
      mbar_init(bar_kv_full + i, 1);
      mbar_init(bar_kv_empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_s_full + i, 1);
      mbar_init(bar_p_full + i, BR);
    }
    mbar_init(bar_o_done + 0, 1);
    mbar_init(bar_o_done + 1, 1);
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
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      mbar_arrive_expect_tx(bar_q, C::Q_BYTES);
      for (int c = 0; c < C::KCH; ++c)
        tma_load_3d(sQ + c * BR * 128, &tmQ, bar_q, c * 64, q_row0, bh);
      int cnt = 0;
      bool ok = true;
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
          tma_load_3d(dst + c * BC * 128, tm, bar_kv_full + slot, c * 64, j * BC, bkv);
        ++cnt;
      };
      load(&tmK, 0);
      for (int j = 1; j < n_blocks && ok; ++j) {
        load(&tmK, j);
        if (ok) load(&tmV, j - 1);
      }
      if (ok) load(&tmV, n_blocks - 1);
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
    if (lane == 0) {
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
      auto mma_s = [&](int j) {
        int slot;
        if (!acquire(slot)) { ok = false; return; }
        const uint32_t d_tm = tmem + C::TM_S + (j & 1) * BC;
        const uint32_t kbase = sKV_addr + slot * C::KV_BYTES;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t a = sdesc_sw128(sQ_addr + (kk >> 2) * BR * 128 + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = sdesc_sw128(kbase + (kk >> 2) * BC * 128 + (kk & 3) * 32, 16, 1024);
          umma_ss(d_tm, a, bd, IDESC_S, kk > 0);
        }
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
        const uint32_t vbase = sKV_addr + slot * C::KV_BYTES;
#pragma unroll
        for (int kk = 0; kk < BC / 16; ++kk) {
          const uint64_t bd = sdesc_sw128(vbase + kk * 16 * 128, BC * 128, 1024);
          umma_ts(tmem + C::TM_O, a_tm + kk * 8, bd, IDESC_O, (j > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(bar_o_done + (j & 1));
        release(slot);
      };
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
    const float sl2 = p.scale_log2;
    // l: fp32 sum of the probabilities (for the log-sum-exp); lr: sum of the
    // same probabilities after rounding to bf16, i.e. of the weights that
    // actually multiply V, so that O = sum(p~ v) / sum(p~) is a convex
    // combination even when one key dominates a row.
    float m = -INFINITY, l = 0.f, lr = 0.f;
    bool ok = true;
    for (int j = 0; j < n_blocks; ++j) {
      ok = mbar_wait(bar_s_full + (j & 1), (j >> 1) & 1, abort_flag, p.status, W_S_FULL);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      float s[BC];
      {
        uint32_t* r = reinterpret_cast<uint32_t*>(s);
#pragma unroll
        for (int c = 0; c < BC / 32; ++c) FA_TMEM_LD32(tl + C::TM_S + (j & 1) * BC + c * 32, (r + c * 32));
        tmem_wait_ld();
      }
      const int key0 = j * BC;
      const bool need_mask = (key0 + BC > p.Nk) || (CAUSAL && key0 + BC - 1 > q_row0);
      if (need_mask) {
        const int lim = CAUSAL ? min(p.Nk - key0, grow - key0 + 1) : (p.Nk - key0);
#pragma unroll
        for (int c = 0; c < BC; ++c)
          if (c >= lim) s[c] = -INFINITY;
      }
      float mx = s[0];
#pragma unroll
      for (int c = 1; c < BC; ++c) mx = fmaxf(mx, s[c]);
      const float mc = mx * sl2;
      if (j == 0) {
        m = mc;
      } else {
        const bool need = mc > m + FA_RESCALE_LOG2_THRESHOLD;
        if (__any_sync(0xffffffffu, need)) {
          const float mn = need ? mc : m;
          const float alpha = ex2(m - mn);
          ok = mbar_wait(bar_o_done + ((j - 1) & 1), ((j - 1) >> 1) & 1, abort_flag, p.status,
                         W_O_DONE);
          if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t r[32];
            FA_TMEM_LD32(tl + C::TM_O + c * 32, r);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
            FA_TMEM_ST32(tl + C::TM_O + c * 32, r);
          }
          tmem_wait_st();
          l *= alpha;
          lr *= alpha;
          m = mn;
        }
      }
      const float neg = (m == -INFINITY) ? 0.f : -m;
      uint32_t pk[BC / 2];
      float ls = 0.f, lrs = 0.f;
#pragma unroll
      for (int c = 0; c < BC; c += 2) {
        const float p0 = ex2(fmaf(s[c], sl2, neg));
        const float p1 = ex2(fmaf(s[c + 1], sl2, neg));
        ls += p0 + p1;
        const uint32_t pr = pack_bf16(p0, p1);
        lrs += __uint_as_float(pr << 16) + __uint_as_float(pr & 0xFFFF0000u);
        pk[c / 2] = pr;
      }
      l += ls;
      lr += lrs;
#pragma unroll
      for (int c = 0; c < BC / 64; ++c) FA_TMEM_ST32(tl + C::TM_S + (j & 1) * BC + c * 32, (pk + c * 32));
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar_p_full + (j & 1));
    }
    if (ok)
      ok = mbar_wait(bar_o_done + ((n_blocks - 1) & 1), ((n_blocks - 1) >> 1) & 1, abort_flag,
                     p.status, W_O_DONE);
    if (__all_sync(0xffffffffu, ok)) {
      tc_fence_after();
      const float inv = 1.0f / lr;
      // Stage this warp's 32 rows of O (bf16) in the Q buffer in the 128-byte
      // swizzled layout the TMA store expects, one 4 KiB box per 64 columns.
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        FA_TMEM_LD32(tl + C::TM_O + c * 32, r);
        tmem_wait_ld();
        uint32_t pk2[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk2[i] = pack_bf16(__uint_as_float(r[2 * i]) * inv, __uint_as_float(r[2 * i + 1]) * inv);
        uint8_t* box = sQ + ((c >> 1) * 4 + warp) * 4096 + lane * 128;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int unit = (c & 1) * 4 + u;
          *reinterpret_cast<uint4*>(box + ((unit ^ (lane & 7)) * 16)) =
              make_uint4(pk2[4 * u], pk2[4 * u + 1], pk2[4 * u + 2], pk2[4 * u + 3]);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0 && q_row0 + warp * 32 < p.Nq) {
        for (int c = 0; c < C::KCH; ++c)
          tma_store_3d(&tmO, sQ + (c * 4 + warp) * 4096, c * 64, q_row0 + warp * 32, bh);
        bulk_commit();
        bulk_wait0();
      }
      if (grow < p.Nq) p.lse[size_t(bh) * p.Nq + grow] = (m + __log2f(l)) * 0.69314718055994531f;
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
