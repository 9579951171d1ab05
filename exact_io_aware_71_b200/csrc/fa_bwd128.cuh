// Backward main kernel with 128-query steps (d = 64, 128).
//
// Same computation as fa_bwd_main_kernel (one CTA per 128-key block of a kv
// group; see fa_bwd.cuh), organised so that every tensor-core instruction
// has N = 128: an M = 128, N = 64 tcgen05.mma costs as many cycles as an
// N = 128 one, so the 64-query steps of the general kernel leave half of
// the tensor pipe unused on S^T, dP^T and dQ^T.
//
// At d = 128, TMEM (512 columns) cannot hold S^T, dP^T, dQ^T, dK and dV of
// a 128-query step side by side, so regions are reused within a step:
//   SP  [0, 128)    S^T (fp32)  -> P^T as 16-bit pairs (per group)
//   DP  [128, 256)  dP^T (fp32) -> dS^T as 16-bit pairs -> dQ^T (fp32)
//   DK  [256, 256 + d), DV [256 + d, 256 + 2d)
// At d = 64, dQ^T has its own columns [384, 512).
// MMA order per step t (one issuing thread; tcgen05 MMAs run in issue
// order, so a later MMA never overwrites a region an earlier one reads):
//   S_0, dP_0, then per step: [P_t] dV_t, S_{t+1}, [dS_t] dK_t, dQ_t,
//   [dQ_t read out] dP_{t+1}
// (d = 64: [dQ_{t-1} read out] dQ_t, then dP_{t+1} without a wait).
// The compute warps form P_t while dP_t runs and dS_t while dV_t and
// S_{t+1} run; the read-out warpgroup empties dQ^T_t from TMEM right away
// (then reduce-adds it into the fp32 accumulator from registers), which
// frees DP for dP_{t+1}.  Waiting for dP_t also proves that dQ_{t-1}, which
// reads the shared dS^T tile, has finished before dS_t overwrites it.
//
// P goes to TMEM rounded once for dV (bf16; fp16 with the F16 operands of
// GQA / MQA groups) and stays in the thread's registers in fp32 for dS,
// because S^T_{t+1} overwrites the P^T columns while dS_t is being formed.
// With ALL16 (wide groups) every product takes fp16 operands and dS goes
// in as fp16 (op_scales, fa_bwd.cuh).  The LSE
// and D rows are read straight from the workspace (L1-resident broadcast
// loads) rather than staged, which keeps shared memory within 227 KB.
#pragma once

namespace fa {

template <int D>
struct Bwd128Cfg {
  static_assert(D == 64 || D == 128, "128-query steps are for d = 64, 128");
  static constexpr int BC = 128;                        // keys per CTA (TMEM lanes)
  static constexpr int BR = 128;                        // query rows per step
  static constexpr int DH = D;
  static constexpr int KCH = D / 64;
  static constexpr int QS = (D == 64) ? 3 : 2;          // Q/dO pipeline stages
  static constexpr int K_BYTES = BC * D * 2;
  static constexpr int QT_BYTES = BR * D * 2;           // one Q or dO tile
  static constexpr int STAGE_BYTES = 2 * QT_BYTES;      // Q | dO
  static constexpr int DS_BYTES = BC * BR * 2;          // dS^T: [2][128 keys][64 queries] bf16
  static constexpr int TM_SP = 0;
  static constexpr int TM_DP = 128;
  static constexpr int TM_DK = 256;
  static constexpr int TM_DV = 256 + DH;
  // dQ^T: its own columns when d = 64 leaves them free, else the DP region.
  static constexpr bool DQ_OWN = (D == 64);
  static constexpr int TM_DQ = DQ_OWN ? TM_DV + DH : TM_DP;
  static constexpr int TMEM_COLS = 512;
  static constexpr int NTHREADS = 512;
  static constexpr int REGS_COMPUTE = 144;              // warpgroups 0-1
  static constexpr int REGS_OTHER = 80;                 // warpgroup 2 (producer, MMA)
  static constexpr int REGS_READ = 144;                 // warpgroup 3 (dQ read-out)
  static constexpr int REGS_NEEDED = 256 * REGS_COMPUTE + 128 * REGS_OTHER + 128 * REGS_READ;
  static constexpr int REGS_LAUNCH = 65536 / NTHREADS;  // per thread at launch (1 CTA per SM)
  static constexpr int SMEM_BYTES = 2 * K_BYTES + QS * STAGE_BYTES + DS_BYTES + 1024 + 1024;
  static_assert(REGS_NEEDED <= 65536, "register split");
  static_assert(TM_DV + DH <= TMEM_COLS, "TMEM budget");
  static_assert(!DQ_OWN || TM_DQ + BR <= TMEM_COLS, "TMEM budget (dQ^T)");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
  static_assert(QS * STAGE_BYTES >= 2 * BC * DH * 2, "dK/dV staging fits in the Q/dO stages");
};

template <int D, bool CAUSAL, int MODE, bool ALL16, bool F16>
__global__ void __launch_bounds__(Bwd128Cfg<D>::NTHREADS, 1)
    fa_bwd_main128_kernel(const __grid_constant__ CUtensorMap tmQ,
                          const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV,
                          const __grid_constant__ CUtensorMap tmdO,
                          const __grid_constant__ CUtensorMap tmdK,
                          const __grid_constant__ CUtensorMap tmdV, const BwdParams p) {
  using C = Bwd128Cfg<D>;
  constexpr int BR = C::BR, BC = C::BC, DH = C::DH, QS = C::QS;
  constexpr bool SPARSE = MODE == BMODE_SPARSE, VARLEN = MODE == BMODE_VARLEN;
  static_assert(BC == MASK_BLOCK && BR == MASK_BLOCK, "one block-mask entry per step");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sK = smem;                                   // [KCH][BC][128B]
  uint8_t* sV = sK + C::K_BYTES;
  uint8_t* sStage = sV + C::K_BYTES;                    // QS x {Q | dO}
  uint8_t* sdS = sStage + QS * C::STAGE_BYTES;          // [2][BC][128B] dS^T, 64 queries per row
  uint64_t* bars = reinterpret_cast<uint64_t*>(sdS + C::DS_BYTES);
  uint64_t* bar_kv = bars + 0;
  uint64_t* bar_qfull = bars + 1;                       // [QS]
  uint64_t* bar_qempty = bars + 1 + QS;                 // [QS]
  uint64_t* bar_s = bars + 1 + 2 * QS;
  uint64_t* bar_dp = bars + 2 + 2 * QS;
  uint64_t* bar_p = bars + 3 + 2 * QS;
  uint64_t* bar_ds = bars + 4 + 2 * QS;
  uint64_t* bar_dqfull = bars + 5 + 2 * QS;
  uint64_t* bar_dqempty = bars + 6 + 2 * QS;
  uint64_t* bar_final = bars + 7 + 2 * QS;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 8 + 2 * QS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  int* sparse_ni = reinterpret_cast<int*>(tmem_holder + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Work unit: (batch, kv head, key block[, group share]).  The dense causal
  // d = 128 instance takes bwd_cta's longest-first order; the others keep
  // the plain decode inline (sharing bwd_cta cost the d = 64 causal kernel
  // 3-4 % through its code generation, although the order is the same).
  int gs, kb, bkv;
  if constexpr (CAUSAL && D == 128 && MODE == BMODE_DENSE) {
    bwd_cta(p, blockIdx.x, gs, kb, bkv);
  } else {
    gs = blockIdx.x % p.gsplit;
    const int rest = blockIdx.x / p.gsplit;
    kb = rest % p.n_kblocks;
    bkv = rest / p.n_kblocks;
  }
  const int b = bkv / p.Hkv;
  const int hkv = bkv - b * p.Hkv;
  const int key0 = kb * BC;
  int nq = p.Nq, nk = p.Nk, qoff = 0, koff = 0;
  if constexpr (VARLEN) {
    varlen_rows(p.cu_q, b, p.total_q, qoff, nq);
    varlen_rows(p.cu_k, b, p.total_k, koff, nk);
    if (key0 >= nk) return;                             // past this sequence's keys
  }
  const int tkv = VARLEN ? hkv : bkv;
  const int n_qblocks = (nq + BR - 1) / BR;
  const int i0 = CAUSAL ? (key0 / BR) : 0;              // first query block that sees key0
  const int span = max(0, n_qblocks - i0);
  int n_i = span;
  const int head0 = hkv * p.group + gs * p.hps;
  const int rot = CAUSAL ? 0 : int((long long)kb * span / p.n_kblocks);
  auto step_q = [&](int t, int& hh, int& qi) {
    hh = t / n_i;
    int li = t - hh * n_i + rot;
    if (li >= n_i) li -= n_i;
    qi = i0 + li;
  };
  auto qvis = [&](int i) -> bool { return __ldg(p.mask + size_t(i) * p.mask_ld + kb) != 0; };
  auto qnext = [&](int i) -> int {
    for (int k = 0; k < span; ++k, ++i) {
      if (i >= n_qblocks) i = i0;
      if (qvis(i)) return i;
    }
    return i0;
  };
  struct Seq { int hh, qi, c; };
  auto seq_begin = [&](Seq& q) { q.hh = 0; q.c = 0; q.qi = qnext(i0 + rot); };
  auto seq_next = [&](Seq& q) {
    if (++q.c == n_i) { q.c = 0; ++q.hh; q.qi = qnext(i0 + rot); }
    else q.qi = qnext(q.qi + 1);
  };
  auto step_at = [&](Seq& q, int t, int& hh, int& qi) {
    if constexpr (SPARSE) {
      hh = q.hh;
      qi = q.qi;
      seq_next(q);
    } else {
      step_q(t, hh, qi);
    }
  };
  // First entry of the LSE*log2(e) / D rows of step (hh, qi) in the workspace.
  auto lrow = [&](int hh, int qi) -> size_t {
    return VARLEN ? size_t((head0 + hh) * p.lpad_ld + varlen_pad_start(qoff, b) + qi * BR)
                  : size_t(b * p.Hq + head0 + hh) * p.Nq_pad + size_t(qi) * BR;
  };

  if (threadIdx.x == 0) {
    mbar_init(bar_kv, 1);
    for (int i = 0; i < QS; ++i) {
      mbar_init(bar_qfull + i, 1);
      mbar_init(bar_qempty + i, 1);
    }
    mbar_init(bar_s, 1);
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
    if (warp == 10) {
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
    regs_to<C::REGS_OTHER, C::REGS_LAUNCH>();
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
        step_at(sq, t, hh, qi);
        const int tq = VARLEN ? head0 + hh : b * p.Hq + head0 + hh;
        const int st = t % QS;
        if (!mbar_wait(bar_qempty + st, ((t / QS) & 1) ^ 1, abort_flag, p.status, WB_QEMPTY))
          break;
        uint8_t* s_q = sStage + st * C::STAGE_BYTES;
        uint8_t* s_do = s_q + C::QT_BYTES;
        mbar_arrive_expect_tx(bar_qfull + st, C::STAGE_BYTES);
        for (int c = 0; c < C::KCH; ++c) {
          tma_load_bh(s_q + c * BR * 128, &tmQ, bar_qfull + st, c * 64, qoff + qi * BR, tq, p.Hq);
          tma_load_bh(s_do + c * BR * 128, &tmdO, bar_qfull + st, c * 64, qoff + qi * BR, tq,
                      p.Hq);
        }
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
      constexpr uint32_t STG = C::STAGE_BYTES >> 4, QT = C::QT_BYTES >> 4;
      // A-operand column of k-step kk (16 queries) within a P^T / dS^T
      // region: each 32-query chunk (32 columns of S^T / dP^T) holds its
      // queries' fp16 P / bf16 dS pairs in its first 16 columns (dS lo in
      // the next 16).
      auto pcol = [](int kk) { return uint32_t((kk >> 1) * 32 + (kk & 1) * 8); };
      auto kst = [&](int t) { return kS0 + uint32_t(t % QS) * STG; };   // Q of step t, K-major
      auto mst = [&](int t) { return mS0 + uint32_t(t % QS) * STG; };   // Q of step t, MN-major
      auto mma_kq = [&](uint32_t d_tm, uint32_t a_lo, uint32_t b_lo, uint32_t idesc) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ko = ((kk >> 2) * BC * 128 + (kk & 3) * 32) >> 4;
          const uint32_t qo = ((kk >> 2) * BR * 128 + (kk & 3) * 32) >> 4;
          umma_ss_lo(d_tm, a_lo + ko, b_lo + qo, idesc, kk > 0);
        }
      };
      bool ok = mbar_wait(bar_kv, 0, abort_flag, p.status, WB_KV) &&
                mbar_wait(bar_qfull + 0, 0, abort_flag, p.status, WB_QFULL);
      tc_fence_after();
      if (ok) {
        mma_kq(tmem + C::TM_SP, kK, kst(0), ID_S);
        umma_commit(bar_s);
        mma_kq(tmem + C::TM_DP, kV, kst(0) + QT, ID_DP);
        umma_commit(bar_dp);
      }
      for (int t = 0; t < n_steps && ok; ++t) {
        const int st = t % QS;
        const uint32_t mQ = mst(t), mdO = mQ + QT;
        // dV += P^T dO  (fp16 P and dO)
        if (!(ok = mbar_wait(bar_p, t & 1, abort_flag, p.status, WB_P))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BR / 16; ++kk)
          umma_ts_lo(tmem + C::TM_DV, tmem + C::TM_SP + pcol(kk), mdO + kk * 128, ID_V,
                     (t > 0 || kk > 0) ? 1u : 0u);
        // S^T of the next step (SP is free once dV_t has read P_t)
        if (t + 1 < n_steps) {
          if (!(ok = mbar_wait(bar_qfull + (t + 1) % QS, ((t + 1) / QS) & 1, abort_flag,
                               p.status, WB_QFULL)))
            break;
          tc_fence_after();
          mma_kq(tmem + C::TM_SP, kK, kst(t + 1), ID_S);
          umma_commit(bar_s);
        }
        // dK += dS^T Q
        if (!(ok = mbar_wait(bar_ds, t & 1, abort_flag, p.status, WB_DS))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BR / 16; ++kk)
          umma_ts_lo(tmem + C::TM_DK, tmem + C::TM_DP + pcol(kk), mQ + kk * 128, ID_KV,
                     (t > 0 || kk > 0) ? 1u : 0u);
        umma_commit(bar_qempty + st);
        // dQ^T = K^T dS^T (M = 128 rows of d, N = 128 queries, K = 128 keys);
        // for d = 64 the upper 64 rows of M read the V tile's 16-bit elements (whatever
        // their type) and are ignored.
        // In its own columns it only waits for the read-out of dQ^T_{t-1}.
        if constexpr (C::DQ_OWN) {
          if (t > 0 &&
              !(ok = mbar_wait(bar_dqempty, (t - 1) & 1, abort_flag, p.status, WB_DQEMPTY)))
            break;
          tc_fence_after();
        }
#pragma unroll
        for (int kk = 0; kk < BC / 16; ++kk)
          umma_ss_lo(tmem + C::TM_DQ, mK + kk * 128, mdS + kk * 128, ID_DQ, kk > 0);
        umma_commit(bar_dqfull);
        // dP^T of the next step; in the DP region it waits until dQ^T_t has
        // left TMEM
        if (t + 1 < n_steps) {
          if constexpr (!C::DQ_OWN) {
            if (!(ok = mbar_wait(bar_dqempty, t & 1, abort_flag, p.status, WB_DQEMPTY))) break;
            tc_fence_after();
          }
          mma_kq(tmem + C::TM_DP, kV, kst(t + 1) + QT, ID_DP);
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
    regs_to<C::REGS_READ, C::REGS_LAUNCH>();
    // ------------------------------------------------------------ dQ read-out
    // Warp 12 + w takes TMEM lane quarter w of dQ^T (lanes = d rows, all 128
    // query columns) into registers, releases DP, then reduce-adds the rows
    // into the fp32 accumulator (coalesced over d).
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
      step_at(sq, u, hh, qi);
      const bool okk = mbar_wait(bar_dqfull, u & 1, abort_flag, p.status, WB_DQFULL);
      if (!__all_sync(0xffffffffu, okk)) break;
      tc_fence_after();
      uint32_t v[BR];
      if (r < DH) {
#pragma unroll
        for (int c = 0; c < BR / 32; ++c) FA_TMEM_LD32(tl + C::TM_DQ + c * 32, (v + c * 32));
        tmem_wait_ld();
      }
      tc_fence_before();
      mbar_arrive(bar_dqempty);
      if (r < DH) {
        const int q0 = qi * BR;
        float* dst = p.dqacc +
                     (VARLEN ? (size_t(head0 + hh) * p.total_q + qoff + q0) * D
                             : (size_t(b * p.Hq + head0 + hh) * p.Nq + q0) * D) + r;
        if (q0 + BR <= nq) {
#pragma unroll
          for (int i = 0; i < BR; ++i) atomicAdd(dst + i * D, dqv(v[i]));
        } else {
          const int nvalid = nq - q0;
#pragma unroll
          for (int i = 0; i < BR; ++i)
            if (i < nvalid) atomicAdd(dst + i * D, dqv(v[i]));
        }
      }
    }
  } else {
    regs_to<C::REGS_COMPUTE, C::REGS_LAUNCH>();
    // ------------------------------------------------------------ compute warps
    const int g = warp >> 2;                       // query columns [64g, 64g+64) of each step
    const int w = warp & 3;                        // TMEM lane quarter
    const int r = w * 32 + lane;                   // key row == TMEM lane
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
      step_at(sq, t, hh, qi);
      const size_t lr = lrow(hh, qi) + g * 64;
      const float4* lse4 = reinterpret_cast<const float4*>(p.Lpad + lr);
      const float4* dd4 = reinterpret_cast<const float4*>(p.Dpad + lr);
      const uint32_t tSP = tl + C::TM_SP + g * 64;
      const uint32_t tDP = tl + C::TM_DP + g * 64;
      // ---- P^T for this key row and the group's 64 queries, 32 at a time:
      // fp16(P) over the chunk's first 16 S^T columns (each chunk is read
      // before written): the A operand of dV, whose fp16 rounding keeps dV
      // within the bound over the query rows of a whole GQA group.
      ok = mbar_wait(bar_s, t & 1, abort_flag, p.status, WB_S);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      float pf[64];                                 // P (fp32), kept for dS
      const float2 sl22 = make_float2(sl2, sl2);
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t u[32];
        FA_TMEM_LD32(tSP + c * 32, u);
        tmem_wait_ld();
        const int qg = qi * BR + g * 64 + c * 32;            // first query of these 32 columns
        const bool need_mask = (CAUSAL && key0 + BC - 1 > qg) || (key0 + BC > nk);
        const int cstart = key >= nk ? 32 : (CAUSAL ? key - qg : 0);
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          const float4 l4 = __ldg(lse4 + (c * 32 + i) / 4);
          const float2 x0 = ffma2(make_float2(__uint_as_float(u[i]), __uint_as_float(u[i + 1])),
                                  sl22, make_float2(-l4.x, -l4.y));
          const float2 x1 = ffma2(make_float2(__uint_as_float(u[i + 2]),
                                              __uint_as_float(u[i + 3])),
                                  sl22, make_float2(-l4.z, -l4.w));
          float pv[4] = {ex2(x0.x), ex2(x0.y), ex2(x1.x), ex2(x1.y)};
          if (need_mask) {
#pragma unroll
            for (int e = 0; e < 4; ++e) pv[e] = (i + e < cstart) ? 0.f : pv[e];
          }
#pragma unroll
          for (int e = 0; e < 4; ++e) pf[c * 32 + i + e] = pv[e];
        }
        uint32_t ph[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          ph[i] = F16 ? pack_f16(pf[c * 32 + 2 * i], pf[c * 32 + 2 * i + 1])
                      : pack_bf16(pf[c * 32 + 2 * i], pf[c * 32 + 2 * i + 1]);
        FA_TMEM_ST16(tSP + c * 32, ph);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar_p);

      // ---- dS^T = P^T o (dP - D), 16 columns at a time (dP unscaled from
      // the fp16 product).
      ok = mbar_wait(bar_dp, t & 1, abort_flag, p.status, WB_DP);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t dpv[16];
          FA_TMEM_LD16(tDP + c * 16, dpv);
          tmem_wait_ld();
          uint32_t pk[8];
#pragma unroll
          for (int i = 0; i < 8; i += 2) {
            const float4 d4 = __ldg(dd4 + (c * 16 + 2 * i) / 4);
            const float dsub[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const float2 pp =
                  make_float2(pf[c * 16 + 2 * (i + e)], pf[c * 16 + 2 * (i + e) + 1]);
              const float2 dp2 = make_float2(__uint_as_float(dpv[2 * (i + e)]),
                                             __uint_as_float(dpv[2 * (i + e) + 1]));
              const float2 nd = make_float2(-dsub[2 * e], -dsub[2 * e + 1]);
              const float2 x = F16 ? ffma2(dp2, inv_vd2, nd) : fadd2(dp2, nd);
              if constexpr (ALL16) {             // fp16(dS * 2^e_dS)
                const float2 y = fmul2(fmul2(pp, x), s_ds2);
                pk[i + e] = pack_f16(y.x, y.y);
              } else {
                const float2 y = fmul2(pp, x);
                pk[i + e] = pack_bf16(y.x, y.y);
              }
            }
          }
          // dS^T pairs over already read dP^T columns of this 32-query chunk
          // (the chunk's first 16 columns, 8 per 16 queries) ...
          FA_TMEM_ST8(tDP + (c >> 1) * 32 + (c & 1) * 8, pk);
          // ... and into the shared tile for dQ: row r, queries [64g + 16c, +16)
          uint8_t* rowp = sdS + g * (BC * 128) + r * 128;
#pragma unroll
          for (int q4 = 0; q4 < 2; ++q4) {
            const int unit = c * 2 + q4;
            *reinterpret_cast<uint4*>(rowp + ((unit ^ (r & 7)) * 16)) =
                make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
          }
        }
      }
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar_ds);
    }

    // ---- epilogue: group 0 writes dK = scale * dK_acc, group 1 writes dV
    if (ok && n_steps > 0) {
      ok = mbar_wait(bar_final, 0, abort_flag, p.status, WB_FINAL);
      ok = __all_sync(0xffffffffu, ok);
      if (ok) tc_fence_after();
    }
    if (ok && p.gsplit > 1) {
      if (n_steps > 0) {
        const int tcol = g == 0 ? C::TM_DK : C::TM_DV;
        const float mul = g == 0 ? os.mul_dk : os.mul_dv;
        float* dst = (g == 0 ? p.dkacc : p.dvacc) +
                     (VARLEN ? size_t(hkv) * p.total_k + koff + key : size_t(bkv) * p.Nk + key) *
                         D;
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
                                                  (long long)(koff + key) * so.n + c * 32);
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
          tma_store_bh(tm, stage + (c * 4 + w) * 4096, c * 64, koff + key0 + w * 32, tkv, p.Hkv);
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
