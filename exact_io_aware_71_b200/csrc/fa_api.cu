// C ABI of libfa: argument checks, TMA descriptor encoding and kernel launch.
// Every step of the attention computation runs in the kernels included here;
// this file only validates, describes the tensors to the TMA unit and launches.
#include <cmath>
#include <cstdint>
#include <cstddef>
#include <cstring>
#include <mutex>
#include <algorithm>

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "fa.h"
#include "fa_fwd.cuh"

#include "fa_bwd.cuh"

namespace fa {
__device__ DevStatus g_status;   // one status word per device (module global)
}
static_assert(FA_MASK_BLOCK == fa::MASK_BLOCK, "block-mask granularity of the C ABI");

namespace {

using namespace fa;

// ---------------------------------------------------------------- checks
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// Element strides of contiguous [B, H, N, d].
Strides contiguous(int H, int N, int d) {
  return Strides{(long long)H * N * d, (long long)N * d, (long long)d};
}

// Each stride positive, a multiple of 8 elements (16 bytes) and below the
// TMA limit of 2^40 bytes.
bool strides_ok(const fa_strides* s, int n) {
  for (int i = 0; i < n; ++i) {
    const long long v[3] = {s[i].batch, s[i].head, s[i].row};
    for (long long x : v)
      if (x <= 0 || (x & 7) != 0 || x >= (1LL << 39)) return false;
  }
  return true;
}

int check_sizes(int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal, float scale) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || Nk < 1) return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (!(std::isfinite(scale) && scale > 0.f)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
  // Grid and index arithmetic use 32-bit ints for (batch*head) and rows.
  const int64_t bhq = int64_t(B) * Hq;
  const int64_t tiles = bhq * ((int64_t(Nq) + 127) / 128);
  if (bhq > (int64_t(1) << 24) || tiles >= (int64_t(1) << 31)) return FA_ERR_UNSUPPORTED;
  if (int64_t(B) * Hkv * ((int64_t(Nk) + 127) / 128) * 2 >= (int64_t(1) << 31))
    return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

// ---------------------------------------------------------------- TMA maps
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

}  // namespace

// A bf16 tensor seen as [batch, heads, rows, d] (d contiguous, the other
// dimensions at element strides st) as a 4-D TMA tensor (d, rows, heads,
// batch): 64-element (128-byte) inner boxes of box_rows rows, 128-byte
// swizzle; rows outside [0, rows) read as zero and are not written.
bool fa::make_map_bf16(CUtensorMap* m, const void* base, int d, int rows, int heads, int batch,
                       const Strides& st, int box_rows) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[4] = {cuuint64_t(d), cuuint64_t(rows), cuuint64_t(heads), cuuint64_t(batch)};
  cuuint64_t strides[3] = {cuuint64_t(st.n) * 2, cuuint64_t(st.h) * 2, cuuint64_t(st.b) * 2};
  cuuint32_t box[4] = {64u, cuuint32_t(box_rows), 1u, 1u};
  cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

namespace {

// Scratch of fa_bwd_noalloc (see fa.h).  In host code this name is only a
// host-side stand-in for the array; its device address comes from
// cudaGetSymbolAddress, looked up on every call with the caller's device and
// context current.  The lookup allocates nothing, and it is not cached: after
// a device reset, or in another context, the module (and the array) can sit
// at another address.
__device__ __align__(256) unsigned char g_noalloc_scratch[FA_NOALLOC_SCRATCH_BYTES];

void* noalloc_scratch() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
  return p;
}

DevStatus* status_ptr() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return nullptr;
  return static_cast<DevStatus*>(p);
}

// ---------------------------------------------------------------- forward
template <class KernelT>
int launch_kernel(KernelT kern, int smem, int threads, unsigned grid, const CUtensorMap& mq,
                  const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mo,
                  const FwdParams& p, cudaStream_t stream) {
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return FA_ERR_CUDA;
  kern<<<grid, threads, smem, stream>>>(mq, mk, mv, mo, p);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// d = 64 / 128: two query tiles per CTA; d = 256: one.  MODE: dense,
// block-sparse (p.mask) or packed variable-length batch (p.cu_q, p.cu_k).
// EPI: the epilogue (O and LSE, plus the residual, or D only).
template <int D, bool CAUSAL, int MODE, int EPI>
int launch_fwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
               const CUtensorMap& mo, FwdParams p, cudaStream_t stream) {
  if constexpr (D == 256) {
    using C = FwdCfg<D>;
    p.n_units = p.n_qblocks;
    return launch_kernel(fa_fwd_kernel<D, CAUSAL, MODE, EPI>, C::SMEM_BYTES, C::NTHREADS,
                         unsigned(p.n_units) * unsigned(p.B * p.Hq), mq, mk, mv, mo, p, stream);
  } else {
    using C = FwdPairCfg<D>;
    // The warpgroups' register split must fit in what the block is launched
    // with, or the setmaxnreg.inc would wait forever: refuse to launch.
    static int regs = -1;
    if (regs < 0) {
      cudaFuncAttributes fattr;
      if (cudaFuncGetAttributes(&fattr, fa_fwd_pair_kernel<D, CAUSAL, MODE, EPI>) != cudaSuccess)
        return FA_ERR_CUDA;
      regs = fattr.numRegs;
    }
    if (regs * C::NTHREADS < C::REGS_NEEDED) return FA_ERR_UNSUPPORTED;
    p.n_units = (p.n_qblocks + 1) / 2;

    // Persistent (one CTA per SM, each walking a strided unit list) for short
    // rows, where unit boundaries are frequent, and for causal rows up to 16k,
    // whose units differ in length; one CTA per unit otherwise (measured
    // faster for long rows, where the hardware's own CTA dispatch balances
    // the units).  The kernel is the same; a CTA whose stride covers the
    // whole list runs exactly one unit.
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long units = (long long)p.n_units * p.B * p.Hq;
    const bool persistent = p.Nk <= 4096 || (CAUSAL && p.Nk <= 16384);
    const unsigned grid = unsigned(persistent ? std::min<long long>(units, sms) : units);
    return launch_kernel(fa_fwd_pair_kernel<D, CAUSAL, MODE, EPI>, C::SMEM_BYTES, C::NTHREADS,
                         grid, mq, mk, mv, mo, p, stream);
  }
}

// The residual output exists for fixed-length batches without a block mask;
// the D epilogue for every mode.
template <int D, bool CAUSAL, int MODE>
int launch_fwd_epi(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                   const CUtensorMap& mo, const FwdParams& p, cudaStream_t stream) {
  if (p.d_out) return launch_fwd<D, CAUSAL, MODE, EPI_D>(mq, mk, mv, mo, p, stream);
  if constexpr (MODE == MODE_DENSE) {
    if (p.o_res) return launch_fwd<D, CAUSAL, MODE, EPI_RES>(mq, mk, mv, mo, p, stream);
  }
  return launch_fwd<D, CAUSAL, MODE, EPI_O>(mq, mk, mv, mo, p, stream);
}

template <int D, bool CAUSAL>
int launch_fwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
               const CUtensorMap& mo, const FwdParams& p, cudaStream_t stream) {
  return p.cu_q ? launch_fwd_epi<D, CAUSAL, MODE_VARLEN>(mq, mk, mv, mo, p, stream)
         : p.mask ? launch_fwd_epi<D, CAUSAL, MODE_SPARSE>(mq, mk, mv, mo, p, stream)
                  : launch_fwd_epi<D, CAUSAL, MODE_DENSE>(mq, mk, mv, mo, p, stream);
}

int launch_fwd_any(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                   const CUtensorMap& mo, const FwdParams& p, int d, int causal,
                   cudaStream_t stream) {
  if (d == 64) return causal ? launch_fwd<64, true>(mq, mk, mv, mo, p, stream)
                             : launch_fwd<64, false>(mq, mk, mv, mo, p, stream);
  if (d == 128) return causal ? launch_fwd<128, true>(mq, mk, mv, mo, p, stream)
                              : launch_fwd<128, false>(mq, mk, mv, mo, p, stream);
  return causal ? launch_fwd<256, true>(mq, mk, mv, mo, p, stream)
                : launch_fwd<256, false>(mq, mk, mv, mo, p, stream);
}

// The forward pass on strided tensors, with an optional block mask.
// o_res: optional residual output at o's strides (null: none).
int fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse,
             const fa_strides* strides, const unsigned char* mask, int B, int Hq, int Hkv,
             int Nq, int Nk, int d, int causal, float scale, cudaStream_t stream,
             void* o_res = nullptr) {
  if (!q || !k || !v || !o || !lse || !strides) return FA_ERR_INVALID_ARG;
  int st = check_sizes(B, Hq, Hkv, Nq, Nk, d, causal, scale);
  if (st != FA_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned4(lse) ||
      !strides_ok(strides, 4) || (o_res && !aligned16(o_res)) || (mask && !aligned16(mask)))
    return FA_ERR_MISALIGNED;
  Strides sq{strides[0].batch, strides[0].head, strides[0].row};
  Strides sk{strides[1].batch, strides[1].head, strides[1].row};
  Strides sv{strides[2].batch, strides[2].head, strides[2].row};
  Strides so{strides[3].batch, strides[3].head, strides[3].row};

  const int bc = (d == 256) ? 64 : 128;
  CUtensorMap mq, mk, mv, mo;
  if (!make_map_bf16(&mq, q, d, Nq, Hq, B, sq, 128) ||
      !make_map_bf16(&mk, k, d, Nk, Hkv, B, sk, bc) ||
      !make_map_bf16(&mv, v, d, Nk, Hkv, B, sv, bc) ||
      !make_map_bf16(&mo, o, d, Nq, Hq, B, so, 32))
    return FA_ERR_CUDA;

  FwdParams p;
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.Nq = Nq; p.Nk = Nk;
  p.group = Hq / Hkv;
  p.n_qblocks = (Nq + 127) / 128;
  p.causal = causal;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.lse = lse;
  p.status = status_ptr();
  if (!p.status) return FA_ERR_CUDA;
  p.mask = mask;
  p.mask_ld = (Nk + MASK_BLOCK - 1) / MASK_BLOCK;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.o_sb = so.b; p.o_sh = so.h; p.o_sn = so.n;
  p.cu_q = p.cu_k = nullptr;
  p.total_q = Nq;
  p.total_k = Nk;
  p.o_res = static_cast<__nv_bfloat16*>(o_res);
  p.d_out = nullptr;
  p.d_ld = 0;
  p.dO = nullptr;
  p.do_sb = p.do_sh = p.do_sn = 0;
  return launch_fwd_any(mq, mk, mv, mo, p, d, causal, stream);
}

// Checks shared by the packed variable-length entry points.
int check_varlen(const int* cu_q, const int* cu_k, int B, int max_q, int max_k, int total_q,
                 int total_k, int Hq, int Hkv, int d, int causal, float scale) {
  if (!cu_q || !cu_k) return FA_ERR_INVALID_ARG;
  if (total_q < 1 || total_k < 1) return FA_ERR_INVALID_ARG;
  int st = check_sizes(B, Hq, Hkv, max_q, max_k, d, causal, scale);
  if (st != FA_OK) return st;
  if (!aligned4(cu_q) || !aligned4(cu_k)) return FA_ERR_MISALIGNED;
  if (int64_t(Hq) * total_q * d >= (int64_t(1) << 40) || int64_t(B) + 1 >= (int64_t(1) << 24))
    return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

// Element strides of packed [total, H, d] tensors, seen as [1, H, total, d].
Strides packed(int H, int total, int d) {
  return Strides{(long long)total * H * d, (long long)d, (long long)H * d};
}

int fwd_varlen_impl(const void* q, const void* k, const void* v, void* o, float* lse,
                    const int* cu_q, const int* cu_k, int B, int max_q, int max_k, int total_q,
                    int total_k, int Hq, int Hkv, int d, int causal, float scale,
                    cudaStream_t stream) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  int st = check_varlen(cu_q, cu_k, B, max_q, max_k, total_q, total_k, Hq, Hkv, d, causal, scale);
  if (st != FA_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned4(lse))
    return FA_ERR_MISALIGNED;
  const Strides sq = packed(Hq, total_q, d), sk = packed(Hkv, total_k, d);
  const int bc = (d == 256) ? 64 : 128;
  CUtensorMap mq, mk, mv, mo;
  if (!make_map_bf16(&mq, q, d, total_q, Hq, 1, sq, 128) ||
      !make_map_bf16(&mk, k, d, total_k, Hkv, 1, sk, bc) ||
      !make_map_bf16(&mv, v, d, total_k, Hkv, 1, sk, bc) ||
      !make_map_bf16(&mo, o, d, total_q, Hq, 1, sq, 32))
    return FA_ERR_CUDA;
  FwdParams p;
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.Nq = max_q; p.Nk = max_k;
  p.group = Hq / Hkv;
  p.n_qblocks = (max_q + 127) / 128;
  p.causal = causal;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.lse = lse;
  p.status = status_ptr();
  if (!p.status) return FA_ERR_CUDA;
  p.mask = nullptr;
  p.mask_ld = 0;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.o_sb = sq.b; p.o_sh = sq.h; p.o_sn = sq.n;
  p.cu_q = cu_q;
  p.cu_k = cu_k;
  p.total_q = total_q;
  p.total_k = total_k;
  p.o_res = nullptr;
  p.d_out = nullptr;
  p.d_ld = 0;
  p.dO = nullptr;
  p.do_sb = p.do_sh = p.do_sn = 0;
  return launch_fwd_any(mq, mk, mv, mo, p, d, causal, stream);
}

// Exact D for the backward of a wide GQA / MQA group: the forward pass runs
// again with the D epilogue and overwrites the workspace's D rows (written
// from the bf16 O by the preprocess) with D = rowsum(dO o O), O in fp32.
// st: strides of q, k, v, o, dO (fixed-length) as [B, H, N, d] views; vl:
// packed batch or null; mask: block mask or null.  O and the LSE are read
// by nobody here and written by nobody.
int recompute_d(const void* q, const void* k, const void* v, const void* o, const float* lse,
                const void* dO, const Strides* st, int B, int Hq, int Hkv, int Nq, int Nk, int d,
                int causal, float scale, const unsigned char* mask, const Varlen* vl,
                void* workspace, DevStatus* status, cudaStream_t stream) {
  const int rows_q = vl ? vl->total_q : Nq, rows_k = vl ? vl->total_k : Nk;
  const int map_b = vl ? 1 : B;
  const int bc = (d == 256) ? 64 : 128;
  const BwdWorkspace w = vl ? bwd_workspace_layout_varlen(B, Hq, Hkv, vl->total_q, vl->total_k, d)
                            : bwd_workspace_layout(B, Hq, Hkv, Nq, Nk, d);
  // d <= 128: the tile-pair kernel multiplies P (as fp16) by the preprocess
  // stage's fp16 copy of V (these groups always have one); d = 256 keeps
  // bf16 V with P as hi + lo.
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const bool v16 = d <= 128;
  const Strides s_v16{(long long)Hkv * rows_k * d, (long long)rows_k * d, d};
  CUtensorMap mq, mk, mv, mo;
  if (!make_map_bf16(&mq, q, d, rows_q, Hq, map_b, st[0], 128) ||
      !make_map_bf16(&mk, k, d, rows_k, Hkv, map_b, st[1], bc) ||
      !make_map_bf16(&mv, v16 ? static_cast<const void*>(ws + w.v16_off) : v, d, rows_k, Hkv,
                     map_b, v16 ? s_v16 : st[2], bc) ||
      !make_map_bf16(&mo, o, d, rows_q, Hq, map_b, st[3], 32))
    return FA_ERR_CUDA;
  FwdParams p;
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.Nq = Nq; p.Nk = Nk;
  p.group = Hq / Hkv;
  p.n_qblocks = (Nq + 127) / 128;
  p.causal = causal;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.lse = const_cast<float*>(lse);
  p.status = status;
  p.mask = mask;
  p.mask_ld = (Nk + MASK_BLOCK - 1) / MASK_BLOCK;
  p.o = static_cast<__nv_bfloat16*>(const_cast<void*>(o));
  p.o_sb = st[3].b; p.o_sh = st[3].h; p.o_sn = st[3].n;
  p.cu_q = vl ? vl->cu_q : nullptr;
  p.cu_k = vl ? vl->cu_k : nullptr;
  p.total_q = rows_q;
  p.total_k = rows_k;
  p.o_res = nullptr;
  p.d_out = reinterpret_cast<float*>(ws + w.d_off);
  p.d_ld = vl ? varlen_lpad_ld(B, vl->total_q) : (long long)round_up(Nq, 128);
  p.dO = static_cast<const __nv_bfloat16*>(dO);
  p.do_sb = st[4].b; p.do_sh = st[4].h; p.do_sn = st[4].n;
  p.v_amax = v16 ? reinterpret_cast<const unsigned*>(ws + w.amax_off) + 1 : nullptr;
  return launch_fwd_any(mq, mk, mv, mo, p, d, causal, stream);
}

// Element strides of the contiguous layouts of q, k, v, o.
void contiguous4(fa_strides* s, int Hq, int Hkv, int Nq, int Nk, int d) {
  const Strides a = contiguous(Hq, Nq, d), b = contiguous(Hkv, Nk, d);
  s[0] = {a.b, a.h, a.n};
  s[1] = {b.b, b.h, b.n};
  s[2] = {b.b, b.h, b.n};
  s[3] = {a.b, a.h, a.n};
}

}  // namespace

extern "C" {

const char* fa_status_string(int s) {
  switch (s) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED";
    case FA_ERR_MISALIGNED: return "FA_ERR_MISALIGNED";
    case FA_ERR_WORKSPACE: return "FA_ERR_WORKSPACE";
    case FA_ERR_CUDA: return "FA_ERR_CUDA";
    case FA_ERR_DEVICE_TIMEOUT: return "FA_ERR_DEVICE_TIMEOUT";
    case FA_ERR_TOO_LARGE: return "FA_ERR_TOO_LARGE";
    default: return "FA_ERR_UNKNOWN";
  }
}

int fa_fwd_strided(const void* q, const void* k, const void* v, void* o, float* lse,
                   const fa_strides* strides, int B, int Hq, int Hkv, int Nq, int Nk, int d,
                   int causal, float scale, cudaStream_t stream) {
  return fwd_impl(q, k, v, o, lse, strides, nullptr, B, Hq, Hkv, Nq, Nk, d, causal, scale,
                  stream);
}

int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
           int Hkv, int Nq, int Nk, int d, int causal, float scale, cudaStream_t stream) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || Nk < 1) return FA_ERR_INVALID_ARG;
  fa_strides s[4];
  contiguous4(s, Hq, Hkv, Nq, Nk, d);
  return fwd_impl(q, k, v, o, lse, s, nullptr, B, Hq, Hkv, Nq, Nk, d, causal, scale, stream);
}

int fa_fwd_block_sparse(const void* q, const void* k, const void* v, void* o, float* lse,
                        const fa_strides* strides, const unsigned char* block_mask, int B, int Hq,
                        int Hkv, int Nq, int Nk, int d, int causal, float scale,
                        cudaStream_t stream) {
  if (!block_mask) return FA_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || Nk < 1) return FA_ERR_INVALID_ARG;
  fa_strides s[4];
  if (!strides) {
    contiguous4(s, Hq, Hkv, Nq, Nk, d);
    strides = s;
  }
  return fwd_impl(q, k, v, o, lse, strides, block_mask, B, Hq, Hkv, Nq, Nk, d, causal, scale,
                  stream);
}

size_t fa_bwd_workspace_size(int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal) {
  if (check_sizes(B, Hq, Hkv, Nq, Nk, d, causal, 1.0f) != FA_OK) return 0;
  return bwd_workspace_bytes(B, Hq, Hkv, Nq, Nk, d);
}

}  // extern "C"

namespace {

// The backward pass on strided tensors, stage by stage (see fa_bwd_stage).
int bwd_impl(int stage, const void* q, const void* k, const void* v, const void* o,
             const float* lse, const void* dO, void* dq, void* dk, void* dv,
             const fa_strides* strides, int B, int Hq, int Hkv, int Nq, int Nk, int d,
             int causal, float scale, void* workspace, size_t workspace_bytes,
             cudaStream_t stream, const unsigned char* mask = nullptr,
             const void* o_res = nullptr) {
  int stages;
  switch (stage) {
    case FA_BWD_ALL: stages = 7; break;
    case FA_BWD_PRE: stages = 1; break;
    case FA_BWD_MAIN: stages = 2; break;
    case FA_BWD_DQ: stages = 4; break;
    default: return FA_ERR_INVALID_ARG;
  }
  if (!q || !k || !v || !o || !lse || !dO || !dq || !dk || !dv || !strides)
    return FA_ERR_INVALID_ARG;
  int st = check_sizes(B, Hq, Hkv, Nq, Nk, d, causal, scale);
  if (st != FA_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned4(lse) ||
      !aligned16(dO) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
      !strides_ok(strides, 8) || (o_res && !aligned16(o_res)) || (mask && !aligned16(mask)))
    return FA_ERR_MISALIGNED;
  const size_t need = bwd_workspace_bytes(B, Hq, Hkv, Nq, Nk, d);
  if (!workspace || workspace_bytes < need) return FA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return FA_ERR_MISALIGNED;
  DevStatus* sp = status_ptr();
  if (!sp) return FA_ERR_CUDA;
  Strides s8[8];
  for (int i = 0; i < 8; ++i) s8[i] = Strides{strides[i].batch, strides[i].head, strides[i].row};
  if (stages & 1) {
    int r = launch_bwd(1, q, k, v, o, o_res, lse, dO, dq, dk, dv, s8, B, Hq, Hkv, Nq, Nk, d,
                       causal, scale, mask, nullptr, workspace, sp, stream);
    if (r != FA_OK) return r;
    // Wide groups without the forward's residual: exact D by recomputation.
    if (!o_res && exact_dk(Hq / Hkv, d)) {
      r = recompute_d(q, k, v, o, lse, dO, s8, B, Hq, Hkv, Nq, Nk, d, causal, scale, mask,
                      nullptr, workspace, sp, stream);
      if (r != FA_OK) return r;
    }
  }
  if (!(stages & 6)) return FA_OK;
  return launch_bwd(stages & 6, q, k, v, o, o_res, lse, dO, dq, dk, dv, s8, B, Hq, Hkv, Nq, Nk,
                    d, causal, scale, mask, nullptr, workspace, sp, stream);
}

void contiguous8(fa_strides* s, int Hq, int Hkv, int Nq, int Nk, int d) {
  const Strides a = contiguous(Hq, Nq, d), b = contiguous(Hkv, Nk, d);
  const fa_strides qa{a.b, a.h, a.n}, kb{b.b, b.h, b.n};
  // q, k, v, o, dO, dq, dk, dv
  s[0] = qa; s[1] = kb; s[2] = kb; s[3] = qa; s[4] = qa; s[5] = qa; s[6] = kb; s[7] = kb;
}

}  // namespace

extern "C" {

int fa_bwd_strided(const void* q, const void* k, const void* v, const void* o, const float* lse,
                   const void* dO, void* dq, void* dk, void* dv, const fa_strides* strides, int B,
                   int Hq, int Hkv, int Nq, int Nk, int d, int causal, float scale,
                   void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  return bwd_impl(FA_BWD_ALL, q, k, v, o, lse, dO, dq, dk, dv, strides, B, Hq, Hkv, Nq, Nk, d,
                  causal, scale, workspace, workspace_bytes, stream);
}

int fa_bwd_block_sparse(const void* q, const void* k, const void* v, const void* o,
                        const float* lse, const void* dO, void* dq, void* dk, void* dv,
                        const fa_strides* strides, const unsigned char* block_mask, int B, int Hq,
                        int Hkv, int Nq, int Nk, int d, int causal, float scale, void* workspace,
                        size_t workspace_bytes, cudaStream_t stream) {
  if (!block_mask) return FA_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || Nk < 1) return FA_ERR_INVALID_ARG;
  fa_strides s[8];
  if (!strides) {
    contiguous8(s, Hq, Hkv, Nq, Nk, d);
    strides = s;
  }
  return bwd_impl(FA_BWD_ALL, q, k, v, o, lse, dO, dq, dk, dv, strides, B, Hq, Hkv, Nq, Nk, d,
                  causal, scale, workspace, workspace_bytes, stream, block_mask);
}

int fa_bwd_stage(int stage, const void* q, const void* k, const void* v, const void* o,
                 const float* lse, const void* dO, void* dq, void* dk, void* dv, int B, int Hq,
                 int Hkv, int Nq, int Nk, int d, int causal, float scale, void* workspace,
                 size_t workspace_bytes, cudaStream_t stream) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || Nk < 1) return FA_ERR_INVALID_ARG;
  fa_strides s[8];
  contiguous8(s, Hq, Hkv, Nq, Nk, d);
  return bwd_impl(stage, q, k, v, o, lse, dO, dq, dk, dv, s, B, Hq, Hkv, Nq, Nk, d, causal,
                  scale, workspace, workspace_bytes, stream);
}

int fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
           const void* dO, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Nq, int Nk,
           int d, int causal, float scale, void* workspace, size_t workspace_bytes,
           cudaStream_t stream) {
  return fa_bwd_stage(FA_BWD_ALL, q, k, v, o, lse, dO, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d, causal,
                      scale, workspace, workspace_bytes, stream);
}

int fa_fwd_residual(const void* q, const void* k, const void* v, void* o, void* o_res,
                    float* lse, const fa_strides* strides, int B, int Hq, int Hkv, int Nq,
                    int Nk, int d, int causal, float scale, cudaStream_t stream) {
  if (!o_res) return FA_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || Nk < 1) return FA_ERR_INVALID_ARG;
  fa_strides s[4];
  if (!strides) {
    contiguous4(s, Hq, Hkv, Nq, Nk, d);
    strides = s;
  }
  return fwd_impl(q, k, v, o, lse, strides, nullptr, B, Hq, Hkv, Nq, Nk, d, causal, scale, stream,
                  o_res);
}

int fa_bwd_residual(const void* q, const void* k, const void* v, const void* o,
                    const void* o_res, const float* lse, const void* dO, void* dq, void* dk,
                    void* dv, const fa_strides* strides, int B, int Hq, int Hkv, int Nq, int Nk,
                    int d, int causal, float scale, void* workspace, size_t workspace_bytes,
                    cudaStream_t stream) {
  if (!o_res) return FA_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || Nk < 1) return FA_ERR_INVALID_ARG;
  fa_strides s[8];
  if (!strides) {
    contiguous8(s, Hq, Hkv, Nq, Nk, d);
    strides = s;
  }
  return bwd_impl(FA_BWD_ALL, q, k, v, o, lse, dO, dq, dk, dv, strides, B, Hq, Hkv, Nq, Nk, d,
                  causal, scale, workspace, workspace_bytes, stream, nullptr, o_res);
}

int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                   const void* dO, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Nq,
                   int Nk, int d, int causal, float scale, cudaStream_t stream) {
  if (!q || !k || !v || !o || !lse || !dO || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
  int st = check_sizes(B, Hq, Hkv, Nq, Nk, d, causal, scale);
  if (st != FA_OK) return st;
  if (bwd_workspace_bytes(B, Hq, Hkv, Nq, Nk, d) > FA_NOALLOC_SCRATCH_BYTES)
    return FA_ERR_TOO_LARGE;
  void* scratch = noalloc_scratch();
  if (!scratch) return FA_ERR_CUDA;
  return fa_bwd_stage(FA_BWD_ALL, q, k, v, o, lse, dO, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d, causal,
                      scale, scratch, FA_NOALLOC_SCRATCH_BYTES, stream);
}

size_t fa_bwd_varlen_workspace_size(int B, int total_q, int total_k, int Hq, int Hkv, int d) {
  if (B < 1 || total_q < 1 || total_k < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return 0;
  if (d != 64 && d != 128 && d != 256) return 0;
  return bwd_workspace_layout_varlen(B, Hq, Hkv, total_q, total_k, d).total;
}

int fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                  const int* cu_seqlens_q, const int* cu_seqlens_k, int B, int max_seqlen_q,
                  int max_seqlen_k, int total_q, int total_k, int Hq, int Hkv, int d, int causal,
                  float scale, cudaStream_t stream) {
  return fwd_varlen_impl(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, B, max_seqlen_q,
                         max_seqlen_k, total_q, total_k, Hq, Hkv, d, causal, scale, stream);
}

int fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const float* lse,
                  const void* dO, void* dq, void* dk, void* dv, const int* cu_seqlens_q,
                  const int* cu_seqlens_k, int B, int max_seqlen_q, int max_seqlen_k,
                  int total_q, int total_k, int Hq, int Hkv, int d, int causal, float scale,
                  void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (!q || !k || !v || !o || !lse || !dO || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
  int st = check_varlen(cu_seqlens_q, cu_seqlens_k, B, max_seqlen_q, max_seqlen_k, total_q,
                        total_k, Hq, Hkv, d, causal, scale);
  if (st != FA_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned4(lse) ||
      !aligned16(dO) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return FA_ERR_MISALIGNED;
  const size_t need = bwd_workspace_layout_varlen(B, Hq, Hkv, total_q, total_k, d).total;
  if (!workspace || workspace_bytes < need) return FA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return FA_ERR_MISALIGNED;
  DevStatus* sp = status_ptr();
  if (!sp) return FA_ERR_CUDA;
  const Strides a = packed(Hq, total_q, d), b = packed(Hkv, total_k, d);
  const Strides s8[8] = {a, b, b, a, a, a, b, b};   // q, k, v, o, dO, dq, dk, dv
  const Varlen vl{cu_seqlens_q, cu_seqlens_k, total_q, total_k};
  int r = launch_bwd(1, q, k, v, o, nullptr, lse, dO, dq, dk, dv, s8, B, Hq, Hkv, max_seqlen_q,
                     max_seqlen_k, d, causal, scale, nullptr, &vl, workspace, sp, stream);
  if (r != FA_OK) return r;
  if (exact_dk(Hq / Hkv, d)) {   // wide groups: exact D by recomputation
    r = recompute_d(q, k, v, o, lse, dO, s8, B, Hq, Hkv, max_seqlen_q, max_seqlen_k, d, causal,
                    scale, nullptr, &vl, workspace, sp, stream);
    if (r != FA_OK) return r;
  }
  return launch_bwd(6, q, k, v, o, nullptr, lse, dO, dq, dk, dv, s8, B, Hq, Hkv, max_seqlen_q,
                    max_seqlen_k, d, causal, scale, nullptr, &vl, workspace, sp, stream);
}

int fa_device_status(cudaStream_t stream, int* where) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return FA_ERR_CUDA;
  unsigned int h[2] = {0u, 0u};
  const unsigned int zero[2] = {0u, 0u};
  // Only the two report words; the test controls behind them are left alone.
  if (cudaMemcpyFromSymbol(h, g_status, sizeof(h)) != cudaSuccess) return FA_ERR_CUDA;
  if (cudaMemcpyToSymbol(g_status, zero, sizeof(zero)) != cudaSuccess) return FA_ERR_CUDA;
  if (where) *where = int(h[1]);
  return h[0] ? FA_ERR_DEVICE_TIMEOUT : FA_OK;
}

int fa_debug_inject(int stall_kv_loads, double wait_limit_seconds) {
  if ((stall_kv_loads != 0 && stall_kv_loads != 1) || !(wait_limit_seconds >= 0.0) ||
      wait_limit_seconds > 60.0)
    return FA_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return FA_ERR_CUDA;
  const unsigned long long ns = (unsigned long long)(wait_limit_seconds * 1e9);
  const int stall = stall_kv_loads;
  if (cudaMemcpyToSymbol(g_status, &ns, sizeof(ns), offsetof(DevStatus, wait_limit_ns)) !=
          cudaSuccess ||
      cudaMemcpyToSymbol(g_status, &stall, sizeof(stall), offsetof(DevStatus, stall_kv)) !=
          cudaSuccess)
    return FA_ERR_CUDA;
  return cudaDeviceSynchronize() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // extern "C"
