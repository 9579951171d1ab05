/*
 * libfa: exact, IO-aware tiled attention for one NVIDIA B200 (sm_100a).
 *
 * What it computes.  Exact softmax(scale * Q K^T) V and its gradients, the
 * same result as standard attention up to rounding ("FlashAttention-2" post,
 * t.iss.one/s/quant_prune_distill/56, section "Введение"; QbitAI FA1
 * article, 52ps.vip, section "FlashAttention").  Q, K and V are streamed
 * tile by tile from HBM into on-chip memory and the N x N score matrix is
 * never written to HBM (same FA1 article, section "FlashAttention", figure
 * caption; QbitAI FA2 article, baiyundou.net, section "具体实现").  The
 * backward pass recomputes the probabilities block by block from Q, K, V and
 * the saved log-sum-exp (FA1 article, section "FlashAttention": "recalculate
 * attention in backward").
 *
 * Conventions shared by every entry point.
 *  - Element types: q, k, v, o, dO, dq, dk, dv are bf16; lse is fp32.
 *  - Layout: contiguous row-major [B, H, N, d]; H = Hq for q, o, dO, dq and
 *    H = Hkv for k, v, dk, dv.  lse is [B, Hq, Nq].
 *  - GQA / MQA (FA2 article, section "具体实现", second small change): Hkv
 *    divides Hq and query head h reads kv head h / (Hq / Hkv).
 *  - Causal masking is top-left aligned: key j is visible to query i iff
 *    j <= i.  Key blocks that lie wholly above the diagonal are skipped, not
 *    computed and zeroed (FA2 post, section "Алгоритм вычисления").
 *  - lse[i] = ln sum_j exp(scale * q_i . k_j) over the visible keys.
 *  - Head dims d in {64, 128, 256} (FA2 article: head dimension up to 256).
 *  - Every pointer is a device pointer owned by the caller; the library
 *    allocates and frees nothing.  q, k, v, o, dO, dq, dk, dv and the
 *    workspace must be 16-byte aligned (TMA); lse 4-byte aligned.
 *  - Calls are asynchronous on `stream` (0 = legacy default stream) and never
 *    synchronise.  Arguments are checked before anything is launched; a
 *    failed check returns a status and launches nothing.
 *  - A kernel whose internal pipeline wait exceeds its time limit records an
 *    error on the device and returns instead of hanging; fa_device_status()
 *    reports it.
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Element strides of a tensor seen as [B, H, N, d] with d contiguous
 * (stride 1).  Contiguous [B, H, N, d] is {H*N*d, N*d, d}; [B, N, H, d] is
 * {N*H*d, d, H*d}; q, k, v taken from one packed [B, N, 3, H, d] tensor use
 * {N*3*H*d, d, 3*H*d} with base pointers offset by 0, H*d and 2*H*d.  Each
 * stride must be a positive multiple of 8 elements (16 bytes, a TMA rule).
 */
typedef struct {
  long long batch, head, row;
} fa_strides;

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1,    /* null pointer, size < 1, Hq % Hkv != 0, bad scale */
  FA_ERR_UNSUPPORTED = 2,    /* d not in {64, 128, 256}, or sizes beyond int range */
  FA_ERR_MISALIGNED = 3,     /* a pointer or stride breaks the alignment rules above */
  FA_ERR_WORKSPACE = 4,      /* workspace null or smaller than fa_bwd_workspace_size() */
  FA_ERR_CUDA = 5,           /* a CUDA runtime/driver call or launch failed */
  FA_ERR_DEVICE_TIMEOUT = 6, /* a kernel gave up on a pipeline wait (see fa_device_status) */
  FA_ERR_TOO_LARGE = 7       /* fa_bwd_noalloc: the problem needs more than its built-in scratch */
} fa_status;

/*
 * Forward pass.  O = softmax(scale * Q K^T [masked]) V and the per-row
 * natural-log log-sum-exp.
 *   q   [B, Hq, Nq, d] bf16 (in)      k, v [B, Hkv, Nk, d] bf16 (in)
 *   o   [B, Hq, Nq, d] bf16 (out)     lse  [B, Hq, Nq] fp32 (out)
 *   causal: 0 or 1.   scale: finite, > 0 (usually 1/sqrt(d)).
 * Returns FA_OK or an fa_status code.
 */
int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
           int Hkv, int Nq, int Nk, int d, int causal, float scale, cudaStream_t stream);

/*
 * Forward pass on strided tensors (layouts such as [B, N, H, d] or views of
 * a packed QKV tensor; see fa_strides).  strides[0..3] describe q, k, v, o.
 * lse stays contiguous [B, Hq, Nq].  Otherwise identical to fa_fwd.
 */
int fa_fwd_strided(const void* q, const void* k, const void* v, void* o, float* lse,
                   const fa_strides* strides, int B, int Hq, int Hkv, int Nq, int Nk, int d,
                   int causal, float scale, cudaStream_t stream);

/*
 * Bytes of caller-owned device workspace fa_bwd needs for these sizes: the
 * fp32 dQ accumulator [B, Hq, Nq, d] and two fp32 row vectors (D =
 * rowsum(dO * O) and LSE * log2 e) padded to 128 rows per head; for GQA /
 * MQA groups also fp32 dK / dV partial sums [B, Hkv, Nk, d], and for GQA /
 * MQA groups and d = 256 fp16 copies of dO and V, for wide groups also of
 * Q and K (see fa_bwd).
 * Returns 0 for invalid sizes.
 */
size_t fa_bwd_workspace_size(int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal);

/*
 * Backward pass.  Given the forward inputs, its outputs o and lse, and dO,
 * writes dq [B, Hq, Nq, d], dk and dv [B, Hkv, Nk, d] (all bf16).  For GQA
 * dk/dv sum over the query heads of each group.  `workspace` must hold
 * fa_bwd_workspace_size(...) bytes; its contents need not be initialised
 * and are clobbered.  The same `scale` and `causal` as the forward pass.
 * Wide groups (Hq / Hkv >= 16, e.g. MQA; at d = 256 every Hq / Hkv >= 2):
 * dk sums dS^T q over every query row of the group, so the rounding of
 * D = rowsum(dO * O) from the bf16 o adds up; the pass then recomputes D
 * from the fp32 output with one more forward pass (below the forward's
 * time: at d <= 128 it multiplies P, as fp16, by the fp16 copy of v).  fa_fwd_residual / fa_bwd_residual give the same precision
 * without it.  For these groups every product takes fp16 operands (q and
 * k are copied like dO and v below) and dS goes in rounded to fp16, scaled
 * by a power of two chosen from the bound |dS| <= 2 d max|dO| max|v|.
 * GQA / MQA groups and d = 256: dV = P^T dO and dP = dO V^T take fp16
 * operands (P rounded to fp16, 8x finer than bf16, which dV sums over every
 * query row of the group).  The preprocess copies dO and V into the
 * workspace as fp16, each scaled by one power of two chosen from its
 * largest magnitude, so the copy is exact for every element within a factor
 * 2^24 of that magnitude; smaller elements keep an absolute error below
 * 2^-25 of it.  (The scale stops at 2^60 and 2^-60: a largest magnitude
 * below 2^-46 or above 2^75 keeps less precision.)  Non-finite dO or V give
 * non-finite results, as in bf16.
 */
int fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
           const void* dO, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Nq, int Nk,
           int d, int causal, float scale, void* workspace, size_t workspace_bytes,
           cudaStream_t stream);

/*
 * Backward pass on strided tensors.  strides[0..7] describe q, k, v, o, dO,
 * dq, dk, dv (see fa_strides); lse is contiguous [B, Hq, Nq].  The workspace
 * is the same as for fa_bwd.  Otherwise identical to fa_bwd.
 */
int fa_bwd_strided(const void* q, const void* k, const void* v, const void* o, const float* lse,
                   const void* dO, void* dq, void* dk, void* dv, const fa_strides* strides, int B,
                   int Hq, int Hkv, int Nq, int Nk, int d, int causal, float scale,
                   void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Block-sparse attention (QbitAI FA1 article, results section: block-sparse
 * FlashAttention).  A block mask removes whole blocks of the score matrix:
 *   block_mask  device bytes, row-major [ceil(Nq / FA_MASK_BLOCK)]
 *               [ceil(Nk / FA_MASK_BLOCK)], shared by every batch and head;
 *               entry (I, J) != 0 keeps the FA_MASK_BLOCK x FA_MASK_BLOCK
 *               block of query rows [I*128, I*128+128) and keys
 *               [J*128, J*128+128) (clipped to Nq, Nk).  Read-only, owned by
 *               the caller, unchanged until the kernels have finished.  The
 *               kernels read it in aligned 16-byte chunks: it must start on
 *               a 16-byte boundary (else FA_ERR_MISALIGNED) and its
 *               allocation must extend to the next multiple of 16 bytes
 *               (torch and cudaMalloc allocations do).
 * A removed block's scores count as -inf: the kernels neither load its K/V
 * nor compute it, so the work shrinks with the fraction of blocks kept.
 * With causal = 1 both masks apply.  A query row left with no visible key
 * gets O = 0 and lse = -inf (the limits of an empty softmax), and adds
 * nothing to any gradient.  An all-ones mask computes the dense result.
 * strides: as for fa_fwd_strided / fa_bwd_strided (4 or 8 entries), or NULL
 * for contiguous [B, H, N, d] tensors.  Everything else is as for fa_fwd and
 * fa_bwd; the backward workspace is fa_bwd_workspace_size(...).  The same
 * mask must be passed to both passes.
 */
#define FA_MASK_BLOCK 128

int fa_fwd_block_sparse(const void* q, const void* k, const void* v, void* o, float* lse,
                        const fa_strides* strides, const unsigned char* block_mask, int B, int Hq,
                        int Hkv, int Nq, int Nk, int d, int causal, float scale,
                        cudaStream_t stream);

int fa_bwd_block_sparse(const void* q, const void* k, const void* v, const void* o,
                        const float* lse, const void* dO, void* dq, void* dk, void* dv,
                        const fa_strides* strides, const unsigned char* block_mask, int B, int Hq,
                        int Hkv, int Nq, int Nk, int d, int causal, float scale, void* workspace,
                        size_t workspace_bytes, cudaStream_t stream);

/*
 * Variable-length batches: B sequences of different lengths packed back to
 * back, with no padding.  The pages do not name this; it serves the
 * small-batch, long-sequence case that the FA2 article's section on
 * parallelising over the sequence length addresses.
 *   q, o, dO, dq  [total_q, Hq, d] bf16, contiguous (row n, head h at
 *                 (n * Hq + h) * d)
 *   k, v, dk, dv  [total_k, Hkv, d] bf16, contiguous
 *   lse           [Hq, total_q] fp32
 *   cu_seqlens_q, cu_seqlens_k  device int32 [B + 1]: sequence b is rows
 *                 cu_seqlens_q[b] .. cu_seqlens_q[b+1] of q (and likewise of
 *                 k, v); non-decreasing, starting at 0 and ending at total_q
 *                 (total_k).  Read on the device only; out-of-range offsets
 *                 are clamped to [0, total], never followed.
 *   max_seqlen_q, max_seqlen_k  at least the longest sequence (they size the
 *                 grid; rows beyond them are not computed).
 * Attention stays within each sequence; causal masking is top-left aligned
 * within the sequence.  A sequence with queries but no keys gets O = 0 and
 * lse = -inf.  Other conventions as for fa_fwd / fa_bwd.
 */
int fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                  const int* cu_seqlens_q, const int* cu_seqlens_k, int B, int max_seqlen_q,
                  int max_seqlen_k, int total_q, int total_k, int Hq, int Hkv, int d, int causal,
                  float scale, cudaStream_t stream);

/* Bytes of workspace fa_bwd_varlen needs (0 for invalid sizes). */
size_t fa_bwd_varlen_workspace_size(int B, int total_q, int total_k, int Hq, int Hkv, int d);

int fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const float* lse,
                  const void* dO, void* dq, void* dk, void* dv, const int* cu_seqlens_q,
                  const int* cu_seqlens_k, int B, int max_seqlen_q, int max_seqlen_k,
                  int total_q, int total_k, int Hq, int Hkv, int d, int causal, float scale,
                  void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Forward pass that also writes the output's rounding residual
 *   o_res [B, Hq, Nq, d] bf16 (out), at o's strides: bf16(O - o), the part
 *   of the fp32 output that rounding it to bf16 dropped,
 * so that o + o_res holds the output to about 16 bits.  To make that the
 * exact output to 16 bits, this pass also multiplies V by P as bf16 hi + lo
 * (one more tensor-core product per key block, so it is slower than
 * fa_fwd; o itself is then the exact output rounded once).  fa_bwd_residual
 * takes o_res to form D = rowsum(dO * O) without recomputing the forward
 * pass; that matters for wide GQA / MQA groups (see fa_bwd).  The pages have no
 * counterpart; it serves their GQA / MQA setting (QbitAI FA2 article,
 * section "具体实现", second small change).  strides: q, k, v, o as for
 * fa_fwd_strided, or NULL for contiguous tensors.  Otherwise as fa_fwd.
 */
int fa_fwd_residual(const void* q, const void* k, const void* v, void* o, void* o_res,
                    float* lse, const fa_strides* strides, int B, int Hq, int Hkv, int Nq,
                    int Nk, int d, int causal, float scale, cudaStream_t stream);

/*
 * Backward pass with the forward's residual o_res (from fa_fwd_residual,
 * same strides as o): D = rowsum(dO * (o + o_res)).  strides: 8 entries as
 * for fa_bwd_strided, or NULL for contiguous tensors.  Otherwise as fa_bwd,
 * with the same workspace.
 */
int fa_bwd_residual(const void* q, const void* k, const void* v, const void* o,
                    const void* o_res, const float* lse, const void* dO, void* dq, void* dk,
                    void* dv, const fa_strides* strides, int B, int Hq, int Hkv, int Nq, int Nk,
                    int d, int causal, float scale, void* workspace, size_t workspace_bytes,
                    cudaStream_t stream);

/* Stages of fa_bwd, for callers that time or schedule them separately. */
typedef enum {
  FA_BWD_ALL = 0,   /* the whole backward pass (same as fa_bwd) */
  FA_BWD_PRE = 1,   /* D = rowsum(dO * O), LSE copy, dQ accumulator := 0 (in the workspace);
                       GQA / MQA and d = 256: the fp16 copies of dO and V; wide groups:
                       those of Q and K and the forward pass that recomputes D (see fa_bwd) */
  FA_BWD_MAIN = 2,  /* dK, dV written; dQ accumulated into the workspace */
  FA_BWD_DQ = 3     /* dq = scale * dQ accumulator, as bf16 */
} fa_bwd_stage_t;

/*
 * One stage of the backward pass, same arguments and checks as fa_bwd.
 * Issuing FA_BWD_PRE, FA_BWD_MAIN and FA_BWD_DQ in that order on one stream
 * (with the same workspace, untouched in between) is exactly fa_bwd.
 * Returns FA_ERR_INVALID_ARG for an unknown stage.
 */
int fa_bwd_stage(int stage, const void* q, const void* k, const void* v, const void* o,
                 const float* lse, const void* dO, void* dq, void* dk, void* dv, int B, int Hq,
                 int Hkv, int Nq, int Nk, int d, int causal, float scale, void* workspace,
                 size_t workspace_bytes, cudaStream_t stream);

/*
 * Size of the scratch area built into the library for fa_bwd_noalloc: a
 * file-scope device array of this many bytes, which every GPU that loads the
 * library holds until the process exits.
 */
#define FA_NOALLOC_SCRATCH_BYTES (64ull << 20)

/*
 * Backward pass for callers that cannot allocate device memory.  The pages
 * have no counterpart to this entry point; it exists for callers that may
 * not call cudaMalloc themselves, for instance a plug-in inside a host
 * application that owns every device allocation, or code on a
 * latency-critical path where cudaMalloc (which may synchronise the device)
 * is not acceptable.  Same arguments and results as fa_bwd without the
 * workspace: its scratch (the fp32 dQ accumulator, the two fp32 row vectors
 * and, for GQA / MQA groups and d = 256, the fp16 operand copies; all that
 * fa_bwd_workspace_size() counts) lives in the library's built-in array of
 * FA_NOALLOC_SCRATCH_BYTES instead.  The call allocates nothing and calls no allocating routine.
 *  - Problems whose fa_bwd_workspace_size() exceeds FA_NOALLOC_SCRATCH_BYTES
 *    are rejected with FA_ERR_TOO_LARGE before anything is launched.
 *  - Every call looks up the array's device address in the caller's current
 *    device and context (nothing is cached, so a device reset or another
 *    context is followed).  The first lookup on a device may load the
 *    library's device code; make that first call before any stream capture.
 *  - Every call shares the one array per device, and it keeps the last
 *    call's contents; the call re-initialises every part it reads.  Calls
 *    whose kernels overlap on the GPU (e.g. on two streams, or from two host
 *    threads) race on the array: serialise them.
 */
int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                   const void* dO, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Nq,
                   int Nk, int d, int causal, float scale, cudaStream_t stream);

/*
 * Test control for the timeout path (for tests; not for production use).
 * With stall_kv_loads = 1, forward launches on the current device withhold
 * their K/V tiles, so the kernels' bounded pipeline waits expire: each CTA
 * records FA_ERR_DEVICE_TIMEOUT (see fa_device_status), frees its resources
 * and returns without writing o or lse.  wait_limit_seconds > 0 replaces the
 * default 4 s limit of every pipeline wait; 0 restores it.  Synchronous;
 * call fa_debug_inject(0, 0) to return to normal operation.
 */
int fa_debug_inject(int stall_kv_loads, double wait_limit_seconds);

/* Human-readable name of a status code (static string, never NULL). */
const char* fa_status_string(int status);

/*
 * Synchronises `stream`, then reads and clears the current device's kernel
 * status word.  Returns FA_OK, FA_ERR_DEVICE_TIMEOUT (a kernel gave up on a
 * pipeline wait; *where, if non-NULL, receives the code of the wait) or
 * FA_ERR_CUDA.
 */
int fa_device_status(cudaStream_t stream, int* where);

#ifdef __cplusplus
}
#endif
#endif /* FA_H_ */
