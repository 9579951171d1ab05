// Block-sparse attention (QbitAI FA1 article, results section: block-sparse
// FlashAttention is faster than every other attention implementation at all
// sequence lengths).  The caller's block mask holds one byte per
// MASK_BLOCK x MASK_BLOCK (query, key) block, row-major
// [ceil(Nq / MASK_BLOCK)][ceil(Nk / MASK_BLOCK)], shared by every batch and
// head; a zero entry removes the block from the score matrix (its scores
// count as -inf) and the kernels neither load nor compute it.
//
// Mask rows are read 32 entries at a time (independent byte loads packed
// into a bit word), so a thread that issues TMA copies does not wait on a
// global load per block.
#pragma once
#include <cstdint>

namespace fa {

constexpr int MASK_BLOCK = 128;
constexpr int MASK_NONE = 1 << 30;   // "no further kept block"

// Bit i set iff byte i of x is nonzero.
__device__ __forceinline__ uint32_t nonzero_bytes(uint32_t x) {
  const uint32_t t = (((x & 0x7F7F7F7Fu) + 0x7F7F7F7Fu) | x) & 0x80808080u;
  return ((t >> 7) & 1u) | ((t >> 14) & 2u) | ((t >> 21) & 4u) | ((t >> 28) & 8u);
}

// Entries [32 w, 32 w + 32) of a mask row that lie below n, one bit each.
// The bytes are fetched as the (at most three) aligned 16-byte chunks that
// hold them, with independent vector loads, and the chunks' other bytes are
// discarded.  The mask starts on a 16-byte boundary and its allocation
// extends to the next multiple of 16 bytes (the C ABI requires both), so
// every chunk lies inside the caller's allocation.
__device__ __forceinline__ uint32_t mask_word(const uint8_t* row, int w, int n) {
  const int j0 = w * 32;
  const int cnt = min(32, n - j0);                   // entries wanted
  if (cnt <= 0) return 0u;
  const uintptr_t a = reinterpret_cast<uintptr_t>(row + j0);
  const uint4* base = reinterpret_cast<const uint4*>(a & ~uintptr_t(15));
  const int sh = int(a & 15u);
  const int chunks = (sh + cnt + 15) >> 4;           // 1 to 3
  uint64_t all = 0u;
#pragma unroll
  for (int c = 0; c < 3; ++c) {
    if (c < chunks) {
      const uint4 v = __ldg(base + c);
      const uint32_t b = nonzero_bytes(v.x) | (nonzero_bytes(v.y) << 4) |
                         (nonzero_bytes(v.z) << 8) | (nonzero_bytes(v.w) << 12);
      all |= uint64_t(b) << (16 * c);
    }
  }
  uint32_t r = uint32_t(all >> sh);
  if (cnt < 32) r &= (1u << cnt) - 1u;
  return r;
}

// Kept entries of a mask row in [0, n).
__device__ __forceinline__ int mask_count(const uint8_t* row, int n) {
  int c = 0;
  for (int w = 0; w * 32 < n; ++w) c += __popc(mask_word(row, w, n));
  return c;
}

// A walk over the kept entries of one mask row, in increasing order.
struct RowWalk {
  const uint8_t* row;
  int n;              // entries in range: [0, n)
  int w;              // word held in `bits` (-1: none)
  uint32_t bits;

  __device__ __forceinline__ void init(const uint8_t* r, int n_) {
    row = r;
    n = n_;
    w = -1;
    bits = 0u;
  }
  // Smallest kept entry >= j, or MASK_NONE.
  __device__ __forceinline__ int next(int j) {
    while (j < n) {
      const int ww = j >> 5;
      if (ww != w) {
        w = ww;
        bits = mask_word(row, ww, n);
      }
      const uint32_t m = bits & (0xFFFFFFFFu << (j & 31));
      if (m) return (ww << 5) + __ffs(m) - 1;
      j = (ww + 1) << 5;
    }
    return MASK_NONE;
  }
};

// A walk over the union of two mask rows (row0 and row0 + ld, with n0 and
// n1 entries in range), in increasing order; f0 / f1 report which rows keep
// the returned entry.
struct PairWalk {
  const uint8_t* row0;
  int ld, n0, n1, w;
  uint32_t b0, b1;

  __device__ __forceinline__ void init(const uint8_t* r0, int ld_, int n0_, int n1_) {
    row0 = r0;
    ld = ld_;
    n0 = n0_;
    n1 = n1_;
    w = -1;
    b0 = b1 = 0u;
  }
  __device__ __forceinline__ int next(int j, bool& f0, bool& f1) {
    const int n = max(n0, n1);
    while (j < n) {
      const int ww = j >> 5;
      if (ww != w) {
        w = ww;
        b0 = mask_word(row0, ww, n0);
        b1 = mask_word(row0 + ld, ww, n1);
      }
      const uint32_t m = (b0 | b1) & (0xFFFFFFFFu << (j & 31));
      if (m) {
        const int i = __ffs(m) - 1;
        f0 = (b0 >> i) & 1u;
        f1 = (b1 >> i) & 1u;
        return (ww << 5) + i;
      }
      j = (ww + 1) << 5;
    }
    f0 = f1 = false;
    return MASK_NONE;
  }
  // Entries kept by row 0 (c0), by row 1 (c1) and by either (returned).
  __device__ __forceinline__ int counts(int& c0, int& c1) const {
    int cu = 0;
    c0 = c1 = 0;
    for (int ww = 0; ww * 32 < max(n0, n1); ++ww) {
      const uint32_t x = mask_word(row0, ww, n0), y = mask_word(row0 + ld, ww, n1);
      c0 += __popc(x);
      c1 += __popc(y);
      cu += __popc(x | y);
    }
    return cu;
  }
};

}  // namespace fa
