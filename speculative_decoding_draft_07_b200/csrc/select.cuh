// Warp-level selection on 64-bit keys (larger key = better), shared by the
// PCTree merge kernels.
#pragma once

#include "common.cuh"

namespace pct {

// Bitonic sort of the warp's 32 keys (one per lane), descending.
__device__ __forceinline__ unsigned long long warp_sort_desc(unsigned long long x, int lane) {
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const unsigned long long y = __shfl_xor_sync(0xffffffffu, x, stride);
      const bool keep_max = ((lane & stride) == 0) == ((lane & size) == 0 || size == 32);
      x = keep_max ? (x > y ? x : y) : (x < y ? x : y);
    }
  }
  return x;
}

// a, b sorted descending across the warp (one key per lane): the 32 largest of
// their union, sorted descending (elementwise max against b reversed is a
// bitonic sequence holding them; one bitonic merge sorts it).
__device__ __forceinline__ unsigned long long warp_merge_top(unsigned long long a,
                                                             unsigned long long b_rev, int lane) {
  unsigned long long x = a > b_rev ? a : b_rev;
#pragma unroll
  for (int stride = 16; stride > 0; stride >>= 1) {
    const unsigned long long y = __shfl_xor_sync(0xffffffffu, x, stride);
    x = ((lane & stride) == 0) ? (x > y ? x : y) : (x < y ? x : y);
  }
  return x;
}

// Candidate key of a beam: larger = better under (score desc, parent position
// asc, token asc); tokens < 2^22, parent positions < 1024.
__device__ __forceinline__ unsigned long long beam_key(float s, int ppos, int tok) {
  return ((unsigned long long)f2ord(s) << 32) | ((unsigned long long)(1023 - ppos) << 22) |
         (unsigned long long)(0x3fffff - tok);
}
__device__ __forceinline__ int beam_key_ppos(unsigned long long x) {
  return 1023 - (int)((x >> 22) & 1023ull);
}
__device__ __forceinline__ int beam_key_tok(unsigned long long x) {
  return 0x3fffff - (int)(x & 0x3fffffull);
}

}  // namespace pct
