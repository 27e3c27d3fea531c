// Seed columns for the PCTree scoring gate: for every (request, depth) row of
// the drafter logits L_d, a handful of columns with large L_d, with L_d and the
// W column at each.
//
// PCTree article (qiita), section on the tree that replaces the chain draft:
// z_d(p) = L_d + Markov(p) for every parent of a depth, so the columns where
// L_d is largest are the natural place to look for each parent's top-k. The
// columns only seed a lower bound (the bound is exact whatever columns are
// chosen), so the search need not be exact either. Three kernels:
//  * drafter_topk_kernel (pct_tree_build): one streaming pass over L (HBM
//    bound); each thread keeps the best 8-column group of its strided share of
//    a slice of the row, the column of that group's maximum is recovered with
//    one reload, each block keeps the ks best of its 256 thread winners and the
//    row's last block merges the slices' picks and gathers their W columns;
//  * seed_columns_kernel (pct_tree_build_seeded): the columns are given (for
//    example the CaDDTree row pass's top-k of the same L); it drops invalid and
//    repeated entries and gathers L and the W columns, from W's transpose when
//    the caller has it (one contiguous row per column);
//  * markov_transpose_kernel: that transpose, once per model.
#include <algorithm>
#include <climits>

#include "common.cuh"
#include "internal.h"
#include "seed.cuh"
#include "select.cuh"

namespace pct {
namespace {

constexpr int kSeedThreads = 256;
constexpr int kSeedParts = 8;   // most slices of a row

template <typename TL>
__device__ __forceinline__ void load8(const TL* p, float (&x)[8]);
template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, float (&x)[8]) {
  const uint4 w = ld_stream16(p);
  x[0] = bf16_lo(w.x); x[1] = bf16_hi(w.x); x[2] = bf16_lo(w.y); x[3] = bf16_hi(w.y);
  x[4] = bf16_lo(w.z); x[5] = bf16_hi(w.z); x[6] = bf16_lo(w.w); x[7] = bf16_hi(w.w);
}
template <>
__device__ __forceinline__ void load8<float>(const float* p, float (&x)[8]) {
  const uint4 a = ld_stream16(p), b = ld_stream16(p + 4);
  x[0] = __uint_as_float(a.x); x[1] = __uint_as_float(a.y);
  x[2] = __uint_as_float(a.z); x[3] = __uint_as_float(a.w);
  x[4] = __uint_as_float(b.x); x[5] = __uint_as_float(b.y);
  x[6] = __uint_as_float(b.z); x[7] = __uint_as_float(b.w);
}

// Elementwise max of two packed bf16 pairs.
__device__ __forceinline__ uint32_t bf16x2_max2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

__device__ __forceinline__ float max8(const float (&x)[8]) {
  return fmaxf(fmax3(x[0], x[1], x[2]), fmax3(fmax3(x[3], x[4], x[5]), x[6], x[7]));
}

// One row of L ([rows][V], V % 8 == 0, 16-byte aligned rows) cut into `parts`
// fixed slices, one block per (row, slice): grid (rows, parts). Each block
// keeps the ks best of its 256 thread winners; with more than one part it
// writes them to pkeys and the last block of the row to finish (a counter per
// row, reset by that block) merges the parts' keys. Nothing waits on another
// block; the counters start at zero (the launcher clears them). Per row: cols[ks] distinct columns, best first (-1 where fewer than
// ks thread winners exist), lval[ks] = L at them, wcol[ks][r_pad] = W[.][col]
// (bf16, zero past r), wmax[ks] = max_j |W[j][col]|.
template <typename TL>
__global__ void __launch_bounds__(kSeedThreads) drafter_topk_kernel(
    int V, int ks, const TL* __restrict__ L, const __nv_bfloat16* __restrict__ W, int r,
    int r_pad, int32_t* __restrict__ cols, float* __restrict__ lval, float* __restrict__ wmax,
    __nv_bfloat16* __restrict__ wcol, unsigned* __restrict__ cnt,
    unsigned long long* __restrict__ pkeys) {
  pdl_wait();
  pdl_trigger();
  __shared__ unsigned long long keys[kSeedThreads];
  __shared__ int s_last;
  const int rowi = (int)blockIdx.x;
  const int parts = (int)gridDim.y, part = (int)blockIdx.y;
  const TL* row = L + (size_t)rowi * V;
  const int Gall = V / 8;
  const int gbeg = (int)((long long)Gall * part / parts);
  const int gend = (int)((long long)Gall * (part + 1) / parts);
  row += (size_t)gbeg * 8;
  const int G = gend - gbeg;
  float best = neg_inf();
  int bg = -1;
  constexpr int U = 8;   // 16-byte groups in flight per thread
  if constexpr (sizeof(TL) == 2) {
    // bf16: every load of a pass issued before any is used, maxima on packed pairs
    for (int g0 = threadIdx.x; g0 < G; g0 += U * kSeedThreads) {
      uint4 q[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int g = g0 + u * kSeedThreads;
        q[u] = g < G ? ld_stream16(row + (size_t)g * 8)
                     : make_uint4(0xff80ff80u, 0xff80ff80u, 0xff80ff80u, 0xff80ff80u);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const uint32_t mx = bf16x2_max2(bf16x2_max2(q[u].x, q[u].y), bf16x2_max2(q[u].z, q[u].w));
        const float gm = fmaxf(bf16_lo(mx), bf16_hi(mx));
        if (gm > best) { best = gm; bg = g0 + u * kSeedThreads; }
      }
    }
  } else
  for (int g0 = threadIdx.x; g0 < G; g0 += U * kSeedThreads) {
    float x[U][8];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int g = g0 + u * kSeedThreads;
      if (g < G) {
        load8<TL>(row + (size_t)g * 8, x[u]);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) x[u][j] = neg_inf();
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const float gm = max8(x[u]);
      if (gm > best) { best = gm; bg = g0 + u * kSeedThreads; }
    }
  }
  int col = -1;
  if (bg >= 0) {
    float x[8];
    load8<TL>(row + (size_t)bg * 8, x);
#pragma unroll
    for (int j = 7; j >= 0; --j)
      if (x[j] == best) col = (gbeg + bg) * 8 + j;
  }
  // the 32 best of the 256 thread winners, sorted: a warp sort each, then
  // warp 0 merges the eight sorted lists
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  {
    unsigned long long x =
        col >= 0 ? ((unsigned long long)f2ord(best) << 32) | (unsigned long long)(0xffffffffu - (uint32_t)col)
                 : 0ull;
    keys[threadIdx.x] = warp_sort_desc(x, lane);
    __syncthreads();
    if (warp == 0) {
      unsigned long long acc = keys[lane];
#pragma unroll
      for (int w = 1; w < kSeedThreads / 32; ++w) acc = warp_merge_top(acc, keys[32 * w + 31 - lane], lane);
      keys[lane] = acc;   // lanes read only keys[32..] after their first read
    }
    __syncthreads();
  }
  if (parts > 1) {
    // publish this part's ks best; the row's last block to arrive merges
    unsigned long long* pk = pkeys + (size_t)rowi * kSeedParts * kSeedMaxK;
    if (threadIdx.x < ks) pk[part * kSeedMaxK + threadIdx.x] = keys[threadIdx.x];
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(&cnt[rowi], 1u) == (unsigned)(parts - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (warp == 0) {
      // every part's sorted list (ks <= 16 entries, padded with zero keys) in
      // registers at once, then merged pairwise
      unsigned long long b[kSeedParts];
#pragma unroll
      for (int q = 0; q < kSeedParts; ++q) {
        const int j = q == 0 ? lane : 31 - lane;
        b[q] = (q < parts && j < ks) ? __ldcg(pk + q * kSeedMaxK + j) : 0ull;
      }
      unsigned long long acc = b[0];
#pragma unroll
      for (int q = 1; q < kSeedParts; ++q)
        if (q < parts) acc = warp_merge_top(acc, b[q], lane);
      keys[lane] = acc;
      if (lane == 0) cnt[rowi] = 0u;   // ready for the next launch
    }
    __syncthreads();
  }
  // W columns of the seed columns: 16 threads per column (a half warp)
  const size_t e0 = (size_t)rowi * ks;
  const int c = threadIdx.x >> 4, sub = threadIdx.x & 15;
  const unsigned long long key = c < ks ? keys[c] : 0ull;
  const int cc = key ? (int)(0xffffffffu - (uint32_t)(key & 0xffffffffull)) : -1;
  float m = 0.f;
  if (cc >= 0) {
    __nv_bfloat16 w[kSeedMaxR / 16];
#pragma unroll
    for (int i = 0; i < kSeedMaxR / 16; ++i) {
      const int j = sub + 16 * i;
      w[i] = j < r ? W[(size_t)j * V + cc] : __float2bfloat16(0.f);
    }
#pragma unroll
    for (int i = 0; i < kSeedMaxR / 16; ++i) {
      const int j = sub + 16 * i;
      if (j < r_pad) wcol[(e0 + c) * r_pad + j] = w[i];
      m = fmaxf(m, fabsf(__bfloat162float(w[i])));
    }
  }
  // max over the column's half warp (every thread takes part)
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (c < ks && sub == 0) {
    cols[e0 + c] = cc;
    lval[e0 + c] = cc >= 0 ? ord2f((uint32_t)(key >> 32)) : neg_inf();
    wmax[e0 + c] = m;
  }
}

// Seed data from given columns, one block per row of L: in[row][ks] are the
// caller's columns; entries outside [0, V) and repeats of an earlier entry of
// the row are dropped (-1), so the kept columns are distinct. W's columns are
// gathered kColLoads strided loads per thread at a time (one 2-byte value of
// each of r rows of W per column); their largest magnitude is a warp max (a
// warp's 32 consecutive entries lie in one column, r_pad being a multiple of
// 32) and one shared-memory max per warp.
constexpr int kColThreads = 128;
constexpr int kColLoads = 16;

// With Wt (W transposed, [V][r_pad], zero past r) a column is one contiguous
// run of r_pad values instead: 16-byte loads, r_pad / 8 per column.
template <typename TL>
__global__ void __launch_bounds__(kColThreads) seed_columns_kernel(
    int V, int ks, const TL* __restrict__ L, const __nv_bfloat16* __restrict__ W,
    const __nv_bfloat16* __restrict__ Wt, int r, int r_pad, const int32_t* __restrict__ in,
    int32_t* __restrict__ cols, float* __restrict__ lval, float* __restrict__ wmax,
    __nv_bfloat16* __restrict__ wcol) {
  pdl_wait();
  pdl_trigger();
  __shared__ int sc[kSeedMaxK];
  __shared__ unsigned smax[kSeedMaxK];
  const int rowi = (int)blockIdx.x;
  const size_t e0 = (size_t)rowi * ks;
  if (threadIdx.x < ks) {
    int c = in[e0 + threadIdx.x];
    if (c < 0 || c >= V) c = -1;
    for (int j = 0; j < (int)threadIdx.x; ++j)
      if (c >= 0 && in[e0 + j] == c) c = -1;   // the first occurrence stays
    sc[threadIdx.x] = c;
    smax[threadIdx.x] = 0u;
  }
  __syncthreads();
  const int n = ks * r_pad;   // a multiple of 32: the loop below is warp-uniform
  __nv_bfloat16* dst = wcol + e0 * r_pad;
  if (Wt) {
    const int cpc = r_pad / 8;   // 16-byte chunks per column
    for (int e = threadIdx.x; e < ks * cpc; e += kColThreads) {
      const int c = e / cpc, j = e - c * cpc;
      const int col = sc[c];
      uint4 q = make_uint4(0u, 0u, 0u, 0u);
      if (col >= 0) q = *reinterpret_cast<const uint4*>(Wt + (size_t)col * r_pad + 8 * j);
      *reinterpret_cast<uint4*>(dst + (size_t)c * r_pad + 8 * j) = q;
      const uint32_t w[4] = {q.x, q.y, q.z, q.w};
      float m = 0.f;
#pragma unroll
      for (int h = 0; h < 4; ++h) m = fmaxf(m, fmaxf(fabsf(bf16_lo(w[h])), fabsf(bf16_hi(w[h]))));
      atomicMax(&smax[c], __float_as_uint(m));
    }
  } else
  for (int e = threadIdx.x; e < n; e += kColLoads * kColThreads) {
    __nv_bfloat16 w[kColLoads];
#pragma unroll
    for (int u = 0; u < kColLoads; ++u) {
      const int f = e + u * kColThreads;
      w[u] = __float2bfloat16(0.f);
      if (f < n) {
        const int c = f / r_pad, j = f - c * r_pad;
        const int col = sc[c];
        if (col >= 0 && j < r) w[u] = W[(size_t)j * V + col];
      }
    }
#pragma unroll
    for (int u = 0; u < kColLoads; ++u) {
      const int f = e + u * kColThreads;
      if (f < n) {
        dst[f] = w[u];
        const unsigned m = __reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(__bfloat162float(w[u]))));
        if ((threadIdx.x & 31) == 0) atomicMax(&smax[f / r_pad], m);
      }
    }
  }
  __syncthreads();
  if (threadIdx.x < ks) {
    const int c = sc[threadIdx.x];
    cols[e0 + threadIdx.x] = c;
    lval[e0 + threadIdx.x] = c >= 0 ? load_f(L + (size_t)rowi * V + c) : neg_inf();
    wmax[e0 + threadIdx.x] = __uint_as_float(smax[threadIdx.x]);
  }
}

}  // namespace

cudaError_t launch_seed_columns(int rows, int V, int ks, int logits_dtype, const void* L,
                                const void* W, const void* Wt, int r, int r_pad,
                                const int32_t* in, int32_t* cols, float* lval, float* wmax,
                                void* wcol, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  if (ks < 1 || ks > kSeedMaxK || r > kSeedMaxR || r_pad > kSeedMaxR || r_pad % 32 != 0)
    return cudaErrorInvalidValue;
  const __nv_bfloat16* Wb = static_cast<const __nv_bfloat16*>(W);
  const __nv_bfloat16* Wtb = static_cast<const __nv_bfloat16*>(Wt);
  __nv_bfloat16* wc = static_cast<__nv_bfloat16*>(wcol);
  TraceScope t(s, "seed_columns");
  if (logits_dtype == PCT_BF16)
    return launch_pdl(seed_columns_kernel<__nv_bfloat16>, dim3((unsigned)rows), dim3(kColThreads),
                      0, s, 1, V, ks, static_cast<const __nv_bfloat16*>(L), Wb, Wtb, r, r_pad, in,
                      cols, lval, wmax, wc);
  return launch_pdl(seed_columns_kernel<float>, dim3((unsigned)rows), dim3(kColThreads), 0, s, 1,
                    V, ks, static_cast<const float*>(L), Wb, Wtb, r, r_pad, in, cols, lval, wmax,
                    wc);
}

// W [r][V] -> Wt [V][r_pad] (bf16, zero past r): a block per 64 columns of W,
// staged through shared memory so that both sides move in 16-byte pieces.
constexpr int kTrCols = 64;
__global__ void __launch_bounds__(256) markov_transpose_kernel(int V, int r, int r_pad,
                                                              const __nv_bfloat16* __restrict__ W,
                                                              __nv_bfloat16* __restrict__ Wt) {
  __shared__ __align__(16) __nv_bfloat16 tile[kSeedMaxR][kTrCols + 8];   // rows of 144 bytes
  const int v0 = (int)blockIdx.x * kTrCols;
  const int nv = min(kTrCols, V - v0);   // a multiple of 8 (V % 8 == 0)
  for (int i = threadIdx.x; i < r * (kTrCols / 8); i += blockDim.x) {
    const int j = i / (kTrCols / 8), c = i - j * (kTrCols / 8);
    if (8 * c < nv)
      *reinterpret_cast<uint4*>(&tile[j][8 * c]) =
          *reinterpret_cast<const uint4*>(W + (size_t)j * V + v0 + 8 * c);
  }
  __syncthreads();
  const int cpc = r_pad / 8;
  for (int i = threadIdx.x; i < nv * cpc; i += blockDim.x) {
    const int cc = i / cpc, jc = i - cc * cpc;
    uint32_t w[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const int j = 8 * jc + 2 * h;
      const uint32_t lo = j < r ? __bfloat16_as_ushort(tile[j][cc]) : 0u;
      const uint32_t hi = j + 1 < r ? __bfloat16_as_ushort(tile[j + 1][cc]) : 0u;
      w[h] = lo | (hi << 16);
    }
    *reinterpret_cast<uint4*>(Wt + (size_t)(v0 + cc) * r_pad + 8 * jc) =
        make_uint4(w[0], w[1], w[2], w[3]);
  }
}

cudaError_t launch_markov_transpose(int V, int r, int r_pad, const void* W, void* Wt,
                                    cudaStream_t s) {
  if (V <= 0 || V % 8 != 0 || r < 1 || r > kSeedMaxR || r_pad < r || r_pad > kSeedMaxR ||
      r_pad % 8 != 0)
    return cudaErrorInvalidValue;
  TraceScope t(s, "markov_transpose");
  markov_transpose_kernel<<<(V + kTrCols - 1) / kTrCols, 256, 0, s>>>(
      V, r, r_pad, static_cast<const __nv_bfloat16*>(W), static_cast<__nv_bfloat16*>(Wt));
  return cudaGetLastError();
}

size_t drafter_topk_scratch(int rows) {
  return ((size_t)rows * sizeof(unsigned) + 255) / 256 * 256 +
         (size_t)rows * kSeedParts * kSeedMaxK * sizeof(unsigned long long);
}

cudaError_t launch_drafter_topk(int rows, int V, int ks, int logits_dtype, const void* L,
                                const void* W, int r, int r_pad, int32_t* cols, float* lval,
                                float* wmax, void* wcol, void* scratch, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  if (ks > kSeedMaxK || r > kSeedMaxR || r_pad > kSeedMaxR || r_pad % 8 != 0 || V % 8 != 0)
    return cudaErrorInvalidValue;
  const __nv_bfloat16* Wb = static_cast<const __nv_bfloat16*>(W);
  __nv_bfloat16* wc = static_cast<__nv_bfloat16*>(wcol);
  // parts of at least two passes of loads each (one when there are few rows),
  // up to kSeedParts per row: the grid then covers the SMs in many short
  // blocks instead of one wave of rows and a tail
  const int passes = V / 8 / (8 * kSeedThreads);
  int parts = std::max(1, std::min(kSeedParts, passes / 2));
  if ((long long)rows * parts < 2LL * num_sms()) parts = std::max(1, std::min(kSeedParts, passes));
  unsigned* cnt = static_cast<unsigned*>(scratch);
  unsigned long long* pkeys = reinterpret_cast<unsigned long long*>(
      static_cast<char*>(scratch) + ((size_t)rows * sizeof(unsigned) + 255) / 256 * 256);
  if (parts > 1) {
    cudaError_t e = cudaMemsetAsync(cnt, 0, sizeof(unsigned) * (size_t)rows, s);
    if (e != cudaSuccess) return e;
  }
  TraceScope t(s, "drafter_topk");
  const dim3 grid((unsigned)rows, (unsigned)parts);
  if (logits_dtype == PCT_BF16)
    return launch_pdl(drafter_topk_kernel<__nv_bfloat16>, grid, dim3(kSeedThreads), 0, s, 1, V, ks,
                      static_cast<const __nv_bfloat16*>(L), Wb, r, r_pad, cols, lval, wmax, wc, cnt,
                      pkeys);
  return launch_pdl(drafter_topk_kernel<float>, grid, dim3(kSeedThreads), 0, s, 1, V, ks,
                    static_cast<const float*>(L), Wb, r, r_pad, cols, lval, wmax, wc, cnt, pkeys);
}

}  // namespace pct
