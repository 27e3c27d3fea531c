// Seed columns for the PCTree scoring gate: for every (request, depth) row of
// the drafter logits L_d, a handful of columns with large L_d.
//
// PCTree article (qiita), section on the tree that replaces the chain draft:
// z_d(p) = L_d + Markov(p) for every parent of a depth, so the columns where
// L_d is largest are the natural place to look for each parent's top-k. The
// columns found here only seed a lower bound (the bound is exact whatever
// columns are chosen), so the search need not be exact either: each thread
// keeps the best 8-column group of its strided share of the row, the column of
// that group's maximum is recovered with one reload, and the block keeps the
// ks best of its 256 thread winners. One streaming pass over L (HBM bound).
#include <climits>

#include "common.cuh"
#include "internal.h"
#include "seed.cuh"

namespace pct {
namespace {

constexpr int kSeedThreads = 256;

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

__device__ __forceinline__ uint32_t seed_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void seed_cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
// Descending bitonic sort of keys[0..P) by the block (P a power of two).
__device__ void seed_sort_desc(unsigned long long* keys, int P) {
  for (int size = 2; size <= P; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const int t = threadIdx.x;
      if (t < P / 2) {
        const int lo = 2 * t - (t & (stride - 1));
        const int hi = lo + stride;
        const bool desc = ((lo & size) == 0);
        const unsigned long long a = keys[lo], b = keys[hi];
        if (desc ? (a < b) : (a > b)) { keys[lo] = b; keys[hi] = a; }
      }
      __syncthreads();
    }
  }
}

// One row of L ([rows][V], V % 8 == 0, 16-byte aligned rows) per block, or per
// cluster of CL blocks when there are few rows (each block scans a fixed
// 1/CL of the row; rank 0 merges the blocks' candidates through distributed
// shared memory). Per row: cols[ks] distinct columns, best first (-1 where
// fewer than ks thread winners exist), lval[ks] = L at them,
// wcol[ks][r_pad] = W[.][col] (bf16, zero past r), wmax[ks] = max_j |W[j][col]|.
template <typename TL, int CL>
__global__ void __launch_bounds__(kSeedThreads) drafter_topk_kernel(
    int V, int ks, const TL* __restrict__ L, const __nv_bfloat16* __restrict__ W, int r,
    int r_pad, int32_t* __restrict__ cols, float* __restrict__ lval, float* __restrict__ wmax,
    __nv_bfloat16* __restrict__ wcol) {
  __shared__ unsigned long long keys[kSeedThreads];
  const int rowi = (int)blockIdx.x / CL;
  const uint32_t rank = CL > 1 ? seed_ctarank() : 0u;
  const TL* row = L + (size_t)rowi * V;
  const int Gall = V / 8;
  const int gbeg = (int)((long long)Gall * rank / CL), gend = (int)((long long)Gall * (rank + 1) / CL);
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
  keys[threadIdx.x] =
      col >= 0 ? ((unsigned long long)f2ord(best) << 32) | (unsigned long long)(0xffffffffu - (uint32_t)col)
               : 0ull;
  __syncthreads();
  // descending bitonic sort of the 256 thread winners
  seed_sort_desc(keys, kSeedThreads);
  if constexpr (CL > 1) {
    // rank 0 takes every block's ks best (distinct columns) and sorts them
    __shared__ unsigned long long others[CL * kSeedMaxK];
    seed_cluster_sync();
    if (rank == 0) {
      for (int i = threadIdx.x; i < (CL - 1) * ks; i += blockDim.x) {
        const uint32_t src = 1u + (uint32_t)(i / ks);
        uint32_t a;
        asm volatile("mapa.shared::cluster.u32 %0, %1, %2;"
                     : "=r"(a) : "r"((uint32_t)__cvta_generic_to_shared(keys + (i % ks))), "r"(src));
        unsigned long long v;
        asm volatile("ld.shared::cluster.u64 %0, [%1];" : "=l"(v) : "r"(a) : "memory");
        others[i] = v;
      }
    }
    seed_cluster_sync();   // no block leaves while rank 0 reads its keys
    if (rank != 0) return;
    for (int i = threadIdx.x; i < (CL - 1) * ks; i += blockDim.x) keys[ks + i] = others[i];
    int P = 1;
    while (P < CL * ks) P <<= 1;
    for (int i = CL * ks + threadIdx.x; i < P; i += blockDim.x) keys[i] = 0ull;
    __syncthreads();
    seed_sort_desc(keys, P);
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

}  // namespace

cudaError_t launch_drafter_topk(int rows, int V, int ks, int logits_dtype, const void* L,
                                const void* W, int r, int r_pad, int32_t* cols, float* lval,
                                float* wmax, void* wcol, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  if (ks > kSeedMaxK || r > kSeedMaxR || r_pad > kSeedMaxR || r_pad % 8 != 0 || V % 8 != 0)
    return cudaErrorInvalidValue;
  TraceScope t(s, "drafter_topk");
  const __nv_bfloat16* Wb = static_cast<const __nv_bfloat16*>(W);
  __nv_bfloat16* wc = static_cast<__nv_bfloat16*>(wcol);
  // few rows: a cluster of 8 blocks per row keeps more of the GPU streaming
  if ((long long)rows * 8 <= 2LL * num_sms() && V / 8 >= 8 * kSeedThreads) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)rows * 8);
    cfg.blockDim = dim3(kSeedThreads);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 8;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e;
    if (logits_dtype == PCT_BF16)
      e = cudaLaunchKernelEx(&cfg, drafter_topk_kernel<__nv_bfloat16, 8>, V, ks,
                             static_cast<const __nv_bfloat16*>(L), Wb, r, r_pad, cols, lval, wmax, wc);
    else
      e = cudaLaunchKernelEx(&cfg, drafter_topk_kernel<float, 8>, V, ks, static_cast<const float*>(L),
                             Wb, r, r_pad, cols, lval, wmax, wc);
    if (e != cudaSuccess) (void)cudaGetLastError();
    return e;
  }
  if (logits_dtype == PCT_BF16)
    drafter_topk_kernel<__nv_bfloat16, 1><<<rows, kSeedThreads, 0, s>>>(
        V, ks, static_cast<const __nv_bfloat16*>(L), Wb, r, r_pad, cols, lval, wmax, wc);
  else
    drafter_topk_kernel<float, 1><<<rows, kSeedThreads, 0, s>>>(
        V, ks, static_cast<const float*>(L), Wb, r, r_pad, cols, lval, wmax, wc);
  return cudaGetLastError();
}

}  // namespace pct
