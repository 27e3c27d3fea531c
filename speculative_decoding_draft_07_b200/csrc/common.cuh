// Device helpers shared by the kernels of libpctree (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/pctree.h"

namespace pct {

constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float neg_inf() { return __int_as_float(0xff800000); }

// Programmatic dependent launch. A kernel started by launch_pdl may begin while
// the previous kernel of its stream is still running: pdl_wait() returns once
// that kernel has completed and its memory operations are visible, so it comes
// before every global-memory access of the kernel (reads and writes). Only
// set-up that touches shared memory, TMEM or the kernel's parameters runs
// before it. pdl_trigger() lets the next kernel start launching; its own
// pdl_wait() still waits for this one to complete. Every launch_pdl kernel
// calls pdl_wait() then pdl_trigger() at its start, so a dependent grid can
// start only once every block of this grid is resident or done: its early
// blocks never hold resources that blocks of this grid still need.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Launch with programmatic stream serialization allowed (and a cluster shape
// when cluster_x > 1).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t s, unsigned cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  int n = 1;
  if (cluster_x > 1) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cluster_x;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    n = 2;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
  if (e != cudaSuccess) (void)cudaGetLastError();
  return e;
}

// 2^x on the special-function unit (hardware approximation, flushes subnormal
// results to zero; relative error a few ulp), used for the softmax sums.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Order-preserving map float -> uint32 (larger float -> larger key). -0 is
// folded onto +0 first so that equal values give equal keys.
__device__ __forceinline__ uint32_t f2ord(float f) {
  uint32_t u = __float_as_uint(f + 0.0f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float ord2f(uint32_t o) {
  uint32_t u = (o & 0x80000000u) ? (o & 0x7fffffffu) : ~o;
  return __uint_as_float(u);
}

// Packed fp32 pairs (sm_100: add/fma on .f32x2, each lane IEEE round to
// nearest even) and the three-input max.
__device__ __forceinline__ float2 f2_add(float2 a, float2 b) {
  float2 r;
  asm("{\n\t.reg .b64 a_, b_, r_;\n\tmov.b64 a_, {%2, %3};\n\tmov.b64 b_, {%4, %5};\n\t"
      "add.rn.f32x2 r_, a_, b_;\n\tmov.b64 {%0, %1}, r_;\n\t}"
      : "=f"(r.x), "=f"(r.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}
__device__ __forceinline__ float2 f2_fma(float2 a, float2 b, float2 c) {
  float2 r;
  asm("{\n\t.reg .b64 a_, b_, c_, r_;\n\tmov.b64 a_, {%2, %3};\n\tmov.b64 b_, {%4, %5};\n\t"
      "mov.b64 c_, {%6, %7};\n\tfma.rn.f32x2 r_, a_, b_, c_;\n\tmov.b64 {%0, %1}, r_;\n\t}"
      : "=f"(r.x), "=f"(r.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return r;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Exact bf16 -> fp32 widening of a raw 16-bit pattern.
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

template <typename T> __device__ __forceinline__ float load_f(const T* p);
template <> __device__ __forceinline__ float load_f<float>(const float* p) { return *p; }
template <> __device__ __forceinline__ float load_f<__nv_bfloat16>(const __nv_bfloat16* p) {
  return bf16_lo(*reinterpret_cast<const uint16_t*>(p));
}

// Streaming 16-byte load that does not allocate in L1.
__device__ __forceinline__ uint4 ld_stream16(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

// 8-byte shared-memory store/load that other warps observe as one unit.
__device__ __forceinline__ void st_shared_vol2(float2* p, float a, float b) {
  asm volatile("st.volatile.shared.v2.f32 [%0], {%1, %2};" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(p))),
               "f"(a), "f"(b)
               : "memory");
}
__device__ __forceinline__ float2 ld_shared_vol2(const float2* p) {
  float2 r;
  asm volatile("ld.volatile.shared.v2.f32 {%0, %1}, [%2];"
               : "=f"(r.x), "=f"(r.y)
               : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(p)))
               : "memory");
  return r;
}

// Key order used by every top-k in this library: larger value first, then
// lower index. Returns true when (va, ia) goes before (vb, ib).
__device__ __forceinline__ bool better(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

// Sorted (descending by `better`) top-k list kept in registers. K is the
// compile-time capacity and k <= K the live length: the k live entries sit in
// the LAST k slots, behind K - k (+inf, -1) markers that nothing displaces, so
// the admission threshold is always slot K - 1. Every index is a compile-time
// constant (a runtime k-th index would force the array into local memory).
// Empty live slots hold (-inf, INT_MAX) so that -inf values still enter in
// index order. finish(k) moves the live entries to slots 0..k-1.
template <int K>
struct TopK {
  float v[K];
  int i[K];
  __device__ __forceinline__ void init(int k) {
#pragma unroll
    for (int j = 0; j < K; ++j) {
      const bool marker = j < K - k;
      v[j] = marker ? __int_as_float(0x7f800000) : neg_inf();
      i[j] = marker ? -1 : 0x7fffffff;
    }
  }
  // admission threshold: the k-th live entry
  __device__ __forceinline__ float tv() const { return v[K - 1]; }
  __device__ __forceinline__ int ti() const { return i[K - 1]; }
  __device__ __forceinline__ bool admits(float z, int idx) const {
    return better(z, idx, v[K - 1], i[K - 1]);
  }
  // Bubble the new element through the sorted list; the last one falls out.
  __device__ __forceinline__ void insert(float z, int idx) {
    float cz = z; int ci = idx;
#pragma unroll
    for (int j = 0; j < K; ++j) {
      const bool sw = better(cz, ci, v[j], i[j]);
      const float tv_ = v[j]; const int ti_ = i[j];
      v[j] = sw ? cz : tv_; i[j] = sw ? ci : ti_;
      cz = sw ? tv_ : cz; ci = sw ? ti_ : ci;
    }
  }
  // Remove the head (shift left).
  __device__ __forceinline__ void pop() {
#pragma unroll
    for (int j = 0; j + 1 < K; ++j) { v[j] = v[j + 1]; i[j] = i[j + 1]; }
    v[K - 1] = neg_inf(); i[K - 1] = 0x7fffffff;
  }
  __device__ __forceinline__ void finish(int k) {
    for (int s = 0; s < K - k; ++s) pop();
  }
};

// Online log-sum-exp state: sum = sum_j exp(z_j - m).
struct LseState {
  float m, s;
  __device__ __forceinline__ void init() { m = neg_inf(); s = 0.f; }
};
__device__ __forceinline__ void lse_combine(float& m, float& s, float m2, float s2) {
  if (m2 == neg_inf()) return;
  if (m == neg_inf()) { m = m2; s = s2; return; }
  if (m2 > m) { s = s * ex2((m - m2) * kLog2e) + s2; m = m2; }
  else        { s = s + s2 * ex2((m2 - m) * kLog2e); }
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ int warp_min_i(int x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = min(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ int warp_sum_i(int x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}
__device__ __forceinline__ unsigned long long warp_max_u64(unsigned long long x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    unsigned long long y = __shfl_xor_sync(0xffffffffu, x, o);
    x = y > x ? y : x;
  }
  return x;
}
// Warp-wide best (value desc, index asc).
__device__ __forceinline__ void warp_best(float& v, int& i) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    float v2 = __shfl_xor_sync(0xffffffffu, v, o);
    int i2 = __shfl_xor_sync(0xffffffffu, i, o);
    if (better(v2, i2, v, i)) { v = v2; i = i2; }
  }
}

}  // namespace pct
