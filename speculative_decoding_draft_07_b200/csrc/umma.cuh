// Device and host helpers of the tcgen05 scoring kernels: mbarriers with
// bounded waits, TMA tile loads, shared-memory matrix descriptors, MMA issue
// and commit, split TMEM loads, the epilogue's chunk reductions, and 2D bf16
// tensor maps (encoded through the driver entry point, no libcuda link).
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace pct {
namespace {

constexpr long long kTimeoutCycles = 4000000000ll;   // ~2 s at 2 GHz

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t addr, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok) : "r"(addr), "r"(parity) : "memory");
  return ok != 0;
}
// Bounded wait. Gives up when another role has aborted or after the timeout.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                         int32_t* err) {
  const uint32_t addr = smem_u32(bar);
  if (mbar_try_wait(addr, parity)) return true;
  const long long t0 = clock64();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(addr, parity)) return true;
    if ((it & 255u) == 0u) {
      if (*abort_flag) return false;
      if (clock64() - t0 > kTimeoutCycles) {
        *abort_flag = 1;
        atomicExch(err, 1);
        return false;
      }
    }
  }
}
// Bounded wait used while draining after an abort (no abort check).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint32_t addr = smem_u32(bar);
  const long long t0 = clock64();
  while (!mbar_try_wait(addr, parity))
    if (clock64() - t0 > kTimeoutCycles) return;
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle, sm_100 layout (version 1).
// layout: 2 = 128-byte swizzle, 6 = 32-byte swizzle.
__device__ __forceinline__ uint64_t make_desc(uint32_t addr, uint32_t lbo, uint32_t sbo,
                                              uint32_t layout = 2) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)(layout & 7u) << 61;
  return d;
}
__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Split forms: the load is issued and its registers are consumed only after
// tmem_wait() on the same array, whose asm takes every register as an in-out
// operand so that no use can be scheduled above the wait. Between the two the
// thread does other work (the previous chunk).
__device__ __forceinline__ void tmem_issue(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait(uint32_t (&r)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                 "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                 "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15])
               :
               : "memory");
}
__device__ __forceinline__ void tmem_issue(uint32_t taddr, uint32_t (&r)[32]) {
  tmem_issue(taddr, *reinterpret_cast<uint32_t(*)[16]>(&r[0]));
  tmem_issue(taddr + 16, *reinterpret_cast<uint32_t(*)[16]>(&r[16]));
}
__device__ __forceinline__ void tmem_wait(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                 "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                 "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]),
                 "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
                 "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]),
                 "+r"(r[30]), "+r"(r[31])
               :
               : "memory");
}

__device__ __forceinline__ void tmem_issue(uint32_t taddr, uint32_t (&r)[64]) {
  tmem_issue(taddr, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
  tmem_issue(taddr + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
}
// (the second wait finds no load outstanding; it only fences the upper half)
__device__ __forceinline__ void tmem_wait(uint32_t (&r)[64]) {
  tmem_wait(*reinterpret_cast<uint32_t(*)[32]>(&r[0]));
  tmem_wait(*reinterpret_cast<uint32_t(*)[32]>(&r[32]));
}

__device__ __forceinline__ uint4 ld_shared16(uint32_t addr) {
  uint4 r;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(addr));
  return r;
}


// 2^t of a pair on the FMA pipe (no SFU). t is clamped below at -125 (the
// smaller terms of a softmax sum underflow anyway); t <= 92 holds for every
// caller (values exceed the running reference by at most 64 nats). Cody-Waite
// style split t = n + f with n = round(t), taken from the low mantissa bits of
// t + 1.5 * 2^23, and f in [-1/2, 1/2]; 2^f by the degree-5 polynomial that
// interpolates 2^f at the six Chebyshev nodes of [-1/2, 1/2] (coefficients
// rounded to fp32; relative error below 1.1e-7, about 2.2e-7 with the fp32
// Horner evaluation); n is added to the exponent field.
constexpr float kExp2C0 = 1.00000012f, kExp2C1 = 0.693147182f, kExp2C2 = 0.240221068f,
                kExp2C3 = 0.0555035695f, kExp2C4 = 0.00967603177f, kExp2C5 = 0.00133908633f;
__device__ __forceinline__ float2 soft_exp2x2(float2 t) {
  constexpr float kRound = 12582912.0f;   // 1.5 * 2^23
  t.x = fmaxf(t.x, -125.0f);
  t.y = fmaxf(t.y, -125.0f);
  const float2 r = f2_add(t, make_float2(kRound, kRound));
  const float2 n = f2_add(r, make_float2(-kRound, -kRound));
  const float2 f = f2_fma(n, make_float2(-1.0f, -1.0f), t);
  float2 q = f2_fma(make_float2(kExp2C5, kExp2C5), f, make_float2(kExp2C4, kExp2C4));
  q = f2_fma(q, f, make_float2(kExp2C3, kExp2C3));
  q = f2_fma(q, f, make_float2(kExp2C2, kExp2C2));
  q = f2_fma(q, f, make_float2(kExp2C1, kExp2C1));
  q = f2_fma(q, f, make_float2(kExp2C0, kExp2C0));
  return make_float2(__uint_as_float(__float_as_uint(q.x) + (__float_as_uint(r.x) << 23)),
                     __uint_as_float(__float_as_uint(q.y) + (__float_as_uint(r.y) << 23)));
}

// sum_j 2^(x_j log2 e - m log2 e) over N values, arguments and partial sums
// in fp32 pairs. The last SOFT values of the chunk take soft_exp2x2 (FMA
// pipe), the rest the SFU, so that the two units share the work.
template <int N, int SOFT = 0>
__device__ __forceinline__ float chunk_exp_sum(const float (&x)[N], float m) {
  static_assert(SOFT % 2 == 0 && SOFT <= N, "soft share in pairs");
  const float2 l2e = make_float2(kLog2e, kLog2e);
  const float2 nmb = make_float2(-m * kLog2e, -m * kLog2e);
  // four independent partial sums (pairs) keep several SFU results in flight
  float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                   make_float2(0.f, 0.f)};
#pragma unroll
  for (int j = 0; j < N; j += 2) {
    const float2 a = f2_fma(make_float2(x[j], x[j + 1]), l2e, nmb);
    float2 e;
    if (j >= N - SOFT) e = soft_exp2x2(a);
    else e = make_float2(ex2(a.x), ex2(a.y));
    acc[(j >> 1) & 3] = f2_add(acc[(j >> 1) & 3], e);
  }
  const float2 t = f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3]));
  return t.x + t.y;
}

// max of N values as a tree of three-input maxima
template <int N>
__device__ __forceinline__ float chunk_max(const float (&x)[N]) {
  float t[(N + 2) / 3];
#pragma unroll
  for (int j = 0; j < N / 3; ++j) t[j] = fmax3(x[3 * j], x[3 * j + 1], x[3 * j + 2]);
  if (N % 3 == 1) t[N / 3] = x[N - 1];
  if (N % 3 == 2) t[N / 3] = fmaxf(x[N - 2], x[N - 1]);
  constexpr int T = (N + 2) / 3;
  float u[(T + 2) / 3];
#pragma unroll
  for (int j = 0; j < T / 3; ++j) u[j] = fmax3(t[3 * j], t[3 * j + 1], t[3 * j + 2]);
  if (T % 3 == 1) u[T / 3] = t[T - 1];
  if (T % 3 == 2) u[T / 3] = fmaxf(t[T - 2], t[T - 1]);
  constexpr int U = (T + 2) / 3;
  float r = u[0];
#pragma unroll
  for (int j = 1; j < U; ++j) r = fmaxf(r, u[j]);
  return r;
}

// N drafter logits of one row starting at column col0 (col0 % N == 0, N a
// multiple of 8). Columns at or past V read as -inf.
template <typename TL, int N>
__device__ __forceinline__ void load_logits(const TL* row, int col0, int V, float (&x)[N]) {
  if constexpr (sizeof(TL) == 4) {
#pragma unroll
    for (int j = 0; j < N; ++j) {
      const int c = col0 + j;
      x[j] = c < V ? load_f(row + c) : neg_inf();
    }
  } else {
#pragma unroll
    for (int q = 0; q < N / 8; ++q) {
      const int c = col0 + q * 8;
      if (c < V) {   // V % 8 == 0: a 16-byte group is entirely in or out
        const uint4 w = __ldg(reinterpret_cast<const uint4*>(row + c));
        x[q * 8 + 0] = bf16_lo(w.x); x[q * 8 + 1] = bf16_hi(w.x);
        x[q * 8 + 2] = bf16_lo(w.y); x[q * 8 + 3] = bf16_hi(w.y);
        x[q * 8 + 4] = bf16_lo(w.z); x[q * 8 + 5] = bf16_hi(w.z);
        x[q * 8 + 6] = bf16_lo(w.w); x[q * 8 + 7] = bf16_hi(w.w);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) x[q * 8 + j] = neg_inf();
      }
    }
  }
}

// ---- host: tensor maps ------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// 2D bf16 tensor map: `inner` contiguous elements per row, rows `row_bytes`
// apart (0: dense), 128-byte swizzle or none.
bool encode_2d_bf16(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                    uint32_t box_inner, uint32_t box_outer, uint64_t row_bytes = 0,
                    bool swizzle128 = true) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes ? row_bytes : inner * 2};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace
}  // namespace pct
