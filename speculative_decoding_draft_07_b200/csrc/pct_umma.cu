// Batched parent scoring on the tcgen05 tensor cores (bf16 Markov parameters).
//
// PCTree article (qiita), section on the chain draft's weakness and the tree
// built in its place: for every frontier parent p of a depth, in one batched
// call, z_d(p) = L_d + Markov(p), followed by the softmax over the vocabulary
// and the parent's local top-k. With the rank-r stand-in Markov(p) = E[p] . W
// the batched call is the contraction Eg[M][r] . W[r][V] (Eg = E rows of the
// parents' tokens), the only dense contraction on the path.
//
// Design (one CTA per SM, 320 threads):
//  * warp 0, one thread: TMA producer. The CTA's parent rows (up to 256 = two
//    128-row UMMA tiles) of Eg are loaded once (K-major, 128-byte swizzle);
//    W is streamed through a 4-stage ring of [64 K][128 V] tiles (V-major,
//    128-byte swizzle), each W tile serving both row tiles.
//  * warp 1, one thread: issues tcgen05.mma (kind::f16, bf16 x bf16 -> fp32,
//    M=128, N=128, K=16) into a double-buffered TMEM accumulator (2 row tiles
//    x 2 buffers x 128 columns = all 512 columns), commits each ring slot back
//    to the producer and each finished accumulator to the epilogue.
//  * warps 2..9: epilogue. Warp w reads TMEM lane quarter (w % 4), so every
//    thread owns one parent row (with 16 epilogue warps two warps share a
//    quarter, each taking half of every N-tile's columns, and the halves are
//    folded at the end; 8 measured faster); it loads 32 accumulator columns at a time,
//    adds the row's drafter logits L_d (bf16, shared by the request's parents,
//    served from L2), and keeps an online log-sum-exp (chunk max, one rescale,
//    32 exp2 on the SFU) and a register top-k admitted by a threshold test.
//    The Markov product never reaches HBM.
// Each CTA covers a contiguous V-slice; its per-row (max, sum, top-k) partial
// goes to global memory and the merge kernel folds the slices.
// Every mbarrier wait is bounded: on expiry the CTA raises an abort flag, sets
// the device error word, drains its own TMA loads and MMAs and frees TMEM.
#include <cuda.h>

#include <algorithm>
#include <climits>

#include "common.cuh"
#include "internal.h"

namespace pct {

cudaError_t launch_score_simt(const ScoreArgs& a, cudaStream_t s);

namespace {

constexpr int BM = 128;                  // UMMA M (rows per tile)
constexpr int BN = 128;                  // UMMA N (vocabulary columns per tile)
constexpr int BK = 64;                   // K per ring slot: one 128-byte swizzle row of bf16
constexpr int STAGES = 4;
constexpr int KBMAX = 4;                 // r_pad <= 256
constexpr int NSUBMAX = 2;               // row tiles per CTA
constexpr int A_TILE_BYTES = BM * BK * 2;        // 16 KB
constexpr int B_STAGE_BYTES = BK * BN * 2;       // 16 KB
constexpr int NUM_EPI_WARPS = 16;                // 1 or 2 per (row tile, TMEM lane quarter)
constexpr int SPLIT = NUM_EPI_WARPS / 8;         // warps sharing a lane quarter: column parts
constexpr int CH = SPLIT == 2 ? 16 : 32;         // accumulator columns per TMEM load
constexpr int THREADS = 64 + 32 * NUM_EPI_WARPS; // producer + MMA warps + epilogue
constexpr int TMEM_COLS = 512;
constexpr int LBMAX = 64;                        // request rows of L_d staged per N-tile
constexpr int L_SLOT_BYTES = 2 * 64 * LBMAX * 2; // two [LB][64] bf16 boxes = 16 KB
constexpr size_t SMEM_BYTES = 1024 + (size_t)NSUBMAX * KBMAX * A_TILE_BYTES +
                              (size_t)STAGES * B_STAGE_BYTES + 2 * (size_t)L_SLOT_BYTES + 256;
constexpr long long kTimeoutCycles = 4000000000ll;   // ~2 s at 2 GHz

// Instruction descriptor, kind::f16: D = f32, A = B = bf16, A K-major,
// B MN-major (W is [r][V], V contiguous), N = 128, M = 128.
constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | (0u << 15) | (1u << 16) |
                           ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);

struct UmmaParams {
  int M, nsub, rows_per_cta, n_par, V, kblocks, S, tiles_total, k;
  int LB;          // L_d rows staged per N-tile (requests a CTA touches, <= LBMAX)
  const void* L;
  long long L_req_stride;
  float2* pms;
  float* pval;
  int32_t* pidx;
  int32_t* err;
  uint32_t* row_thr;   // [M] best published k-th value per row (ordered key, 0 = none)
};

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
__device__ __forceinline__ uint64_t make_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
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
// 16 consecutive fp32 accumulator columns of this thread's TMEM lane (load
// and wait in one asm statement).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld(uint32_t taddr, uint32_t (&r)[16]) { tmem_ld16(taddr, r); }
__device__ __forceinline__ void tmem_ld(uint32_t taddr, uint32_t (&r)[32]);

// 32 consecutive fp32 accumulator columns of this thread's TMEM lane. The
// load and its wait sit in one asm statement so that no use of the outputs can
// be scheduled before the data has arrived.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ uint4 ld_shared16(uint32_t addr) {
  uint4 r;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(addr));
  return r;
}

__device__ __forceinline__ void tmem_ld(uint32_t taddr, uint32_t (&r)[32]) { tmem_ld32(taddr, r); }

// sum_j 2^(x_j log2 e - m log2 e) over N values, arguments and partial sums
// in fp32 pairs.
template <int N>
__device__ __forceinline__ float chunk_exp_sum(const float (&x)[N], float m) {
  const float2 l2e = make_float2(kLog2e, kLog2e);
  const float2 nmb = make_float2(-m * kLog2e, -m * kLog2e);
  float2 sa = make_float2(0.f, 0.f), sb = make_float2(0.f, 0.f);
#pragma unroll
  for (int j = 0; j < N; j += 4) {
    const float2 a0 = f2_fma(make_float2(x[j], x[j + 1]), l2e, nmb);
    const float2 a1 = f2_fma(make_float2(x[j + 2], x[j + 3]), l2e, nmb);
    sa = f2_add(sa, make_float2(ex2(a0.x), ex2(a0.y)));
    sb = f2_add(sb, make_float2(ex2(a1.x), ex2(a1.y)));
  }
  const float2 t = f2_add(sa, sb);
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
  if (sizeof(TL) == 4) {
#pragma unroll
    for (int j = 0; j < N; ++j) {
      const int c = col0 + j;
      x[j] = c < V ? load_f(row + c) : neg_inf();
    }
    return;
  }
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

// STAGE: the drafter logits of each N-tile arrive in shared memory by TMA
// (bf16 logits, every CTA touching at most LBMAX requests); otherwise the
// epilogue reads them from global memory (L2) itself.
template <typename TL, int KMAX, bool STAGE>
__global__ void __launch_bounds__(THREADS, 1)
    score_umma_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const __grid_constant__ CUtensorMap tmL, const UmmaParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + NSUBMAX * KBMAX * A_TILE_BYTES;
  uint8_t* sL = sB + STAGES * B_STAGE_BYTES;                     // [2] L_d slots
  uint64_t* full = reinterpret_cast<uint64_t*>(sL + 2 * L_SLOT_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* afull = empty + STAGES;
  uint64_t* tfull = afull + 1;      // [2]
  uint64_t* tempty = tfull + 2;     // [2]
  uint64_t* lfull = tempty + 2;     // [2]
  uint64_t* lempty = lfull + 2;     // [2]
  uint64_t* drain = lempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sl = blockIdx.x, mt = blockIdx.y;
  const int t_begin = (int)((long long)sl * p.tiles_total / p.S);
  const int t_end = (int)((long long)(sl + 1) * p.tiles_total / p.S);
  const int ntiles = t_end - t_begin;
  const int row0 = mt * p.rows_per_cta;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    mbar_init(afull, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], NUM_EPI_WARPS * 32);
      mbar_init(&lfull[i], 1);
      mbar_init(&lempty[i], NUM_EPI_WARPS * 32);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      uint32_t armed = 0, armed_par = 0;   // per ring slot: loads issued, parity of the last
      mbar_expect_tx(afull, (uint32_t)(p.nsub * p.kblocks * A_TILE_BYTES));
      for (int st = 0; st < p.nsub; ++st)
        for (int kb = 0; kb < p.kblocks; ++kb)
          tma_load_2d(sA + (st * KBMAX + kb) * A_TILE_BYTES, &tmA, kb * BK, row0 + st * BM, afull);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      const int req0 = row0 / p.n_par;
      uint32_t larmed = 0;
      for (int it = 0; it < ntiles && ok; ++it) {
        const int n0 = (t_begin + it) * BN;
        if (STAGE) {
          const int slot = it & 1;
          if (!wait_bar(&lempty[slot], (((uint32_t)it >> 1) & 1u) ^ 1u, abort_flag, p.err)) { ok = false; break; }
          mbar_expect_tx(&lfull[slot], (uint32_t)(2 * 64 * p.LB * 2));
          uint8_t* dst = sL + slot * L_SLOT_BYTES;
          tma_load_2d(dst, &tmL, n0, req0, &lfull[slot]);
          tma_load_2d(dst + 64 * p.LB * 2, &tmL, n0 + 64, req0, &lfull[slot]);
          larmed = (uint32_t)it + 1;
        }
        for (int kb = 0; kb < p.kblocks; ++kb) {
          if (!wait_bar(&empty[stage], phase ^ 1u, abort_flag, p.err)) { ok = false; break; }
          mbar_expect_tx(&full[stage], B_STAGE_BYTES);
          uint8_t* dst = sB + stage * B_STAGE_BYTES;
          tma_load_2d(dst, &tmB, n0, kb * BK, &full[stage]);
          tma_load_2d(dst + B_STAGE_BYTES / 2, &tmB, n0 + 64, kb * BK, &full[stage]);
          armed |= 1u << stage;
          armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      // every load this thread issued has landed before the CTA may exit
      drain_wait(afull, 0);
#pragma unroll
      for (int i = 0; i < STAGES; ++i)
        if (armed & (1u << i)) drain_wait(&full[i], (armed_par >> i) & 1u);
      // the last one or two L_d slots armed (tiles larmed-1 and larmed-2)
      for (int t = (int)larmed - 2; t < (int)larmed; ++t)
        if (t >= 0) drain_wait(&lfull[t & 1], ((uint32_t)t >> 1) & 1u);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      // The issue loop is kept to a few instructions per MMA: a 128x128x16
      // MMA lasts 64 cycles, and a longer dependent instruction chain here
      // (descriptor assembly, runtime loops) leaves the tensor pipe idle.
      // Descriptors are built once; the start-address field holds addr >> 4
      // in the low 14 bits and shared addresses stay below 256 KB, so adding
      // (offset >> 4) to a descriptor never carries out of the field.
      bool ok = wait_bar(afull, 0, abort_flag, p.err);
      tc_fence_after();
      int stage = 0;
      uint32_t phase = 0;
      const uint64_t a_desc0 = make_desc(smem_u32(sA), 16, 1024);      // row tile 0, K block 0
      const uint64_t b_desc0 = make_desc(smem_u32(sB), 8192, 1024);    // ring slot 0
      const bool two = p.nsub == 2;
      for (int it = 0; it < ntiles && ok; ++it) {
        const int buf = it & 1;
        const uint32_t use = (uint32_t)(it >> 1);
        if (!wait_bar(&tempty[buf], (use & 1u) ^ 1u, abort_flag, p.err)) break;
        tc_fence_after();
        const uint32_t d0 = tmem_base + (uint32_t)(buf * NSUBMAX * BN);
        const uint32_t d1 = d0 + BN;
        for (int kb = 0; kb < p.kblocks; ++kb) {
          if (!wait_bar(&full[stage], phase, abort_flag, p.err)) { ok = false; break; }
          const uint64_t bd = b_desc0 + (uint64_t)((stage * B_STAGE_BYTES) >> 4);
          const uint64_t ad = a_desc0 + (uint64_t)((kb * A_TILE_BYTES) >> 4);
          const uint32_t acc0 = kb != 0;
          // B: [64 K][2 x 64 V] V-major, +2048 bytes per 16 K rows;
          // A: [128 rows][64 K] K-major, +32 bytes per 16 K columns
          umma_f16(d0, ad, bd, IDESC, acc0);
          if (two) umma_f16(d1, ad + (KBMAX * A_TILE_BYTES >> 4), bd, IDESC, acc0);
#pragma unroll
          for (int k4 = 1; k4 < BK / 16; ++k4) {
            umma_f16(d0, ad + (uint64_t)(k4 * 2), bd + (uint64_t)(k4 * 128), IDESC, 1u);
            if (two)
              umma_f16(d1, ad + (uint64_t)((KBMAX * A_TILE_BYTES >> 4) + k4 * 2),
                       bd + (uint64_t)(k4 * 128), IDESC, 1u);
          }
          umma_commit(&empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(&tfull[buf]);
      }
      // all issued MMAs complete before TMEM is released
      umma_commit(drain);
      drain_wait(drain, 0);
    }
  } else {
    // ---------------- epilogue ----------------
    // warp group g = (warp - 2) / 4 covers TMEM lane quarters 0..3 once:
    // row tile st = g / 2, column half h = g % 2 of every N-tile
    const int e = warp - 2;
    const int g = e >> 2;
    const int st = g / SPLIT, h = g % SPLIT;
    const int quad = warp & 3;
    const int r_in = st * BM + quad * 32 + lane;
    const int row = row0 + r_in;
    const bool valid = (st < p.nsub) && (row < p.M);
    const int req = valid ? row / p.n_par : row0 / p.n_par;
    const int req_local = req - row0 / p.n_par;       // < LB when STAGE
    const TL* Lr = static_cast<const TL*>(p.L) + (size_t)req * p.L_req_stride;
    const uint32_t sL_row = smem_u32(sL) + (uint32_t)(req_local * 128);
    const int k = p.k, V = p.V;
    float m = neg_inf(), s = 0.f;
    TopK<KMAX> tk;
    tk.init(k);
    // admission gate: max(own k-th value, best k-th value any slice of this
    // row has published). Every slice's k-th value is a lower bound of the
    // row's k-th, so values below the gate cannot be in the row's top-k.
    float gth = neg_inf();
    uint32_t* thr = p.row_thr + (valid ? row : 0);
    uint32_t pub_prev = 0;   // loaded at the end of the previous tile, used one tile later
    for (int it = 0; it < ntiles; ++it) {
      const int buf = it & 1;
      const uint32_t par = (uint32_t)((it >> 1) & 1);
      if (!wait_bar(&tfull[buf], par, abort_flag, p.err)) break;
      if (STAGE && !wait_bar(&lfull[buf], par, abort_flag, p.err)) break;
      tc_fence_after();
      const int n0 = (t_begin + it) * BN;
      const uint32_t tbase =
          tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)((buf * NSUBMAX + st) * BN);
#pragma unroll 1
      for (int c = h * (BN / CH / SPLIT); c < (h + 1) * (BN / CH / SPLIT); ++c) {
        const int col0 = n0 + c * CH;
        float x[CH];
        if (STAGE) {
          // [LB][64] box (c * CH) / 64, columns (c * CH) % 64 .. of this request's row
          const uint32_t a = sL_row + (uint32_t)(buf * L_SLOT_BYTES + ((c * CH) >> 6) * (64 * p.LB * 2) +
                                                 ((c * CH) & 63) * 2);
          uint4 w[CH / 8];
#pragma unroll
          for (int q = 0; q < CH / 8; ++q) w[q] = ld_shared16(a + 16 * q);
#pragma unroll
          for (int q = 0; q < CH / 8; ++q) {
            x[q * 8 + 0] = bf16_lo(w[q].x); x[q * 8 + 1] = bf16_hi(w[q].x);
            x[q * 8 + 2] = bf16_lo(w[q].y); x[q * 8 + 3] = bf16_hi(w[q].y);
            x[q * 8 + 4] = bf16_lo(w[q].z); x[q * 8 + 5] = bf16_hi(w[q].z);
            x[q * 8 + 6] = bf16_lo(w[q].w); x[q * 8 + 7] = bf16_hi(w[q].w);
          }
        } else if (valid) {
          load_logits<TL, CH>(Lr, col0, V, x);
        }
        uint32_t acc[CH];
        tmem_ld(tbase + (uint32_t)(c * CH), acc);
        if (valid) {
          // z = L + E[p].W in fp32 pairs
#pragma unroll
          for (int j = 0; j < CH; j += 2) {
            const float2 z2 = f2_add(make_float2(x[j], x[j + 1]),
                                     make_float2(__uint_as_float(acc[j]), __uint_as_float(acc[j + 1])));
            x[j] = z2.x;
            x[j + 1] = z2.y;
          }
          if (col0 + CH > V) {
#pragma unroll
            for (int j = 0; j < CH; ++j) x[j] = (col0 + j < V) ? x[j] : neg_inf();
          }
          const float cm = chunk_max<CH>(x);
          // sum of 2^(z log2 e - m log2 e) against the running reference m,
          // computed before (and independent of) this chunk's max; m moves
          // only when a value exceeds it by more than 64 (exp(64) keeps the
          // fp32 sum far from overflow), which recomputes the chunk
          float csum = 0.f;
          if (m != neg_inf()) csum = chunk_exp_sum<CH>(x, m);
          if (cm > m + 64.f) {
            s = (m == neg_inf()) ? 0.f : s * ex2((m - cm) * kLog2e);
            m = cm;
            csum = chunk_exp_sum<CH>(x, m);
          }
          s += csum;
          if (cm >= gth) {
            // superset gate (x >= gate); the exact order test runs per
            // candidate. The gate only rises, so positions outside the mask
            // never need a second look.
            uint32_t cand = 0;
#pragma unroll
            for (int j = 0; j < CH; ++j) cand |= (uint32_t)(x[j] >= gth) << j;
            while (cand) {
              const int j = __ffs(cand) - 1;
              cand &= cand - 1;
              float z = x[0];
#pragma unroll
              for (int jj = 1; jj < CH; ++jj) z = (j == jj) ? x[jj] : z;
              if (z >= gth && tk.admits(z, col0 + j)) {
                tk.insert(z, col0 + j);
                gth = fmaxf(gth, tk.tv());
              }
            }
          }
        }
      }
      // publish this slice's k-th value for the row and pick up the best one
      // published by any slice (stale values are still valid lower bounds)
      if (valid) {
        if (pub_prev > f2ord(neg_inf())) gth = fmaxf(gth, ord2f(pub_prev));
        const float own = tk.tv();
        if (own != neg_inf()) atomicMax(thr, f2ord(own));
        pub_prev = *reinterpret_cast<volatile uint32_t*>(thr);
      }
      tc_fence_before();
      mbar_arrive(&tempty[buf]);
      if (STAGE) mbar_arrive(&lempty[buf]);
    }
    // fold the two column halves of each row through shared memory (the Eg
    // tile region is idle once the last MMA has completed)
    wait_bar(afull, 0, abort_flag, p.err);
    float2* xms = reinterpret_cast<float2*>(sA);                       // [256]
    float* xv = reinterpret_cast<float*>(sA + 256 * sizeof(float2));   // [256][KMAX]
    int* xi = reinterpret_cast<int*>(xv + 256 * KMAX);                 // [256][KMAX]
    if (SPLIT == 1) {
      if (valid) {
        tk.finish(k);
        const size_t ps = (size_t)row * p.S + sl;
        p.pms[ps] = make_float2(m, s);
#pragma unroll
        for (int j = 0; j < KMAX; ++j)
          if (j < k) { p.pval[ps * k + j] = tk.v[j]; p.pidx[ps * k + j] = tk.i[j]; }
      }
    } else if (h == 1) {
      tk.finish(k);
      xms[r_in] = make_float2(m, s);
#pragma unroll
      for (int j = 0; j < KMAX; ++j) { xv[r_in * KMAX + j] = tk.v[j]; xi[r_in * KMAX + j] = tk.i[j]; }
    }
    if (SPLIT > 1) asm volatile("bar.sync 1, %0;" ::"n"(NUM_EPI_WARPS * 32) : "memory");
    if (SPLIT > 1 && h == 0 && valid) {
      const float2 o = xms[r_in];
      lse_combine(m, s, o.x, o.y);
#pragma unroll
      for (int j = 0; j < KMAX; ++j) {
        const float v = xv[r_in * KMAX + j];
        const int i = xi[r_in * KMAX + j];
        if (j < k && tk.admits(v, i)) tk.insert(v, i);
      }
      tk.finish(k);
      const size_t ps = (size_t)row * p.S + sl;
      p.pms[ps] = make_float2(m, s);
#pragma unroll
      for (int j = 0; j < KMAX; ++j)
        if (j < k) { p.pval[ps * k + j] = tk.v[j]; p.pidx[ps * k + j] = tk.i[j]; }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(TMEM_COLS));
  }
}

// ---------------------------------------------------------------------------
// Host: tensor maps through the driver entry point (no libcuda link needed).
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

int umma_nsub(int rows) { return rows > BM ? 2 : 1; }

}  // namespace

int score_slices(int rows, int V, int markov_dtype) {
  const int sms = num_sms();
  if (markov_dtype == PCT_BF16) {
    const int rpc = BM * umma_nsub(rows);
    const int mtiles = (rows + rpc - 1) / rpc;
    const int tiles = (V + BN - 1) / BN;
    return std::max(1, std::min(tiles, sms / std::max(mtiles, 1)));
  }
  const int target = 4 * sms;
  const int max_s = (V + 127) / 128;
  return std::max(1, std::min((target + rows - 1) / rows, max_s));
}

size_t score_smem_bytes() { return SMEM_BYTES; }

cudaError_t launch_score(const ScoreArgs& a, cudaStream_t s) {
  if (a.markov_dtype != PCT_BF16) return launch_score_simt(a, s);
  const int rows = a.n_req * a.n_par;
  CUtensorMap tmA, tmB;
  if (!encode_2d_bf16(&tmA, a.Eg, (uint64_t)a.r_pad, (uint64_t)a.M_pad, BK, BM)) return cudaErrorInvalidValue;
  if (!encode_2d_bf16(&tmB, a.W, (uint64_t)a.V, (uint64_t)a.r, 64, BK)) return cudaErrorInvalidValue;
  UmmaParams p;
  p.M = rows;
  p.nsub = umma_nsub(rows);
  p.rows_per_cta = BM * p.nsub;
  p.n_par = a.n_par;
  p.V = a.V;
  p.kblocks = a.r_pad / BK;
  p.S = a.S;
  p.tiles_total = (a.V + BN - 1) / BN;
  p.k = a.k;
  p.L = a.L;
  p.L_req_stride = a.L_req_stride;
  p.pms = a.part.ms;
  p.pval = a.part.val;
  p.pidx = a.part.idx;
  p.err = a.err;
  p.row_thr = a.row_thr;
  if (cudaMemsetAsync(a.row_thr, 0, sizeof(uint32_t) * (size_t)rows, s) != cudaSuccess)
    return cudaErrorInvalidValue;
  const int mtiles = (rows + p.rows_per_cta - 1) / p.rows_per_cta;
  // requests any CTA's rows span: stage L_d by TMA when that fits a slot
  int span = 0;
  for (int mt = 0; mt < mtiles; ++mt) {
    const int r0 = mt * p.rows_per_cta, r1 = std::min(rows, r0 + p.rows_per_cta) - 1;
    span = std::max(span, r1 / a.n_par - r0 / a.n_par + 1);
  }
  const bool stage = a.logits_dtype == PCT_BF16 && span <= LBMAX;
  p.LB = stage ? (span + 7) / 8 * 8 : 0;
  CUtensorMap tmL;
  if (stage) {
    if (!encode_2d_bf16(&tmL, a.L, (uint64_t)a.V, (uint64_t)a.n_req, 64, (uint32_t)p.LB,
                        (uint64_t)a.L_req_stride * 2, false))
      return cudaErrorInvalidValue;
  } else {
    tmL = tmB;   // unused
  }
  dim3 grid(a.S, mtiles);
  TraceScope t(s, "pct_score_umma");
#define PCT_UMMA(TL, KM, ST)                                                                    \
  do {                                                                                          \
    auto kern = score_umma_kernel<TL, KM, ST>;                                                  \
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,     \
                                         (int)SMEM_BYTES);                                      \
    if (e != cudaSuccess) return e;                                                             \
    kern<<<grid, THREADS, SMEM_BYTES, s>>>(tmA, tmB, tmL, p);                                   \
  } while (0)
  if (stage) {
    if (a.k <= 4) PCT_UMMA(__nv_bfloat16, 4, true); else if (a.k <= 8) PCT_UMMA(__nv_bfloat16, 8, true); else PCT_UMMA(__nv_bfloat16, 16, true);
  } else if (a.logits_dtype == PCT_BF16) {
    if (a.k <= 4) PCT_UMMA(__nv_bfloat16, 4, false); else if (a.k <= 8) PCT_UMMA(__nv_bfloat16, 8, false); else PCT_UMMA(__nv_bfloat16, 16, false);
  } else {
    if (a.k <= 4) PCT_UMMA(float, 4, false); else if (a.k <= 8) PCT_UMMA(float, 8, false); else PCT_UMMA(float, 16, false);
  }
#undef PCT_UMMA
  return cudaGetLastError();
}

}  // namespace pct
