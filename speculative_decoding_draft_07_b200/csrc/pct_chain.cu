// PCTree for small frontiers in one persistent launch (bf16 Markov parameters,
// bf16 drafter logits, at most 16 requests and 128 parent rows per depth).
//
// PCTree article (qiita), section on the chain draft's weakness and the tree
// built in its place: for every frontier parent p of depth d,
// z_d(p) = L_d + Markov(p), all parents in one batched call; the softmax over
// the vocabulary; each parent's local top-k; path scores s = s(p) + log pi;
// the beam per depth. With the rank-r stand-in Markov(p) = E[p] . W each depth
// is the contraction Eg[M][r] . W[r][V] with M = (requests x frontier) <= 128.
//
// At these sizes the contraction is a stream of W (r x V bf16, 77.8 MB at
// r = 256, V = 151936) per depth, and the per-depth beam merge is short but
// sequential. So the whole build of all depths is one cooperative launch with
// one CTA per SM:
//  * every CTA owns a fixed slice of the vocabulary (128-column N-tiles). Warp
//    0 streams its W tiles through a ring depth after depth (W does not depend
//    on the frontier, so the next depth's tiles load while the current depth
//    is merged, and a W that fits in L2 is read from L2 after the first depth),
//    with the requests' L_d tile of every N-tile; warp 1 issues the tcgen05
//    MMAs (M = 128, N = 128, K = 16) into a double-buffered TMEM accumulator,
//    and L_d joins the product as one more K = 16 step (one-hot request
//    indicator x L_d tile), so the accumulator holds z;
//  * warps 2..5 are the epilogue (one TMEM lane quarter each): online
//    log-sum-exp and a register top-k per row behind a gate that every CTA
//    raises with atomicMax to the best known k-th value of the row. Frontiers
//    of at most 32 (64) rows are written into the A tile four (two) times, so
//    that every lane quarter holds a copy and the four (two) warps split each
//    tile's columns; the copies are folded through shared memory;
//  * at the end of a depth each CTA writes its (max, sum) per row and appends
//    its top-k entries that reach the row's gate to the row's candidate list
//    (the union holds the row's exact top-k: the gate never exceeds the row's
//    k-th value), then arrives at a grid barrier (a counter; bounded wait).
//    Every CTA then merges all rows itself (the same inputs and code give the
//    same bits everywhere): lse from the partials, each row's k best
//    candidates, the beam over path scores, canonical order, and the next
//    depth's A tile gathered from E. CTA 0 writes the level arrays the global
//    top-N kernel reads. One barrier per depth, no launch per depth.
// Every wait is bounded: an mbarrier wait or the grid barrier that gives up
// sets the grid's error word, the CTA stops, drains its loads and MMAs and
// frees TMEM; the others see the word at their next wait.
#include <cuda.h>

#include <algorithm>
#include <climits>

#include "common.cuh"
#include "internal.h"
#include "seed.cuh"
#include "select.cuh"
#include "umma.cuh"

namespace pct {
namespace {

constexpr int C_BM = 128;                            // A rows (TMEM lanes)
constexpr int C_BN = 128;                            // columns per N-tile
constexpr int C_BK = 64;                             // K per W ring slot
constexpr int C_STAGES = 6;
constexpr int C_KBMAX = 4;                           // r_pad <= 256
constexpr int C_A_KB = C_BM * C_BK * 2;              // 16 KB per K block of A
constexpr int C_B_STAGE = C_BK * C_BN * 2;           // 16 KB per W slot
constexpr int C_LFOLD = 16;                          // requests (K of the L_d step)
constexpr int C_LPART = C_LFOLD * C_BN * 2;          // [16][128] L_d tile, 4 KB
constexpr int C_ONEHOT = C_BM * C_LFOLD * 2;         // [128][16] one-hot, 4 KB
constexpr int C_EPI = 4;                             // epilogue warps
constexpr int C_THREADS = 64 + 32 * C_EPI;
constexpr int C_ROWS = 128;                          // parent rows per depth, at most
constexpr int C_MAXBEAM = 32;
constexpr int C_KEYS = 2048;                         // rows x k beam candidates
constexpr int C_CH = 32;                             // accumulator columns per TMEM load
constexpr int C_TMEM_COLS = 2 * C_BN;
// the next depth's seed data, prefetched while the current depth is scored
// when every request's fits: W columns (k x r_pad bf16 per request), then the
// columns, L_d there and max|W| there (k each per request)
constexpr int C_PRE = 8192 + 3 * 4 * 256;

// kind::f16 instruction descriptor: D f32, A = B = bf16, A K-major, B
// MN-major, N = 128, M = 128.
constexpr uint32_t C_IDESC = (1u << 4) | (1u << 7) | (1u << 10) | (0u << 15) | (1u << 16) |
                             ((uint32_t)(C_BN >> 3) << 17) | ((uint32_t)(C_BM >> 4) << 24);

template <int KMAX>
constexpr size_t chain_smem_bytes() {
  return 1024 + (size_t)C_KBMAX * C_A_KB + (size_t)C_STAGES * C_B_STAGE + 2 * (size_t)C_LPART +
         C_ONEHOT + C_KEYS * 8 + C_ROWS * (8 + 8 * KMAX) + C_ROWS * 16 + C_PRE + 64 + 256;
}

struct ChainParams {
  int batch, D, V, k, beam, kblocks, G, tiles_total, r, r_pad, cap;
  int F[65];                      // frontier sizes, F[0] = 1
  const __nv_bfloat16* E;         // [V][r]
  const int32_t* anchor;          // [batch]
  float2* ms;                     // [2][C_ROWS][G] (max, sum) per row and CTA
  unsigned long long* cand;       // [2][C_ROWS][cap] appended candidate keys
  int32_t* cand_cnt;              // [D][C_ROWS]
  uint32_t* row_thr;              // [D][C_ROWS] gate (ordered key, 0 = none)
  unsigned* arrive;               // [D] grid barrier counters
  int32_t* err;                   // grid error word
  int32_t* lvl_tok;               // [D][batch][beam]
  int32_t* lvl_ppos;
  float* lvl_s;
  int32_t* status;                // [batch]
  // admission seeds per (request, depth): the k best drafter-logit columns,
  // L_d and max|W| there, and W's columns (bf16, r_pad wide)
  const int32_t* scol;
  const float* slval;
  const float* swmax;
  const __nv_bfloat16* swcol;
};

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}
// Tile load of W kept in L2 (evict-last): W is read again at every depth.
__device__ __forceinline__ void tma_load_2d_keep(void* dst, const CUtensorMap* map, int x, int y,
                                                 uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}
__device__ __forceinline__ void epi_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(C_EPI * 32) : "memory");
}
__device__ __forceinline__ void red_max_u32(uint32_t* p, uint32_t v) {
  asm volatile("red.relaxed.gpu.global.max.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
// Copies per lane quarter of an A tile holding m rows.
__device__ __forceinline__ int copies_for(int m) { return m <= 32 ? 4 : (m <= 64 ? 2 : 1); }

// The A tile and the one-hot request indicator of a depth whose M rows are the
// frontier ftok (row r of request r / Fd): A row a holds copy a / (128 / R) of
// row a % (128 / R) (K-major, 128-byte swizzle, zero past r and past M).
// Every epilogue thread writes one A row's one-hot entry and a share of A.
__device__ void build_a_tile(const ChainParams& p, int M, int Fd, const int* ftok, uint8_t* sA,
                             uint8_t* sOneHot) {
  const int t = threadIdx.x - 64;                  // 0..127
  const int R = copies_for(M), rpc = C_BM / R;
  // every (row, chunk) of the M rows is loaded once and stored to each of the
  // R copies; the rest of the tile (rows past M in each copy) is zero
  const int per_row = p.kblocks * 8;               // 16-byte chunks per A row
  const int total = M * per_row;
  constexpr int B = 8;                             // chunks in flight per thread
  for (int i0 = t; i0 < total; i0 += B * C_EPI * 32) {
    uint4 v[B];
#pragma unroll
    for (int j = 0; j < B; ++j) {
      const int idx = i0 + j * C_EPI * 32;
      v[j] = make_uint4(0u, 0u, 0u, 0u);
      if (idx < total) {
        const int r = idx / per_row, rem = idx - r * per_row;
        const int kk = (rem >> 3) * C_BK + (rem & 7) * 8;
        if (kk < p.r) {
          const int tok = (unsigned)ftok[r] < (unsigned)p.V ? ftok[r] : 0;
          v[j] = __ldg(reinterpret_cast<const uint4*>(p.E + (size_t)tok * p.r + kk));
        }
      }
    }
#pragma unroll
    for (int j = 0; j < B; ++j) {
      const int idx = i0 + j * C_EPI * 32;
      if (idx < total) {
        const int r = idx / per_row, rem = idx - r * per_row;
        const int kb = rem >> 3, c8 = rem & 7;
        for (int cp = 0; cp < R; ++cp) {
          const int a = cp * rpc + r;
          *reinterpret_cast<uint4*>(sA + kb * C_A_KB + a * 128 + ((c8 ^ (a & 7)) << 4)) = v[j];
        }
      }
    }
  }
  {
    // thread t clears row t of the tile when it lies past M in its copy
    const int a = t;
    if (a - (a / rpc) * rpc >= M)
      for (int rem = 0; rem < per_row; ++rem)
        *reinterpret_cast<uint4*>(sA + (rem >> 3) * C_A_KB + a * 128 + (((rem & 7) ^ (a & 7)) << 4)) =
            make_uint4(0u, 0u, 0u, 0u);
  }
  {
    // one-hot row a (K-major, 32-byte swizzle: the two 16-byte halves of a row
    // swap in rows 4..7 of each 8-row group)
    const int a = t;
    const int r = a - (a / rpc) * rpc;
    const int kq = r < M ? r / Fd : -1;
    uint8_t* rowp = sOneHot + (a >> 3) * 256 + (a & 7) * 32;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int kl = kq - 8 * half;
      const uint32_t one = 0x3F80u << (16 * (kl & 1));   // bf16 1.0 in its half word
      const int wi = (kl >= 0 && kl < 8) ? (kl >> 1) : -1;
      const int phys = half ^ ((a >> 2) & 1);
      *reinterpret_cast<uint4*>(rowp + 16 * phys) =
          make_uint4(wi == 0 ? one : 0u, wi == 1 ? one : 0u, wi == 2 ? one : 0u, wi == 3 ? one : 0u);
    }
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Seed gates of the M rows of depth dd (frontier of Fd per request, A tile
// built): row r's gate is a lower bound of its k-th value, the least of the
// exact z at the request's k seed columns less the rounding allowance of the
// tensor-core sum (seed.cuh); ordered keys, 0 where there is no seed. Every
// epilogue thread takes (row, column) pairs; the parent embedding is read from
// copy 0 of the row in the A tile.
// Whether depth dd's seed data of every request fits the prefetch buffer.
__device__ __forceinline__ bool seed_prefetchable(const ChainParams& p) {
  return p.batch * p.k * p.r_pad * 2 <= 8192 && p.batch * p.k <= 256;
}
// Every epilogue thread: asynchronous copies of depth dd's seed data into pre
// (layout above); seed_wait() before use.
__device__ void seed_prefetch_depth(const ChainParams& p, int dd, uint8_t* pre) {
  const int t = threadIdx.x - 64;
  const int k = p.k, n16 = k * p.r_pad / 8;
  for (int i = t; i < p.batch * n16; i += C_EPI * 32) {
    const int b = i / n16, j = i - b * n16;
    const size_t e0 = ((size_t)b * p.D + (dd - 1)) * k;
    const uint32_t dst = smem_u32(pre + (size_t)i * 16);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst),
                 "l"(p.swcol + e0 * p.r_pad + (size_t)j * 8) : "memory");
  }
  for (int i = t; i < 3 * p.batch * k; i += C_EPI * 32) {
    const int w = i / (p.batch * k), bc = i - w * p.batch * k;
    const int b = bc / k, c = bc - b * k;
    const size_t e = ((size_t)b * p.D + (dd - 1)) * k + c;
    const void* src = w == 0 ? static_cast<const void*>(p.scol + e)
                             : w == 1 ? static_cast<const void*>(p.slval + e)
                                      : static_cast<const void*>(p.swmax + e);
    const uint32_t dst = smem_u32(pre + 8192 + (size_t)i * 4);
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
}

__device__ void chain_seeds(const ChainParams& p, int dd, int M, int Fd, const uint8_t* sA,
                            uint32_t* sseed, __nv_bfloat16* swc, const uint8_t* pre) {
  const int t = threadIdx.x - 64;
  for (int r = t; r < C_ROWS; r += C_EPI * 32) sseed[r] = 0xffffffffu;
  const int k = p.k;
  if (pre != nullptr) {
    asm volatile("cp.async.wait_all;" ::: "memory");
    epi_sync();
  }
  const int32_t* pcol = reinterpret_cast<const int32_t*>(pre + 8192);
  const float* plval = reinterpret_cast<const float*>(pre + 8192) + p.batch * k;
  const float* pwmax = plval + p.batch * k;
  for (int b = 0; b < p.batch; ++b) {
    const size_t e0 = ((size_t)b * p.D + (dd - 1)) * k;
    const __nv_bfloat16* wsrc;
    if (pre != nullptr) {
      wsrc = reinterpret_cast<const __nv_bfloat16*>(pre) + (size_t)b * k * p.r_pad;
    } else {
      // the request's k W columns for this depth, once per CTA (k x r_pad bf16)
      const int n16 = k * p.r_pad / 8;
      for (int i = t; i < n16; i += C_EPI * 32)
        reinterpret_cast<uint4*>(swc)[i] = __ldg(reinterpret_cast<const uint4*>(p.swcol + e0 * p.r_pad) + i);
      epi_sync();
      wsrc = swc;
    }
    // column-major tasks: a warp's lanes share one or two W columns (broadcast
    // reads) and take consecutive rows (conflict-free in the swizzled A tile)
    for (int pr = t; pr < Fd * k; pr += C_EPI * 32) {
      const int c = pr / Fd, i = pr - c * Fd;
      const int r = b * Fd + i;
      const size_t e = e0 + c;
      const int col = pre != nullptr ? pcol[b * k + c] : p.scol[e];
      uint32_t key = 0u;
      if (col >= 0) {
        const __nv_bfloat16* wc = wsrc + (size_t)c * p.r_pad;
        float dot = 0.f, e1 = 0.f;
        for (int j0 = 0; j0 < p.r; j0 += 8) {
          const int kb = j0 / C_BK, c8 = (j0 % C_BK) >> 3;
          const uint4 ev = *reinterpret_cast<const uint4*>(sA + kb * C_A_KB + r * 128 + ((c8 ^ (r & 7)) << 4));
          const uint4 wv = *reinterpret_cast<const uint4*>(wc + j0);
          const float ee[8] = {bf16_lo(ev.x), bf16_hi(ev.x), bf16_lo(ev.y), bf16_hi(ev.y),
                               bf16_lo(ev.z), bf16_hi(ev.z), bf16_lo(ev.w), bf16_hi(ev.w)};
          const float ww[8] = {bf16_lo(wv.x), bf16_hi(wv.x), bf16_lo(wv.y), bf16_hi(wv.y),
                               bf16_lo(wv.z), bf16_hi(wv.z), bf16_lo(wv.w), bf16_hi(wv.w)};
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            dot = fmaf(ee[q], ww[q], dot);
            e1 += fabsf(ee[q]);
          }
        }
        const float l = pre != nullptr ? plval[b * k + c] : p.slval[e];
        const float wm = pre != nullptr ? pwmax[b * k + c] : p.swmax[e];
        const float lo = (l + dot) - (fabsf(l) + e1 * wm) * kSeedSlack;
        key = (lo == lo && lo != __int_as_float(0x7f800000) && lo > neg_inf()) ? f2ord(lo) : 0u;
      }
      atomicMin(&sseed[r], key);
    }
    if (pre == nullptr || b + 1 == p.batch) epi_sync();
  }
}

template <int KMAX>
__global__ void __launch_bounds__(C_THREADS, 1)
    pct_chain_kernel(const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmL,
                     const ChainParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + C_KBMAX * C_A_KB;
  uint8_t* sL = sB + C_STAGES * C_B_STAGE;
  uint8_t* sOneHot = sL + 2 * C_LPART;
  unsigned long long* mkeys = reinterpret_cast<unsigned long long*>(sOneHot + C_ONEHOT);  // [C_KEYS]
  float* xm = reinterpret_cast<float*>(mkeys + C_KEYS);      // [C_ROWS] copies' max
  float* xs = xm + C_ROWS;                                   // [C_ROWS] copies' sum
  float* xv = xs + C_ROWS;                                   // [C_ROWS][KMAX]
  int* xi = reinterpret_cast<int*>(xv + C_ROWS * KMAX);      // [C_ROWS][KMAX]
  int* ftok = xi + C_ROWS * KMAX;                            // [C_ROWS] frontier tokens
  float* fs = reinterpret_cast<float*>(ftok + C_ROWS);       // [C_ROWS] frontier scores
  uint32_t* sseed = reinterpret_cast<uint32_t*>(fs + C_ROWS); // [C_ROWS] seed gates (ordered keys)
  int* misc = reinterpret_cast<int*>(sseed + C_ROWS);         // [16]
  uint8_t* spre = reinterpret_cast<uint8_t*>(misc + 16);       // [C_PRE] (16-byte aligned)
  uint64_t* full = reinterpret_cast<uint64_t*>(spre + C_PRE);
  uint64_t* empty = full + C_STAGES;
  uint64_t* lfull = empty + C_STAGES;    // [2]
  uint64_t* lempty = lfull + 2;          // [2]
  uint64_t* tfull = lempty + 2;          // [2]
  uint64_t* tempty = tfull + 2;          // [2]
  uint64_t* aready = tempty + 2;
  uint64_t* drain = aready + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cta = blockIdx.x;
  const int t_begin = (int)((long long)cta * p.tiles_total / p.G);
  const int t_end = (int)((long long)(cta + 1) * p.tiles_total / p.G);
  const int ntiles = t_end - t_begin;
  const int k = p.k;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C_STAGES; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&lfull[i], 1);
      mbar_init(&lempty[i], 1);
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], C_EPI);
    }
    mbar_init(aready, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp >= 2) {
    // depth 1: the frontier is each request's anchor
    const int t = threadIdx.x - 64;
    if (t < p.batch) {
      int a = p.anchor[t];
      if (a < 0 || a >= p.V) {
        if (cta == 0) atomicOr(&p.status[t], PCT_DEV_BAD_TOKEN);
        a = 0;
      }
      ftok[t] = a;
      fs[t] = 0.f;
    }
    epi_sync();
    build_a_tile(p, p.batch, 1, ftok, sA, sOneHot);
    epi_sync();
    chain_seeds(p, 1, p.batch, 1, sA, sseed, reinterpret_cast<__nv_bfloat16*>(mkeys), nullptr);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(C_TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  if (threadIdx.x == 64) mbar_arrive(aready);   // depth 1's A tile is written

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer: W tiles (and L_d tiles), depth after depth
      uint32_t armed = 0, armed_par = 0;
      int stage = 0;
      uint32_t phase = 0;
      int git = 0;
      bool ok = true;
      uint64_t keep;
      asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(keep));
      for (int d = 1; d <= p.D && ok; ++d) {
        for (int it = 0; it < ntiles && ok; ++it, ++git) {
          const int n0 = (t_begin + it) * C_BN;
          const int ls = git & 1;
          if (!wait_bar(&lempty[ls], (((uint32_t)git >> 1) & 1u) ^ 1u, abort_flag, p.err)) { ok = false; break; }
          mbar_expect_tx(&lfull[ls], (uint32_t)C_LPART);
          tma_load_3d(sL + ls * C_LPART, &tmL, n0, d - 1, 0, &lfull[ls]);
          tma_load_3d(sL + ls * C_LPART + C_LPART / 2, &tmL, n0 + 64, d - 1, 0, &lfull[ls]);
          for (int kb = 0; kb < p.kblocks; ++kb) {
            if (!wait_bar(&empty[stage], phase ^ 1u, abort_flag, p.err)) { ok = false; break; }
            mbar_expect_tx(&full[stage], (uint32_t)C_B_STAGE);
            uint8_t* dst = sB + stage * C_B_STAGE;
            tma_load_2d_keep(dst, &tmB, n0, kb * C_BK, &full[stage], keep);
            tma_load_2d_keep(dst + C_B_STAGE / 2, &tmB, n0 + 64, kb * C_BK, &full[stage], keep);
            armed |= 1u << stage;
            armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
            if (++stage == C_STAGES) { stage = 0; phase ^= 1u; }
          }
        }
      }
      // every load issued has landed before the CTA may exit
#pragma unroll 1
      for (int i = 0; i < C_STAGES; ++i)
        if (armed & (1u << i)) drain_wait(&full[i], (armed_par >> i) & 1u);
      for (int g = git - 2; g < git; ++g)
        if (g >= 0) drain_wait(&lfull[g & 1], ((uint32_t)g >> 1) & 1u);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      int git = 0;
      bool ok = true;
      const uint64_t a_desc0 = make_desc(smem_u32(sA), 16, 1024);
      const uint64_t b_desc0 = make_desc(smem_u32(sB), 8192, 1024);
      const uint64_t x_desc = make_desc(smem_u32(sOneHot), 16, 256, 6);
      const uint64_t l_desc0 = make_desc(smem_u32(sL), C_LPART / 2, 1024);
      for (int d = 1; d <= p.D && ok; ++d) {
        if (!wait_bar(aready, (uint32_t)(d - 1) & 1u, abort_flag, p.err)) break;
        tc_fence_after();
        for (int it = 0; it < ntiles; ++it, ++git) {
          const int buf = git & 1;
          if (!wait_bar(&tempty[buf], (((uint32_t)git >> 1) & 1u) ^ 1u, abort_flag, p.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t dt = tmem_base + (uint32_t)(buf * C_BN);
          for (int kb = 0; kb < p.kblocks; ++kb) {
            if (!wait_bar(&full[stage], phase, abort_flag, p.err)) { ok = false; break; }
            const uint64_t bd = b_desc0 + (uint64_t)((stage * C_B_STAGE) >> 4);
            const uint64_t ad = a_desc0 + (uint64_t)((kb * C_A_KB) >> 4);
            umma_f16(dt, ad, bd, C_IDESC, kb != 0);
            umma_f16(dt, ad + 2, bd + 128, C_IDESC, 1u);
            umma_f16(dt, ad + 4, bd + 256, C_IDESC, 1u);
            umma_f16(dt, ad + 6, bd + 384, C_IDESC, 1u);
            umma_commit(&empty[stage]);
            if (++stage == C_STAGES) { stage = 0; phase ^= 1u; }
          }
          if (!ok) break;
          const int ls = git & 1;
          if (!wait_bar(&lfull[ls], ((uint32_t)git >> 1) & 1u, abort_flag, p.err)) { ok = false; break; }
          umma_f16(dt, x_desc, l_desc0 + (uint64_t)((ls * C_LPART) >> 4), C_IDESC, 1u);
          umma_commit(&lempty[ls]);
          umma_commit(&tfull[buf]);
        }
      }
      umma_commit(drain);
      drain_wait(drain, 0);
    }
  } else {
    // ---------------- epilogue, merge and the next A tile (warps 2..5)
    const int ew = warp - 2;                  // 0..3
    const int quad = warp & 3;                // TMEM lane quarter this warp may read
    const int a_row = quad * 32 + lane;       // A row = TMEM lane
    int git = 0;
    for (int d = 1; d <= p.D; ++d) {
      const int Fp = p.F[d - 1], M = p.batch * Fp;
      const int R = copies_for(M), rpc = C_BM / R;
      const int copy = a_row / rpc, r = a_row - copy * rpc;
      const bool valid = r < M;
      const int ncols = C_BN / R;             // columns of each tile for this copy
      const int par = d & 1;
      uint32_t* thr = p.row_thr + (size_t)(d - 1) * C_ROWS + (valid ? r : 0);
      float m = neg_inf(), s = 0.f;
      TopK<KMAX> tk;
      tk.init(k);
      if (d < p.D && seed_prefetchable(p)) seed_prefetch_depth(p, d + 1, spre);
      const uint32_t seed_key = valid ? sseed[r] : 0u;
      const float seed_gate =
          (seed_key > f2ord(neg_inf()) && seed_key != 0xffffffffu) ? ord2f(seed_key) : neg_inf();
      float gth = seed_gate;
      bool ok = true;
      for (int it = 0; it < ntiles; ++it, ++git) {
        const int buf = git & 1;
        if (ok && !wait_bar(&tfull[buf], ((uint32_t)git >> 1) & 1u, abort_flag, p.err)) ok = false;
        ok = __all_sync(0xffffffffu, ok);   // the TMEM loads below need the whole warp
        if (!ok) continue;
        tc_fence_after();
        const int n0 = (t_begin + it) * C_BN + copy * ncols;
        const uint32_t tbase = tmem_base + ((uint32_t)(quad * 32) << 16) +
                               (uint32_t)(buf * C_BN + copy * ncols);
#pragma unroll 1
        for (int c = 0; c < ncols / C_CH; ++c) {
          uint32_t acc[C_CH];
          tmem_issue(tbase + (uint32_t)(c * C_CH), acc);
          tmem_wait(acc);
          if (!valid) continue;
          const int col0 = n0 + c * C_CH;
          float x[C_CH];
#pragma unroll
          for (int j = 0; j < C_CH; ++j) x[j] = (col0 + j < p.V) ? __uint_as_float(acc[j]) : neg_inf();
          const float cm = chunk_max<C_CH>(x);
          // sum against the running reference m, which moves only when a value
          // exceeds it by more than 64 (the chunk is then summed again)
          float csum = 0.f;
          if (m != neg_inf()) csum = chunk_exp_sum<C_CH>(x, m);
          if (cm > m + 64.f) {
            s = (m == neg_inf()) ? 0.f : s * ex2((m - cm) * kLog2e);
            m = cm;
            csum = chunk_exp_sum<C_CH>(x, m);
          }
          s += csum;
          if (cm >= gth) {
            uint32_t cand = 0;
#pragma unroll
            for (int j = 0; j < C_CH; ++j) cand |= (uint32_t)(x[j] >= gth) << j;
            while (cand) {
              const int j = __ffs(cand) - 1;
              cand &= cand - 1;
              float z = x[0];
#pragma unroll
              for (int jj = 1; jj < C_CH; ++jj) z = (j == jj) ? x[jj] : z;
              if (z >= gth && tk.admits(z, col0 + j)) {
                tk.insert(z, col0 + j);
                gth = fmaxf(gth, tk.tv());
              }
            }
          }
        }
        if (valid) {
          // publish this copy's k-th value (a reduction nothing waits for); the
          // row's gate is read once, at the end of the depth
          const float own = tk.tv();
          if (own != neg_inf()) red_max_u32(thr, f2ord(own));
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[buf]);
      }
      // fold the copies of each row (copy 0 keeps the result; only a finished
      // list is handed over, copy 0 keeps inserting into its own)
      if (copy > 0) tk.finish(k);
      if (valid && copy > 0) {
        const int o = (copy - 1) * rpc + r;
        xm[o] = m;
        xs[o] = s;
#pragma unroll
        for (int j = 0; j < KMAX; ++j) { xv[o * KMAX + j] = tk.v[j]; xi[o * KMAX + j] = tk.i[j]; }
      }
      epi_sync();
      if (valid && copy == 0) {
        for (int c = 1; c < R; ++c) {
          const int o = (c - 1) * rpc + r;
          lse_combine(m, s, xm[o], xs[o]);
#pragma unroll
          for (int j = 0; j < KMAX; ++j) {
            const float v = xv[o * KMAX + j];
            const int i = xi[o * KMAX + j];
            if (j < k && tk.admits(v, i)) tk.insert(v, i);
          }
        }
        tk.finish(k);
        p.ms[((size_t)par * C_ROWS + r) * p.G + cta] = make_float2(m, s);
        // entries at or above the row's gate join the row's candidates
        const uint32_t g = *reinterpret_cast<volatile uint32_t*>(thr);
        const float gate = fmaxf(g > f2ord(neg_inf()) ? ord2f(g) : neg_inf(), seed_gate);
        int n = 0;
#pragma unroll
        for (int j = 0; j < KMAX; ++j) n += (j < k && tk.v[j] != neg_inf() && tk.v[j] >= gate);
        if (n > 0) {
          const int pos = atomicAdd(&p.cand_cnt[(size_t)(d - 1) * C_ROWS + r], n);
          unsigned long long* dst = p.cand + ((size_t)par * C_ROWS + r) * p.cap + pos;
#pragma unroll
          for (int j = 0; j < KMAX; ++j)
            if (j < n) dst[j] = ((unsigned long long)f2ord(tk.v[j]) << 32) | (uint32_t)(~tk.i[j]);
        }
      }
      // grid barrier: every CTA's partials of this depth are written
      __threadfence();
      epi_sync();
      if (threadIdx.x == 64) {
        int fail = *abort_flag;
        if (!fail) {
          atomicAdd(&p.arrive[d - 1], 1u);
          const long long t0 = clock64();
          for (uint32_t spin = 0;; ++spin) {
            if (ld_acquire(&p.arrive[d - 1]) >= (unsigned)p.G) break;
            if (*reinterpret_cast<volatile int32_t*>(p.err)) { fail = 1; break; }
            if ((spin & 63u) == 63u && clock64() - t0 > kTimeoutCycles) {
              atomicExch(p.err, 1);
              fail = 1;
              break;
            }
          }
        } else {
          atomicExch(p.err, 1);
        }
        if (fail) *abort_flag = 1;
        misc[0] = fail;
      }
      epi_sync();
      if (misc[0]) break;

      // merge, step 1 (a warp per row, four rows of a warp at a time, every
      // load of the four issued before any is used): lse over the CTAs'
      // partials, the row's k best candidates, and their beam keys
      // s(p) + z - lse
      for (int r0 = ew; r0 < M; r0 += 4 * C_EPI) {
        constexpr int PL = 5;                    // partials per lane per pass (G <= 160)
        float lm[4], lsum[4];
        int ncand[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          lm[q] = neg_inf();
          lsum[q] = 0.f;
          const int rr = r0 + q * C_EPI;
          ncand[q] = rr < M ? __ldcg(p.cand_cnt + (size_t)(d - 1) * C_ROWS + rr) : 0;
        }
        // the first 32 candidates of each row are loaded with the counts
        unsigned long long first[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int rr = r0 + q * C_EPI;
          first[q] = (rr < M && lane < p.cap)
                         ? __ldcg(p.cand + ((size_t)par * C_ROWS + rr) * p.cap + lane) : 0ull;
        }
        for (int c0 = 0; c0 < p.G; c0 += 32 * PL) {
          float2 v[4][PL];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int rr = r0 + q * C_EPI;
            const float2* msr = p.ms + ((size_t)par * C_ROWS + (rr < M ? rr : 0)) * p.G;
#pragma unroll
            for (int i = 0; i < PL; ++i) {
              const int c = c0 + i * 32 + lane;
              v[q][i] = (rr < M && c < p.G) ? __ldcg(msr + c) : make_float2(neg_inf(), 0.f);
            }
          }
#pragma unroll
          for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int i = 0; i < PL; ++i) lse_combine(lm[q], lsum[q], v[q][i].x, v[q][i].y);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (lane >= min(ncand[q], p.cap)) first[q] = 0ull;   // entries past the count are stale
#pragma unroll 1
        for (int q = 0; q < 4; ++q) {
          const int rr = r0 + q * C_EPI;
          if (rr >= M) break;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) {
            const float m2 = __shfl_xor_sync(0xffffffffu, lm[q], o);
            const float s2 = __shfl_xor_sync(0xffffffffu, lsum[q], o);
            lse_combine(lm[q], lsum[q], m2, s2);
          }
          const float lse = (lm[q] == neg_inf()) ? neg_inf() : lm[q] + logf(lsum[q]);
          const int n = min(ncand[q], p.cap);
          const unsigned long long* cr = p.cand + ((size_t)par * C_ROWS + rr) * p.cap;
          unsigned long long top = warp_sort_desc(first[q], lane);
          for (int base = 32; base < n; base += 32) {
            unsigned long long x = base + lane < n ? __ldcg(cr + base + lane) : 0ull;
            x = warp_sort_desc(x, lane);
            top = warp_merge_top(top, __shfl_sync(0xffffffffu, x, 31 - lane), lane);
          }
          if (lane < k) {
            const int b = rr / Fp, i = rr - b * Fp;
            const float z = ord2f((uint32_t)(top >> 32));
            const int tok = (int)(~(uint32_t)top);
            mkeys[rr * k + lane] = top != 0ull ? beam_key(fs[rr] + (z - lse), i, tok) : 0ull;
            // every candidate may enter the beam: its E row heads to L2 now, so
            // the next A tile's gather finds it there
            if (top != 0ull && (unsigned)tok < (unsigned)p.V && d < p.D)
              for (int j = 0; j < p.r; j += 64)
                asm volatile("prefetch.global.L2 [%0];" ::"l"(p.E + (size_t)tok * p.r + j));
          }
        }
      }
      epi_sync();
      // merge, step 2 (a warp per request): the beam, then canonical order
      const int Fn = p.F[d];
      for (int b = ew; b < p.batch; b += C_EPI) {
        const int C = Fp * k;
        const unsigned long long* kb_ = mkeys + (size_t)b * C;
        unsigned long long top = 0ull;
        for (int base = 0; base < C; base += 32) {
          unsigned long long x = base + lane < C ? kb_[base + lane] : 0ull;
          x = warp_sort_desc(x, lane);
          top = base == 0 ? x : warp_merge_top(top, __shfl_sync(0xffffffffu, x, 31 - lane), lane);
        }
        // lanes t < Fn hold the beam, best first; sort them by (position, token)
        const unsigned long long ppos = (unsigned long long)beam_key_ppos(top);
        const unsigned long long tk_ = (unsigned long long)beam_key_tok(top);
        const unsigned long long ck = lane < Fn ? ~((ppos << 42) | (tk_ << 10) | (unsigned)lane) : 0ull;
        const unsigned long long srt = ~warp_sort_desc(ck, lane);
        const int rank = (int)(srt & 1023ull);
        const uint32_t shi = __shfl_sync(0xffffffffu, (uint32_t)(top >> 32), lane < Fn ? rank : 0);
        __syncwarp();
        // a beam entry without a candidate (non-finite logits) carries no token
        const bool real = __shfl_sync(0xffffffffu, top, lane < Fn ? rank : 0) != 0ull;
        if (lane < Fn && !real && cta == 0) atomicOr(&p.status[b], PCT_DEV_BAD_TOKEN);
        if (lane < Fn) {
          const int tok = real ? (int)((srt >> 10) & 0x3fffffull) : 0;
          const int pp = (int)(srt >> 42);
          const float sc = ord2f(shi);
          ftok[b * Fn + lane] = tok;   // rows of depth d + 1 (request-major)
          fs[b * Fn + lane] = sc;
          if (cta == 0) {
            const size_t o = ((size_t)(d - 1) * p.batch + b) * p.beam + lane;
            p.lvl_tok[o] = tok;
            p.lvl_ppos[o] = pp;
            p.lvl_s[o] = sc;
          }
        }
      }
      epi_sync();
      if (d < p.D) {
        build_a_tile(p, p.batch * Fn, Fn, ftok, sA, sOneHot);
        epi_sync();
        if (threadIdx.x == 64) mbar_arrive(aready);
        chain_seeds(p, d + 1, p.batch * Fn, Fn, sA, sseed, reinterpret_cast<__nv_bfloat16*>(mkeys),
                    seed_prefetchable(p) ? spre : nullptr);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(C_TMEM_COLS));
  }
}

// 3D bf16 tensor map over L [batch][D][V]: box {64 columns, 1 depth, 16
// requests}, 128-byte swizzle; requests past the batch read as zero.
bool encode_l3d(CUtensorMap* map, const void* L, int V, int D, int batch) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)V, (cuuint64_t)D, (cuuint64_t)batch};
  const cuuint64_t strides[2] = {(cuuint64_t)V * 2, (cuuint64_t)D * V * 2};
  const cuuint32_t box[3] = {64, 1, (cuuint32_t)C_LFOLD};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(L), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int KMAX>
cudaError_t set_chain_smem() {
  return cudaFuncSetAttribute(pct_chain_kernel<KMAX>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)chain_smem_bytes<KMAX>());
}

int chain_grid(int V) {
  const int tiles = (V + C_BN - 1) / C_BN;
  return std::max(1, std::min(num_sms(), tiles));
}

}  // namespace

bool chain_eligible(const ChainShape& c) {
  if (c.markov_dtype != PCT_BF16 || c.logits_dtype != PCT_BF16) return false;
  if (c.batch < 1 || c.batch > C_LFOLD || c.k > 16 || c.beam > C_MAXBEAM) return false;
  if (c.r % 8 != 0 || c.r_pad > C_KBMAX * C_BK || c.V % 8 != 0) return false;
  int F = 1;
  for (int d = 1; d <= c.D; ++d) {
    if (c.batch * F > C_ROWS || F * c.k > C_KEYS / c.batch) return false;
    F = std::min(c.beam, F * c.k);
  }
  if (c.batch * F > C_ROWS) return false;   // the last frontier is held too
  int dev = 0, coop = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev) != cudaSuccess || !coop)
    return false;
  int per_sm = 0;
  const size_t smem = c.k <= 4 ? chain_smem_bytes<4>() : c.k <= 8 ? chain_smem_bytes<8>()
                                                                  : chain_smem_bytes<16>();
  const cudaError_t e = c.k <= 4 ? set_chain_smem<4>() : c.k <= 8 ? set_chain_smem<8>()
                                                                  : set_chain_smem<16>();
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return false;
  }
  cudaError_t q;
  if (c.k <= 4) q = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, pct_chain_kernel<4>, C_THREADS, smem);
  else if (c.k <= 8) q = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, pct_chain_kernel<8>, C_THREADS, smem);
  else q = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, pct_chain_kernel<16>, C_THREADS, smem);
  if (q != cudaSuccess) {
    (void)cudaGetLastError();
    return false;
  }
  return per_sm >= 1 && chain_grid(c.V) <= per_sm * num_sms();
}

size_t chain_workspace(const ChainShape& c) {
  const size_t G = (size_t)chain_grid(c.V);
  const size_t cap = G * (size_t)c.k;
  size_t o = 0;
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  o += up(2 * C_ROWS * G * sizeof(float2));                 // ms
  o += up(2 * C_ROWS * cap * sizeof(unsigned long long));   // cand
  o += up((size_t)c.D * C_ROWS * 4 * 2 + (size_t)c.D * 4 + 4);   // cnt, thr, arrive, err (cleared)
  return o;
}

cudaError_t launch_chain(const ChainShape& c, const void* L, const int32_t* anchor, const void* E,
                         const void* W, void* ws, int32_t* lvl_tok, int32_t* lvl_ppos, float* lvl_s,
                         int32_t** err_out, int32_t* status, const int32_t* scol,
                         const float* slval, const float* swmax, const void* swcol,
                         cudaStream_t s) {
  const int G = chain_grid(c.V);
  const size_t cap = (size_t)G * c.k;
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  char* w = static_cast<char*>(ws);
  ChainParams p;
  p.batch = c.batch; p.D = c.D; p.V = c.V; p.k = c.k; p.beam = c.beam;
  p.r = c.r; p.r_pad = c.r_pad; p.kblocks = c.r_pad / C_BK; p.G = G;
  p.tiles_total = (c.V + C_BN - 1) / C_BN;
  p.cap = (int)cap;
  p.F[0] = 1;
  for (int d = 1; d <= c.D; ++d) p.F[d] = std::min(c.beam, p.F[d - 1] * c.k);
  p.E = static_cast<const __nv_bfloat16*>(E);
  p.anchor = anchor;
  p.ms = reinterpret_cast<float2*>(w);
  w += up(2 * C_ROWS * (size_t)G * sizeof(float2));
  p.cand = reinterpret_cast<unsigned long long*>(w);
  w += up(2 * C_ROWS * cap * sizeof(unsigned long long));
  char* cleared = w;
  const size_t cleared_bytes = (size_t)c.D * C_ROWS * 4 * 2 + (size_t)c.D * 4 + 4;
  p.cand_cnt = reinterpret_cast<int32_t*>(w);
  p.row_thr = reinterpret_cast<uint32_t*>(w + (size_t)c.D * C_ROWS * 4);
  p.arrive = reinterpret_cast<unsigned*>(w + (size_t)c.D * C_ROWS * 8);
  p.err = reinterpret_cast<int32_t*>(w + (size_t)c.D * C_ROWS * 8 + (size_t)c.D * 4);
  p.lvl_tok = lvl_tok; p.lvl_ppos = lvl_ppos; p.lvl_s = lvl_s;
  p.status = status;
  p.scol = scol; p.slval = slval; p.swmax = swmax;
  p.swcol = static_cast<const __nv_bfloat16*>(swcol);
  *err_out = p.err;
  CUtensorMap tmB, tmL;
  if (!encode_2d_bf16(&tmB, W, (uint64_t)c.V, (uint64_t)c.r, 64, C_BK)) return cudaErrorInvalidValue;
  if (!encode_l3d(&tmL, L, c.V, c.D, c.batch)) return cudaErrorInvalidValue;
  cudaError_t e = cudaMemsetAsync(cleared, 0, cleared_bytes, s);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(G);
  cfg.blockDim = dim3(C_THREADS);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  TraceScope t(s, "pct_chain");
  if (c.k <= 4) {
    cfg.dynamicSmemBytes = chain_smem_bytes<4>();
    e = cudaLaunchKernelEx(&cfg, pct_chain_kernel<4>, tmB, tmL, p);
  } else if (c.k <= 8) {
    cfg.dynamicSmemBytes = chain_smem_bytes<8>();
    e = cudaLaunchKernelEx(&cfg, pct_chain_kernel<8>, tmB, tmL, p);
  } else {
    cfg.dynamicSmemBytes = chain_smem_bytes<16>();
    e = cudaLaunchKernelEx(&cfg, pct_chain_kernel<16>, tmB, tmL, p);
  }
  if (e != cudaSuccess) (void)cudaGetLastError();
  return e;
}

}  // namespace pct
