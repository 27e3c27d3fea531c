// Batched parent scoring on CTA pairs (tcgen05 cta_group::2, bf16 Markov
// parameters): the form used for more than 128 parent rows.
//
// PCTree article (qiita), section on the chain draft's weakness and the tree
// built in its place: for every frontier parent p of a depth, in one batched
// call, z_d(p) = L_d + Markov(p), followed by the softmax over the vocabulary
// and the parent's local top-k. With the rank-r stand-in Markov(p) = E[p] . W
// the batched call is the contraction Eg[M][r] . W[r][V].
//
// Design: a cluster of two CTAs on two SMs computes 256 parent rows against
// 256-column N-tiles with pair MMAs (M = 256, N = 256, K = 16: each SM owns
// 128 rows and all 256 columns of the accumulator, and holds half of the W
// tile). One pair MMA keeps both SMs' tensor cores busy for 128 cycles, so the
// issue loop and its per-stage handshakes cost little next to the math.
//  * warp 0, one thread per CTA: TMA producer. The CTA's 128 Eg rows once
//    (K-major, 128-byte swizzle); W through an 8-slot ring of [64 K][128 V]
//    half tiles (V-major, 128-byte swizzle); with folded L_d, the requests'
//    [16][128] L_d half tile per N-tile through a 2-slot ring. Every load
//    signals the leader CTA's barrier, which counts both halves.
//  * warp 1, one thread of the leader CTA: issues the pair MMAs into a
//    double-buffered accumulator (2 x 256 TMEM columns), commits each ring slot
//    and each finished accumulator to the barriers of both CTAs.
//  * warps 2..17 of each CTA: epilogue. Warp w reads TMEM lane quarter w % 4
//    and one 64-column quarter of every N-tile: L_d add (unless folded),
//    online log-sum-exp, and a register top-k behind an admission gate seeded
//    with a lower bound of the row's k-th value. The four column quarters of a
//    row are folded at the end and one partial per (row, V-slice) is written.
// Every mbarrier wait is bounded; on expiry the CTA raises an abort flag, sets
// the device error word and leaves its loops; the leader drains its MMAs and
// both CTAs meet at a cluster barrier before TMEM is released.
#include <cuda.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "umma.cuh"

namespace pct {

namespace {

constexpr int P_BM = 128;                  // rows per CTA (pair: 256)
constexpr int P_BN = 256;                  // columns per N-tile (each CTA loads 128)
constexpr int P_HALF = 128;
constexpr int P_BK = 64;
constexpr int P_STAGES = 8;
constexpr int P_KBMAX = 4;                 // r_pad <= 256
constexpr int P_A_BLOCK = P_BM * P_BK * 2;           // 16 KB per K block
constexpr int P_B_STAGE = P_BK * P_HALF * 2;         // 16 KB per ring slot
constexpr int P_EPI_WARPS = 16;                      // 4 per TMEM lane quarter
constexpr int P_THREADS = 64 + 32 * P_EPI_WARPS;
constexpr int P_CH = 32;                             // accumulator columns per chunk
constexpr bool P_PREFETCH = false;                   // next chunk's TMEM load in flight
static_assert(P_CH == 16 || P_CH == 32, "a chunk's candidate mask is one 32-bit word");
constexpr int P_COLS_PER_WARP = P_BN / 4;            // 64
constexpr int P_SOFT = 0;   // of every 16 exponentials on the FMA pipe (0, 2, 4, 6 measured: 0 fastest)
constexpr int P_LFOLD = 16;
constexpr int P_LPART = P_LFOLD * P_HALF * 2;        // [16 K][128 N] = 4 KB per slot
constexpr int P_ONEHOT = P_BM * P_LFOLD * 2;         // [128 rows][16 K] = 4 KB
constexpr size_t P_SMEM = 1024 + (size_t)P_KBMAX * P_A_BLOCK + (size_t)P_STAGES * P_B_STAGE +
                          2 * (size_t)P_LPART + P_ONEHOT + 512;

// kind::f16 instruction descriptor: D f32, A = B = bf16, A K-major, B
// MN-major, N = 256, M = 256 (pair).
constexpr uint32_t P_IDESC = (1u << 4) | (1u << 7) | (1u << 10) | (0u << 15) | (1u << 16) |
                             ((uint32_t)(P_BN >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);

struct PairParams {
  int M, n_par, V, kblocks, S, tiles_total, k;
  const void* L;
  long long L_req_stride;
  float2* pms;
  float* pval;
  int32_t* pidx;
  int32_t* err;
  uint32_t* row_thr;
};

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// The same shared-memory object in CTA 0 of the cluster (shared::cluster address).
__device__ __forceinline__ uint32_t leader_addr(const void* p) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, 0;" : "=r"(r) : "r"(smem_u32(p)));
  return r;
}
// Arrivals on the leader's barriers use the default (CTA-scope) semantics: what
// they publish is either TMEM reads already ordered by a tcgen05 fence (the
// epilogue's release of an accumulator) or bulk tensor copy bytes counted
// by the barrier itself (the producers' loads), so no cluster-scope memory
// fence is needed in front of them.
__device__ __forceinline__ void arrive_leader(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void arrive_expect_leader(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cluster.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
// Tile load into this CTA's shared memory; completion counted on the leader's barrier.
__device__ __forceinline__ void tma_load_pair(void* dst, const CUtensorMap* map, int x, int y,
                                              uint32_t leader_bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(leader_bar)
      : "memory");
}
__device__ __forceinline__ void umma_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %3, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %4, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(accumulate), "r"(P_IDESC));
}
// Arrives on the barrier at this offset in both CTAs once the leader's prior MMAs complete.
__device__ __forceinline__ void commit_pair(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], m;\n\t}" ::"r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}

template <typename TL, int KMAX, bool FOLD>
__global__ void __launch_bounds__(P_THREADS, 1)
    score_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const __grid_constant__ CUtensorMap tmL, const PairParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + P_KBMAX * P_A_BLOCK;
  uint8_t* sL = sB + P_STAGES * P_B_STAGE;       // [2] L_d half tiles (folded L_d)
  uint8_t* sOneHot = sL + 2 * P_LPART;
  uint64_t* full = reinterpret_cast<uint64_t*>(sOneHot + P_ONEHOT);   // [STAGES] leader: 2 producers
  uint64_t* empty = full + P_STAGES;                                  // [STAGES] each CTA
  uint64_t* lfull = empty + P_STAGES;                                 // [2] leader
  uint64_t* lempty = lfull + 2;                                       // [2] each CTA
  uint64_t* afull = lempty + 2;                                       // leader
  uint64_t* tfull = afull + 1;                                        // [2] each CTA
  uint64_t* tempty = tfull + 2;                                       // [2] leader: all epilogue warps
  uint64_t* fin = tempty + 2;                                         // each CTA
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int sl = blockIdx.x >> 1, mt = blockIdx.y;
  const int t_begin = (int)((long long)sl * p.tiles_total / p.S);
  const int t_end = (int)((long long)(sl + 1) * p.tiles_total / p.S);
  const int ntiles = t_end - t_begin;
  const int prow0 = mt * 2 * P_BM;                  // first row of the pair
  const int row0 = prow0 + (int)rank * P_BM;        // first row of this CTA
  const int req0 = prow0 / p.n_par;                 // first request of the pair

  if (threadIdx.x == 0) {
    for (int i = 0; i < P_STAGES; ++i) { mbar_init(&full[i], 2); mbar_init(&empty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&lfull[i], 2);
      mbar_init(&lempty[i], 1);
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 2 * P_EPI_WARPS);
    }
    mbar_init(afull, 2);
    mbar_init(fin, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (FOLD && warp >= 2 && warp < 6) {
    // one-hot request indicator of this CTA's rows (K-major, 32-byte swizzle:
    // the two 16-byte halves of a row swap in rows 4..7 of each 8-row group)
    const int i = (warp & 3) * 32 + lane;
    const int rr = row0 + i;
    const int kk = rr < p.M ? rr / p.n_par - req0 : -1;
    uint8_t* rowp = sOneHot + (i >> 3) * 256 + (i & 7) * 32;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int kl = kk - 8 * half;
      const uint32_t one = 0x3F80u << (16 * (kl & 1));   // bf16 1.0 in its half word
      const int wi = (kl >= 0 && kl < 8) ? (kl >> 1) : -1;
      const int phys = half ^ ((i >> 2) & 1);
      *reinterpret_cast<uint4*>(rowp + 16 * phys) =
          make_uint4(wi == 0 ? one : 0u, wi == 1 ? one : 0u, wi == 2 ? one : 0u, wi == 3 ? one : 0u);
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();   // barriers, one-hot tiles and TMEM of both CTAs are ready
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();   // the set-up above touches only shared memory and TMEM
  pdl_trigger();

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (each CTA) ----------------
      const uint32_t l_afull = leader_addr(afull);
      arrive_expect_leader(l_afull, (uint32_t)(p.kblocks * P_A_BLOCK));
      for (int kb = 0; kb < p.kblocks; ++kb)
        tma_load_pair(sA + kb * P_A_BLOCK, &tmA, kb * P_BK, row0, l_afull);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      uint32_t armed = 0, armed_par = 0;   // leader's drain: ring slots loaded, parity of the last
      int larmed = 0;
      for (int it = 0; it < ntiles && ok; ++it) {
        const int n0 = (t_begin + it) * P_BN + (int)rank * P_HALF;
        if (FOLD) {
          const int ls = it & 1;
          if (!wait_bar(&lempty[ls], (((uint32_t)it >> 1) & 1u) ^ 1u, abort_flag, p.err)) break;
          const uint32_t lb = leader_addr(&lfull[ls]);
          arrive_expect_leader(lb, (uint32_t)P_LPART);
          tma_load_pair(sL + ls * P_LPART, &tmL, n0, req0, lb);
          tma_load_pair(sL + ls * P_LPART + P_LPART / 2, &tmL, n0 + 64, req0, lb);
          larmed = it + 1;
        }
        for (int kb = 0; kb < p.kblocks; ++kb) {
          if (!wait_bar(&empty[stage], phase ^ 1u, abort_flag, p.err)) { ok = false; break; }
          const uint32_t fb = leader_addr(&full[stage]);
          arrive_expect_leader(fb, (uint32_t)P_B_STAGE);
          uint8_t* dst = sB + stage * P_B_STAGE;
          tma_load_pair(dst, &tmB, n0, kb * P_BK, fb);
          tma_load_pair(dst + P_B_STAGE / 2, &tmB, n0 + 64, kb * P_BK, fb);
          armed |= 1u << stage;
          armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
          if (++stage == P_STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (rank == 0) {
        // every load of either CTA counted on the leader's barriers has landed
        drain_wait(afull, 0);
#pragma unroll 1
        for (int i = 0; i < P_STAGES; ++i)
          if (armed & (1u << i)) drain_wait(&full[i], (armed_par >> i) & 1u);
        for (int t = larmed - 2; t < larmed; ++t)
          if (t >= 0) drain_wait(&lfull[t & 1], ((uint32_t)t >> 1) & 1u);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ---------------- pair MMA issuer (leader CTA) ----------------
      bool ok = wait_bar(afull, 0, abort_flag, p.err);
      tc_fence_after();
      int stage = 0;
      uint32_t phase = 0;
      const uint64_t a_desc0 = make_desc(smem_u32(sA), 16, 1024);
      const uint64_t b_desc0 = make_desc(smem_u32(sB), 8192, 1024);
      const uint64_t x_desc = make_desc(smem_u32(sOneHot), 16, 256, 6);
      const uint64_t l_desc0 = make_desc(smem_u32(sL), P_LPART / 2, 1024);
      for (int it = 0; it < ntiles && ok; ++it) {
        const int buf = it & 1;
        if (!wait_bar(&tempty[buf], (((uint32_t)it >> 1) & 1u) ^ 1u, abort_flag, p.err)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + (uint32_t)(buf * P_BN);
        for (int kb = 0; kb < p.kblocks; ++kb) {
          if (!wait_bar(&full[stage], phase, abort_flag, p.err)) { ok = false; break; }
          const uint64_t bd = b_desc0 + (uint64_t)((stage * P_B_STAGE) >> 4);
          const uint64_t ad = a_desc0 + (uint64_t)((kb * P_A_BLOCK) >> 4);
          umma_pair(d, ad, bd, kb != 0);
          umma_pair(d, ad + 2, bd + 128, 1u);
          umma_pair(d, ad + 4, bd + 256, 1u);
          umma_pair(d, ad + 6, bd + 384, 1u);
          commit_pair(&empty[stage]);
          if (++stage == P_STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        if (FOLD) {
          const int ls = it & 1;
          if (!wait_bar(&lfull[ls], ((uint32_t)it >> 1) & 1u, abort_flag, p.err)) break;
          umma_pair(d, x_desc, l_desc0 + (uint64_t)((ls * P_LPART) >> 4), 1u);
          commit_pair(&lempty[ls]);
        }
        commit_pair(&tfull[buf]);
      }
      // every MMA complete (signalled in both CTAs) before the operands or TMEM go
      commit_pair(fin);
      drain_wait(fin, 0);
    } else if (lane == 0) {
      drain_wait(fin, 0);
    }
  } else {
    // ---------------- epilogue (each CTA) ----------------
    const int quad = warp & 3;
    const int h = (warp - 2) >> 2;                  // 64-column quarter of every N-tile
    const int r_in = quad * 32 + lane;
    const int row = row0 + r_in;
    const bool valid = row < p.M;
    const int req = valid ? row / p.n_par : req0;
    const TL* Lr = static_cast<const TL*>(p.L) + (size_t)req * p.L_req_stride;
    const int k = p.k, V = p.V;
    float m = neg_inf(), s = 0.f;
    TopK<KMAX> tk;
    tk.init(k);
    // admission gate: the largest known lower bound of the row's k-th value
    // (the row's seed, this CTA's own k-th, other slices' published k-th)
    uint32_t* thr = p.row_thr + (valid ? row : 0);
    uint32_t pub_prev = valid ? *reinterpret_cast<volatile uint32_t*>(thr) : 0u;
    float gth = pub_prev > f2ord(neg_inf()) ? ord2f(pub_prev) : neg_inf();
    const uint32_t l_tempty0 = leader_addr(&tempty[0]), l_tempty1 = leader_addr(&tempty[1]);
    for (int it = 0; it < ntiles; ++it) {
      const int buf = it & 1;
      if (!wait_bar(&tfull[buf], ((uint32_t)it >> 1) & 1u, abort_flag, p.err)) break;
      tc_fence_after();
      const int n0 = (t_begin + it) * P_BN + h * P_COLS_PER_WARP;
      const uint32_t tbase = tmem_base + ((uint32_t)(quad * 32) << 16) +
                             (uint32_t)(buf * P_BN + h * P_COLS_PER_WARP);
      auto chunk = [&](int c, const uint32_t (&acc)[P_CH]) {
        const int col0 = n0 + c * P_CH;
        float x[P_CH];
        if (!valid) return;
        if (FOLD) {
#pragma unroll
          for (int j = 0; j < P_CH; ++j) x[j] = __uint_as_float(acc[j]);
        } else {
          load_logits<TL, P_CH>(Lr, col0, V, x);
#pragma unroll
          for (int j = 0; j < P_CH; j += 2) {
            const float2 z2 = f2_add(make_float2(x[j], x[j + 1]),
                                     make_float2(__uint_as_float(acc[j]), __uint_as_float(acc[j + 1])));
            x[j] = z2.x;
            x[j + 1] = z2.y;
          }
        }
        if (col0 + P_CH > V) {
#pragma unroll
          for (int j = 0; j < P_CH; ++j) x[j] = (col0 + j < V) ? x[j] : neg_inf();
        }
        const float cm = chunk_max<P_CH>(x);
        // sum of exp against the running reference m, which moves only when a
        // value exceeds it by more than 64 (the chunk is then summed again)
        float csum = 0.f;
        if (m != neg_inf()) csum = chunk_exp_sum<P_CH, P_SOFT>(x, m);
        if (cm > m + 64.f) {
          s = (m == neg_inf()) ? 0.f : s * ex2((m - cm) * kLog2e);
          m = cm;
          csum = chunk_exp_sum<P_CH, P_SOFT>(x, m);
        }
        s += csum;
        if (cm >= gth) {
          uint32_t cand = 0;
#pragma unroll
          for (int j = 0; j < P_CH; ++j) cand |= (uint32_t)(x[j] >= gth) << j;
          while (cand) {
            const int j = __ffs(cand) - 1;
            cand &= cand - 1;
            float z = x[0];
#pragma unroll
            for (int jj = 1; jj < P_CH; ++jj) z = (j == jj) ? x[jj] : z;
            if (z >= gth && tk.admits(z, col0 + j)) {
              tk.insert(z, col0 + j);
              gth = fmaxf(gth, tk.tv());
            }
          }
        }
      };
      constexpr int NCH = P_COLS_PER_WARP / P_CH;
      if (P_PREFETCH) {
        // the next chunk's accumulator load is in flight while a chunk is processed
        uint32_t acc_a[P_CH], acc_b[P_CH];
        tmem_issue(tbase, acc_a);
#pragma unroll 1
        for (int i = 0; i < NCH; i += 2) {
          tmem_wait(acc_a);
          tmem_issue(tbase + (uint32_t)((i + 1) * P_CH), acc_b);
          chunk(i, acc_a);
          tmem_wait(acc_b);
          if (i + 2 < NCH) tmem_issue(tbase + (uint32_t)((i + 2) * P_CH), acc_a);
          chunk(i + 1, acc_b);
        }
      } else {
#pragma unroll 1
        for (int i = 0; i < NCH; ++i) {
          uint32_t acc[P_CH];
          tmem_issue(tbase + (uint32_t)(i * P_CH), acc);
          tmem_wait(acc);
          chunk(i, acc);
        }
      }
      if (valid) {
        if (pub_prev > f2ord(neg_inf())) gth = fmaxf(gth, ord2f(pub_prev));
        const float own = tk.tv();
        if (own != neg_inf()) atomicMax(thr, f2ord(own));
        pub_prev = *reinterpret_cast<volatile uint32_t*>(thr);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) arrive_leader(buf ? l_tempty1 : l_tempty0);
    }
    // fold the four column quarters of each row through shared memory (the Eg
    // region is idle once the leader's last MMA has completed in both CTAs)
    drain_wait(fin, 0);
    float2* xms = reinterpret_cast<float2*>(sA);                        // [3][128]
    float* xv = reinterpret_cast<float*>(sA + 3 * P_BM * sizeof(float2));  // [3][128][KMAX]
    int* xi = reinterpret_cast<int*>(xv + 3 * P_BM * KMAX);              // [3][128][KMAX]
    if (h > 0) {
      tk.finish(k);
      const int o = (h - 1) * P_BM + r_in;
      xms[o] = make_float2(m, s);
#pragma unroll
      for (int j = 0; j < KMAX; ++j) { xv[o * KMAX + j] = tk.v[j]; xi[o * KMAX + j] = tk.i[j]; }
    }
    asm volatile("bar.sync 1, %0;" ::"n"(P_EPI_WARPS * 32) : "memory");
    if (h == 0 && valid) {
      for (int q = 0; q < 3; ++q) {
        const int o = q * P_BM + r_in;
        const float2 ms = xms[o];
        lse_combine(m, s, ms.x, ms.y);
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
          const float v = xv[o * KMAX + j];
          const int id = xi[o * KMAX + j];
          if (j < k && tk.admits(v, id)) tk.insert(v, id);
        }
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
  cluster_sync_all();   // no MMA or load of the pair still uses either CTA's memory
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(512));
  }
}

}  // namespace

int pair_rows_min() { return P_BM + 1; }

int pair_slices(int rows, int V) {
  const int pairs = num_sms() / 2;
  const int mtiles = (rows + 2 * P_BM - 1) / (2 * P_BM);
  const int tiles = (V + P_BN - 1) / P_BN;
  return std::max(1, std::min(tiles, pairs / std::max(mtiles, 1)));
}

cudaError_t launch_score_pair(const ScoreArgs& a, cudaStream_t s) {
  const int rows = a.n_req * a.n_par;
  if (a.r_pad > P_KBMAX * P_BK) return cudaErrorInvalidValue;
  CUtensorMap tmA, tmB, tmL;
  if (!encode_2d_bf16(&tmA, a.Eg, (uint64_t)a.r_pad, (uint64_t)a.M_pad, P_BK, P_BM))
    return cudaErrorInvalidValue;
  if (!encode_2d_bf16(&tmB, a.W, (uint64_t)a.V, (uint64_t)a.r, 64, P_BK)) return cudaErrorInvalidValue;
  PairParams p;
  p.M = rows;
  p.n_par = a.n_par;
  p.V = a.V;
  p.kblocks = a.r_pad / P_BK;
  p.S = a.S;
  p.tiles_total = (a.V + P_BN - 1) / P_BN;
  p.k = a.k;
  p.L = a.L;
  p.L_req_stride = a.L_req_stride;
  p.pms = a.part.ms;
  p.pval = a.part.val;
  p.pidx = a.part.idx;
  p.err = a.err;
  p.row_thr = a.row_thr;
  if (!a.thr_seeded &&
      cudaMemsetAsync(a.row_thr, 0, sizeof(uint32_t) * (size_t)rows, s) != cudaSuccess)
    return cudaErrorInvalidValue;
  const int mtiles = (rows + 2 * P_BM - 1) / (2 * P_BM);
  int span = 0;   // requests any pair's rows touch
  for (int mt = 0; mt < mtiles; ++mt) {
    const int r0 = mt * 2 * P_BM, r1 = std::min(rows, r0 + 2 * P_BM) - 1;
    span = std::max(span, r1 / a.n_par - r0 / a.n_par + 1);
  }
  const bool fold = a.logits_dtype == PCT_BF16 && span <= P_LFOLD;
  if (fold) {
    // [16 requests][64 columns] boxes, 128-byte swizzle (the MMA's B layout);
    // rows past the last request read as zero
    if (!encode_2d_bf16(&tmL, a.L, (uint64_t)a.V, (uint64_t)a.n_req, 64, (uint32_t)P_LFOLD,
                        (uint64_t)a.L_req_stride * 2, true))
      return cudaErrorInvalidValue;
  } else {
    tmL = tmB;   // unused
  }
  const dim3 grid(2 * a.S, mtiles);
  TraceScope t(s, "pct_score_pair");
#define PCT_PAIR(TL, KM, FD)                                                                  \
  do {                                                                                        \
    auto kern = score_pair_kernel<TL, KM, FD>;                                                \
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,   \
                                         (int)P_SMEM);                                        \
    if (e != cudaSuccess) {                                                                   \
      (void)cudaGetLastError();                                                               \
      return e;                                                                               \
    }                                                                                         \
    e = launch_pdl(kern, grid, dim3(P_THREADS), P_SMEM, s, 2, tmA, tmB, tmL, p);              \
    if (e != cudaSuccess) return e;                                                           \
  } while (0)
#define PCT_PAIR_K(TL, FD)                        \
  do {                                            \
    if (a.k <= 4) PCT_PAIR(TL, 4, FD);            \
    else if (a.k <= 8) PCT_PAIR(TL, 8, FD);       \
    else PCT_PAIR(TL, 16, FD);                    \
  } while (0)
  if (fold) PCT_PAIR_K(__nv_bfloat16, true);
  else if (a.logits_dtype == PCT_BF16) PCT_PAIR_K(__nv_bfloat16, false);
  else PCT_PAIR_K(float, false);
#undef PCT_PAIR_K
#undef PCT_PAIR
  return cudaGetLastError();
}

}  // namespace pct
