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
#include "umma.cuh"

namespace pct {

cudaError_t launch_score_simt(const ScoreArgs& a, cudaStream_t s);
// CTA-pair form (pct_umma2.cu), used from pair_rows_min() rows on
int pair_rows_min();
int pair_slices(int rows, int V);
cudaError_t launch_score_pair(const ScoreArgs& a, cudaStream_t s);

namespace {

constexpr int BM = 128;                  // UMMA M (rows per tile)
constexpr int BN = 128;                  // UMMA N (vocabulary columns per tile)
constexpr int BK = 64;                   // K per ring slot: one 128-byte swizzle row of bf16
constexpr int STAGES = 4;                // ring slots after the A tiles
constexpr int STAGES_MAX = 8;            // with one row tile, the second tile's space holds 4 more
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
// Folded L_d: a CTA whose rows span at most LFOLD requests adds L_d inside the
// MMA, as one more K=16 step whose A operand is the rows' one-hot request
// indicator and whose B operand is the requests' [16][128] L_d tile.
constexpr int LFOLD = 16;
constexpr int LF_PART_BYTES = LFOLD * BN * 2;    // [16 K][128 N] bf16 per ring slot = 4 KB
constexpr int LF_ONEHOT_BYTES = BM * LFOLD * 2;  // [128 rows][16 K] bf16 per row tile = 4 KB
// L_d modes of the scoring kernel
constexpr int L_GLOBAL = 0;   // epilogue loads L_d from global memory (L2)
constexpr int L_STAGE = 1;    // L_d tiles staged in shared memory by TMA, added by the epilogue
constexpr int L_FOLD = 2;     // L_d added by the tensor cores
constexpr size_t SMEM_BYTES = 1024 + (size_t)NSUBMAX * KBMAX * A_TILE_BYTES +
                              (size_t)STAGES * B_STAGE_BYTES + 2 * (size_t)L_SLOT_BYTES + 256;

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
  int b_kmajor;        // 1: W's tiles come from its transpose [V][r_pad] (K-major)
};

// LMODE (L_GLOBAL / L_STAGE / L_FOLD) says how the drafter logits L_d join
// the Markov product: loaded by the epilogue from global memory (L2); staged
// per N-tile in shared memory by TMA (bf16 logits, a CTA touching at most LBMAX
// requests) and added by the epilogue; or folded into the MMA (bf16 logits, at
// most LFOLD requests per CTA), in which case the accumulator already holds z.
template <typename TL, int KMAX, int LMODE>
__global__ void __launch_bounds__(THREADS, 1)
    score_umma_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const __grid_constant__ CUtensorMap tmL, const UmmaParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + NSUBMAX * KBMAX * A_TILE_BYTES;
  uint8_t* sL = sB + STAGES * B_STAGE_BYTES;   // L_STAGE: [2] L_d slots; L_FOLD: [STAGES] L_d
                                               // parts, then [2] one-hot tiles
  uint8_t* sOneHot = sL + STAGES * LF_PART_BYTES;
  constexpr bool STAGE = LMODE == L_STAGE;
  constexpr bool FOLD = LMODE == L_FOLD;
  uint64_t* full = reinterpret_cast<uint64_t*>(sL + 2 * L_SLOT_BYTES);
  uint64_t* empty = full + STAGES_MAX;
  uint64_t* afull = empty + STAGES_MAX;
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
  // W ring: slots 0..3 after the A tiles; with a single row tile (and L_d not
  // folded, whose per-slot parts have room for four) slots 4..7 in the unused
  // second A tile, so that two N-tiles of W are in flight instead of one
  const int nst = (!FOLD && p.nsub == 1) ? STAGES_MAX : STAGES;
  uint8_t* const sB2 = sA + KBMAX * A_TILE_BYTES;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES_MAX; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
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
  if (FOLD && warp >= 2) {
    // one-hot request indicator of every row (K-major, 32-byte swizzle: the
    // two 16-byte halves of a row swap in rows 4..7 of each 8-row group)
    const int e = warp - 2, g = e >> 2, st = g / SPLIT, h = g % SPLIT;
    const int i = (warp & 3) * 32 + lane;        // row within the tile
    const int rr = row0 + st * BM + i;
    if (h == 0 && st < NSUBMAX) {
      const int kk = (st < p.nsub && rr < p.M) ? rr / p.n_par - row0 / p.n_par : -1;
      uint8_t* rowp = sOneHot + st * LF_ONEHOT_BYTES + (i >> 3) * 256 + (i & 7) * 32;
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
  pdl_wait();   // the set-up above touches only shared memory and TMEM
  pdl_trigger();

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
        // W first: its slots free as the MMAs finish, the staged L_d slots only
        // as the epilogue does, so waiting for an L_d slot before a tile's W
        // would hold W back by a tile
        for (int kb = 0; kb < p.kblocks; ++kb) {
          if (!wait_bar(&empty[stage], phase ^ 1u, abort_flag, p.err)) { ok = false; break; }
          const bool lpart = FOLD && kb == 0;
          mbar_expect_tx(&full[stage], B_STAGE_BYTES + (lpart ? LF_PART_BYTES : 0));
          uint8_t* dst = stage < STAGES ? sB + stage * B_STAGE_BYTES
                                        : sB2 + (stage - STAGES) * B_STAGE_BYTES;
          if (p.b_kmajor) {
            // [128 N rows][64 K] of W's transpose: one contiguous 16 KB piece
            tma_load_2d(dst, &tmB, kb * BK, n0, &full[stage]);
          } else {
            tma_load_2d(dst, &tmB, n0, kb * BK, &full[stage]);
            tma_load_2d(dst + B_STAGE_BYTES / 2, &tmB, n0 + 64, kb * BK, &full[stage]);
          }
          if (lpart) {
            // the CTA's requests' L_d rows as the extra K block: [16 K][2 x 64 N]
            uint8_t* ldst = sL + stage * LF_PART_BYTES;
            tma_load_2d(ldst, &tmL, n0, req0, &full[stage]);
            tma_load_2d(ldst + LF_PART_BYTES / 2, &tmL, n0 + 64, req0, &full[stage]);
          }
          armed |= 1u << stage;
          armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
          if (++stage == nst) { stage = 0; phase ^= 1u; }
        }
        if (STAGE && ok) {
          const int slot = it & 1;
          if (!wait_bar(&lempty[slot], (((uint32_t)it >> 1) & 1u) ^ 1u, abort_flag, p.err)) { ok = false; break; }
          mbar_expect_tx(&lfull[slot], (uint32_t)(2 * 64 * p.LB * 2));
          uint8_t* dst = sL + slot * L_SLOT_BYTES;
          tma_load_2d(dst, &tmL, n0, req0, &lfull[slot]);
          tma_load_2d(dst + 64 * p.LB * 2, &tmL, n0 + 64, req0, &lfull[slot]);
          larmed = (uint32_t)it + 1;
        }
      }
      // every load this thread issued has landed before the CTA may exit
      drain_wait(afull, 0);
#pragma unroll
      for (int i = 0; i < STAGES_MAX; ++i)
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
      // B: [64 K][2 x 64 V] V-major (W), +2048 bytes per 16 K rows; or, from
      // W's transpose, [128 V][64 K] K-major like A, +32 bytes per 16 K
      const uint32_t b_lbo = p.b_kmajor ? 16u : 8192u;
      const uint64_t b_desc0 = make_desc(smem_u32(sB), b_lbo, 1024);    // ring slot 0
      const uint64_t b_desc4 = make_desc(smem_u32(sB2), b_lbo, 1024);   // ring slot 4 (one row tile)
      const uint64_t b_k16 = p.b_kmajor ? 2u : 128u;
      const uint32_t idesc_w = p.b_kmajor ? (IDESC & ~(1u << 16)) : IDESC;
      // folded L_d: one-hot rows (K-major, 32-byte swizzle, 8-row groups 256
      // bytes apart) times the L_d part of ring slot `stage` (V-major,
      // 128-byte swizzle, the two 64-column halves 2048 bytes apart)
      const uint64_t x_desc0 = make_desc(smem_u32(sOneHot), 16, 256, 6);
      const uint64_t l_desc0 = make_desc(smem_u32(sL), LF_PART_BYTES / 2, 1024);
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
          const uint64_t bd = stage < STAGES ? b_desc0 + (uint64_t)((stage * B_STAGE_BYTES) >> 4)
                                             : b_desc4 + (uint64_t)(((stage - STAGES) * B_STAGE_BYTES) >> 4);
          const uint64_t ad = a_desc0 + (uint64_t)((kb * A_TILE_BYTES) >> 4);
          const uint32_t acc0 = kb != 0;
          // A: [128 rows][64 K] K-major, +32 bytes per 16 K columns
          umma_f16(d0, ad, bd, idesc_w, acc0);
          if (two) umma_f16(d1, ad + (KBMAX * A_TILE_BYTES >> 4), bd, idesc_w, acc0);
#pragma unroll
          for (int k4 = 1; k4 < BK / 16; ++k4) {
            umma_f16(d0, ad + (uint64_t)(k4 * 2), bd + k4 * b_k16, idesc_w, 1u);
            if (two)
              umma_f16(d1, ad + (uint64_t)((KBMAX * A_TILE_BYTES >> 4) + k4 * 2),
                       bd + k4 * b_k16, idesc_w, 1u);
          }
          if (FOLD && kb == 0) {
            const uint64_t ld = l_desc0 + (uint64_t)((stage * LF_PART_BYTES) >> 4);
            umma_f16(d0, x_desc0, ld, IDESC, 1u);
            if (two) umma_f16(d1, x_desc0 + (uint64_t)(LF_ONEHOT_BYTES >> 4), ld, IDESC, 1u);
          }
          umma_commit(&empty[stage]);
          if (++stage == nst) { stage = 0; phase ^= 1u; }
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
    // admission gate: the largest known lower bound of the row's k-th value:
    // the row's seed (k exact values of the row, stored before the launch),
    // this slice's own k-th value, and the k-th values other slices of the
    // row have published. Values below the gate cannot be in the row's top-k.
    uint32_t* thr = p.row_thr + (valid ? row : 0);
    uint32_t pub_prev = valid ? *reinterpret_cast<volatile uint32_t*>(thr) : 0u;
    float gth = pub_prev > f2ord(neg_inf()) ? ord2f(pub_prev) : neg_inf();
    for (int it = 0; it < ntiles; ++it) {
      const int buf = it & 1;
      const uint32_t par = (uint32_t)((it >> 1) & 1);
      if (!wait_bar(&tfull[buf], par, abort_flag, p.err)) break;
      if (STAGE && !wait_bar(&lfull[buf], par, abort_flag, p.err)) break;
      tc_fence_after();
      const int n0 = (t_begin + it) * BN;
      const uint32_t tbase =
          tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)((buf * NSUBMAX + st) * BN);
      // one chunk of CH accumulator columns (acc already waited for)
      auto chunk = [&](int c, const uint32_t (&acc)[CH]) {
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
        } else if (!FOLD && valid) {
          load_logits<TL, CH>(Lr, col0, V, x);
        }
        if (valid) {
          if (FOLD) {
            // the accumulator holds z = L + E[p].W
#pragma unroll
            for (int j = 0; j < CH; ++j) x[j] = __uint_as_float(acc[j]);
          } else {
            // z = L + E[p].W in fp32 pairs
#pragma unroll
            for (int j = 0; j < CH; j += 2) {
              const float2 z2 = f2_add(make_float2(x[j], x[j + 1]),
                                       make_float2(__uint_as_float(acc[j]), __uint_as_float(acc[j + 1])));
              x[j] = z2.x;
              x[j + 1] = z2.y;
            }
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
      };
      // the next chunk's accumulator load is in flight while a chunk is processed
      constexpr int NCH = BN / CH / SPLIT;
      const int cb = h * NCH;
      uint32_t acc_a[CH], acc_b[CH];
      tmem_issue(tbase + (uint32_t)(cb * CH), acc_a);
#pragma unroll 1
      for (int i = 0; i < NCH; i += 2) {
        tmem_wait(acc_a);
        if (i + 1 < NCH) tmem_issue(tbase + (uint32_t)((cb + i + 1) * CH), acc_b);
        chunk(cb + i, acc_a);
        if (i + 1 < NCH) {
          tmem_wait(acc_b);
          if (i + 2 < NCH) tmem_issue(tbase + (uint32_t)((cb + i + 2) * CH), acc_a);
          chunk(cb + i + 1, acc_b);
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

int umma_nsub(int rows) { return rows > BM ? 2 : 1; }

}  // namespace

int score_slices(int rows, int V, int markov_dtype) {
  const int sms = num_sms();
  if (markov_dtype == PCT_BF16 && rows >= pair_rows_min()) return pair_slices(rows, V);
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
  if (rows >= pair_rows_min()) return launch_score_pair(a, s);
  CUtensorMap tmA, tmB;
  if (!encode_2d_bf16(&tmA, a.Eg, (uint64_t)a.r_pad, (uint64_t)a.M_pad, BK, BM)) return cudaErrorInvalidValue;
  // W's transpose, when the caller has it, is read as K-major tiles: an N-tile
  // is then one contiguous run of 128 rows instead of r strided pieces
  const bool kmaj = a.Wt != nullptr && a.r_pad % BK == 0;
  if (kmaj) {
    if (!encode_2d_bf16(&tmB, a.Wt, (uint64_t)a.r_pad, (uint64_t)a.V, BK, BN))
      return cudaErrorInvalidValue;
  } else if (!encode_2d_bf16(&tmB, a.W, (uint64_t)a.V, (uint64_t)a.r, 64, BK)) {
    return cudaErrorInvalidValue;
  }
  UmmaParams p;
  p.b_kmajor = kmaj ? 1 : 0;
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
  if (!a.thr_seeded &&
      cudaMemsetAsync(a.row_thr, 0, sizeof(uint32_t) * (size_t)rows, s) != cudaSuccess)
    return cudaErrorInvalidValue;
  const int mtiles = (rows + p.rows_per_cta - 1) / p.rows_per_cta;
  // requests any CTA's rows span: stage L_d by TMA when that fits a slot
  int span = 0;
  for (int mt = 0; mt < mtiles; ++mt) {
    const int r0 = mt * p.rows_per_cta, r1 = std::min(rows, r0 + p.rows_per_cta) - 1;
    span = std::max(span, r1 / a.n_par - r0 / a.n_par + 1);
  }
  const bool bf16_l = a.logits_dtype == PCT_BF16;
  const int lmode = !bf16_l ? L_GLOBAL : span <= LFOLD ? L_FOLD : span <= LBMAX ? L_STAGE : L_GLOBAL;
  p.LB = lmode == L_STAGE ? (span + 7) / 8 * 8 : 0;
  CUtensorMap tmL;
  if (lmode == L_STAGE) {
    if (!encode_2d_bf16(&tmL, a.L, (uint64_t)a.V, (uint64_t)a.n_req, 64, (uint32_t)p.LB,
                        (uint64_t)a.L_req_stride * 2, false))
      return cudaErrorInvalidValue;
  } else if (lmode == L_FOLD) {
    // [16 requests][64 columns] boxes, 128-byte swizzle (the MMA's B layout);
    // rows past the last request read as zero
    if (!encode_2d_bf16(&tmL, a.L, (uint64_t)a.V, (uint64_t)a.n_req, 64, (uint32_t)LFOLD,
                        (uint64_t)a.L_req_stride * 2, true))
      return cudaErrorInvalidValue;
  } else {
    tmL = tmB;   // unused
  }
  dim3 grid(a.S, mtiles);
  TraceScope t(s, "pct_score_umma");
#define PCT_UMMA(TL, KM, LM)                                                                    \
  do {                                                                                          \
    auto kern = score_umma_kernel<TL, KM, LM>;                                                  \
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,     \
                                         (int)SMEM_BYTES);                                      \
    if (e != cudaSuccess) {                                                                     \
      (void)cudaGetLastError();                                                                 \
      return e;                                                                                 \
    }                                                                                           \
    e = launch_pdl(kern, grid, dim3(THREADS), SMEM_BYTES, s, 1, tmA, tmB, tmL, p);             \
    if (e != cudaSuccess) return e;                                                             \
  } while (0)
#define PCT_UMMA_K(TL, LM)                                    \
  do {                                                        \
    if (a.k <= 4) PCT_UMMA(TL, 4, LM);                        \
    else if (a.k <= 8) PCT_UMMA(TL, 8, LM);                   \
    else PCT_UMMA(TL, 16, LM);                                \
  } while (0)
  if (lmode == L_FOLD) PCT_UMMA_K(__nv_bfloat16, L_FOLD);
  else if (lmode == L_STAGE) PCT_UMMA_K(__nv_bfloat16, L_STAGE);
  else if (bf16_l) PCT_UMMA_K(__nv_bfloat16, L_GLOBAL);
  else PCT_UMMA_K(float, L_GLOBAL);
#undef PCT_UMMA_K
#undef PCT_UMMA
  return cudaGetLastError();
}

}  // namespace pct
