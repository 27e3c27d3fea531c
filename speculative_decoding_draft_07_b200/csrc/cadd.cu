// CaDDTree: cost-aware best-first draft tree.
//
// "Cost-Aware Diffusion Draft Trees for Speculative Decoding" (gist.science
// summary), technical summary, "Method: CaDDTree": the tree maximises
// (1 + Phi(T)) / (C_d + C_v(|T|; l)); for a fixed size the best tree takes the
// nodes of highest prefix probability (greedy best-first); with convex C_v the
// objective is unimodal, so nodes are added until the marginal gain is
// non-positive.
//
// The row pass gives every (request, depth) row of marginal logits its
// log-sum-exp and the tokens that can ever enter the tree. A node is added at
// size n only if its prefix probability p satisfies
// p > (1 + Phi) dC(n) / C(n) >= theta, where theta = min_n dC(n) / C(n) and
// dC(n) = C(n + 1) - C(n). Since p never exceeds the marginal q_d of its last
// token, tokens with q_d <= theta can be dropped without changing the result.
// At most n_max - 1 tokens of a row can ever be used, so the survivors are
// sorted (value desc, token asc) and cut to n_max - 1; if too many survive
// (theta tiny), an exact radix select finds the n_max - 1 best instead.
//
// Kernels:
//  * bf16 rows (V % 8 == 0, 16-byte aligned): cadd_seg_rowpass_kernel, one
//    block per (row, segment) with the segment in registers, filtering against
//    the segment's own threshold, then cadd_seg_finish_kernel, one block per
//    row, applying the row's exact threshold (details at the kernels);
//  * other rows: cadd_rowpass_kernel, one 256-thread block per row streamed in
//    32 KB register chunks, a running log-sum-exp of the block (a lower bound
//    of the row's) giving after every chunk a threshold for its survivors;
//  * best-first growth, one warp per request: a pool of candidate (next
//    sibling, first child) entries packed into 64-bit keys (score, depth,
//    parent insertion index, rank) so that one warp max-reduction pops the
//    best node under the library's total order; the stop test is evaluated in
//    log form, s > log((1 + Phi) dC(n) / C(n)), before each insertion.
#include <algorithm>
#include <climits>

#include "common.cuh"
#include "internal.h"
#include "select.cuh"

namespace pct {
namespace {

constexpr int kRowThreads = 256;
constexpr int kChunk = 8;             // 16-byte loads per thread per chunk (32 KB per block)
constexpr int kCap = 2048;          // candidate buffer per row (power of two)
constexpr float kThetaSlack = 1e-3f;

__device__ __forceinline__ unsigned long long cand_key(float x, int v) {
  return ((unsigned long long)f2ord(x) << 32) | (unsigned)(~v);
}

// Block reduction of online log-sum-exp pairs; result in every thread.
__device__ void block_lse(float& m, float& s, float* sm, float* ss) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    float m2 = __shfl_xor_sync(0xffffffffu, m, o), s2 = __shfl_xor_sync(0xffffffffu, s, o);
    lse_combine(m, s, m2, s2);
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) { sm[warp] = m; ss[warp] = s; }
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    m = lane < nw ? sm[lane] : neg_inf();
    s = lane < nw ? ss[lane] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      float m2 = __shfl_xor_sync(0xffffffffu, m, o), s2 = __shfl_xor_sync(0xffffffffu, s, o);
      lse_combine(m, s, m2, s2);
    }
    if (lane == 0) { sm[0] = m; ss[0] = s; }
  }
  __syncthreads();
  m = sm[0]; s = ss[0];
  __syncthreads();
}

// Exclusive block scan of one int per thread; returns the prefix, total in *tot.
__device__ int block_excl_scan(int x, int* sbuf, int* tot) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) sbuf[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    int w = lane < nw ? sbuf[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < nw) sbuf[lane] = w;   // inclusive warp totals
  }
  __syncthreads();
  const int before = (warp > 0 ? sbuf[warp - 1] : 0) + incl - x;
  *tot = sbuf[(blockDim.x >> 5) - 1];
  __syncthreads();
  return before;
}

// Descending bitonic sort of keys[0..P) in shared memory, P a power of two.
__device__ void bitonic_desc(unsigned long long* keys, int P) {
  for (int size = 2; size <= P; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int t = threadIdx.x; t < P / 2; t += blockDim.x) {
        const int lo = 2 * t - (t & (stride - 1));
        const int hi = lo + stride;
        const bool desc = ((lo & size) == 0);
        unsigned long long a = keys[lo], b = keys[hi];
        if (desc ? (a < b) : (a > b)) { keys[lo] = b; keys[hi] = a; }
      }
      __syncthreads();
    }
  }
}

template <typename T>
__device__ __forceinline__ float elem(const T* x, int v) { return load_f(x + v); }

// Visit every value of a row: f(value, index). bf16 rows with 16-byte aligned
// starts use vector loads of 8 values; everything else is scalar.
template <typename T, typename F>
__device__ __forceinline__ void for_row(const T* x, int V, bool vec, F&& f) {
  if (sizeof(T) == 2 && vec) {
    const uint4* p = reinterpret_cast<const uint4*>(x);
    const int nvec = V >> 3;
    for (int c = threadIdx.x; c < nvec; c += blockDim.x) {
      const uint4 q = p[c];
      const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int j = 0; j < 8; ++j) f((j & 1) ? bf16_hi(w[j >> 1]) : bf16_lo(w[j >> 1]), c * 8 + j);
    }
    for (int v = (nvec << 3) + threadIdx.x; v < V; v += blockDim.x) f(elem(x, v), v);
  } else {
    for (int v = threadIdx.x; v < V; v += blockDim.x) f(elem(x, v), v);
  }
}

// theta = min over n in [1, n_max - 1] of dC(n) / C(n) for request b, computed
// by one warp in double; returns ln(theta) (-inf when some dC(n) <= 0, i.e. no
// token can be excluded) and reports C(n) <= 0 in the status word.
__device__ float cadd_ln_theta(const CaddParams& p, double ell, int lane, bool report,
                               int32_t* status_b) {
  const double cb = (double)p.C_d + (double)p.a + (double)p.b * ell;
  double th = 1e300;
  int bad = 0, nonpos = 0;
  for (int n = 1 + lane; n <= p.n_max; n += 32) {
    const double Cn = cb + (double)p.c * n + (double)p.e * (double)n * n;
    if (Cn <= 0.0) bad = 1;
    if (n < p.n_max) {
      const double dC = (double)p.c + (double)p.e * (2.0 * n + 1.0);
      if (dC <= 0.0) nonpos = 1; else if (Cn > 0.0) th = fmin(th, dC / Cn);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    th = fmin(th, __shfl_xor_sync(0xffffffffu, th, o));
    bad |= __shfl_xor_sync(0xffffffffu, bad, o);
    nonpos |= __shfl_xor_sync(0xffffffffu, nonpos, o);
  }
  if (report && lane == 0 && bad) atomicOr(status_b, PCT_DEV_BAD_COST);
  return (nonpos || th >= 1e299) ? neg_inf() : (float)log(th);
}

// Keep (value, token) in the candidate buffer; the counter keeps counting past
// the capacity so that an overflow is detected.
__device__ __forceinline__ void cadd_keep(unsigned long long* keys, int* n, float z, int v) {
  const int pos = atomicAdd(n, 1);
  if (pos < kCap) keys[pos] = cand_key(z, v);
}

// Exact selection of the K best values of a row (value desc, token asc) into
// keys[0..K) (unordered): a 4-round radix select on the order-preserving keys
// finds the K-th value, then every larger value and the lowest-index values
// equal to it are taken. Block-wide (every thread calls it).
template <typename T>
__device__ void select_topk_exact(const T* x, int V, bool vec, int K, unsigned long long* keys,
                                  int* hist, int* sbuf, int* s_n) {
  unsigned prefix = 0, pmask = 0;
  int need = K;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int j = threadIdx.x; j < 256; j += blockDim.x) hist[j] = 0;
    __syncthreads();
    for_row(x, V, vec, [&](float z, int v) {
      const unsigned kk = f2ord(z);
      if ((kk & pmask) == prefix) atomicAdd(&hist[(kk >> shift) & 255], 1);
    });
    __syncthreads();
    if (threadIdx.x == 0) {
      int cum = 0, bsel = 0;
      for (int j = 255; j >= 0; --j) {
        if (cum + hist[j] >= need) { bsel = j; break; }
        cum += hist[j];
      }
      need -= cum;
      sbuf[0] = bsel; sbuf[1] = need;
    }
    __syncthreads();
    prefix |= (unsigned)sbuf[0] << shift;
    pmask |= 255u << shift;
    need = sbuf[1];
    __syncthreads();
  }
  // prefix is the exact key of the K-th value; take every larger value and
  // the `need` lowest-index values equal to it (contiguous segments per thread
  // keep index order)
  if (threadIdx.x == 0) *s_n = 0;
  __syncthreads();
  const int seg = (V + blockDim.x - 1) / blockDim.x;
  const int v0 = threadIdx.x * seg, v1 = min(V, v0 + seg);
  int ties = 0;
  for (int v = v0; v < v1; ++v) {
    const float z = elem(x, v);
    const unsigned kk = f2ord(z);
    if (kk > prefix) { const int pos = atomicAdd(s_n, 1); keys[pos] = cand_key(z, v); }
    else if (kk == prefix) ++ties;
  }
  int tot;
  int rank = block_excl_scan(ties, sbuf, &tot);
  const int above = *s_n;    // stable after the scan's barriers
  for (int v = v0; v < v1 && rank < need; ++v) {
    const float z = elem(x, v);
    if (f2ord(z) == prefix) { keys[above + rank] = cand_key(z, v); ++rank; }
  }
  __syncthreads();
}

// Each row's top_k tokens (cadd_tree_grow_topk). The row pass holds, sorted,
// every value of the row above the row's threshold (or the exact n best);
// when there are at least top_k of them their head is the answer, written
// here. Otherwise the row joins the list of rows cadd_topk_fill_kernel
// selects exactly (in any order). Block-wide (every thread calls it, with the
// same n).
__device__ __forceinline__ void cadd_topk_head(const CaddParams& p, size_t row, int n,
                                               const unsigned long long* keys) {
  if (n >= p.top_k) {
    for (int j = threadIdx.x; j < p.top_k; j += blockDim.x)
      p.top_tok[row * p.top_k + j] = (int)(~(unsigned)(keys[j] & 0xffffffffu));
  } else if (threadIdx.x == 0) {
    p.top_list[atomicAdd(p.top_list_n, 1u)] = (int)row;
  }
}

template <typename T>
__global__ __launch_bounds__(kRowThreads, 3) void cadd_rowpass_kernel(
    CaddParams p, const T* __restrict__ L, const int64_t* __restrict__ ctx,
    float* __restrict__ row_lse, int32_t* __restrict__ cand_cnt, float* __restrict__ cand_q,
    int32_t* __restrict__ cand_tok, int32_t* __restrict__ status) {
  pdl_wait();
  pdl_trigger();
  __shared__ unsigned long long keys[kCap];
  __shared__ float sm[32], ss[32];
  __shared__ int sbuf[32];
  __shared__ int hist[256];
  __shared__ int s_n, s_n2;
  __shared__ float s_lnth;
  __shared__ float2 s_pub[kRowThreads / 32];   // per-warp running (max, sum)
  const int d = blockIdx.x, b = blockIdx.y;
  const int V = p.V;
  const size_t row = (size_t)b * p.D + d;
  const T* x = L + row * (size_t)V;
  const int K = p.n_max - 1;               // tokens a row can contribute at most
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool vec = (sizeof(T) == 2) && (V % 8 == 0) && ((reinterpret_cast<uintptr_t>(L) & 15u) == 0);

  if (warp == 0) {
    const float lt = cadd_ln_theta(p, (double)ctx[b], lane, d == 0, &status[b]);
    if (lane == 0) { s_lnth = lt; s_n = 0; }
  }
  if (lane == 0) s_pub[warp] = make_float2(neg_inf(), 0.f);
  __syncthreads();
  const float lnth = s_lnth - kThetaSlack;

  // One pass over the row in chunks held in registers. After each chunk a
  // warp publishes its running (max, sum) to shared memory and combines every
  // warp's latest snapshot: partial sums over disjoint parts of the row, so the
  // combination is a lower bound of the row's log-sum-exp whatever the other
  // warps' progress. That bound gives a threshold every final candidate
  // already passes, and the chunk's survivors are taken straight from
  // registers: no second read of the row and no block barrier in the loop.
  float m = neg_inf(), s = 0.f;
  if (vec) {
    const uint4* pv = reinterpret_cast<const uint4*>(x);
    const int nvec = V >> 3;
    // uniform trip count: the warp shuffles below need every lane
    for (int c0 = 0; c0 < nvec; c0 += kRowThreads * kChunk) {
      const int base = c0 + threadIdx.x;
      uint4 q[kChunk];
#pragma unroll
      for (int u = 0; u < kChunk; ++u) {
        const int c = base + u * kRowThreads;
        q[u] = c < nvec ? ld_stream16(pv + c)
                        : make_uint4(0xff80ff80u, 0xff80ff80u, 0xff80ff80u, 0xff80ff80u);
      }
      float gmax[kChunk];   // each 8-value group's max, reused by the candidate pass
#pragma unroll
      for (int u = 0; u < kChunk; ++u) {
        const uint32_t w[4] = {q[u].x, q[u].y, q[u].z, q[u].w};
        const float cm = fmaxf(fmax3(bf16_lo(w[0]), bf16_hi(w[0]), bf16_lo(w[1])),
                               fmax3(bf16_hi(w[1]), fmax3(bf16_lo(w[2]), bf16_hi(w[2]), bf16_lo(w[3])),
                                     bf16_hi(w[3])));
        gmax[u] = cm;
        if (cm > m) { s = (m == neg_inf()) ? 0.f : s * ex2((m - cm) * kLog2e); m = cm; }
        if (m != neg_inf()) {
          const float mb = m * kLog2e;
          float s0 = 0.f, s1 = 0.f;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            s0 += ex2(fmaf(bf16_lo(w[j]), kLog2e, -mb));
            s1 += ex2(fmaf(bf16_hi(w[j]), kLog2e, -mb));
          }
          s += s0 + s1;
        }
      }
      // warp total -> published snapshot -> bound over all warps' snapshots
      float wm = m, ws = s;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float m2 = __shfl_xor_sync(0xffffffffu, wm, o), s2 = __shfl_xor_sync(0xffffffffu, ws, o);
        lse_combine(wm, ws, m2, s2);
      }
      if (lane == 0) st_shared_vol2(&s_pub[warp], wm, ws);
      float bm = neg_inf(), bs = 0.f;
#pragma unroll
      for (int w2 = 0; w2 < kRowThreads / 32; ++w2) {
        const float2 o = w2 == warp ? make_float2(wm, ws) : ld_shared_vol2(&s_pub[w2]);
        lse_combine(bm, bs, o.x, o.y);
      }
      const float t = (K <= 0 || bm == neg_inf()) ? __int_as_float(0x7f800000)
                                                  : bm + logf(bs) + lnth;
      // survivors of the chunk: counted per thread, one shared-memory atomic
      // per warp reserves their slots (the count keeps running past the
      // buffer so that an overflow is seen)
      int cnt = 0;
#pragma unroll
      for (int u = 0; u < kChunk; ++u) {
        if (gmax[u] > t) {
          const uint32_t w[4] = {q[u].x, q[u].y, q[u].z, q[u].w};
#pragma unroll
          for (int j = 0; j < 8; ++j) cnt += ((j & 1) ? bf16_hi(w[j >> 1]) : bf16_lo(w[j >> 1])) > t;
        }
      }
      if (__ballot_sync(0xffffffffu, cnt > 0)) {
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        int pos = 0;
        if (lane == 31) pos = atomicAdd(&s_n, incl);
        pos = __shfl_sync(0xffffffffu, pos, 31) + incl - cnt;
#pragma unroll
        for (int u = 0; u < kChunk; ++u) {
          if (gmax[u] > t) {
            const uint32_t w[4] = {q[u].x, q[u].y, q[u].z, q[u].w};
            const int v0 = (base + u * kRowThreads) * 8;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float z = (j & 1) ? bf16_hi(w[j >> 1]) : bf16_lo(w[j >> 1]);
              if (z > t) {
                if (pos < kCap) keys[pos] = cand_key(z, v0 + j);
                ++pos;
              }
            }
          }
        }
      }
    }
    // tail (V % 8 values): scalar, folded into the totals below
    for (int v = (nvec << 3) + threadIdx.x; v < V; v += kRowThreads) lse_combine(m, s, elem(x, v), 1.f);
  } else {
    for (int v = threadIdx.x; v < V; v += kRowThreads) lse_combine(m, s, elem(x, v), 1.f);
  }
  block_lse(m, s, sm, ss);
  const float lse = (m == neg_inf()) ? neg_inf() : m + logf(s);
  const float t = (K <= 0) ? __int_as_float(0x7f800000) : lse + lnth;
  // scalar paths (tail or non-vector rows) collect against the exact threshold
  if (K > 0) {
    if (vec) {
      for (int v = ((V >> 3) << 3) + threadIdx.x; v < V; v += kRowThreads) {
        const float z = elem(x, v);
        if (z > t) cadd_keep(keys, &s_n, z, v);
      }
    } else {
      for (int v = threadIdx.x; v < V; v += kRowThreads) {
        const float z = elem(x, v);
        if (z > t) cadd_keep(keys, &s_n, z, v);
      }
    }
  }
  __syncthreads();
  int n = s_n;
  if (n <= kCap) {
    // exact filter of the chunk survivors against the final threshold
    if (threadIdx.x == 0) s_n2 = 0;
    __syncthreads();
    unsigned long long mine[kCap / kRowThreads];
    int cntm = 0;
#pragma unroll
    for (int u = 0; u < kCap / kRowThreads; ++u) {
      const int j = threadIdx.x + u * kRowThreads;
      if (j < n) {
        const unsigned long long kk = keys[j];
        if (ord2f((unsigned)(kk >> 32)) > t) mine[cntm++] = kk;
      }
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < kCap / kRowThreads; ++u)
      if (u < cntm) keys[atomicAdd(&s_n2, 1)] = mine[u];
    __syncthreads();
    n = s_n2;
  } else {
    // more than the buffer survived (theta tiny): exact radix select of the K
    // best (value desc, token asc) over the row
    select_topk_exact(x, V, vec, K, keys, hist, sbuf, &s_n);
    n = K;
  }
  int P = 1;
  while (P < n) P <<= 1;
  for (int j = n + threadIdx.x; j < P; j += kRowThreads) keys[j] = 0ull;
  __syncthreads();
  if (P > 1) bitonic_desc(keys, P);
  const int keep = min(n, max(K, 0));
  const size_t cbase = row * (size_t)max(K, 1);
  for (int j = threadIdx.x; j < keep; j += kRowThreads) {
    const unsigned long long kk = keys[j];
    const float z = ord2f((unsigned)(kk >> 32));
    cand_q[cbase + j] = z - lse;
    cand_tok[cbase + j] = (int)(~(unsigned)(kk & 0xffffffffu));
  }
  if (p.top_k > 0) cadd_topk_head(p, row, n, keys);
  if (threadIdx.x == 0) {
    cand_cnt[row] = keep;
    row_lse[row] = lse;
  }
}

// ---------------------------------------------------------------------------
// Segmented row pass (bf16 rows, 16-byte aligned, V % 8 == 0), two kernels.
//  * cadd_seg_rowpass_kernel: every row is cut into S segments of at most
//    kSegPer 16-byte groups, one kSegThreads-thread block per (row, segment),
//    with no dependence between blocks. The segment is loaded straight into
//    registers (kSegG 16-byte loads per thread in flight) and folded into a
//    partial log-sum-exp; a bitmap then marks each group whose maximum exceeds
//    the segment's own threshold lse_seg + ln(theta). Since lse_seg <= lse of
//    the row, the marks cover every value the row keeps.
//  * cadd_seg_finish_kernel, one block per row: combines the S partials into
//    the row's lse, reads the marked groups again, keeps their values above
//    the exact threshold lse + ln(theta), sorts them (value desc, token asc)
//    and writes the first n_max - 1; if too many groups are marked or too
//    many values pass (theta tiny) it selects them exactly over the row.
// HBM sees every row once; the bitmap adds 1 bit per 16 bytes, the marked
// groups a few KB per row.

constexpr int kSegThreads = 128;
constexpr int kFinThreads = 128;          // finish kernel block
constexpr int kSegG = 10;                 // 16-byte groups per thread (80 values)
constexpr int kSegBlocks = 6;             // resident blocks per SM (register bound)
constexpr int kSegPer = kSegG * kSegThreads;   // 16-byte groups per segment
constexpr int kSegWords = kSegPer / 32;         // bitmap words per segment
static_assert(kSegThreads == 128 && kSegWords <= 64 && kSegWords % 8 == 0,
              "bitmap words of a block: two sets of at most 64 threads, whole sectors");
constexpr int kSegFinCap = 1024;          // exact survivors sorted per row (>= n_max - 1)
constexpr int kFinGroups = 4096;          // marked groups listed per row
constexpr int kFinBatch = 4;              // 16-byte loads in flight per thread (finish)
constexpr int kFinMaxSegs = 256;          // segments per row that may use the tight bitmap
constexpr float kSegMargin = 1e-3f;       // covers the rounding of lse_seg against lse

// Segments of a row of V values (V % 8 == 0).
__host__ __device__ __forceinline__ int seg_count(int V) {
  const int ngroups = V / 8;
  return ngroups <= kSegPer ? 1 : (ngroups + kSegPer - 1) / kSegPer;
}
// 32-bit words of a row's candidate-group bitmap: one bit per 16-byte group,
// rounded up to whole 32-byte sectors (the row's last segment writes the
// padding words, as zeros).
__host__ __device__ __forceinline__ int seg_words(int V) { return ((V / 8 + 31) / 32 + 7) & ~7; }

// Elementwise max of two packed bf16 pairs.
__device__ __forceinline__ uint32_t bf16x2_max(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
// Per half: 0xffff where a > b (bf16 compare), else 0.
__device__ __forceinline__ uint32_t bf16x2_gt(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("set.gt.u32.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
// The largest bf16 value not above t, in both halves. For any bf16 x: x > t
// exactly when x > that value. A NaN t gives +inf (no x passes, as no x > NaN).
__device__ __forceinline__ uint32_t bf16_pair_round_down(float t) {
  uint32_t h;
  if (t != t) {
    h = 0x7f80u;
  } else {
    const uint32_t u = __float_as_uint(t);
    h = u >> 16;                               // truncation: toward zero (infinities exact)
    if ((u & 0xffffu) != 0u && (u & 0x80000000u)) h += 1u;   // negative: one step further down
  }
  return h | (h << 16);
}

// Sum of s_i 2^((m_i - M) log2 e) with M the block-wide max of m_i, in a fixed
// order (thread, then lane tree, then warps in order), so every block that
// reduces the same values gets the same bits. Returns (M, sum) in every thread.
__device__ float2 block_lse_fixed(float m, float s, float2* wred) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float M = m;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float sc = (m == neg_inf()) ? 0.f : s * ex2((m - M) * kLog2e);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sc += __shfl_xor_sync(0xffffffffu, sc, o);
  if (lane == 0) wred[warp] = make_float2(M, sc);
  __syncthreads();
  constexpr int nw = kFinThreads / 32;
  float BM = neg_inf();
#pragma unroll
  for (int w = 0; w < nw; ++w) BM = fmaxf(BM, wred[w].x);
  float BS = 0.f;
#pragma unroll
  for (int w = 0; w < nw; ++w) {
    const float2 e = wred[w];
    if (e.x != neg_inf()) BS += e.y * ex2((e.x - BM) * kLog2e);
  }
  __syncthreads();   // wred is reused by the caller's next reduction
  return make_float2(BM, BS);
}

// Descending bitonic sort of one key per lane across a warp.
__device__ __forceinline__ unsigned long long warp_sort_desc_u64(unsigned long long v, int lane) {
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      const unsigned long long o = __shfl_xor_sync(0xffffffffu, v, j);
      const bool keep_max = ((lane & k) == 0) == ((lane & j) == 0);
      v = keep_max ? (o > v ? o : v) : (o < v ? o : v);
    }
  }
  return v;
}

// ln(theta) for context length ell, theta = min over n in [1, n_max - 1] of
// dC(n) / C(n), in closed form: with c, e >= 0, C is nondecreasing, and
// f(n) = dC(n) / C(n) has f' of the sign of -2e^2 n^2 - 2e(c + e) n + (2eA -
// c^2 - ce) (A = C_d + a + b l), a parabola opening downwards: f only falls,
// or rises and then falls, for n > 0, so its minimum over an interval is at an
// end, and theta = min(f(1), f(n_max - 1)) when C(1) > 0. -inf (no token can be
// excluded) when c = e = 0 or C(1) <= 0 (a cost the growth reports as bad);
// fp32 rounding (about 1e-6 relative) stays far inside the slack the filter
// subtracts.
__device__ __forceinline__ float cadd_ln_theta_closed(const CaddParams& p, float ell) {
  if (p.n_max < 2) return neg_inf();
  const float A = p.C_d + p.a + p.b * ell;
  const float C1 = A + p.c + p.e;
  if (!(p.c > 0.f || p.e > 0.f) || !(C1 > 0.f)) return neg_inf();
  const float n1 = (float)(p.n_max - 1);
  const float f1 = (p.c + 3.f * p.e) / C1;
  const float fN = (p.c + p.e * (2.f * n1 + 1.f)) / (A + p.c * n1 + p.e * n1 * n1);
  return logf(fminf(f1, fN));
}

struct SegWs {
  float* lnth;                 // [rows] filter offset ln(theta) - slack
  float2* part;                // [rows][S] partial (max, sum)
  float* t2;                   // [rows][S] threshold of the tight bitmap
  uint32_t* mask;              // [2][rows][seg_words(V)] candidate groups (loose, tight),
                               // bit g % 32 of word g / 32
};

// One (row, segment) work item of the row pass: segment seg of a row covers
// the 16-byte groups [seg * kSegPer, min(ngroups, (seg + 1) * kSegPer)), so
// every segment but a row's last is full.
struct SegItem {
  int row, seg, g0, ng;
};
__device__ __forceinline__ SegItem seg_item(int row, int seg, int V) {
  SegItem it;
  it.row = row;
  it.seg = seg;
  it.g0 = seg * kSegPer;
  it.ng = min(V >> 3, it.g0 + kSegPer) - it.g0;
  return it;
}
// The item's segment into registers: kSegG independent 16-byte loads per
// thread (groups past a short segment read as -inf).
__device__ __forceinline__ void seg_load(const __nv_bfloat16* __restrict__ L, int V,
                                         const SegItem& it, uint4 (&q)[kSegG]) {
  const uint4* src = reinterpret_cast<const uint4*>(L + (size_t)it.row * V) + it.g0;
  if (it.ng == kSegPer) {
#pragma unroll
    for (int j = 0; j < kSegG; ++j) q[j] = ld_stream16(src + j * kSegThreads + threadIdx.x);
  } else {
#pragma unroll
    for (int j = 0; j < kSegG; ++j) {
      const int g = j * kSegThreads + threadIdx.x;
      q[j] = g < it.ng ? ld_stream16(src + g)
                       : make_uint4(0xff80ff80u, 0xff80ff80u, 0xff80ff80u, 0xff80ff80u);
    }
  }
}

struct SegSmem {
  float2 wred[kSegThreads / 32];
  uint32_t words[2][kSegWords];                // the block's bitmap words (loose, tight)
  uint32_t tpair, tpair2;
};

// Everything after the loads for one item: the partial log-sum-exp, then two
// bits per 16-byte group. The loose bit is set when the group's maximum
// exceeds the segment's own threshold t = lse_seg + ln(theta): lse_seg <= lse
// of the row, so these bits cover every value the row keeps. The tight bit
// uses t2 = t + ln(S) - 1/2, about where the row's threshold falls when the S
// segments hold similar mass; it covers the row's values whenever the row's
// threshold is at least t2, which the finishing kernel checks per segment
// before it tests only the groups one of the two bitmaps marks.
__device__ __forceinline__ void seg_process(const CaddParams& p, const int64_t* __restrict__ ctx,
                                            const SegWs& w, const SegItem& it,
                                            const uint4 (&q)[kSegG], SegSmem& sm) {
  const int S = seg_count(p.V);
  const int row = it.row, seg = it.seg, g0 = it.g0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t slot = (size_t)row * S + seg;

  // packed maxima: gm[j] holds the larger of each half-pair of group j's words,
  // so max(lo, hi) of gm[j] is the group's maximum; their tree gives the thread's
  uint32_t gm[kSegG];
#pragma unroll
  for (int j = 0; j < kSegG; ++j)
    gm[j] = bf16x2_max(bf16x2_max(q[j].x, q[j].y), bf16x2_max(q[j].z, q[j].w));
  uint32_t tmx = gm[0];
#pragma unroll
  for (int j = 1; j < kSegG; ++j) tmx = bf16x2_max(tmx, gm[j]);
  const float m = fmaxf(bf16_lo(tmx), bf16_hi(tmx));

  // partial log-sum-exp against the thread's own maximum (no rescaling), two
  // packed pairs of fp32 sums
  float s = 0.f;
  if (m != neg_inf()) {
    const float nmb = -m * kLog2e;
    float2 p0 = make_float2(0.f, 0.f), p1 = make_float2(0.f, 0.f);
#pragma unroll
    for (int j = 0; j < kSegG; ++j) {
      const uint4 v = q[j];
      const float2 l2 = make_float2(kLog2e, kLog2e), n2 = make_float2(nmb, nmb);
      const float2 t0 = f2_fma(make_float2(bf16_lo(v.x), bf16_hi(v.x)), l2, n2);
      const float2 t1 = f2_fma(make_float2(bf16_lo(v.y), bf16_hi(v.y)), l2, n2);
      const float2 t2 = f2_fma(make_float2(bf16_lo(v.z), bf16_hi(v.z)), l2, n2);
      const float2 t3 = f2_fma(make_float2(bf16_lo(v.w), bf16_hi(v.w)), l2, n2);
      p0 = f2_add(p0, make_float2(ex2(t0.x), ex2(t0.y)));
      p1 = f2_add(p1, make_float2(ex2(t1.x), ex2(t1.y)));
      p0 = f2_add(p0, make_float2(ex2(t2.x), ex2(t2.y)));
      p1 = f2_add(p1, make_float2(ex2(t3.x), ex2(t3.y)));
    }
    s = (p0.x + p1.x) + (p0.y + p1.y);
  }

  // the block's (max, sum) in a fixed order (lane tree, then warps in order);
  // one thread turns it into the segment's threshold and publishes it with
  // the partial, so the per-row scalar work runs once per block
  {
    float M = m;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float sc = (m == neg_inf()) ? 0.f : s * ex2((m - M) * kLog2e);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sc += __shfl_xor_sync(0xffffffffu, sc, o);
    if (lane == 0) sm.wred[warp] = make_float2(M, sc);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    constexpr int nw = kSegThreads / 32;
    float BM = neg_inf();
#pragma unroll
    for (int i = 0; i < nw; ++i) BM = fmaxf(BM, sm.wred[i].x);
    float BS = 0.f;
#pragma unroll
    for (int i = 0; i < nw; ++i) {
      const float2 e = sm.wred[i];
      if (e.x != neg_inf()) BS += e.y * ex2((e.x - BM) * kLog2e);
    }
    const float lnth = cadd_ln_theta_closed(p, (float)ctx[row / p.D]) - kThetaSlack;
    const float lse_seg = (BM == neg_inf()) ? neg_inf() : BM + logf(BS);
    const float t = (p.n_max <= 1) ? __int_as_float(0x7f800000) : lse_seg + lnth - kSegMargin;
    const float t2 = t + (S > 1 ? logf((float)S) - 0.5f : 0.f);
    sm.tpair = bf16_pair_round_down(t);
    sm.tpair2 = bf16_pair_round_down(t2);
    w.t2[slot] = t2;
    w.part[slot] = make_float2(BM, BS);
    if (seg == 0) w.lnth[row] = lnth;
  }
  __syncthreads();

  // A bf16 value exceeds t exactly when it exceeds t rounded down to bf16, so
  // a group is tested with one packed compare of its maximum. Group
  // g0 + j * kSegThreads + 32 * warp + lane is bit lane of one word (kSegPer,
  // kSegThreads and g0 are multiples of 32): the warp's ballot is the word.
  // The block's kSegWords words of each bitmap are contiguous (and start on
  // a 32-byte boundary): staged in shared memory, they leave in whole sectors.
  const uint32_t tpair = sm.tpair, tpair2 = sm.tpair2;
#pragma unroll
  for (int j = 0; j < kSegG; ++j) {
    const unsigned ball = __ballot_sync(0xffffffffu, bf16x2_gt(gm[j], tpair) != 0u);
    const unsigned ball2 = __ballot_sync(0xffffffffu, bf16x2_gt(gm[j], tpair2) != 0u);
    if (lane == 0) {
      sm.words[0][j * (kSegThreads / 32) + warp] = ball;
      sm.words[1][j * (kSegThreads / 32) + warp] = ball2;
    }
  }
  __syncthreads();
  const int nwr = seg_words(p.V);
  const int w0 = g0 >> 5;
  const int i = threadIdx.x & 63, which = threadIdx.x >> 6;
  if (which < 2 && i < kSegWords && w0 + i < nwr)
    w.mask[((size_t)which * p.batch * p.D + row) * nwr + w0 + i] = sm.words[which][i];
}

// One CTA per (row, segment) item (grid: rows x segments), with the whole
// segment's loads in flight at once. Measured at 1024 rows of V = 151936:
// persistent CTAs double-buffering two items in registers fit half as many
// CTAs per SM, and segments staged in shared memory by bulk copies keep fewer
// bytes in flight; both were slower.
__global__ __launch_bounds__(kSegThreads, kSegBlocks) void cadd_seg_rowpass_kernel(
    CaddParams p, const __nv_bfloat16* __restrict__ L, const int64_t* __restrict__ ctx, SegWs w) {
  pdl_wait();
  pdl_trigger();
  __shared__ SegSmem sm;
  const SegItem it = seg_item(blockIdx.x, blockIdx.y, p.V);
  uint4 q[kSegG];
  seg_load(L, p.V, it, q);
  seg_process(p, ctx, w, it, q, sm);
}

__global__ __launch_bounds__(kFinThreads) void cadd_seg_finish_kernel(
    CaddParams p, const __nv_bfloat16* __restrict__ L, const int64_t* __restrict__ ctx, SegWs w,
    float* __restrict__ row_lse, int32_t* __restrict__ cand_cnt, float* __restrict__ cand_q,
    int32_t* __restrict__ cand_tok, int32_t* __restrict__ status) {
  pdl_wait();
  pdl_trigger();
  __shared__ float2 wred[kFinThreads / 32];
  __shared__ unsigned long long keys[kSegFinCap];
  __shared__ int glist[kFinGroups];
  __shared__ int hist[256];
  __shared__ int sbuf[32];
  __shared__ int s_n, s_ng;
  __shared__ bool use_tight[kFinMaxSegs];

  const int V = p.V;
  const int S = seg_count(V);
  const int row = blockIdx.x;
  const int b = row / p.D, d = row - b * p.D;
  const int K = p.n_max - 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const __nv_bfloat16* x = L + (size_t)row * V;

  // C(n) <= 0 for some n: reported once per request
  if (d == 0 && warp == 1) (void)cadd_ln_theta(p, (double)ctx[b], lane, true, &status[b]);

  // the row's lse from the partials in a fixed order
  if (threadIdx.x == 0) {
    s_n = 0;
    s_ng = 0;
  }
  const float lnth = w.lnth[row];
  float pm = neg_inf(), pss = 0.f;
  for (int g = threadIdx.x; g < S; g += kFinThreads) {
    const float2 e = w.part[(size_t)row * S + g];
    lse_combine(pm, pss, e.x, e.y);
  }
  const float2 rl = block_lse_fixed(pm, pss, wred);   // its barriers publish s_n, s_ng
  const float lse = (rl.x == neg_inf()) ? neg_inf() : rl.x + logf(rl.y);
  const float t = (K <= 0) ? __int_as_float(0x7f800000) : lse + lnth;

  // per segment, the tight bitmap when the row's threshold is at least the
  // segment's t2, else the loose one
  for (int g = threadIdx.x; g < S; g += kFinThreads)
    if (g < kFinMaxSegs) use_tight[g] = t >= w.t2[(size_t)row * S + g];
  __syncthreads();

  // the marked groups (list in shared memory), then their values above the
  // row's threshold, kFinBatch independent 16-byte loads per thread at a time
  int n = 0, over = 0;
  if (K > 0) {
    const int nw = seg_words(V);
    const uint32_t* mrow = w.mask + (size_t)row * nw;
    const uint32_t* mrow2 = mrow + (size_t)(p.batch * p.D) * nw;
    for (int i = threadIdx.x; i < nw; i += kFinThreads) {
      const int sg = i / (kSegPer / 32);
      uint32_t bits = (sg < kFinMaxSegs && use_tight[sg]) ? mrow2[i] : mrow[i];
      if (bits == 0u) continue;
      const int at = atomicAdd(&s_ng, __popc(bits));
      for (int k = at; bits; ++k) {
        const int e = __ffs(bits) - 1;
        bits &= bits - 1;
        if (k < kFinGroups) glist[k] = 32 * i + e;
      }
    }
    __syncthreads();
    const int ng = s_ng;
    if (ng > kFinGroups) {
      over = 1;
    } else {
      const uint4* xg = reinterpret_cast<const uint4*>(x);
      for (int i0 = 0; i0 < ng; i0 += kFinBatch * kFinThreads) {
        uint4 v[kFinBatch];
        int g[kFinBatch];
#pragma unroll
        for (int u = 0; u < kFinBatch; ++u) {
          const int i = i0 + u * kFinThreads + threadIdx.x;
          g[u] = i < ng ? glist[i] : -1;
          v[u] = g[u] >= 0 ? ld_stream16(xg + g[u])
                           : make_uint4(0xff80ff80u, 0xff80ff80u, 0xff80ff80u, 0xff80ff80u);
        }
#pragma unroll
        for (int u = 0; u < kFinBatch; ++u) {
          const uint32_t wd[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float z = (e & 1) ? bf16_hi(wd[e >> 1]) : bf16_lo(wd[e >> 1]);
            if (z > t) {
              const int at = atomicAdd(&s_n, 1);
              if (at < kSegFinCap) keys[at] = cand_key(z, 8 * g[u] + e);
            }
          }
        }
      }
    }
    __syncthreads();
    n = s_n;
  }
  over = __syncthreads_or(over);
  if (K > 0 && (over || n > kSegFinCap)) {
    select_topk_exact(x, V, true, K, keys, hist, sbuf, &s_n);
    n = K;
  }
  if (n <= 32) {
    if (warp == 0) {
      unsigned long long v = lane < n ? keys[lane] : 0ull;
      v = warp_sort_desc_u64(v, lane);
      keys[lane] = v;
    }
    __syncthreads();
  } else {
    int P = 1;
    while (P < n) P <<= 1;
    for (int j = n + threadIdx.x; j < P; j += kFinThreads) keys[j] = 0ull;
    __syncthreads();
    bitonic_desc(keys, P);
  }
  const int keep = min(n, max(K, 0));
  const size_t cbase = (size_t)row * (size_t)max(K, 1);
  for (int j = threadIdx.x; j < keep; j += kFinThreads) {
    const unsigned long long kk = keys[j];
    cand_q[cbase + j] = ord2f((unsigned)(kk >> 32)) - lse;
    cand_tok[cbase + j] = (int)(~(unsigned)(kk & 0xffffffffu));
  }
  if (p.top_k > 0) cadd_topk_head(p, (size_t)row, n, keys);
  if (threadIdx.x == 0) {
    cand_cnt[row] = keep;
    row_lse[row] = lse;
  }
}

// ---------------------------------------------------------------------------
// Exact top_k of the rows the row pass listed (fewer than top_k values above
// their threshold), each row cut into parts; a block takes one part of a
// listed row in two reads of it:
//  1. every thread's best key (value desc, token asc: keys are distinct); the
//     top_k-th best of the block's thread bests, g, is at most the part's
//     top_k-th best key (top_k distinct keys of the part reach it);
//  2. every key >= g into shared memory. Only the top_k threads whose best
//     reaches g hold such keys, so there are few; they are sorted and the
//     first top_k kept. Should more than kFillCap arrive (a part whose large
//     values sit in a few threads' strides), every warp instead folds the part
//     into a sorted 32-key list, exact at any size.
// With more than one part the parts' lists are published and the row's last
// block to arrive (a counter per row, cleared by the launcher, reset by that
// block) merges them. Nothing waits on another block.
constexpr int kFillThreads = 256;
constexpr int kFillParts = 16;   // most parts of a row
constexpr int kFillLoads = 8;    // 16-byte (or scalar) loads in flight per thread
constexpr int kFillCap = 2048;   // keys collected in step 2

// f(z, v) for the values of [v0, v1) (vector: 8-value groups [g0, g1)) that
// this thread owns, kFillLoads loads in flight; the trip count is the same
// for every thread of a warp.
template <typename T, typename F>
__device__ __forceinline__ void fill_visit(const T* x, bool vec, int lo, int hi, F&& f) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int step = kFillThreads * kFillLoads;
  if (sizeof(T) == 2 && vec) {
    const uint4* xg = reinterpret_cast<const uint4*>(x);
    for (int base = lo + warp * 32 * kFillLoads; base < hi; base += step) {
      uint4 q[kFillLoads];
#pragma unroll
      for (int u = 0; u < kFillLoads; ++u) {
        const int g = base + 32 * u + lane;
        q[u] = g < hi ? xg[g] : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < kFillLoads; ++u) {
        const int g = base + 32 * u + lane;
        const uint32_t w[4] = {q[u].x, q[u].y, q[u].z, q[u].w};
#pragma unroll
        for (int e = 0; e < 8; ++e)
          f((e & 1) ? bf16_hi(w[e >> 1]) : bf16_lo(w[e >> 1]), 8 * g + e, g < hi);
      }
    }
  } else {
    for (int base = lo + warp * 32 * kFillLoads; base < hi; base += step) {
      float z[kFillLoads];
#pragma unroll
      for (int u = 0; u < kFillLoads; ++u) {
        const int v = base + 32 * u + lane;
        z[u] = v < hi ? load_f(x + v) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < kFillLoads; ++u) {
        const int v = base + 32 * u + lane;
        f(z[u], v, v < hi);
      }
    }
  }
}

struct FillSmem {
  unsigned long long keys[kFillCap];
  unsigned long long g;
  int n, last;
};

// One (row, part) item; every thread of the block calls it.
template <typename T>
__device__ void cadd_topk_fill_item(const CaddParams& p, const T* __restrict__ L, bool vec,
                                    int row, int part, int parts, FillSmem& sm) {
  const int V = p.V, top_k = p.top_k;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int nwarps = kFillThreads / 32;
  unsigned long long* keys = sm.keys;
  const T* x = L + (size_t)row * V;
  const bool groups = sizeof(T) == 2 && vec;
  const int n_units = groups ? V >> 3 : V;
  const int lo = (int)((long long)n_units * part / parts);
  const int hi = (int)((long long)n_units * (part + 1) / parts);

  // 1. thread bests, then the top_k-th best of them
  unsigned long long best = 0ull;
  fill_visit(x, vec, lo, hi, [&](float z, int v, bool ok) {
    const unsigned long long k = ok ? cand_key(z, v) : 0ull;
    best = k > best ? k : best;
  });
  keys[threadIdx.x] = warp_sort_desc(best, lane);
  if (threadIdx.x == 0) sm.n = 0;
  __syncthreads();
  if (warp == 0) {
    unsigned long long acc = keys[lane];
#pragma unroll
    for (int w = 1; w < nwarps; ++w) acc = warp_merge_top(acc, keys[32 * w + 31 - lane], lane);
    if (lane == top_k - 1) sm.g = acc;
  }
  __syncthreads();
  const unsigned long long g = sm.g;   // 0: fewer than top_k values, all of them qualify

  // 2. every key >= g
  fill_visit(x, vec, lo, hi, [&](float z, int v, bool ok) {
    const unsigned long long k = ok ? cand_key(z, v) : 0ull;
    if (k != 0ull && k >= g) {
      const int at = atomicAdd(&sm.n, 1);
      if (at < kFillCap) keys[at] = k;
    }
  });
  __syncthreads();
  const int n = sm.n;
  unsigned long long acc = 0ull;
  if (n <= 32) {
    if (warp == 0) acc = warp_sort_desc(lane < n ? keys[lane] : 0ull, lane);
  } else if (n <= kFillCap) {
    int P = 1;
    while (P < n) P <<= 1;
    for (int j = n + threadIdx.x; j < P; j += kFillThreads) keys[j] = 0ull;
    __syncthreads();
    bitonic_desc(keys, P);
    if (warp == 0) acc = keys[lane];
  } else {
    // exact at any size: each warp folds 32 keys at a time into its sorted list
    unsigned long long list = 0ull, thr = 0ull;
    fill_visit(x, vec, lo, hi, [&](float z, int v, bool ok) {
      unsigned long long k = ok ? cand_key(z, v) : 0ull;
      if (__any_sync(0xffffffffu, k > thr)) {
        k = warp_sort_desc(k, lane);
        list = warp_merge_top(list, __shfl_sync(0xffffffffu, k, 31 - lane), lane);
        thr = __shfl_sync(0xffffffffu, list, top_k - 1);
      }
    });
    __syncthreads();
    keys[32 * warp + lane] = list;
    __syncthreads();
    if (warp == 0) {
      acc = keys[lane];
#pragma unroll
      for (int w = 1; w < nwarps; ++w) acc = warp_merge_top(acc, keys[32 * w + 31 - lane], lane);
    }
  }
  bool write = true;
  if (parts > 1) {
    unsigned long long* pk = p.top_keys + (size_t)row * kFillParts * 32;
    if (warp == 0) pk[part * 32 + lane] = lane < top_k ? acc : 0ull;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) sm.last = atomicAdd(&p.top_cnt[row], 1u) == (unsigned)(parts - 1);
    __syncthreads();
    write = sm.last != 0;
    if (write) {
      __threadfence();
      if (warp == 0) {
        // every part's list in registers at once (the loads overlap), then merged
        unsigned long long b[kFillParts];
#pragma unroll
        for (int q = 0; q < kFillParts; ++q)
          b[q] = q < parts ? __ldcg(pk + q * 32 + (q == 0 ? lane : 31 - lane)) : 0ull;
        acc = b[0];
#pragma unroll
        for (int q = 1; q < kFillParts; ++q)
          if (q < parts) acc = warp_merge_top(acc, b[q], lane);
        if (lane == 0) p.top_cnt[row] = 0u;   // ready for the next launch
      }
    }
  }
  if (write && warp == 0 && lane < top_k)
    p.top_tok[(size_t)row * top_k + lane] = acc ? (int)(~(unsigned)(acc & 0xffffffffu)) : -1;
  __syncthreads();   // the shared memory is free for the block's next item
}

// Items (listed row, part) are spread over a small grid: item i is part
// i % parts of row top_list[i / parts]; blocks take items i = blockIdx.x,
// blockIdx.x + gridDim.x, ...
template <typename T>
__global__ __launch_bounds__(kFillThreads) void cadd_topk_fill_kernel(CaddParams p,
                                                                       const T* __restrict__ L,
                                                                       bool vec, int parts) {
  pdl_wait();
  pdl_trigger();
  __shared__ FillSmem sm;
  const int items = (int)*p.top_list_n * parts;
  for (int i = (int)blockIdx.x; i < items; i += (int)gridDim.x)
    cadd_topk_fill_item(p, L, vec, p.top_list[i / parts], i % parts, parts, sm);
}

// ---------------------------------------------------------------------------
// best-first growth, one warp per request

__device__ __forceinline__ unsigned long long pool_key(float s, int depth, int pidx, int rank) {
  return ((unsigned long long)f2ord(s) << 32) | ((unsigned long long)(63 - depth) << 20) |
         ((unsigned long long)(1023 - pidx) << 10) | (unsigned long long)(1023 - rank);
}

template <bool STAGED>
__global__ __launch_bounds__(32) void cadd_bestfirst_kernel(
    CaddParams p, const int32_t* __restrict__ anchor, const int64_t* __restrict__ ctx,
    const int32_t* __restrict__ cand_cnt, const float* __restrict__ cand_q,
    const int32_t* __restrict__ cand_tok, int32_t* __restrict__ otok, int32_t* __restrict__ opar,
    int32_t* __restrict__ odep, float* __restrict__ oscore, int32_t* __restrict__ ocount,
    float* __restrict__ ophi, int32_t* __restrict__ status) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ unsigned long long pool[];          // [n_max + 1]
  const int nmax = p.n_max;
  const int D = p.D, K1 = max(nmax - 1, 1);
  int* ntok = reinterpret_cast<int*>(pool + nmax + 1);  // [n_max] each
  int* npar = ntok + nmax;
  int* ndep = npar + nmax;
  float* ns = reinterpret_cast<float*>(ndep + nmax);
  int* canon = reinterpret_cast<int*>(ns + nmax);
  int* order = canon + nmax;
  float* sq = reinterpret_cast<float*>(order + nmax);   // [D][K1] the request's candidates
  int* stk = reinterpret_cast<int*>(sq + (size_t)D * K1);
  __shared__ int dstart[66], dfill[66], scnt[64];

  const int b = blockIdx.x, lane = threadIdx.x;
  const size_t row0 = (size_t)b * D;
  const int a0 = anchor[b];
  if (lane == 0 && (a0 < 0 || a0 >= p.V)) atomicOr(&status[b], PCT_DEV_BAD_TOKEN);
  if (lane == 0) { ntok[0] = a0; npar[0] = -1; ndep[0] = 0; ns[0] = 0.f; }

  // the request's candidate lists, staged once when they fit in shared memory:
  // the growth below reads them one pop after another, so each read would
  // otherwise be a dependent trip to L2 on the sequential path
  for (int dd = lane; dd < D; dd += 32) scnt[dd] = min(max(cand_cnt[row0 + dd], 0), K1);
  __syncwarp();
  if (STAGED) {
    // all rows' candidates as one index space (row offsets in dstart), eight
    // loads per lane issued before any is stored
    if (lane == 0) {
      int acc = 0;
      for (int dd = 0; dd < D; ++dd) { dstart[dd] = acc; acc += scnt[dd]; }
      dstart[D] = acc;
    }
    __syncwarp();
    const int total = dstart[D];
    constexpr int U = 8;
    for (int base = 0; base < total; base += 32 * U) {
      float qv[U];
      int tv[U], at[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int f = base + u * 32 + lane;
        at[u] = -1;
        if (f < total) {
          int dd = 0;
          while (dstart[dd + 1] <= f) ++dd;
          const int j = f - dstart[dd];
          const size_t g = (row0 + dd) * K1 + j;
          qv[u] = cand_q[g];
          tv[u] = cand_tok[g];
          at[u] = dd * K1 + j;
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (at[u] >= 0) { sq[at[u]] = qv[u]; stk[at[u]] = tv[u]; }
    }
    __syncwarp();
  }
  auto cnt_at = [&](int depth) { return scnt[depth - 1]; };
  auto q_at = [&](int depth, int rank) {
    return STAGED ? sq[(depth - 1) * K1 + rank] : cand_q[(row0 + depth - 1) * K1 + rank];
  };
  // The pool is unsorted; slot j belongs to lane j % 32, which keeps the best
  // key of its slots (lbest at lslot) in registers. A pop is the warp's
  // largest lbest (keys are distinct), found by two 32-bit warp maxima; then
  // only the owner of the popped slot and the owner of a new slot update.
  int pool_n = 0;
  unsigned long long lbest = 0ull;
  int lslot = -1;
  if (D >= 1 && nmax > 1 && cnt_at(1) > 0) {
    const unsigned long long k0 = pool_key(q_at(1, 0), 1, 0, 0);
    if (lane == 0) { pool[0] = k0; lbest = k0; lslot = 0; }
    pool_n = 1;
  }
  __syncwarp();

  const float ell = (float)ctx[b];
  const float cbase = p.C_d + p.a + p.b * ell;
  int n = 1;
  float phi = 0.f;
  while (n < nmax) {
    const unsigned hi = __reduce_max_sync(0xffffffffu, (unsigned)(lbest >> 32));
    const bool top_hi = lbest != 0ull && (unsigned)(lbest >> 32) == hi;
    const unsigned lo = __reduce_max_sync(0xffffffffu, top_hi ? (unsigned)lbest : 0u);
    const unsigned long long wbest = ((unsigned long long)hi << 32) | lo;
    const unsigned own = __ballot_sync(0xffffffffu, top_hi && (unsigned)lbest == lo);
    if (own == 0u) break;                                         // no candidate left
    const int owner = __ffs(own) - 1;
    const int bslot = __shfl_sync(0xffffffffu, lslot, owner);
    const float s = ord2f((unsigned)(wbest >> 32));
    const int depth = 63 - (int)((wbest >> 20) & 63);
    const int pidx = 1023 - (int)((wbest >> 10) & 1023);
    const int rank = 1023 - (int)(wbest & 1023);
    // stop test: add only if f(n + 1) > f(n)  <=>  s > log((1 + Phi) dC(n) / C(n))
    const float fn = (float)n;
    const float Cn = cbase + p.c * fn + p.e * fn * fn;
    const float dC = p.c + p.e * (2.f * fn + 1.f);
    const float thr = dC > 0.f ? logf((1.f + phi) * dC / Cn) : neg_inf();
    if (!(s > thr)) break;
    const int tk = STAGED ? stk[(depth - 1) * K1 + rank] : cand_tok[(row0 + depth - 1) * K1 + rank];
    const int np = pidx;
    unsigned long long sib = 0ull, child = 0ull;
    if (rank + 1 < cnt_at(depth)) sib = pool_key(ns[np] + q_at(depth, rank + 1), depth, np, rank + 1);
    if (depth < D && cnt_at(depth + 1) > 0) child = pool_key(s + q_at(depth + 1, 0), depth + 1, n, 0);
    __syncwarp();
    if (lane == 0) { ntok[n] = tk; npar[n] = np; ndep[n] = depth; ns[n] = s; }
    if (lane == owner) {
      // the popped slot takes the sibling; the owner's best is found again
      pool[bslot] = sib;
      lbest = 0ull;
      lslot = -1;
      for (int j = lane; j < pool_n; j += 32) {
        const unsigned long long k = j == bslot ? sib : pool[j];
        if (k > lbest) { lbest = k; lslot = j; }
      }
    }
    if (child) {
      if (lane == (pool_n & 31)) {
        pool[pool_n] = child;
        if (child > lbest) { lbest = child; lslot = pool_n; }
      }
      ++pool_n;
    }
    phi += expf(s);
    ++n;
    __syncwarp();
  }

  // canonical BFS order: by depth, then (parent's canonical index, token)
  for (int j = lane; j < 66; j += 32) { dstart[j] = 0; dfill[j] = 0; }
  __syncwarp();
  for (int j = lane; j < n; j += 32) atomicAdd(&dstart[ndep[j] + 1], 1);
  __syncwarp();
  if (lane == 0) for (int j = 1; j < 66; ++j) dstart[j] += dstart[j - 1];
  __syncwarp();
  for (int j = lane; j < n; j += 32) {
    const int dd = ndep[j];
    order[dstart[dd] + atomicAdd(&dfill[dd], 1)] = j;
  }
  __syncwarp();
  if (lane == 0) canon[0] = 0;
  __syncwarp();
  for (int dd = 1; dd <= D && dd < 64; ++dd) {
    const int s0 = dstart[dd], s1 = dstart[dd + 1];
    if (s0 == s1) break;
    for (int jj = s0 + lane; jj < s1; jj += 32) {
      const int j = order[jj];
      const unsigned long long kj = ((unsigned long long)canon[npar[j]] << 32) | (unsigned)ntok[j];
      int r = 0;
      for (int ii = s0; ii < s1; ++ii) {
        const int i2 = order[ii];
        const unsigned long long ki = ((unsigned long long)canon[npar[i2]] << 32) | (unsigned)ntok[i2];
        r += ki < kj;
      }
      canon[j] = s0 + r;
    }
    __syncwarp();
  }
  const size_t ob = (size_t)b * nmax;
  for (int j = lane; j < n; j += 32) {
    const int o = canon[j];
    otok[ob + o] = ntok[j];
    opar[ob + o] = j == 0 ? -1 : canon[npar[j]];
    odep[ob + o] = ndep[j];
    oscore[ob + o] = ns[j];
  }
  for (int o = n + lane; o < nmax; o += 32) {
    otok[ob + o] = -1; opar[ob + o] = -1; odep[ob + o] = -1; oscore[ob + o] = neg_inf();
  }
  if (lane == 0) { ocount[b] = n; ophi[b] = phi; }
}

}  // namespace

size_t cadd_rowpass_bytes_per_row(int n_max) {
  const size_t K1 = (size_t)(n_max > 1 ? n_max - 1 : 1);
  return K1 * (sizeof(float) + sizeof(int32_t)) + sizeof(float) + sizeof(int32_t);
}

static size_t align256(size_t x) { return (x + 255) / 256 * 256; }

size_t cadd_seg_workspace(int batch, int D, int V, int dtype) {
  if (dtype != PCT_BF16 || V % 8 != 0) return 0;
  const size_t rows = (size_t)batch * D, slots = rows * seg_count(V);
  return align256(rows * sizeof(float)) + align256(slots * sizeof(float2)) +
         align256(slots * sizeof(float)) + 2 * rows * seg_words(V) * sizeof(uint32_t);
}

size_t cadd_topk_workspace(size_t rows) {
  return align256(rows * sizeof(int32_t)) + align256((rows + 1) * sizeof(unsigned)) +
         rows * kFillParts * 32 * sizeof(unsigned long long);
}

cudaError_t launch_cadd(const CaddParams& p_in, const void* L, const int32_t* anchor,
                        const int64_t* ctx, int32_t* tok, int32_t* parent, int32_t* depth,
                        float* score, int32_t* count, float* phi, int32_t* status,
                        float* row_lse, int32_t* cand_cnt, float* cand_q, int32_t* cand_tok,
                        void* seg_ws, void* topk_ws, cudaStream_t s) {
  CaddParams p = p_in;
  if (p.top_k > 0) {
    const size_t rows = (size_t)p.batch * p.D;
    char* c = static_cast<char*>(topk_ws);
    if (!c || p.top_k > 32) return cudaErrorInvalidValue;
    p.top_list = reinterpret_cast<int32_t*>(c);            c += align256(rows * sizeof(int32_t));
    p.top_cnt = reinterpret_cast<unsigned*>(c);            // [rows] part counters, then the
    p.top_list_n = p.top_cnt + rows;                       // list's length: cleared together
    c += align256((rows + 1) * sizeof(unsigned));
    p.top_keys = reinterpret_cast<unsigned long long*>(c);
    cudaError_t e = cudaMemsetAsync(p.top_cnt, 0, (rows + 1) * sizeof(unsigned), s);
    if (e != cudaSuccess) return e;
  }
  const bool segmented = seg_ws != nullptr && p.dtype == PCT_BF16 && p.V % 8 == 0 &&
                         (reinterpret_cast<uintptr_t>(L) & 15u) == 0;
  if (segmented) {
    const size_t rows = (size_t)p.batch * p.D, slots = rows * seg_count(p.V);
    char* c = static_cast<char*>(seg_ws);
    SegWs w;
    w.lnth = reinterpret_cast<float*>(c);              c += align256(rows * sizeof(float));
    w.part = reinterpret_cast<float2*>(c);             c += align256(slots * sizeof(float2));
    w.t2 = reinterpret_cast<float*>(c);                c += align256(slots * sizeof(float));
    w.mask = reinterpret_cast<uint32_t*>(c);
    if (rows > 0x7fffffffu || seg_count(p.V) > 65535) return cudaErrorInvalidConfiguration;
    const __nv_bfloat16* Lb = static_cast<const __nv_bfloat16*>(L);
    {
      TraceScope t(s, "cadd_rowpass");
      const dim3 grid((unsigned)rows, (unsigned)seg_count(p.V));
      cudaError_t e = launch_pdl(cadd_seg_rowpass_kernel, grid, dim3(kSegThreads), 0, s, 1, p, Lb,
                                 ctx, w);
      if (e != cudaSuccess) return e;
    }
    TraceScope t(s, "cadd_finish");
    cudaError_t e = launch_pdl(cadd_seg_finish_kernel, dim3((unsigned)rows), dim3(kFinThreads), 0, s,
                               1, p, Lb, ctx, w, row_lse, cand_cnt, cand_q, cand_tok, status);
    if (e != cudaSuccess) return e;
  } else {
    dim3 grid(p.D, p.batch);
    TraceScope t(s, "cadd_rowpass");
    cudaError_t e =
        p.dtype == PCT_BF16
            ? launch_pdl(cadd_rowpass_kernel<__nv_bfloat16>, grid, dim3(kRowThreads), 0, s, 1, p,
                         static_cast<const __nv_bfloat16*>(L), ctx, row_lse, cand_cnt, cand_q,
                         cand_tok, status)
            : launch_pdl(cadd_rowpass_kernel<float>, grid, dim3(kRowThreads), 0, s, 1, p,
                         static_cast<const float*>(L), ctx, row_lse, cand_cnt, cand_q, cand_tok,
                         status);
    if (e != cudaSuccess) return e;
  }
  // exact top_k of the rows with fewer than top_k values above their threshold:
  // it needs only the finishing kernel, like the best-first growth below, so it
  // runs beside the growth on the library's second stream when there is one
  auto launch_fill = [&](cudaStream_t fs) -> cudaError_t {
    // parts of about 8192 values (one or two loads per thread and read);
    // the grid covers the SMs twice and loops over however many items there are
    const int parts = std::max(1, std::min(kFillParts, (p.V + 8191) / 8192));
    const bool vec = p.dtype == PCT_BF16 && p.V % 8 == 0 && (reinterpret_cast<uintptr_t>(L) & 15u) == 0;
    const size_t items = (size_t)p.batch * p.D * parts;
    const unsigned grid = (unsigned)std::min<size_t>(items, (size_t)2 * num_sms());
    TraceScope t(fs, "cadd_topk_fill");
    return p.dtype == PCT_BF16
        ? launch_pdl(cadd_topk_fill_kernel<__nv_bfloat16>, dim3(grid), dim3(kFillThreads), 0, fs, 1,
                     p, static_cast<const __nv_bfloat16*>(L), vec, parts)
        : launch_pdl(cadd_topk_fill_kernel<float>, dim3(grid), dim3(kFillThreads), 0, fs, 1, p,
                     static_cast<const float*>(L), vec, parts);
  };
  const size_t base = (size_t)(p.n_max + 1) * 8 + (size_t)p.n_max * 4 * 6;
  const size_t staged = base + (size_t)p.D * std::max(p.n_max - 1, 1) * 8;
  const bool stage = staged <= 160 * 1024;
  const size_t smem = stage ? staged : base;
  auto kern = stage ? cadd_bestfirst_kernel<true> : cadd_bestfirst_kernel<false>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  AuxStream ax{};
  const bool fork = p.top_k > 0 && aux_stream(&ax) == PCT_OK;
  if (p.top_k > 0 && !fork) {
    cudaError_t e = launch_fill(s);
    if (e != cudaSuccess) return e;
  }
  if (fork) aux_lock(ax);
  cudaError_t fe = cudaSuccess;
  if (fork) {
    fe = cudaEventRecord(ax.fork, s);
    if (fe == cudaSuccess) fe = cudaStreamWaitEvent(ax.s, ax.fork, 0);
    if (fe == cudaSuccess) fe = launch_fill(ax.s);
    if (fe == cudaSuccess) fe = cudaEventRecord(ax.join, ax.s);
    if (fe != cudaSuccess) {
      aux_unlock(ax);
      return fe;
    }
  }
  cudaError_t e;
  {
    TraceScope t(s, "cadd_bestfirst");
    e = launch_pdl(kern, dim3(p.batch), dim3(32), smem, s, 1, p, anchor, ctx, cand_cnt, cand_q,
                   cand_tok, tok, parent, depth, score, count, phi, status);
  }
  if (fork) {
    // the caller's stream goes on only after the selection too
    const cudaError_t je = cudaStreamWaitEvent(s, ax.join, 0);
    aux_unlock(ax);
    if (e == cudaSuccess) e = je;
  }
  return e;
}

}  // namespace pct
