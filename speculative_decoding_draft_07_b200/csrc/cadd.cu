// CaDDTree: cost-aware best-first draft tree.
//
// "Cost-Aware Diffusion Draft Trees for Speculative Decoding" (gist.science
// summary), technical summary, "Method: CaDDTree": the tree maximises
// (1 + Phi(T)) / (C_d + C_v(|T|; l)); for a fixed size the best tree takes the
// nodes of highest prefix probability (greedy best-first); with convex C_v the
// objective is unimodal, so nodes are added until the marginal gain is
// non-positive.
//
// Two kernels:
//  * row pass, one 256-thread block per (request, depth) row of marginal
//    logits, streamed once from HBM in 32 KB register chunks: a running
//    log-sum-exp of the block (a lower bound of the row's) gives after every
//    chunk a threshold with which the chunk's survivors are taken straight from
//    registers; a final exact filter keeps only the tokens that can ever enter
//    the tree. A node is added at size n only if its prefix
//    probability p satisfies p > (1 + Phi) dC(n) / C(n) >= theta, where
//    theta = min_n dC(n) / C(n) and dC(n) = C(n + 1) - C(n); since p never
//    exceeds the marginal q_d of its last token, tokens with q_d <= theta can
//    be dropped without changing the result. At most n_max - 1 tokens of a row
//    can ever be used, so the survivors are sorted (value desc, token asc) and
//    cut to n_max - 1. If more than the buffer survive (theta tiny), an exact
//    radix select finds the n_max - 1 best instead.
//  * best-first growth, one warp per request: a pool of candidate (next
//    sibling, first child) entries packed into 64-bit keys (score, depth,
//    parent insertion index, rank) so that one warp max-reduction pops the
//    best node under the library's total order; the stop test is evaluated in
//    log form, s > log((1 + Phi) dC(n) / C(n)), before each insertion.
#include <climits>

#include "common.cuh"
#include "internal.h"

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
    for (int c = threadIdx.x; c < nvec; c += kRowThreads) {
      const uint4 q = p[c];
      const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int j = 0; j < 8; ++j) f((j & 1) ? bf16_hi(w[j >> 1]) : bf16_lo(w[j >> 1]), c * 8 + j);
    }
    for (int v = (nvec << 3) + threadIdx.x; v < V; v += kRowThreads) f(elem(x, v), v);
  } else {
    for (int v = threadIdx.x; v < V; v += kRowThreads) f(elem(x, v), v);
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

// ln(theta) in fp32 by one warp: its rounding error (about 1e-6 relative) is
// far inside the kThetaSlack subtracted before use, so the filter stays a
// superset of the double-precision one. dC(n) = c + e (2n + 1) >= 0 since
// c, e >= 0 (checked on the host).
__device__ float cadd_ln_theta_f(const CaddParams& p, float ell, int lane) {
  const float cb = p.C_d + p.a + p.b * ell;
  float th = __int_as_float(0x7f800000);
  int nonpos = 0;
  for (int n = 1 + lane; n < p.n_max; n += 32) {
    const float fn = (float)n;
    const float Cn = cb + p.c * fn + p.e * fn * fn;
    const float dC = p.c + p.e * (2.0f * fn + 1.0f);
    if (dC <= 0.0f) nonpos = 1; else if (Cn > 0.0f) th = fminf(th, dC / Cn);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    th = fminf(th, __shfl_xor_sync(0xffffffffu, th, o));
    nonpos |= __shfl_xor_sync(0xffffffffu, nonpos, o);
  }
  return (nonpos || th == __int_as_float(0x7f800000)) ? neg_inf() : logf(th);
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

template <typename T>
__global__ __launch_bounds__(kRowThreads, 3) void cadd_rowpass_kernel(
    CaddParams p, const T* __restrict__ L, const int64_t* __restrict__ ctx,
    float* __restrict__ row_lse, int32_t* __restrict__ cand_cnt, float* __restrict__ cand_q,
    int32_t* __restrict__ cand_tok, int32_t* __restrict__ status) {
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
  if (threadIdx.x == 0) {
    cand_cnt[row] = keep;
    row_lse[row] = lse;
  }
}

// ---------------------------------------------------------------------------
// Row pass on CTA clusters (bf16 rows, 16-byte aligned, V <= kClSegs * 40960):
// a cluster of kClSegs CTAs per (request, depth) row. Each CTA copies its
// segment of the row into shared memory with bulk asynchronous copies (in
// pieces, so the first is reduced while the others land), folds it into a
// partial log-sum-exp, and writes the partial into the leader CTA's shared
// memory. After a cluster barrier every CTA combines the kClSegs partials in
// segment order into the row's log-sum-exp and the exact threshold
// lse + ln(theta), filters its staged segment against it, and appends the
// survivors to the leader's buffer (distributed shared memory). After a second
// barrier the leader sorts them (value desc, token asc) and writes the first
// n_max - 1; if the buffer overflowed (theta tiny) it selects them exactly over
// the row instead. HBM sees the row once.

constexpr int kClSegs = 8;
constexpr int kClPiece = 16384;                 // bytes per bulk copy
constexpr int kClSegMax = 5 * kClPiece;         // segment bytes staged (80 KB)
constexpr int kClCap = 1024;                    // survivors buffered in the leader

// Elementwise max of two packed bf16 pairs.
__device__ __forceinline__ uint32_t bf16x2_max(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

__device__ __forceinline__ uint32_t cl_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cl_map0(const void* p) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, 0;"
               : "=r"(r) : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(p))));
  return r;
}
__device__ __forceinline__ void cl_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
__device__ __forceinline__ uint32_t cl_smem(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__global__ __launch_bounds__(kRowThreads, 2) void cadd_cluster_rowpass_kernel(
    CaddParams p, const __nv_bfloat16* __restrict__ L, const int64_t* __restrict__ ctx,
    float* __restrict__ row_lse, int32_t* __restrict__ cand_cnt, float* __restrict__ cand_q,
    int32_t* __restrict__ cand_tok, int32_t* __restrict__ status) {
  extern __shared__ __align__(128) uint8_t cl_smem_raw[];
  uint8_t* segbuf = cl_smem_raw;                         // this CTA's segment (seg_cap bytes)
  __shared__ __align__(8) uint64_t bars[kClSegMax / kClPiece];
  __shared__ float2 part[kClSegs];       // leader: the segments' partial (max, sum)
  __shared__ int s_cnt;                  // leader: survivors appended
  __shared__ float sm[32], ss[32];
  __shared__ int sbuf[32];
  __shared__ int hist[256];
  __shared__ int s_n;
  __shared__ float s_lnth;
  __shared__ int s_timeout;

  const uint32_t rank = cl_rank();
  const int d = blockIdx.x / kClSegs, b = blockIdx.y;
  const int V = p.V;
  const size_t row = (size_t)b * p.D + d;
  const __nv_bfloat16* x = L + row * (size_t)V;
  const int K = p.n_max - 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ngroups = V / 8;                             // V % 8 == 0 on this path
  const int g_per = (ngroups + kClSegs - 1) / kClSegs;
  const int g_begin = min(ngroups, (int)rank * g_per), g_end = min(ngroups, g_begin + g_per);
  const int seg_bytes = (g_end - g_begin) * 16;
  const int npieces = (seg_bytes + kClPiece - 1) / kClPiece;
  // survivors buffer after the largest segment (same offset in every CTA)
  unsigned long long* keys =
      reinterpret_cast<unsigned long long*>(segbuf + (g_per * 16 + 127) / 128 * 128);   // [kClCap]

  if (threadIdx.x == 0) {
    for (int i = 0; i < npieces; ++i) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(cl_smem(&bars[i])));
    }
    s_cnt = 0;
    s_timeout = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // the whole segment in flight at once: one bulk copy per piece
    const char* src = reinterpret_cast<const char*>(x) + (size_t)g_begin * 16;
    for (int i = 0; i < npieces; ++i) {
      const int bytes = min(kClPiece, seg_bytes - i * kClPiece);
      const uint32_t bar = cl_smem(&bars[i]);
      asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                   : "memory");
      asm volatile(
          "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
              cl_smem(segbuf + i * kClPiece)),
          "l"(src + (size_t)i * kClPiece), "r"(bytes), "r"(bar)
          : "memory");
    }
  }
  if (warp == 1 && rank == 0) {   // the leader's copy is read by the whole cluster
    const float lt = cadd_ln_theta_f(p, (float)ctx[b], lane);
    if (lane == 0) s_lnth = lt - kThetaSlack;
  }
  if (warp == 2 && rank == 0 && d == 0) (void)cadd_ln_theta(p, (double)ctx[b], lane, true, &status[b]);

  // pass 1: partial log-sum-exp of the segment, piece by piece as they land.
  // Each thread sums 2^((z - m) log2 e) against its own reference m, which
  // moves only when a group exceeds it by more than 64 (so no term overflows);
  // m starts finite so that leading -inf values add 0 instead of NaN.
  float m = -1e30f, s = 0.f;
  float2 acc = make_float2(0.f, 0.f);
  float2 nmb = make_float2(1e30f * kLog2e, 1e30f * kLog2e);
  const float2 l2e = make_float2(kLog2e, kLog2e);
  const uint4* sv = reinterpret_cast<const uint4*>(segbuf);
  for (int i = 0; i < npieces; ++i) {
    // bounded wait for piece i by one warp; the others sleep in the block barrier
    if (warp == 0) {
      const uint32_t bar = cl_smem(&bars[i]);
      const long long t0 = clock64();
      uint32_t ok = 0;
      while (!ok) {
        asm volatile(
            "{\n\t.reg .pred q;\n\tmbarrier.try_wait.parity.shared::cta.b64 q, [%1], 0, 20000;\n\t"
            "selp.u32 %0, 1, 0, q;\n\t}"
            : "=r"(ok) : "r"(bar) : "memory");
        if (!ok && clock64() - t0 > 4000000000ll) { s_timeout = 1; break; }
      }
    }
    __syncthreads();
    const int gi0 = i * (kClPiece / 16);
    const int gi1 = min(g_end - g_begin, gi0 + kClPiece / 16);
    for (int g = gi0 + threadIdx.x; g < gi1; g += kRowThreads) {
      const uint4 q = sv[g];
      float f[8];
      f[0] = bf16_lo(q.x); f[1] = bf16_hi(q.x); f[2] = bf16_lo(q.y); f[3] = bf16_hi(q.y);
      f[4] = bf16_lo(q.z); f[5] = bf16_hi(q.z); f[6] = bf16_lo(q.w); f[7] = bf16_hi(q.w);
      const float cm = fmaxf(fmax3(f[0], f[1], f[2]), fmax3(f[3], fmax3(f[4], f[5], f[6]), f[7]));
      if (cm > m + 64.f) {
        s = (s + acc.x + acc.y) * ex2((m - cm) * kLog2e);
        acc = make_float2(0.f, 0.f);
        m = cm;
        nmb = make_float2(-m * kLog2e, -m * kLog2e);
      }
      const float2 a0 = f2_fma(make_float2(f[0], f[1]), l2e, nmb);
      const float2 a1 = f2_fma(make_float2(f[2], f[3]), l2e, nmb);
      const float2 a2 = f2_fma(make_float2(f[4], f[5]), l2e, nmb);
      const float2 a3 = f2_fma(make_float2(f[6], f[7]), l2e, nmb);
      const float2 e01 = f2_add(make_float2(ex2(a0.x), ex2(a0.y)), make_float2(ex2(a1.x), ex2(a1.y)));
      const float2 e23 = f2_add(make_float2(ex2(a2.x), ex2(a2.y)), make_float2(ex2(a3.x), ex2(a3.y)));
      acc = f2_add(acc, f2_add(e01, e23));
    }
  }
  s += acc.x + acc.y;
  if (!(s > 0.f)) { m = neg_inf(); s = 0.f; }   // nothing finite seen
  block_lse(m, s, sm, ss);
  // the segment's partial into the leader, then every CTA sees all of them
  if (threadIdx.x == 0) {
    asm volatile("st.shared::cluster.v2.f32 [%0], {%1, %2};" ::"r"(cl_map0(&part[rank])), "f"(m), "f"(s)
                 : "memory");
  }
  cl_sync();
  float lm = neg_inf(), ls = 0.f;
  for (int g = 0; g < kClSegs; ++g) {   // segment order: independent of arrival
    float pm, ps;
    asm volatile("ld.shared::cluster.v2.f32 {%0, %1}, [%2];" : "=f"(pm), "=f"(ps) : "r"(cl_map0(&part[g])));
    lse_combine(lm, ls, pm, ps);
  }
  const float lse = (lm == neg_inf()) ? neg_inf() : lm + logf(ls);
  float lnth;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(lnth) : "r"(cl_map0(&s_lnth)));
  const float t = (K <= 0) ? __int_as_float(0x7f800000) : lse + lnth;

  // pass 2: the segment's values above the exact threshold, into the leader
  const uint32_t cnt_addr = cl_map0(&s_cnt);
  const uint32_t keys_addr = cl_map0(keys);
  const int ng = g_end - g_begin;
  for (int g0 = 0; g0 < ng; g0 += kRowThreads) {   // uniform trip count for the warp scans
    const int g = g0 + threadIdx.x;
    float f[8];
    int cnt = 0;
    if (g < ng) {
      const uint4 q = sv[g];
      // the group's max by packed bf16 maxima (exact: every bf16 value is an
      // fp32 value), the exact per-value test only for groups that reach t
      const uint32_t mx = bf16x2_max(bf16x2_max(q.x, q.y), bf16x2_max(q.z, q.w));
      if (fmaxf(bf16_lo(mx), bf16_hi(mx)) > t) {
        f[0] = bf16_lo(q.x); f[1] = bf16_hi(q.x); f[2] = bf16_lo(q.y); f[3] = bf16_hi(q.y);
        f[4] = bf16_lo(q.z); f[5] = bf16_hi(q.z); f[6] = bf16_lo(q.w); f[7] = bf16_hi(q.w);
#pragma unroll
        for (int j = 0; j < 8; ++j) cnt += f[j] > t;
      }
    }
    if (__ballot_sync(0xffffffffu, cnt > 0)) {
      int incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      uint32_t pos = 0;
      if (lane == 31)
        asm volatile("atom.shared::cluster.add.u32 %0, [%1], %2;" : "=r"(pos) : "r"(cnt_addr), "r"(incl)
                     : "memory");
      pos = __shfl_sync(0xffffffffu, pos, 31) + (uint32_t)(incl - cnt);
      if (cnt > 0) {
        const int v0 = (g_begin + g) * 8;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (f[j] > t) {
            if (pos < (uint32_t)kClCap) {
              const unsigned long long kk = cand_key(f[j], v0 + j);
              asm volatile("st.shared::cluster.u64 [%0], %1;" ::"r"(keys_addr + 8u * pos), "l"(kk)
                           : "memory");
            }
            ++pos;
          }
        }
      }
    }
  }
  cl_sync();   // every survivor is in the leader; no CTA touches another's memory after this
  if (s_timeout) {
    // a copy that never completed: report it and give it (bounded) time to land
    // before this CTA's shared memory is released
    if (threadIdx.x == 0) {
      atomicOr(&status[b], PCT_DEV_TIMEOUT);
      for (int i = 0; i < npieces; ++i) {
        const uint32_t bar = cl_smem(&bars[i]);
        const long long t0 = clock64();
        uint32_t ok = 0;
        while (!ok && clock64() - t0 < 4000000000ll)
          asm volatile(
              "{\n\t.reg .pred q;\n\tmbarrier.try_wait.parity.shared::cta.b64 q, [%1], 0;\n\t"
              "selp.u32 %0, 1, 0, q;\n\t}"
              : "=r"(ok) : "r"(bar) : "memory");
      }
    }
    __syncthreads();
  }
  if (rank != 0) return;
  int n = s_cnt;
  if (K > 0 && n > kClCap) {
    select_topk_exact(x, V, true, K, keys, hist, sbuf, &s_n);
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
    cand_q[cbase + j] = ord2f((unsigned)(kk >> 32)) - lse;
    cand_tok[cbase + j] = (int)(~(unsigned)(kk & 0xffffffffu));
  }
  if (threadIdx.x == 0) {
    cand_cnt[row] = keep;
    row_lse[row] = lse;
  }
}

// ---------------------------------------------------------------------------
// best-first growth, one warp per request

__device__ __forceinline__ unsigned long long pool_key(float s, int depth, int pidx, int rank) {
  return ((unsigned long long)f2ord(s) << 32) | ((unsigned long long)(63 - depth) << 20) |
         ((unsigned long long)(1023 - pidx) << 10) | (unsigned long long)(1023 - rank);
}

__global__ __launch_bounds__(32) void cadd_bestfirst_kernel(
    CaddParams p, const int32_t* __restrict__ anchor, const int64_t* __restrict__ ctx,
    const int32_t* __restrict__ cand_cnt, const float* __restrict__ cand_q,
    const int32_t* __restrict__ cand_tok, int32_t* __restrict__ otok, int32_t* __restrict__ opar,
    int32_t* __restrict__ odep, float* __restrict__ oscore, int32_t* __restrict__ ocount,
    float* __restrict__ ophi, int32_t* __restrict__ status) {
  extern __shared__ unsigned long long pool[];          // [n_max + 1]
  const int nmax = p.n_max;
  int* ntok = reinterpret_cast<int*>(pool + nmax + 1);  // [n_max] each
  int* npar = ntok + nmax;
  int* ndep = npar + nmax;
  float* ns = reinterpret_cast<float*>(ndep + nmax);
  int* canon = reinterpret_cast<int*>(ns + nmax);
  int* order = canon + nmax;
  __shared__ int dstart[66], dfill[66];

  const int b = blockIdx.x, lane = threadIdx.x;
  const int D = p.D, K1 = max(nmax - 1, 1);
  const size_t row0 = (size_t)b * D;
  const int a0 = anchor[b];
  if (lane == 0 && (a0 < 0 || a0 >= p.V)) atomicOr(&status[b], PCT_DEV_BAD_TOKEN);
  if (lane == 0) { ntok[0] = a0; npar[0] = -1; ndep[0] = 0; ns[0] = 0.f; }

  auto cnt_at = [&](int depth) { return cand_cnt[row0 + depth - 1]; };
  auto q_at = [&](int depth, int rank) { return cand_q[(row0 + depth - 1) * K1 + rank]; };
  int pool_n = 0;
  if (D >= 1 && nmax > 1 && cnt_at(1) > 0) {
    if (lane == 0) pool[0] = pool_key(q_at(1, 0), 1, 0, 0);
    pool_n = 1;
  }
  __syncwarp();

  const float ell = (float)ctx[b];
  const float cbase = p.C_d + p.a + p.b * ell;
  int n = 1;
  float phi = 0.f;
  while (n < nmax) {
    unsigned long long best = 0ull;
    int bslot = -1;
    for (int j = lane; j < pool_n; j += 32) {
      const unsigned long long k = pool[j];
      if (k > best) { best = k; bslot = j; }
    }
    const unsigned long long wbest = warp_max_u64(best);
    if (wbest == 0ull) break;                                     // no candidate left
    const unsigned own = __ballot_sync(0xffffffffu, best == wbest);
    bslot = __shfl_sync(0xffffffffu, bslot, __ffs(own) - 1);
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
    const int tk = cand_tok[(row0 + depth - 1) * K1 + rank];
    const int np = pidx;
    unsigned long long sib = 0ull, child = 0ull;
    if (rank + 1 < cnt_at(depth)) sib = pool_key(ns[np] + q_at(depth, rank + 1), depth, np, rank + 1);
    if (depth < D && cnt_at(depth + 1) > 0) child = pool_key(s + q_at(depth + 1, 0), depth + 1, n, 0);
    __syncwarp();
    if (lane == 0) {
      ntok[n] = tk; npar[n] = np; ndep[n] = depth; ns[n] = s;
      pool[bslot] = sib;
      if (child) pool[pool_n] = child;
    }
    if (child) ++pool_n;
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

cudaError_t launch_cadd(const CaddParams& p, const void* L, const int32_t* anchor,
                        const int64_t* ctx, int32_t* tok, int32_t* parent, int32_t* depth,
                        float* score, int32_t* count, float* phi, int32_t* status,
                        float* row_lse, int32_t* cand_cnt, float* cand_q, int32_t* cand_tok,
                        cudaStream_t s) {
  const int cl_seg = (p.V / 8 + kClSegs - 1) / kClSegs * 16;   // bytes of the largest segment
  const bool cluster = p.dtype == PCT_BF16 && p.V % 8 == 0 &&
                       (reinterpret_cast<uintptr_t>(L) & 15u) == 0 && cl_seg <= kClSegMax;
  if (cluster) {
    const size_t smem = (size_t)(cl_seg + 127) / 128 * 128 + (size_t)kClCap * sizeof(unsigned long long);
    cudaError_t e = cudaFuncSetAttribute(cadd_cluster_rowpass_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) { (void)cudaGetLastError(); return e; }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kClSegs * p.D, p.batch);
    cfg.blockDim = dim3(kRowThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kClSegs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    TraceScope t(s, "cadd_rowpass");
    e = cudaLaunchKernelEx(&cfg, cadd_cluster_rowpass_kernel, p,
                           static_cast<const __nv_bfloat16*>(L), ctx, row_lse, cand_cnt, cand_q,
                           cand_tok, status);
    if (e != cudaSuccess) { (void)cudaGetLastError(); return e; }
  } else {
    dim3 grid(p.D, p.batch);
    TraceScope t(s, "cadd_rowpass");
    if (p.dtype == PCT_BF16)
      cadd_rowpass_kernel<__nv_bfloat16><<<grid, kRowThreads, 0, s>>>(
          p, static_cast<const __nv_bfloat16*>(L), ctx, row_lse, cand_cnt, cand_q, cand_tok, status);
    else
      cadd_rowpass_kernel<float><<<grid, kRowThreads, 0, s>>>(
          p, static_cast<const float*>(L), ctx, row_lse, cand_cnt, cand_q, cand_tok, status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const size_t smem = (size_t)(p.n_max + 1) * 8 + (size_t)p.n_max * 4 * 6;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(cadd_bestfirst_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  TraceScope t(s, "cadd_bestfirst");
  cadd_bestfirst_kernel<<<p.batch, 32, smem, s>>>(p, anchor, ctx, cand_cnt, cand_q, cand_tok, tok,
                                                  parent, depth, score, count, phi, status);
  return cudaGetLastError();
}

}  // namespace pct
