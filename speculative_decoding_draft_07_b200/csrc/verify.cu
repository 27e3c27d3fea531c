// Tree verification and the tree-attention ancestor mask.
//
// DSpark explainer (xiaohu-jiedu), section on one round from drafting to
// confirmation: drafts are checked from the head, consecutive matches are
// kept, the first miss ends the check and the target contributes its own token
// there. On a tree with greedy decoding this is: argmax of the target logits
// at every node, then a walk from the root along children whose token equals
// the current node's argmax; the correction is the argmax where the walk ends.
//
// Kernel layout (B200): one 256-thread block per (request, node row). The row
// (V bf16 values, 303.9 KB at V = 151936) is streamed once with 16-byte
// non-allocating loads, eight in flight per thread; each 8-value chunk is
// reduced with packed bf16 max first, and only a chunk that beats the running
// maximum is searched for its first position, so the common path costs a few
// instructions per 16 bytes. The block that finishes last for a request
// (arrival counter) performs that request's accept walk, so no second launch
// and no grid-wide wait is needed.
#include <cuda.h>

#include <climits>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace pct {
namespace {

constexpr int kVerifyThreads = 256;
constexpr int kUnroll = 8;

// ---------------------------------------------------------------------------
// Ancestor mask: thread = (row i, word w). Ancestors have smaller indices
// (parent[i] < i), so the walk can stop as soon as it drops below the word.
__global__ void ancestor_mask_kernel(int n_stride, int words, const int32_t* __restrict__ parent,
                                     const int32_t* __restrict__ count, uint32_t* __restrict__ mask,
                                     int32_t* __restrict__ status) {
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.y;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= n_stride * words) return;
  const int i = idx / words, w = idx - (idx / words) * words;
  int cnt = count[b];
  if (cnt < 1 || cnt > n_stride) {
    if (idx == 0) atomicOr(&status[b], PCT_DEV_BAD_COUNT);
    cnt = min(max(cnt, 0), n_stride);
  }
  const int32_t* pr = parent + (size_t)b * n_stride;
  uint32_t bits = 0;
  if (i < cnt) {
    const int lo = w * 32, hi = lo + 32;
    int j = i;
    bool bad = false;
    for (int steps = 0; steps <= n_stride; ++steps) {   // j strictly decreases
      if (j < lo && w != 0) break;
      if (j < hi) bits |= 1u << (j - lo);
      const int pj = pr[j];
      if (j == 0) { bad = (pj != -1); break; }
      if (pj < 0 || pj >= j) { bad = true; break; }
      j = pj;
    }
    if (bad && w == 0) atomicOr(&status[b], PCT_DEV_BAD_PARENT);
  }
  mask[((size_t)b * n_stride + i) * words + w] = bits;
}

// ---------------------------------------------------------------------------
// Block-wide (value desc, index asc) reduction; result valid in every thread.
__device__ __forceinline__ void block_best(float& v, int& i, float* sv, int* si) {
  warp_best(v, i);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) { sv[warp] = v; si[warp] = i; }
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    v = lane < nw ? sv[lane] : neg_inf();
    i = lane < nw ? si[lane] : INT_MAX;
    warp_best(v, i);
    if (lane == 0) { sv[0] = v; si[0] = i; }
  }
  __syncthreads();
  v = sv[0]; i = si[0];
  __syncthreads();
}

__device__ __forceinline__ int block_min(int x, int* sm) {
  x = warp_min_i(x);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) sm[warp] = x;
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    x = lane < nw ? sm[lane] : INT_MAX;
    x = warp_min_i(x);
    if (lane == 0) sm[0] = x;
  }
  __syncthreads();
  x = sm[0];
  __syncthreads();
  return x;
}

// Position (0..7) of the first value equal to `m` among 8 packed bf16.
__device__ __forceinline__ int first_eq8(const uint4& q, float m) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
  int pos = 7;
#pragma unroll
  for (int j = 7; j >= 0; --j) {
    const float x = (j & 1) ? bf16_hi(w[j >> 1]) : bf16_lo(w[j >> 1]);
    if (x == m) pos = j;
  }
  return pos;
}

__device__ __forceinline__ float max8_bf16(const uint4& q) {
  __nv_bfloat162 a = __hmax2(*reinterpret_cast<const __nv_bfloat162*>(&q.x),
                             *reinterpret_cast<const __nv_bfloat162*>(&q.y));
  __nv_bfloat162 b = __hmax2(*reinterpret_cast<const __nv_bfloat162*>(&q.z),
                             *reinterpret_cast<const __nv_bfloat162*>(&q.w));
  a = __hmax2(a, b);
  return fmaxf(__low2float(a), __high2float(a));
}

// Row argmax, bf16, 16-byte vector path (row start 16-byte aligned).
__device__ __forceinline__ void row_argmax_bf16_vec(const __nv_bfloat16* row, int V, float& best,
                                                    int& bidx) {
  const uint4* p = reinterpret_cast<const uint4*>(row);
  const int nvec = V >> 3;
  const int tid = threadIdx.x;
  for (int base = tid; base < nvec; base += kVerifyThreads * kUnroll) {
    uint4 q[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int c = base + u * kVerifyThreads;
      q[u] = c < nvec ? ld_stream16(p + c) : make_uint4(0xff80ff80u, 0xff80ff80u, 0xff80ff80u, 0xff80ff80u);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const float cm = max8_bf16(q[u]);
      if (cm > best) {
        best = cm;
        bidx = (base + u * kVerifyThreads) * 8 + first_eq8(q[u], cm);
      }
    }
  }
  // tail (V % 8 values), scalar
  const int tail0 = nvec << 3;
  for (int v = tail0 + tid; v < V; v += kVerifyThreads) {
    const float x = load_f(row + v);
    if (x > best) { best = x; bidx = v; }
  }
}

template <typename T>
__device__ __forceinline__ void row_argmax_scalar(const T* row, int V, float& best, int& bidx) {
  for (int v = threadIdx.x; v < V; v += kVerifyThreads) {
    const float x = load_f(row + v);
    if (x > best) { best = x; bidx = v; }
  }
}

__device__ __forceinline__ void row_argmax_f32_vec(const float* row, int V, float& best, int& bidx) {
  const float4* p = reinterpret_cast<const float4*>(row);
  const int nvec = V >> 2;
  const int tid = threadIdx.x;
  for (int base = tid; base < nvec; base += kVerifyThreads * kUnroll) {
    float4 q[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int c = base + u * kVerifyThreads;
      if (c < nvec) {
        uint4 t = ld_stream16(p + c);
        q[u] = make_float4(__uint_as_float(t.x), __uint_as_float(t.y), __uint_as_float(t.z),
                           __uint_as_float(t.w));
      } else {
        q[u] = make_float4(neg_inf(), neg_inf(), neg_inf(), neg_inf());
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int v0 = (base + u * kVerifyThreads) * 4;
      if (q[u].x > best) { best = q[u].x; bidx = v0; }
      if (q[u].y > best) { best = q[u].y; bidx = v0 + 1; }
      if (q[u].z > best) { best = q[u].z; bidx = v0 + 2; }
      if (q[u].w > best) { best = q[u].w; bidx = v0 + 3; }
    }
  }
  for (int v = (nvec << 2) + tid; v < V; v += kVerifyThreads) {
    const float x = row[v];
    if (x > best) { best = x; bidx = v; }
  }
}

// MODE 0: bf16 vector, 1: bf16 scalar, 2: f32 vector, 3: f32 scalar.
template <int MODE>
__global__ __launch_bounds__(kVerifyThreads) void verify_kernel(
    int n_stride, int V, int max_depth, const int32_t* __restrict__ tok,
    const int32_t* __restrict__ parent, const int32_t* __restrict__ count,
    const void* __restrict__ target, int32_t* __restrict__ argmax, int32_t* __restrict__ alen,
    int32_t* __restrict__ apath, int32_t* __restrict__ corr, int32_t* __restrict__ status,
    unsigned* __restrict__ arrive) {
  pdl_wait();
  pdl_trigger();
  __shared__ float sv[32];
  __shared__ int si[32];
  __shared__ int s_last;
  const int i = blockIdx.x, b = blockIdx.y;
  const int raw_cnt = count[b];
  const int cnt = min(max(raw_cnt, 0), n_stride);

  if (i < cnt) {
    float best = neg_inf();
    int bidx = INT_MAX;
    const size_t off = ((size_t)b * n_stride + i) * (size_t)V;
    if (MODE == 0) row_argmax_bf16_vec(static_cast<const __nv_bfloat16*>(target) + off, V, best, bidx);
    if (MODE == 1) row_argmax_scalar(static_cast<const __nv_bfloat16*>(target) + off, V, best, bidx);
    if (MODE == 2) row_argmax_f32_vec(static_cast<const float*>(target) + off, V, best, bidx);
    if (MODE == 3) row_argmax_scalar(static_cast<const float*>(target) + off, V, best, bidx);
    block_best(best, bidx, sv, si);
    // a row that is entirely -inf: every position is a maximum, the first wins
    if (threadIdx.x == 0) argmax[(size_t)b * n_stride + i] = (best == neg_inf()) ? 0 : bidx;
  } else if (threadIdx.x == 0) {
    argmax[(size_t)b * n_stride + i] = -1;
  }

  // arrival: the last block of this request walks the tree
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned prev = atomicAdd(&arrive[b], 1u);
    s_last = (prev == (unsigned)n_stride - 1u);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  const int32_t* tk = tok + (size_t)b * n_stride;
  const int32_t* pr = parent + (size_t)b * n_stride;
  const int32_t* am = argmax + (size_t)b * n_stride;
  int bad = 0;
  if (raw_cnt < 1 || raw_cnt > n_stride) bad |= PCT_DEV_BAD_COUNT;
  for (int c = threadIdx.x; c < cnt; c += blockDim.x) {
    const int p = pr[c];
    if (c == 0 ? (p != -1) : (p < 0 || p >= c)) bad |= PCT_DEV_BAD_PARENT;
    const int t = tk[c];
    if (t < 0 || t >= V) bad |= PCT_DEV_BAD_TOKEN;
  }
  if (bad) atomicOr(&status[b], bad);

  int u = 0, len = 0;
  int* s_min = si;
  if (cnt > 0) {
    for (int iter = 0; iter <= max_depth; ++iter) {
      const int want = __ldcg(am + u);
      int best = INT_MAX;
      for (int c = 1 + threadIdx.x; c < cnt; c += blockDim.x)
        if (pr[c] == u && tk[c] == want) best = min(best, c);
      best = block_min(best, s_min);
      if (best == INT_MAX) break;
      if (len == max_depth) {
        if (threadIdx.x == 0) atomicOr(&status[b], PCT_DEV_DEPTH_OVERFLOW);
        break;
      }
      if (threadIdx.x == 0) apath[(size_t)b * max_depth + len] = best;
      ++len;
      u = best;
    }
  }
  for (int j = len + threadIdx.x; j < max_depth; j += blockDim.x) apath[(size_t)b * max_depth + j] = -1;
  if (threadIdx.x == 0) {
    alen[b] = len;
    corr[b] = cnt > 0 ? __ldcg(am + u) : -1;
    arrive[b] = 0u;   // leave the counter ready for the next call
  }
}

}  // namespace

cudaError_t launch_ancestor_mask(int batch, int n_stride, const int32_t* parent,
                                 const int32_t* count, uint32_t* mask, int32_t* status,
                                 cudaStream_t s) {
  const int words = (n_stride + 31) / 32;
  const int total = n_stride * words;
  dim3 grid((total + 255) / 256, batch);
  TraceScope t(s, "ancestor_mask");
  return launch_pdl(ancestor_mask_kernel, grid, dim3(256), 0, s, 1, n_stride, words, parent, count,
                    mask, status);
}

cudaError_t launch_verify(int batch, int n_stride, int vocab, int max_depth, const int32_t* tok,
                          const int32_t* parent, const int32_t* count, const void* target,
                          int dtype, int32_t* argmax, int32_t* alen, int32_t* apath,
                          int32_t* corr, int32_t* status, unsigned* arrive, cudaStream_t s) {
  dim3 grid(n_stride, batch);
  const bool aligned16 = (reinterpret_cast<uintptr_t>(target) & 15u) == 0;
  TraceScope t(s, "verify_argmax_walk");
  cudaError_t e;
  if (dtype == PCT_BF16) {
    if (aligned16 && vocab % 8 == 0)
      e = launch_pdl(verify_kernel<0>, grid, dim3(kVerifyThreads), 0, s, 1, n_stride, vocab,
                     max_depth, tok, parent, count, target, argmax, alen, apath, corr, status, arrive);
    else
      e = launch_pdl(verify_kernel<1>, grid, dim3(kVerifyThreads), 0, s, 1, n_stride, vocab,
                     max_depth, tok, parent, count, target, argmax, alen, apath, corr, status, arrive);
  } else {
    if (aligned16 && vocab % 4 == 0)
      e = launch_pdl(verify_kernel<2>, grid, dim3(kVerifyThreads), 0, s, 1, n_stride, vocab,
                     max_depth, tok, parent, count, target, argmax, alen, apath, corr, status, arrive);
    else
      e = launch_pdl(verify_kernel<3>, grid, dim3(kVerifyThreads), 0, s, 1, n_stride, vocab,
                     max_depth, tok, parent, count, target, argmax, alen, apath, corr, status, arrive);
  }
  return e;
}

// ---------------------------------------------------------------------------
// Lazy verification walk (the same acceptance, argmax only along the walk).
//
// DSpark explainer, one round from drafting to confirmation: the drafts are
// checked from the head and checking stops at the first miss, so the only
// target rows whose argmax decides the round are the rows of the nodes the walk
// reaches: the root and each accepted node, at most max_depth + 1 rows.
//
// One cluster of kWalkCluster CTAs per request. Each CTA owns a fixed eighth of
// the vocabulary; per step it scans its part of the current node's row, the
// eight partial (max, first index) pairs are merged through distributed shared
// memory after one cluster barrier, and every CTA finds the same next node in
// its shared-memory copy of the tree. The partial slots alternate between two
// buffers, so one barrier per step keeps a slot from being rewritten before
// every CTA has read it. Cluster barriers are hardware barriers: no CTA waits on
// a flag.
namespace {

constexpr int kWalkCluster = 8;
constexpr int kWalkThreads = 256;

__device__ __forceinline__ uint32_t walk_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void walk_cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
// A value and an index from the same shared-memory object of CTA `rank` of the cluster.
__device__ __forceinline__ void walk_remote_pair(const float* v, const int* i, uint32_t rank,
                                                 float& rv, int& ri) {
  uint32_t av, ai;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;"
               : "=r"(av) : "r"((uint32_t)__cvta_generic_to_shared(v)), "r"(rank));
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;"
               : "=r"(ai) : "r"((uint32_t)__cvta_generic_to_shared(i)), "r"(rank));
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(rv) : "r"(av) : "memory");
  asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(ri) : "r"(ai) : "memory");
}

// Argmax (value desc, index asc) of row[lo, hi) by this thread: MODE 0 bf16 in
// 8-value groups (lo, hi multiples of 8, row 16-byte aligned), 2 fp32 in
// 4-value groups (same for 4), 1 / 3 element by element.
template <int MODE>
__device__ __forceinline__ void walk_scan(const void* rowp, int lo, int hi, float& best, int& bidx) {
  const int tid = threadIdx.x;
  if (MODE == 0) {
    const uint4* p = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(rowp));
    const int g0 = lo >> 3, g1 = hi >> 3;
    for (int base = g0 + tid; base < g1; base += kWalkThreads * kUnroll) {
      uint4 q[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int c = base + u * kWalkThreads;
        q[u] = c < g1 ? ld_stream16(p + c) : make_uint4(0xff80ff80u, 0xff80ff80u, 0xff80ff80u, 0xff80ff80u);
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const float cm = max8_bf16(q[u]);
        if (cm > best) {
          best = cm;
          bidx = (base + u * kWalkThreads) * 8 + first_eq8(q[u], cm);
        }
      }
    }
  } else if (MODE == 2) {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(rowp));
    const int g0 = lo >> 2, g1 = hi >> 2;
    for (int base = g0 + tid; base < g1; base += kWalkThreads * kUnroll) {
      float4 q[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int c = base + u * kWalkThreads;
        if (c < g1) {
          const uint4 t = ld_stream16(p + c);
          q[u] = make_float4(__uint_as_float(t.x), __uint_as_float(t.y), __uint_as_float(t.z),
                             __uint_as_float(t.w));
        } else {
          q[u] = make_float4(neg_inf(), neg_inf(), neg_inf(), neg_inf());
        }
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int v0 = (base + u * kWalkThreads) * 4;
        if (q[u].x > best) { best = q[u].x; bidx = v0; }
        if (q[u].y > best) { best = q[u].y; bidx = v0 + 1; }
        if (q[u].z > best) { best = q[u].z; bidx = v0 + 2; }
        if (q[u].w > best) { best = q[u].w; bidx = v0 + 3; }
      }
    }
  } else {
    for (int v = lo + tid; v < hi; v += kWalkThreads) {
      const float x = MODE == 1 ? load_f(static_cast<const __nv_bfloat16*>(rowp) + v)
                                : load_f(static_cast<const float*>(rowp) + v);
      if (x > best) { best = x; bidx = v; }
    }
  }
}

template <int MODE>
__global__ __launch_bounds__(kWalkThreads) void verify_walk_kernel(
    int n_stride, int V, int max_depth, const int32_t* __restrict__ tok,
    const int32_t* __restrict__ parent, const int32_t* __restrict__ count,
    const void* __restrict__ target, int32_t* __restrict__ argmax, int32_t* __restrict__ alen,
    int32_t* __restrict__ apath, int32_t* __restrict__ corr, int32_t* __restrict__ status) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int32_t walk_tree[];          // [n_stride] tokens, then [n_stride] parents
  __shared__ float part_v[2];
  __shared__ int part_i[2];
  __shared__ float sv[32];
  __shared__ int si[32];
  __shared__ int s_am;
  const uint32_t rank = walk_ctarank();
  const int b = blockIdx.x / kWalkCluster;
  const int raw_cnt = count[b];
  const int cnt = min(max(raw_cnt, 0), n_stride);
  int32_t* stok = walk_tree;
  int32_t* spar = walk_tree + n_stride;
  const int32_t* tk = tok + (size_t)b * n_stride;
  const int32_t* pr = parent + (size_t)b * n_stride;
  int bad = 0;
  for (int c = threadIdx.x; c < cnt; c += blockDim.x) {
    const int t = tk[c], p = pr[c];
    stok[c] = t;
    spar[c] = p;
    if (c == 0 ? (p != -1) : (p < 0 || p >= c)) bad |= PCT_DEV_BAD_PARENT;
    if (t < 0 || t >= V) bad |= PCT_DEV_BAD_TOKEN;
  }
  if (rank == 0) {
    if (threadIdx.x == 0 && (raw_cnt < 1 || raw_cnt > n_stride)) bad |= PCT_DEV_BAD_COUNT;
    if (bad) atomicOr(&status[b], bad);
    for (int c = threadIdx.x; c < n_stride; c += blockDim.x) argmax[(size_t)b * n_stride + c] = -1;
  }
  // this CTA's part of every row, in whole 16-byte groups where the mode uses them
  const int unit = MODE == 0 ? 8 : (MODE == 2 ? 4 : 1);
  const int units = V / unit;
  const int lo = (int)((long long)units * rank / kWalkCluster) * unit;
  const int hi = (int)((long long)units * (rank + 1) / kWalkCluster) * unit;
  const size_t esz = (MODE == 0 || MODE == 1) ? 2 : 4;
  const char* tb = static_cast<const char*>(target) + (size_t)b * n_stride * V * esz;
  __syncthreads();

  int u = 0, len = 0;
  bool go = cnt > 0;
  for (int step = 0; go; ++step) {
    const int par = step & 1;
    float best = neg_inf();
    int bidx = INT_MAX;
    walk_scan<MODE>(tb + (size_t)u * V * esz, lo, hi, best, bidx);
    block_best(best, bidx, sv, si);
    if (threadIdx.x == 0) { part_v[par] = best; part_i[par] = bidx; }
    walk_cluster_sync();
    if (threadIdx.x < 32) {
      float v = neg_inf();
      int i = INT_MAX;
      if (threadIdx.x < kWalkCluster) walk_remote_pair(&part_v[par], &part_i[par], threadIdx.x, v, i);
      warp_best(v, i);
      // a row that is entirely -inf: every position is a maximum, the first wins
      if (threadIdx.x == 0) s_am = (v == neg_inf()) ? 0 : i;
    }
    __syncthreads();
    const int am = s_am;
    if (rank == 0 && threadIdx.x == 0) argmax[(size_t)b * n_stride + u] = am;
    int nxt = INT_MAX;
    for (int c = 1 + threadIdx.x; c < cnt; c += blockDim.x)
      if (spar[c] == u && stok[c] == am) nxt = min(nxt, c);
    nxt = block_min(nxt, si);
    if (nxt == INT_MAX) {
      go = false;
      if (rank == 0 && threadIdx.x == 0) corr[b] = am;
    } else if (len == max_depth) {
      go = false;
      if (rank == 0 && threadIdx.x == 0) {
        atomicOr(&status[b], PCT_DEV_DEPTH_OVERFLOW);
        corr[b] = am;
      }
    } else {
      if (rank == 0 && threadIdx.x == 0) apath[(size_t)b * max_depth + len] = nxt;
      ++len;
      u = nxt;
    }
  }
  if (rank == 0) {
    for (int j = len + threadIdx.x; j < max_depth; j += blockDim.x) apath[(size_t)b * max_depth + j] = -1;
    if (threadIdx.x == 0) {
      alen[b] = len;
      if (cnt == 0) corr[b] = -1;
    }
  }
  walk_cluster_sync();   // no CTA leaves while another may still read its partial slots
}

}  // namespace

cudaError_t launch_verify_walk(int batch, int n_stride, int vocab, int max_depth,
                               const int32_t* tok, const int32_t* parent, const int32_t* count,
                               const void* target, int dtype, int32_t* argmax, int32_t* alen,
                               int32_t* apath, int32_t* corr, int32_t* status, cudaStream_t s) {
  const bool aligned16 = (reinterpret_cast<uintptr_t>(target) & 15u) == 0;
  int mode;
  if (dtype == PCT_BF16) mode = (aligned16 && vocab % 8 == 0) ? 0 : 1;
  else mode = (aligned16 && vocab % 4 == 0) ? 2 : 3;
  const dim3 grid(batch * kWalkCluster), block(kWalkThreads);
  const size_t smem = 2 * sizeof(int32_t) * (size_t)n_stride;
  TraceScope t(s, "verify_walk");
#define PCT_WALK(M)                                                                              \
  launch_pdl(verify_walk_kernel<M>, grid, block, smem, s, kWalkCluster, n_stride, vocab,         \
             max_depth, tok, parent, count, target, argmax, alen, apath, corr, status)
  switch (mode) {
    case 0: return PCT_WALK(0);
    case 1: return PCT_WALK(1);
    case 2: return PCT_WALK(2);
    default: return PCT_WALK(3);
  }
#undef PCT_WALK
}

}  // namespace pct

// ---------------------------------------------------------------------------
// Allocation-free verification entry point.
//
// For callers that cannot allocate device memory (see the header): the only
// scratch the verification kernel needs, one arrival counter per request,
// lives in this file-scope device array instead of a caller workspace. Every
// GPU that loads the library holds it (16 KB) until the process exits, and
// every call shares it.
namespace pct {
namespace {

__device__ __align__(256) unsigned g_noalloc_arrive[PCT_NOALLOC_MAX_BATCH];

std::mutex g_noalloc_mu;
struct NoallocSlot {
  CUcontext ctx;   // context the address belongs to
  void* ptr;
};
NoallocSlot g_noalloc_slot[64] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  }
  return fn;
}

// Device address of the counters in the current context. Host code may not use
// the array's name as a device pointer, so the address is looked up with
// cudaGetSymbolAddress the first time a context calls in, and kept per device
// together with that context: a different context on the same device (after
// cudaDeviceReset, or one the caller made current) is looked up again.
int noalloc_counters(unsigned** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PCT_ECUDA;
  if (dev < 0 || dev >= 64) return PCT_EUNSUPPORTED;
  CtxGetCurrentFn cur = ctx_get_current();
  if (!cur) return PCT_ECUDA;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  CUcontext ctx = nullptr;
  if (cur(&ctx) != CUDA_SUCCESS) return PCT_ECUDA;
  NoallocSlot& slot = g_noalloc_slot[dev];
  if (ctx == nullptr || slot.ptr == nullptr || slot.ctx != ctx) {
    void* p = nullptr;   // the lookup makes the device's context current if none was
    if (cudaGetSymbolAddress(&p, g_noalloc_arrive) != cudaSuccess || p == nullptr) return PCT_ECUDA;
    if (cur(&ctx) != CUDA_SUCCESS || ctx == nullptr) return PCT_ECUDA;
    slot.ctx = ctx;
    slot.ptr = p;
  }
  *out = static_cast<unsigned*>(slot.ptr);
  return PCT_OK;
}

}  // namespace
}  // namespace pct

extern "C" int32_t tree_verify_accept_noalloc(int32_t batch, int32_t n_stride, int32_t vocab,
                                              int32_t max_depth, const int32_t* tok,
                                              const int32_t* parent, const int32_t* count,
                                              const void* target, int32_t target_dtype,
                                              int32_t* argmax, int32_t* accept_len,
                                              int32_t* accept_path, int32_t* correction,
                                              int32_t* dev_status, void* cuda_stream) {
  if (batch < 1 || n_stride < 1 || n_stride > 4096) return PCT_EINVAL;
  if (batch > PCT_NOALLOC_MAX_BATCH) return PCT_EUNSUPPORTED;
  if (vocab < 1 || max_depth < 1 || max_depth > 4096) return PCT_EINVAL;
  if (target_dtype != PCT_F32 && target_dtype != PCT_BF16) return PCT_EINVAL;
  if (!tok || !parent || !count || !target || !argmax || !accept_len || !accept_path ||
      !correction || !dev_status)
    return PCT_EINVAL;
  if (!pct::device_ok()) return PCT_EDEVICE;
  unsigned* arrive = nullptr;
  const int st = pct::noalloc_counters(&arrive);
  if (st != PCT_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  // the counters keep the previous call's contents: clear the ones this call uses
  if (cudaMemsetAsync(dev_status, 0, sizeof(int32_t) * batch, s) != cudaSuccess) return PCT_ECUDA;
  if (cudaMemsetAsync(arrive, 0, sizeof(unsigned) * batch, s) != cudaSuccess) return PCT_ECUDA;
  if (pct::launch_verify(batch, n_stride, vocab, max_depth, tok, parent, count, target,
                         target_dtype, argmax, accept_len, accept_path, correction, dev_status,
                         arrive, s) != cudaSuccess)
    return PCT_ECUDA;
  return PCT_OK;
}
