// Monte Carlo acceptance length of a round's trees (tau, tokens per round).
//
// DSpark explainer (xiaohu-jiedu), one round from drafting to confirmation:
// drafts are checked from the head, the first miss ends the round, and the
// target adds one token of its own. On a tree, a walk starts at the root; at
// node u the target's token for the next position is drawn and the walk moves
// to the child of u that carries it, or stops. Only which child the draw hits
// matters, so a step draws one uniform x and moves to the first child c (in
// index order) whose running sum of p(c) exceeds x, where p(c) is the
// probability that the target's token equals c's token given agreement up to
// u. PCTree article (qiita), numbers table: tau is the pages' headline measure.
//
// Random numbers: Philox4x32-10 (Salmon et al., "Parallel random numbers: as
// easy as 1, 2, 3", SC 2011), written from its definition: draw j of trial t
// of request b uses the counter (t, b, j, 0) and the key (seed low, seed high)
// and the uniform is the first word's top 24 bits times 2^-24. Running sums
// and comparisons are fp32 in child index order, so a host implementation of
// the same definition reproduces every walk.
//
// Layout: one 256-thread block per (request, chunk of trials). Thread 0 links
// the request's children into index-ordered lists in shared memory (first
// child, next sibling), the block counts accepted lengths in a shared
// histogram, and the counts are added to the request's global histogram.
#include "common.cuh"
#include "internal.h"

namespace pct {
namespace {

constexpr int kSimThreads = 256;

__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint32_t hi0 = __umulhi(0xD2511F53u, c.x), lo0 = 0xD2511F53u * c.x;
    const uint32_t hi1 = __umulhi(0xCD9E8D57u, c.z), lo1 = 0xCD9E8D57u * c.z;
    c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
  }
  return c;
}

__global__ __launch_bounds__(kSimThreads) void accept_sim_kernel(
    int n_stride, int max_depth, const int32_t* __restrict__ parent,
    const int32_t* __restrict__ count, const float* __restrict__ p_child, long long trials,
    uint32_t k0, uint32_t k1, unsigned long long* __restrict__ hist, int32_t* __restrict__ status) {
  extern __shared__ int sim_sm[];
  int* first = sim_sm;                                        // [n_stride]
  int* next = first + n_stride;                               // [n_stride]
  float* pc = reinterpret_cast<float*>(next + n_stride);      // [n_stride]
  unsigned* h = reinterpret_cast<unsigned*>(pc + n_stride);   // [max_depth + 1]
  __shared__ int s_bad;
  const int b = blockIdx.y;
  const int raw = count[b];
  const int cnt = min(max(raw, 0), n_stride);
  const int32_t* pr = parent + (size_t)b * n_stride;
  if (threadIdx.x == 0) s_bad = (raw < 1 || raw > n_stride) ? PCT_DEV_BAD_COUNT : 0;
  for (int i = threadIdx.x; i < n_stride; i += blockDim.x) {
    first[i] = -1;
    next[i] = -1;
    pc[i] = p_child[(size_t)b * n_stride + i];
  }
  for (int i = threadIdx.x; i <= max_depth; i += blockDim.x) h[i] = 0u;
  __syncthreads();
  for (int c = threadIdx.x; c < cnt; c += blockDim.x) {
    const int p = pr[c];
    if (c == 0 ? (p != -1) : (p < 0 || p >= c)) atomicOr(&s_bad, PCT_DEV_BAD_PARENT);
  }
  __syncthreads();
  if (s_bad) {
    if (threadIdx.x == 0 && blockIdx.x == 0) atomicOr(&status[b], s_bad);
    return;
  }
  if (threadIdx.x == 0) {
    // children in increasing index order: link from the last node down
    for (int c = cnt - 1; c >= 1; --c) {
      const int p = pr[c];
      next[c] = first[p];
      first[p] = c;
    }
  }
  __syncthreads();
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x; t < trials; t += stride) {
    int u = 0, acc = 0;
    for (int j = 0; j < max_depth; ++j) {
      const uint4 r = philox4x32_10(make_uint4((uint32_t)t, (uint32_t)b, (uint32_t)j, 0u), k0, k1);
      const float x = __uint2float_rn(r.x >> 8) * (1.0f / 16777216.0f);
      float cum = 0.f;
      int nxt = -1;
      for (int c = first[u]; c >= 0; c = next[c]) {
        cum = __fadd_rn(cum, pc[c]);
        if (x < cum) {
          nxt = c;
          break;
        }
      }
      if (nxt < 0) break;
      u = nxt;
      ++acc;
    }
    atomicAdd(&h[acc], 1u);
  }
  __syncthreads();
  for (int i = threadIdx.x; i <= max_depth; i += blockDim.x)
    if (h[i]) atomicAdd(&hist[(size_t)b * (max_depth + 1) + i], (unsigned long long)h[i]);
}

}  // namespace

size_t accept_sim_smem(int n_stride, int max_depth) {
  return 3 * sizeof(int) * (size_t)n_stride + sizeof(unsigned) * (size_t)(max_depth + 1);
}

cudaError_t launch_accept_sim(int batch, int n_stride, int max_depth, const int32_t* parent,
                              const int32_t* count, const float* p_child, long long trials,
                              unsigned long long seed, unsigned long long* hist, int32_t* status,
                              cudaStream_t s) {
  const size_t smem = accept_sim_smem(n_stride, max_depth);
  cudaError_t e = cudaFuncSetAttribute(accept_sim_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return e;
  }
  // enough chunks of trials per request to fill the GPU a few times over
  const long long per_block = kSimThreads;
  long long chunks = (trials + per_block - 1) / per_block;
  const long long want = (4LL * num_sms() + batch - 1) / batch;
  chunks = chunks < want ? chunks : want;
  chunks = chunks < 1 ? 1 : (chunks > 65535 ? 65535 : chunks);
  dim3 grid((unsigned)chunks, (unsigned)batch);
  TraceScope t(s, "accept_sim");
  accept_sim_kernel<<<grid, kSimThreads, smem, s>>>(n_stride, max_depth, parent, count, p_child,
                                                     trials, (uint32_t)(seed & 0xffffffffull),
                                                     (uint32_t)(seed >> 32), hist, status);
  return cudaGetLastError();
}

}  // namespace pct
