// PCTree selection kernels: partial merge, per-depth beam, global top-N.
//
// PCTree article (qiita), section on the chain draft's weakness and the tree
// built in its place: after every frontier parent p has been scored,
// z_d(p) = L_d + Markov(p), each parent keeps its local top-k children,
// candidates are ranked by s(c) = s(p) + log pi(c|p), each depth is pruned to
// the beam, and a final global top-N keeps the tree inside the verification
// budget.
//
//  * gather:  Eg[row] = E[token of the row's parent] (the batched Markov call's
//             A operand for the next depth), zero-padded to the MMA's K tile.
//  * merge:   one 512-thread block per request and depth. A warp per parent
//             row folds the V-slice partials into the row's log-sum-exp and
//             top-k; the |F| * k candidates become 64-bit keys ordered by the
//             total order (score desc, parent position asc, token asc) and are
//             bitonic-sorted; the best `beam` are re-sorted into canonical
//             order (parent position, token), which within one depth is the
//             lexicographic order of the token paths.
//  * final:   one block per request; the kept nodes of all depths are ranked
//             by (score desc, depth asc, canonical position asc), the best N-1
//             selected, and an exclusive scan over the depth-major flattening
//             gives every selected node its canonical BFS index; parents are
//             remapped through the same scan.
#include <climits>
#include <type_traits>

#include "common.cuh"
#include "internal.h"
#include "seed.cuh"
#include "select.cuh"

namespace pct {
namespace {

template <typename TE>
__global__ void gather_rows_kernel(int rows, const int32_t* __restrict__ toks, int V, int r,
                                   int r_pad, const TE* __restrict__ E, TE* __restrict__ Eg,
                                   int32_t* __restrict__ status, int status_div, SeedArgs seed) {
  pdl_wait();
  pdl_trigger();
  const int row = blockIdx.x;
  if (row >= rows) return;
  int t = toks[row];
  if (t < 0 || t >= V) {
    if (threadIdx.x == 0) atomicOr(&status[row / status_div], PCT_DEV_BAD_TOKEN);
    t = 0;
  }
  const TE* src = E + (size_t)t * r;
  TE* dst = Eg + (size_t)row * r_pad;
  for (int j = threadIdx.x; j < r_pad; j += blockDim.x) dst[j] = j < r ? src[j] : TE(0.f);
  if constexpr (std::is_same<TE, __nv_bfloat16>::value) {
    if (seed.thr == nullptr) return;
    // one row per request: its seed from the request's seed data
    __shared__ __align__(16) SeedSmem sm;
    const size_t e = (size_t)row * seed.req_stride;
    const SeedData sd{seed.cols + e, seed.lval + e, seed.wmax + e,
                      static_cast<const __nv_bfloat16*>(seed.wcol) + e * r_pad};
    seed_prefetch(sd, seed.ks, r_pad, &sm);
    seed_prefetch_wait();   // also orders the Eg row written above
    seed_rows(1, [&](int) { return static_cast<const __nv_bfloat16*>(dst); }, &sm, seed.ks, r_pad,
              seed.thr + row);
  }
}

// Fold the S partials of one row with a group of G lanes (G = 16 or 32, the
// group aligned within the warp; every lane of the warp calls it). Returns lse
// and writes the row's k best (value desc, token asc) to out_v / out_i. Each
// lane takes its slices' lists (sorted by the scoring kernel: a lane with a
// single slice copies it, more are merged into it), then k rounds of "take the
// best head across the group, the owner pops".
template <int KMAX, int G>
__device__ __forceinline__ float merge_row(const Partials& part, size_t row, int S, int k,
                                           float* out_v, int* out_i) {
  const int gl = threadIdx.x & (G - 1);
  float m = neg_inf(), s = 0.f;
  TopK<KMAX> tk;
  tk.init(k);
  bool first = true;
  for (int sl = gl; sl < S; sl += G) {
    const size_t ps = row * S + sl;
    const float2 ms = part.ms[ps];
    lse_combine(m, s, ms.x, ms.y);
    float v[KMAX];
    int id[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      v[j] = j < k ? part.val[ps * k + j] : neg_inf();
      id[j] = j < k ? part.idx[ps * k + j] : 0x7fffffff;
    }
    if (first && k == KMAX) {
#pragma unroll
      for (int j = 0; j < KMAX; ++j) { tk.v[j] = v[j]; tk.i[j] = id[j]; }
    } else {
#pragma unroll
      for (int j = 0; j < KMAX; ++j)
        if (j < k && tk.admits(v[j], id[j])) tk.insert(v[j], id[j]);
    }
    first = false;
  }
  tk.finish(k);
#pragma unroll
  for (int o = G / 2; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o), s2 = __shfl_xor_sync(0xffffffffu, s, o);
    lse_combine(m, s, m2, s2);
  }
  const float lse = (m == neg_inf()) ? neg_inf() : m + logf(s);
  // rolled: this code runs once per launch, so its size (instruction fetch)
  // costs more than the loop
#pragma unroll 1
  for (int j = 0; j < k; ++j) {
    float v = tk.v[0];
    int i = tk.i[0];
#pragma unroll
    for (int o = G / 2; o > 0; o >>= 1) {
      const float v2 = __shfl_xor_sync(0xffffffffu, v, o);
      const int i2 = __shfl_xor_sync(0xffffffffu, i, o);
      if (better(v2, i2, v, i)) { v = v2; i = i2; }
    }
    if (tk.v[0] == v && tk.i[0] == i) tk.pop();
    if (gl == 0) { out_v[j] = v; out_i[j] = i; }
  }
  return lse;
}

constexpr int kMergeThreads = 512;
constexpr int kMaxCand = 1024;

// Descending bitonic sort of keys[0..P) (P a power of two) by the block.
__device__ void bitonic_desc_block(unsigned long long* keys, int P) {
  for (int size = 2; size <= P; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int t = threadIdx.x; t < P / 2; t += blockDim.x) {
        const int lo = 2 * t - (t & (stride - 1));
        const int hi = lo + stride;
        const bool desc = ((lo & size) == 0);
        const unsigned long long x = keys[lo], y = keys[hi];
        if (desc ? (x < y) : (x > y)) { keys[lo] = y; keys[hi] = x; }
      }
      __syncthreads();
    }
  }
}

template <int KMAX, typename TE>
__global__ __launch_bounds__(kMergeThreads, 1) void merge_kernel(MergeArgs a) {
  pdl_wait();
  pdl_trigger();
  __shared__ unsigned long long keys[kMaxCand];
  __shared__ unsigned long long ck[256];
  __shared__ float kept_s[256];
  __shared__ float wv[kMergeThreads / 32][32];
  __shared__ int wi[kMergeThreads / 32][32];
  // the next depth's parent embeddings (bf16), kept for the seeds (up to 32
  // rows; the row stride's extra 16 bytes keep the seed product's fragment
  // loads free of bank conflicts)
  constexpr int kEgsStride = kSeedMaxR + 8;
  __shared__ __align__(16) uint16_t egs[kSeedMmaRows * kEgsStride];
  __shared__ float e1s[kSeedMmaRows];
  const int b = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = kMergeThreads / 32;
  const int F = a.F_prev, k = a.k, C = F * k;
  if (threadIdx.x == 0 && *a.err) atomicOr(&a.status[b], PCT_DEV_TIMEOUT);
  // the next depth's seed data (W columns) arrive while the merge runs
  __shared__ __align__(16) SeedSmem seed_sm;
  const size_t se = (size_t)b * a.seed.req_stride;
  if constexpr (std::is_same<TE, __nv_bfloat16>::value) {
    if (a.seed.thr != nullptr) {
      const SeedData sd{a.seed.cols + se, a.seed.lval + se, a.seed.wmax + se,
                        static_cast<const __nv_bfloat16*>(a.seed.wcol) + se * a.r_pad};
      seed_prefetch(sd, a.seed.ks, a.r_pad, &seed_sm);
    }
  }

  // candidates (score, parent position, token) as ordered keys: a half warp
  // per parent row when a row has at most 16 V-slices, else a warp
  if (a.S <= 16) {
    const int h = lane >> 4, gl = lane & 15;
    for (int i0 = 2 * warp; i0 < F; i0 += 2 * nwarps) {
      const int i = i0 + h;
      const size_t row = (size_t)b * F + min(i, F - 1);   // both halves take part in the shuffles
      const float sp = (a.prev_s && i < F) ? a.prev_s[(size_t)b * a.prev_stride + i] : 0.f;
      const float lse = merge_row<KMAX, 16>(a.part, row, a.S, k, wv[warp] + 16 * h, wi[warp] + 16 * h);
      __syncwarp();
      if (i < F) {
        for (int j = gl; j < k; j += 16)
          keys[i * k + j] = beam_key(sp + (wv[warp][16 * h + j] - lse), i, wi[warp][16 * h + j]);
      }
      __syncwarp();
    }
  } else {
    for (int i = warp; i < F; i += nwarps) {
      const size_t row = (size_t)b * F + i;
      const float sp = a.prev_s ? a.prev_s[(size_t)b * a.prev_stride + i] : 0.f;
      const float lse = merge_row<KMAX, 32>(a.part, row, a.S, k, wv[warp], wi[warp]);
      __syncwarp();
      for (int j = lane; j < k; j += 32) keys[i * k + j] = beam_key(sp + (wv[warp][j] - lse), i, wi[warp][j]);
      __syncwarp();
    }
  }
  int P = 32;
  while (P < C) P <<= 1;
  for (int t = C + threadIdx.x; t < P; t += blockDim.x) keys[t] = 0ull;
  __syncthreads();
  // beam: the best `beam` candidates under (score desc, parent position asc, token asc)
  const int kept = min(a.beam, C);
  if (kept <= 32) {
    // every 32-key chunk sorted by a warp, then pairs of chunks merged to their
    // top 32 until one chunk is left (keys are distinct: parent, token)
    for (int c = warp; c < P / 32; c += nwarps)
      keys[32 * c + lane] = warp_sort_desc(keys[32 * c + lane], lane);
    __syncthreads();
    for (int width = 1; width < P / 32; width <<= 1) {
      for (int c = warp * 2 * width; c < P / 32; c += nwarps * 2 * width) {
        if (c + width < P / 32) {
          const unsigned long long x = keys[32 * c + lane], y = keys[32 * (c + width) + 31 - lane];
          keys[32 * c + lane] = warp_merge_top(x, y, lane);
        }
      }
      __syncthreads();
    }
  } else {
    bitonic_desc_block(keys, P);
  }
  // canonical order of the kept: ascending (parent position, token); the beam
  // rank rides along in the low bits to find the score again
  int Q = 1;
  while (Q < kept) Q <<= 1;
  for (int t = threadIdx.x; t < Q; t += blockDim.x) {
    if (t < kept) {
      const unsigned long long x = keys[t];
      const unsigned long long ppos = 1023ull - ((x >> 22) & 1023ull);
      const unsigned long long tok = 0x3fffffull - (x & 0x3fffffull);
      kept_s[t] = ord2f((unsigned)(x >> 32));
      ck[t] = ~((ppos << 42) | (tok << 10) | (unsigned long long)t);   // descending sort -> ascending
    } else {
      ck[t] = 0ull;
    }
  }
  __syncthreads();
  if (Q <= 32) {
    if (warp == 0) {
      const unsigned long long x = lane < Q ? ck[lane] : 0ull;
      const unsigned long long y = warp_sort_desc(x, lane);
      if (lane < Q) ck[lane] = y;
    }
    __syncthreads();
  } else {
    bitonic_desc_block(ck, Q);
  }
  for (int t = threadIdx.x; t < kept; t += blockDim.x) {
    const unsigned long long x = ~ck[t];
    const size_t o = (size_t)b * a.beam + t;
    a.lvl_tok[o] = (int)((x >> 10) & 0x3fffffull);
    a.lvl_ppos[o] = (int)(x >> 42);
    a.lvl_s[o] = kept_s[x & 1023ull];
  }
  if (a.Eg_next == nullptr) return;
  // next depth's Markov operand rows: Eg[b * F_new + pos] = E[token], 16-byte copies
  const int Fn = a.F_new;
  const TE* E = static_cast<const TE*>(a.E);
  TE* Eg = static_cast<TE*>(a.Eg_next);
  constexpr int per16 = 16 / (int)sizeof(TE);
  const bool vec = (a.r % per16 == 0) && (a.r_pad % per16 == 0) &&
                   ((reinterpret_cast<uintptr_t>(E) & 15u) == 0);
  const bool stash = std::is_same<TE, __nv_bfloat16>::value && a.seed.thr != nullptr &&
                     kept <= 32 && a.r_pad <= kSeedMaxR;
  if (vec) {
    const int rv = a.r / per16, rpv = a.r_pad / per16;
    for (int idx = threadIdx.x; idx < kept * rpv; idx += blockDim.x) {
      const int t = idx / rpv, j = idx - t * rpv;
      const unsigned long long x = ~ck[t];
      int tok = (int)((x >> 10) & 0x3fffffull);
      tok = (tok < 0 || tok >= a.V) ? 0 : tok;
      const uint4 val = j < rv ? reinterpret_cast<const uint4*>(E + (size_t)tok * a.r)[j]
                               : make_uint4(0u, 0u, 0u, 0u);
      reinterpret_cast<uint4*>(Eg + ((size_t)b * Fn + t) * a.r_pad)[j] = val;
      if (stash) reinterpret_cast<uint4*>(egs + t * kEgsStride)[j] = val;
    }
  } else {
    for (int idx = threadIdx.x; idx < kept * a.r_pad; idx += blockDim.x) {
      const int t = idx / a.r_pad, j = idx - t * a.r_pad;
      const unsigned long long x = ~ck[t];
      int tok = (int)((x >> 10) & 0x3fffffull);
      tok = (tok < 0 || tok >= a.V) ? 0 : tok;
      Eg[((size_t)b * Fn + t) * a.r_pad + j] = j < a.r ? E[(size_t)tok * a.r + j] : TE(0.f);
    }
  }
  if constexpr (std::is_same<TE, __nv_bfloat16>::value) {
    if (a.seed.thr == nullptr) return;
    // next depth's admission seeds for this request's new parents
    seed_prefetch_wait();   // also orders the Eg rows written above
    if (stash && vec && a.seed.ks <= kSeedMmaCols && a.r_pad % 16 == 0)
      seed_rows_mma(kept, reinterpret_cast<const __nv_bfloat16*>(egs), kEgsStride, &seed_sm,
                    a.seed.ks, a.r_pad, a.seed.thr + (size_t)b * Fn, e1s);
    else if (stash && vec)
      seed_rows<KMAX>(kept, [&](int t) { return reinterpret_cast<const __nv_bfloat16*>(egs + t * kEgsStride); },
                      &seed_sm, a.seed.ks, a.r_pad, a.seed.thr + (size_t)b * Fn);
    else
      seed_rows<KMAX>(kept, [&](int t) { return static_cast<const __nv_bfloat16*>(Eg) + ((size_t)b * Fn + t) * a.r_pad; },
                      &seed_sm, a.seed.ks, a.r_pad, a.seed.thr + (size_t)b * Fn);
  }
}

constexpr int kFinalThreads = 1024;
constexpr int kMaxUnion = 4096;

__global__ __launch_bounds__(kFinalThreads) void final_kernel(FinalArgs a) {
  pdl_wait();
  pdl_trigger();
  __shared__ float us[kMaxUnion];
  __shared__ int oidx[kMaxUnion];
  __shared__ int off[66];
  __shared__ int sbuf[32];
  const int b = blockIdx.x;
  if (threadIdx.x == 0) {
    off[0] = 0;
    for (int d = 1; d <= a.D; ++d) off[d] = off[d - 1] + a.F[d];
  }
  __syncthreads();
  const int U = off[a.D];
  const int keepN = a.N - 1;
  const size_t lvl_stride = (size_t)a.batch * a.beam;
  auto depth_of = [&](int u) {
    int d = 1;
    while (u >= off[d]) ++d;
    return d;
  };
  for (int u = threadIdx.x; u < U; u += blockDim.x) {
    const int d = depth_of(u), pos = u - off[d - 1];
    us[u] = a.lvl_s[(d - 1) * lvl_stride + (size_t)b * a.beam + pos];
  }
  __syncthreads();
  // selection flag: rank under (score desc, depth asc, position asc) < N - 1;
  // the flattened index u is depth-major, so (depth, position) order is u order.
  // The U x U comparisons are spread over every thread: S threads per u, each
  // over a stride-S share of the v (counts added in shared memory)
  constexpr int PER = kMaxUnion / kFinalThreads;
  const bool all_kept = U <= keepN;
  if (!all_kept) {
    for (int u = threadIdx.x; u < U; u += blockDim.x) oidx[u] = 0;
    __syncthreads();
    const int S = max(1, (int)blockDim.x / U);
    for (int task = threadIdx.x; task < U * S; task += blockDim.x) {
      const int u = task % U, part = task / U;
      const float su = us[u];
      int rank = 0;
#pragma unroll 4
      for (int v = part; v < U; v += S) rank += (us[v] > su) || (us[v] == su && v < u);
      if (rank) atomicAdd(&oidx[u], rank);
    }
    __syncthreads();
  }
  int flag[PER];
  int mine = 0;
#pragma unroll
  for (int q = 0; q < PER; ++q) {
    const int u = threadIdx.x * PER + q;
    const int f = u < U && (all_kept || oidx[u] < keepN);
    flag[q] = f;
    mine += f;
  }
  __syncthreads();   // oidx is rewritten below
  // exclusive scan of the per-thread counts (threads own consecutive u)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) sbuf[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = sbuf[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    sbuf[lane] = w;
  }
  __syncthreads();
  int run = (warp > 0 ? sbuf[warp - 1] : 0) + incl - mine;
  const int total = sbuf[31];
#pragma unroll
  for (int q = 0; q < PER; ++q) {
    const int u = threadIdx.x * PER + q;
    if (u < U) oidx[u] = flag[q] ? 1 + run : -1;
    run += flag[q];
  }
  __syncthreads();
  const size_t ob = (size_t)b * a.N;
  int bad = 0;
  for (int u = threadIdx.x; u < U; u += blockDim.x) {
    const int o = oidx[u];
    if (o < 0) continue;
    const int d = depth_of(u), pos = u - off[d - 1];
    const size_t li = (d - 1) * lvl_stride + (size_t)b * a.beam + pos;
    int par = 0;
    if (d > 1) {
      par = oidx[off[d - 2] + a.lvl_ppos[li]];
      if (par < 0) { bad = 1; par = 0; }
    }
    a.tok[ob + o] = a.lvl_tok[li];
    a.parent[ob + o] = par;
    a.depth[ob + o] = d;
    a.score[ob + o] = us[u];
  }
  const int cnt = 1 + total;
  for (int o = cnt + threadIdx.x; o < a.N; o += blockDim.x) {
    a.tok[ob + o] = -1; a.parent[ob + o] = -1; a.depth[ob + o] = -1; a.score[ob + o] = neg_inf();
  }
  if (threadIdx.x == 0) {
    a.tok[ob] = a.anchor[b]; a.parent[ob] = -1; a.depth[ob] = 0; a.score[ob] = 0.f;
    a.count[b] = cnt;
  }
  if (bad) atomicOr(&a.status[b], PCT_DEV_BAD_PARENT);
  if (threadIdx.x == 0 && a.err && *a.err) atomicOr(&a.status[b], PCT_DEV_TIMEOUT);
}

template <int KMAX>
__global__ void rows_finalize_kernel(int rows, int k, int S, Partials part, float* lse_out,
                                     int32_t* top_tok, float* top_logpi, const int32_t* err,
                                     int32_t* status, int n_par) {
  pdl_wait();
  pdl_trigger();
  __shared__ float wv[8][16];
  __shared__ int wi[8][16];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + warp;
  if (row >= rows) return;
  const float lse = merge_row<KMAX, 32>(part, row, S, k, wv[warp], wi[warp]);
  __syncwarp();
  for (int j = lane; j < k; j += 32) {
    top_tok[(size_t)row * k + j] = wi[warp][j];
    top_logpi[(size_t)row * k + j] = wv[warp][j] - lse;
  }
  if (lane == 0) {
    lse_out[row] = lse;
    if (*err) atomicOr(&status[row / n_par], PCT_DEV_TIMEOUT);
  }
}

}  // namespace

cudaError_t launch_gather_rows(int rows, const int32_t* toks, int V, int r, int r_pad,
                               int markov_dtype, const void* E, void* Eg, int32_t* status,
                               int status_div, const SeedArgs& seed, cudaStream_t s) {
  if (seed.thr != nullptr && (status_div != 1 || markov_dtype != PCT_BF16 || seed.ks > kSeedMaxK ||
                              r_pad > kSeedMaxR))
    return cudaErrorInvalidValue;
  TraceScope t(s, "gather_rows");
  if (markov_dtype == PCT_BF16)
    return launch_pdl(gather_rows_kernel<__nv_bfloat16>, dim3(rows), dim3(128), 0, s, 1, rows, toks,
                      V, r, r_pad, static_cast<const __nv_bfloat16*>(E),
                      static_cast<__nv_bfloat16*>(Eg), status, status_div, seed);
  return launch_pdl(gather_rows_kernel<float>, dim3(rows), dim3(128), 0, s, 1, rows, toks, V, r,
                    r_pad, static_cast<const float*>(E), static_cast<float*>(Eg), status,
                    status_div, seed);
}

cudaError_t launch_merge(const MergeArgs& a, cudaStream_t s) {
  if (a.seed.thr != nullptr && (a.seed.ks > kSeedMaxK || a.r_pad > kSeedMaxR ||
                                a.Eg_next == nullptr || a.markov_dtype != PCT_BF16))
    return cudaErrorInvalidValue;
  TraceScope t(s, "pct_merge_beam");
  const bool bf = a.markov_dtype == PCT_BF16;
#define PCT_MERGE(KM)                                                                        \
  (bf ? launch_pdl(merge_kernel<KM, __nv_bfloat16>, dim3(a.batch), dim3(kMergeThreads), 0, s, 1, a) \
      : launch_pdl(merge_kernel<KM, float>, dim3(a.batch), dim3(kMergeThreads), 0, s, 1, a))
  if (a.k <= 4) return PCT_MERGE(4);
  if (a.k <= 8) return PCT_MERGE(8);
  return PCT_MERGE(16);
#undef PCT_MERGE
}

cudaError_t launch_final(const FinalArgs& a, cudaStream_t s) {
  TraceScope t(s, "pct_global_topn");
  return launch_pdl(final_kernel, dim3(a.batch), dim3(kFinalThreads), 0, s, 1, a);
}

cudaError_t launch_rows_finalize(int rows, int k, int S, Partials part, float* lse,
                                 int32_t* top_tok, float* top_logpi, const int32_t* err,
                                 int32_t* status, int n_par, cudaStream_t s) {
  TraceScope t(s, "pct_rows_finalize");
  const dim3 grid((rows + 7) / 8);
  if (k <= 4)
    return launch_pdl(rows_finalize_kernel<4>, grid, dim3(256), 0, s, 1, rows, k, S, part, lse,
                      top_tok, top_logpi, err, status, n_par);
  if (k <= 8)
    return launch_pdl(rows_finalize_kernel<8>, grid, dim3(256), 0, s, 1, rows, k, S, part, lse,
                      top_tok, top_logpi, err, status, n_par);
  return launch_pdl(rows_finalize_kernel<16>, grid, dim3(256), 0, s, 1, rows, k, S, part, lse,
                    top_tok, top_logpi, err, status, n_par);
}

}  // namespace pct
