// Admission seeds for the scoring kernel's top-k (PCTree parent scoring).
//
// PCTree article (qiita), section on the tree that replaces the chain draft:
// every frontier parent p keeps the k largest z_d(p) = L_d + Markov(p). The
// scoring kernel admits a value to its running top-k only at or above a gate,
// and any k actual values of the row bound the row's k-th largest from below.
// The seed evaluates z exactly at k columns that are likely to be near the top
// (the request's best drafter-logit columns of that depth, shared by all of its
// parents) and stores their minimum, less a rounding allowance that covers the
// difference between this fp32 dot product and the tensor-core accumulation of
// the same sum, as the row's starting gate. A loose seed only costs speed; it
// never excludes a value that belongs to the row's top-k.
#pragma once

#include "common.cuh"

namespace pct {

// Rounding allowance relative to |L| + sum_j |E_j W_j|: two fp32 sums of the
// same r <= 256 exact bf16 products (in any order, rounded or truncated) differ
// by at most about (r + 2) * 2^-23 of that magnitude, below 2^-14; the
// allowance is 2^-12. sum_j |E_j W_j| is bounded by sum_j |E_j| * max_j |W_j|.
constexpr float kSeedSlack = 1.0f / 4096.0f;
constexpr int kSeedMaxK = 16;
constexpr int kSeedMaxR = 256;

// Per (request, depth) seed data, written by the drafter top-k kernel:
//   cols [ks]            seed columns (distinct; any entry < 0: no seed)
//   lval [ks]            L_d at those columns
//   wmax [ks]            max_j |W[j][col]|
//   wcol [ks][r_pad]     W[.][col] as bf16, zero padded past r
struct SeedData {
  const int32_t* cols;
  const float* lval;
  const float* wmax;
  const __nv_bfloat16* wcol;
};

// Shared-memory copy of one (request, depth) seed entry.
struct SeedSmem {
  __nv_bfloat16 wcol[kSeedMaxK * kSeedMaxR];   // first: 16-byte aligned
  int32_t cols[kSeedMaxK];
  float lval[kSeedMaxK];
  float wmax[kSeedMaxK];
};

// Copies one seed entry (W columns: ks * r_pad bf16, 16-byte aligned) into
// shared memory with asynchronous copies, so that their latency overlaps the
// caller's other work; the caller waits with seed_prefetch_wait() before
// seed_rows().
__device__ __forceinline__ void seed_prefetch(const SeedData& sd, int ks, int r_pad,
                                              SeedSmem* sm) {
  const int n16 = ks * r_pad / 8;
  for (int i = threadIdx.x; i < n16; i += blockDim.x) {
    const uint32_t dst = static_cast<uint32_t>(__cvta_generic_to_shared(sm->wcol + 8 * i));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(sd.wcol + 8 * i)
                 : "memory");
  }
  for (int i = threadIdx.x; i < 3 * ks; i += blockDim.x) {
    const int w = i / ks, c = i - w * ks;
    const void* src = w == 0 ? static_cast<const void*>(sd.cols + c)
                             : w == 1 ? static_cast<const void*>(sd.lval + c)
                                      : static_cast<const void*>(sd.wmax + c);
    void* dstp = w == 0 ? static_cast<void*>(sm->cols + c)
                        : w == 1 ? static_cast<void*>(sm->lval + c) : static_cast<void*>(sm->wmax + c);
    const uint32_t dst = static_cast<uint32_t>(__cvta_generic_to_shared(dstp));
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void seed_prefetch_wait() {
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();
}

// One warp per row: rows t < nrows of one request, parent embedding rows
// eg_row(t) (bf16, r_pad wide, zero padded, 16-byte aligned) written by this
// block before a __syncthreads. sm holds the seed entry (seed_prefetch).
// Writes thr[t] = ordered key of the row's bound, 0 when there is none.
// KS bounds ks at compile time (the unrolled per-column work).
template <int KS = kSeedMaxK, typename EgFn>
__device__ __forceinline__ void seed_rows(int nrows, EgFn eg_row, const SeedSmem* sm, int ks,
                                          int r_pad, uint32_t* __restrict__ thr) {
  static_assert(KS <= kSeedMaxK, "seed columns");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const __nv_bfloat16* ws = sm->wcol;
  bool usable = true;
#pragma unroll
  for (int c = 0; c < KS; ++c) usable &= (c >= ks) || sm->cols[c] >= 0;
  for (int t = warp; t < nrows; t += nw) {
    const int j0 = 8 * lane;
    float e[8];
    if (j0 < r_pad) {
      const uint4 w = *reinterpret_cast<const uint4*>(eg_row(t) + j0);
      e[0] = bf16_lo(w.x); e[1] = bf16_hi(w.x); e[2] = bf16_lo(w.y); e[3] = bf16_hi(w.y);
      e[4] = bf16_lo(w.z); e[5] = bf16_hi(w.z); e[6] = bf16_lo(w.w); e[7] = bf16_hi(w.w);
    } else {
#pragma unroll
      for (int q = 0; q < 8; ++q) e[q] = 0.f;
    }
    float e1 = 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q) e1 += fabsf(e[q]);
    float d[KS];
#pragma unroll
    for (int c = 0; c < KS; ++c) {
      d[c] = 0.f;
      if (c < ks && j0 < r_pad) {
        const uint4 w = *reinterpret_cast<const uint4*>(ws + c * r_pad + j0);
        d[c] = fmaf(e[0], bf16_lo(w.x), d[c]); d[c] = fmaf(e[1], bf16_hi(w.x), d[c]);
        d[c] = fmaf(e[2], bf16_lo(w.y), d[c]); d[c] = fmaf(e[3], bf16_hi(w.y), d[c]);
        d[c] = fmaf(e[4], bf16_lo(w.z), d[c]); d[c] = fmaf(e[5], bf16_hi(w.z), d[c]);
        d[c] = fmaf(e[6], bf16_lo(w.w), d[c]); d[c] = fmaf(e[7], bf16_hi(w.w), d[c]);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      e1 += __shfl_xor_sync(0xffffffffu, e1, o);
#pragma unroll
      for (int c = 0; c < KS; ++c)
        if (c < ks) d[c] += __shfl_xor_sync(0xffffffffu, d[c], o);
    }
    float lo_min = __int_as_float(0x7f800000);
    bool finite = usable;
#pragma unroll
    for (int c = 0; c < KS; ++c) {
      if (c < ks) {
        const float l = sm->lval[c];
        const float lo = (l + d[c]) - (fabsf(l) + e1 * sm->wmax[c]) * kSeedSlack;
        finite = finite && (lo == lo) && lo != __int_as_float(0x7f800000);
        lo_min = fminf(lo_min, lo);
      }
    }
    if (lane == 0) thr[t] = (finite && lo_min > neg_inf()) ? f2ord(lo_min) : 0u;
  }
}

// The same bounds for up to 32 rows and ks <= 8 columns at once, for the merge
// kernel (the rows are a request's new parents). The products E_t . W[:, c]
// form a [32 x r_pad] x [r_pad x 8] matrix product, done with mma.sync
// m16n8k16 (bf16 operands, fp32 accumulation) by warps 0 and 1, one 16-row
// half each: far too small for the tcgen05 path's set-up to pay. The slack
// covers any accumulation order, so the bound is the one seed_rows computes.
// eg: shared memory, row t at eg + t * eg_stride (eg_stride >= r_pad, a
// multiple of 8; rows nrows..31 may hold anything); r_pad % 16 == 0;
// e1s: 32 floats of shared memory. Every thread of the block calls it.
constexpr int kSeedMmaRows = 32;
constexpr int kSeedMmaCols = 8;
__device__ __forceinline__ uint32_t seed_lds32(const __nv_bfloat16* p) {
  return *reinterpret_cast<const uint32_t*>(p);
}
__device__ __forceinline__ void seed_rows_mma(int nrows, const __nv_bfloat16* eg, int eg_stride, const SeedSmem* sm,
                              int ks, int r_pad, uint32_t* __restrict__ thr, float* e1s) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  // sum_j |E_tj| per row: one warp per row at a time, 8 values per lane
  for (int t = warp; t < nrows; t += nw) {
    float e1 = 0.f;
    for (int j0 = 8 * lane; j0 < r_pad; j0 += 256) {
      const uint4 w = *reinterpret_cast<const uint4*>(eg + t * eg_stride + j0);
      e1 += fabsf(bf16_lo(w.x)) + fabsf(bf16_hi(w.x)) + fabsf(bf16_lo(w.y)) + fabsf(bf16_hi(w.y)) +
            fabsf(bf16_lo(w.z)) + fabsf(bf16_hi(w.z)) + fabsf(bf16_lo(w.w)) + fabsf(bf16_hi(w.w));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) e1 += __shfl_xor_sync(0xffffffffu, e1, o);
    if (lane == 0) e1s[t] = e1;
  }
  __syncthreads();
  if (warp >= 2) return;
  // D = A . B with A = rows 16 * warp .. +15 of eg and B[k][n] = W[k][col n]
  // (the seed columns, stored n-major: a column-major B fragment)
  const int g = lane >> 2, q = lane & 3;
  const __nv_bfloat16* a_lo = eg + (16 * warp + g) * eg_stride + 2 * q;
  const __nv_bfloat16* a_hi = a_lo + 8 * eg_stride;
  const __nv_bfloat16* bcol = sm->wcol + g * r_pad + 2 * q;   // column g (zero where g >= ks)
  float c0 = 0.f, c1 = 0.f, c2 = 0.f, c3 = 0.f;
#pragma unroll 4
  for (int k0 = 0; k0 < r_pad; k0 += 16) {
    const uint32_t a0 = seed_lds32(a_lo + k0), a1 = seed_lds32(a_hi + k0);
    const uint32_t a2 = seed_lds32(a_lo + k0 + 8), a3 = seed_lds32(a_hi + k0 + 8);
    const uint32_t b0 = g < ks ? seed_lds32(bcol + k0) : 0u;
    const uint32_t b1 = g < ks ? seed_lds32(bcol + k0 + 8) : 0u;
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c0), "+f"(c1), "+f"(c2), "+f"(c3)
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  }
  // lane (g, q) holds rows 16w + g (c0, c1) and 16w + g + 8 (c2, c3), columns
  // 2q and 2q + 1; the row's minimum over columns is across the quad
  bool usable = true;
#pragma unroll
  for (int c = 0; c < kSeedMmaCols; ++c) usable &= (c >= ks) || sm->cols[c] >= 0;
  const float d[4] = {c0, c1, c2, c3};
  float lo_min[2] = {__int_as_float(0x7f800000), __int_as_float(0x7f800000)};
  bool fin[2] = {usable, usable};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int hrow = i >> 1, c = 2 * q + (i & 1);
    const int t = 16 * warp + g + 8 * hrow;
    if (c < ks && t < nrows) {
      const float l = sm->lval[c];
      const float lo = (l + d[i]) - (fabsf(l) + e1s[t] * sm->wmax[c]) * kSeedSlack;
      fin[hrow] = fin[hrow] && (lo == lo) && lo != __int_as_float(0x7f800000);
      lo_min[hrow] = fminf(lo_min[hrow], lo);
    }
  }
#pragma unroll
  for (int hrow = 0; hrow < 2; ++hrow) {
#pragma unroll
    for (int o = 1; o < 4; o <<= 1) {
      lo_min[hrow] = fminf(lo_min[hrow], __shfl_xor_sync(0xffffffffu, lo_min[hrow], o));
      fin[hrow] = __shfl_xor_sync(0xffffffffu, (int)fin[hrow], o) && fin[hrow];
    }
    const int t = 16 * warp + g + 8 * hrow;
    if (q == 0 && t < nrows)
      thr[t] = (fin[hrow] && lo_min[hrow] > neg_inf()) ? f2ord(lo_min[hrow]) : 0u;
  }
}

}  // namespace pct
