// Host-side interfaces between the translation units of libpctree.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/pctree.h"

namespace pct {

// ---- kernel trace (api.cu) ------------------------------------------------
// Brackets one launch with events when the trace is on. Usage:
//   { TraceScope t(stream, "name"); kernel<<<...>>>(...); }
struct TraceScope {
  TraceScope(cudaStream_t s, const char* name);
  ~TraceScope();
  cudaStream_t stream;
  int slot;
};

// ---- device queries (api.cu) ----------------------------------------------
int num_sms();          // SMs of the current device (cached per device)
bool device_ok();       // compute capability 10.x

// ---- auxiliary stream (api.cu) -----------------------------------------------
// A second stream of the current device and context (created on first use,
// kept for the process) with two events, for work inside one call that does
// not depend on the caller's stream's next kernel: record `fork` on the
// caller's stream, make `s` wait for it, launch there, record `join` on `s`,
// make the caller's stream wait for it, all under `mu` (calls from several
// host threads share the stream and events). A graph capture of the caller's
// stream takes the forked work in as a branch.
struct AuxStream {
  cudaStream_t s;
  cudaEvent_t fork, join;
  void* mu;   // std::mutex*
};
int aux_stream(AuxStream* out);   // PCT_OK or an error code
void aux_lock(const AuxStream& a);
void aux_unlock(const AuxStream& a);

// ---- verify.cu --------------------------------------------------------------
cudaError_t launch_ancestor_mask(int batch, int n_stride, const int32_t* parent,
                                 const int32_t* count, uint32_t* mask, int32_t* status,
                                 cudaStream_t s);
cudaError_t launch_verify(int batch, int n_stride, int vocab, int max_depth, const int32_t* tok,
                          const int32_t* parent, const int32_t* count, const void* target,
                          int dtype, int32_t* argmax, int32_t* alen, int32_t* apath,
                          int32_t* corr, int32_t* status, unsigned* arrive, cudaStream_t s);

// Lazy walk: argmax only of the rows the walk reaches (no workspace).
cudaError_t launch_verify_walk(int batch, int n_stride, int vocab, int max_depth,
                               const int32_t* tok, const int32_t* parent, const int32_t* count,
                               const void* target, int dtype, int32_t* argmax, int32_t* alen,
                               int32_t* apath, int32_t* corr, int32_t* status, cudaStream_t s);

// ---- accept_sim.cu ----------------------------------------------------------
size_t accept_sim_smem(int n_stride, int max_depth);
cudaError_t launch_accept_sim(int batch, int n_stride, int max_depth, const int32_t* parent,
                              const int32_t* count, const float* p_child, long long trials,
                              unsigned long long seed, unsigned long long* hist, int32_t* status,
                              cudaStream_t s);

// ---- cadd.cu ----------------------------------------------------------------
struct CaddParams {
  int batch, D, V, n_max, dtype;
  float C_d, a, b, c, e;
  int top_k;                      // > 0: each row's top_k tokens into top_tok [rows][top_k]
  int32_t* top_tok;
  int32_t* top_list;              // [rows] rows the row pass left to the exact selection
  unsigned* top_list_n;           // their number
  unsigned* top_cnt;              // [rows] part counters of the exact selection
  unsigned long long* top_keys;   // [rows][parts][32] the parts' lists
};
// Workspace of the top_k output (cadd_tree_grow_topk): top_list, top_cnt and
// top_list_n, top_keys for `rows` rows, 256-byte aligned pieces.
size_t cadd_topk_workspace(size_t rows);
size_t cadd_rowpass_bytes_per_row(int n_max);
// Workspace of the segmented row pass (bf16 rows with V % 8 == 0; else 0).
size_t cadd_seg_workspace(int batch, int D, int V, int dtype);
cudaError_t launch_cadd(const CaddParams& p, const void* L, const int32_t* anchor,
                        const int64_t* ctx, int32_t* tok, int32_t* parent, int32_t* depth,
                        float* score, int32_t* count, float* phi, int32_t* status,
                        float* row_lse, int32_t* cand_cnt, float* cand_q, int32_t* cand_tok,
                        void* seg_ws, void* topk_ws, cudaStream_t s);

// ---- PCTree (pct_*.cu) ------------------------------------------------------
// Partial results of one (row, V-slice): online log-sum-exp state and the
// slice's top-k (value desc, token asc).
struct Partials {
  float2* ms;      // [rows][S]    (max, sum exp(z - max))
  float* val;      // [rows][S][k] z values
  int32_t* idx;    // [rows][S][k] token ids
};

// One depth of batched parent scoring: rows = n_req * n_par; row r belongs
// to request r / n_par and its parent embedding row is Eg[r].
struct ScoreArgs {
  int n_req, n_par, V, r, r_pad, k;
  int logits_dtype, markov_dtype;
  const void* L;          // logits base for request 0
  long long L_req_stride; // elements between consecutive requests' rows
  const void* Eg;         // [M_pad][r_pad] (bf16) or [M_pad][r] (f32)
  int M_pad;
  const void* W;          // [r][V]
  const void* Wt;         // null, or W transposed [V][r_pad] (bf16): read instead of W
  Partials part;
  int S;                  // V-slices (partials per row)
  int32_t* err;           // device word, set on a timed-out wait
  uint32_t* row_thr;      // [rows] best known lower bound of each row's k-th value
                          // (ordered key, 0 = none)
  bool thr_seeded;        // row_thr holds seeds; otherwise launch_score clears it
};
// Slices the scoring kernel will use for `rows` rows (deterministic per device).
int score_slices(int rows, int V, int markov_dtype);
cudaError_t launch_score(const ScoreArgs& a, cudaStream_t s);

// Admission seeds of the next scoring launch (seed.cuh). Seed data of the
// (request b, depth) entry in use: cols/lval/wmax + b * req_stride [ks] and
// wcol + b * req_stride * r_pad [ks][r_pad]. Null thr: no seeds.
struct SeedArgs {
  const int32_t* cols;
  const float* lval;
  const float* wmax;
  const void* wcol;        // bf16
  long long req_stride;
  int ks;
  uint32_t* thr;
};

// Gather E rows of tokens into Eg (zero padded to r_pad for bf16); with
// seeds, one row per request (status_div == 1).
cudaError_t launch_gather_rows(int rows, const int32_t* toks, int V, int r, int r_pad,
                               int markov_dtype, const void* E, void* Eg, int32_t* status,
                               int status_div, const SeedArgs& seed, cudaStream_t s);

// Non-negative least-squares fit of C_v(n; l) = a + b l + c n + e n^2 to m
// samples: out = (a, b, c, e, rms), device float64 [5] (cost_fit.cu).
cudaError_t launch_cost_fit(long long m, const float* n, const float* ell, const float* lat,
                            double* out, int32_t* status, cudaStream_t s);

// Seed data for every row of the logits [rows][V] (V % 8 == 0, bf16 W [r][V]):
// the ks best columns (approximately), L at them, W's columns (bf16, zero
// padded to r_pad) and their largest magnitude. scratch: drafter_topk_scratch
// bytes (256-byte aligned), any contents.
size_t drafter_topk_scratch(int rows);
cudaError_t launch_drafter_topk(int rows, int V, int ks, int logits_dtype, const void* L,
                                const void* W, int r, int r_pad, int32_t* cols, float* lval,
                                float* wmax, void* wcol, void* scratch, cudaStream_t s);

// Seed data for every row of the logits from caller-given columns in[rows][ks]
// (dropped: entries outside [0, V) and repeats within a row); the same
// outputs as launch_drafter_topk.
// Wt: null, or W transposed [V][r_pad] (launch_markov_transpose), read instead of W.
cudaError_t launch_seed_columns(int rows, int V, int ks, int logits_dtype, const void* L,
                                const void* W, const void* Wt, int r, int r_pad,
                                const int32_t* in, int32_t* cols, float* lval, float* wmax,
                                void* wcol, cudaStream_t s);
// Wt [V][r_pad] = W [r][V] transposed (bf16, zero past r; V % 8 == 0).
cudaError_t launch_markov_transpose(int V, int r, int r_pad, const void* W, void* Wt,
                                    cudaStream_t s);

struct MergeArgs {
  int batch, F_prev, F_new, k, beam, S, V, r, r_pad, markov_dtype, depth;
  Partials part;
  const int32_t* prev_tok;   // [batch][F_prev] (depth 1: anchors, stride 1)
  const float* prev_s;       // [batch][F_prev] (depth 1: null -> 0)
  int prev_stride;           // elements between requests in prev arrays
  int32_t* lvl_tok;          // [batch][beam] this depth
  int32_t* lvl_ppos;
  float* lvl_s;
  const void* E;
  void* Eg_next;             // null at the last depth
  const int32_t* err;
  int32_t* status;
  SeedArgs seed;             // next depth's seeds (thr null: none)
};
cudaError_t launch_merge(const MergeArgs& a, cudaStream_t s);

// PCTree in one persistent launch for small frontiers (pct_chain.cu): bf16
// logits and Markov parameters, at most 16 requests and 128 parent rows per
// depth, beam <= 32. The level arrays are those launch_final reads.
struct ChainShape {
  int batch, D, V, r, r_pad, k, beam, logits_dtype, markov_dtype;
};
bool chain_eligible(const ChainShape& c);           // shape and current device
size_t chain_workspace(const ChainShape& c);
// Seeds: [batch][D][k] columns, L_d and max|W| there, W's columns [..][r_pad]
// (launch_drafter_topk's output).
cudaError_t launch_chain(const ChainShape& c, const void* L, const int32_t* anchor, const void* E,
                         const void* W, void* ws, int32_t* lvl_tok, int32_t* lvl_ppos, float* lvl_s,
                         int32_t** err_out, int32_t* status, const int32_t* scol,
                         const float* slval, const float* swmax, const void* swcol,
                         cudaStream_t s);

struct FinalArgs {
  int batch, D, beam, N;
  int F[65];                 // F[d] for d = 1..D
  const int32_t* anchor;
  const int32_t* lvl_tok;    // [D][batch][beam]
  const int32_t* lvl_ppos;
  const float* lvl_s;
  int32_t *tok, *parent, *depth, *count;
  float* score;
  int32_t* status;
  const int32_t* err;        // optional: nonzero -> PCT_DEV_TIMEOUT for every request
};
cudaError_t launch_final(const FinalArgs& a, cudaStream_t s);

// pct_score_parents: per-row merge of partials into lse + top-k.
cudaError_t launch_rows_finalize(int rows, int k, int S, Partials part, float* lse,
                                 int32_t* top_tok, float* top_logpi, const int32_t* err,
                                 int32_t* status, int n_par, cudaStream_t s);

}  // namespace pct
