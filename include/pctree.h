/*
 * pctree.h -- C ABI of the draft-tree hot path (libpctree.so, sm_100a).
 *
 * One round of tree-based speculative decoding on one GPU:
 *   pct_tree_build      parent-conditioned drafting tree (PCTree)
 *   pct_tree_build_seeded   the same, with each row's gate seeded by given columns
 *   pct_markov_transpose    W transposed once per model, for the seeded build
 *   cadd_tree_grow      cost-aware best-first tree (CaDDTree)
 *   cadd_tree_grow_topk the same, plus each logits row's top-k tokens
 *   tree_ancestor_mask  self-plus-ancestor bitmask for tree attention
 *   tree_verify_accept  greedy verification: argmax, accept walk, correction
 *   pct_score_parents   one depth of PCTree's batched parent scoring
 *
 * Conventions shared by every call
 * --------------------------------
 * - Every data pointer is DEVICE memory owned by the caller (allocated and
 *   freed by the caller; the library never allocates device memory). Arrays are
 *   dense, row-major, in the layouts given per argument.
 * - Calls are asynchronous on `cuda_stream` (a cudaStream_t passed as void*;
 *   NULL means the legacy default stream). No host synchronisation happens
 *   inside a call, so a call can be captured in a CUDA graph. The library keeps
 *   no state between calls (apart from the optional kernel trace below) and is
 *   re-entrant; two calls may share a workspace only if they are ordered.
 * - Workspace: calls that need scratch memory take `workspace` / `ws_bytes`;
 *   the size comes from the matching *_workspace() query, evaluated for the
 *   current device. The workspace must be 256-byte aligned. Its contents on
 *   entry are irrelevant and on exit unspecified.
 * - Return value: PCT_OK, or an error detected on the host BEFORE anything is
 *   launched (PCT_EINVAL, PCT_EWORKSPACE, PCT_EUNSUPPORTED, PCT_EDEVICE), or
 *   PCT_ECUDA when a launch fails. Data errors found on the device are written
 *   to the caller's per-request `dev_status` word (bits PCT_DEV_*; 0 = fine);
 *   other requests still complete. There is no device trap, assert or
 *   unbounded wait; a bounded wait that gives up sets PCT_DEV_TIMEOUT.
 * - Node tables (tok, parent, depth, score), per request, slot 0 is the root:
 *   tok = anchor, parent = -1, depth = 0, score = 0. Nodes are in canonical
 *   BFS order: by depth, then by (parent index, token); parent[i] < i. Slots at
 *   or past `count` hold tok = -1, parent = -1, depth = -1, score = -inf.
 * - Total order used by every selection: higher score first, then lower depth,
 *   then the lexicographically smaller token path (siblings: lower token id).
 * - dtypes: PCT_F32 = IEEE binary32, PCT_BF16 = bfloat16 (upper half of a
 *   binary32). Arithmetic is fp32 throughout (bf16 inputs are widened exactly).
 */
#ifndef PCTREE_H
#define PCTREE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Host return codes. */
enum {
  PCT_OK = 0,
  PCT_EINVAL = 1,        /* bad argument or shape; nothing launched            */
  PCT_EWORKSPACE = 2,    /* workspace NULL, misaligned or smaller than needed   */
  PCT_ECUDA = 3,         /* a CUDA runtime/driver call or a launch failed       */
  PCT_EDEVICE = 4,       /* current device is not compute capability 10.x       */
  PCT_ETIMEOUT = 5,      /* reserved for host-visible timeouts                  */
  PCT_EUNSUPPORTED = 6   /* valid combination outside this build's limits       */
};

/* Element types. */
enum { PCT_F32 = 0, PCT_BF16 = 1 };

/* Device status bits, OR-ed into dev_status[request]. */
enum {
  PCT_DEV_BAD_PARENT = 1,     /* parent[i] not in [0, i) for 0 < i < count, or parent[0] != -1 */
  PCT_DEV_BAD_TOKEN = 2,      /* a token or anchor outside [0, vocab)                         */
  PCT_DEV_BAD_COUNT = 4,      /* count outside [1, n_stride]                                  */
  PCT_DEV_DEPTH_OVERFLOW = 8, /* accept walk longer than max_depth                            */
  PCT_DEV_BAD_COST = 16,      /* CaDDTree cost C(n) <= 0 for some n in [1, n_max]             */
  PCT_DEV_TIMEOUT = 32        /* a bounded device wait gave up                                */
};

/* ------------------------------------------------------------------------ *
 * PCTree: parent-conditioned drafting tree.
 * Source: PCTree article (qiita), section on the chain draft's weakness and
 * the tree built in its place: for every frontier parent p at depth d the
 * drafter's logits are z_d(p) = L_d + Markov(p), all parents scored in one
 * batched Markov call; each parent keeps its local top-k children; candidates
 * are ranked by s(c) = sum log pi(v|u) along the path; each depth is pruned to
 * a beam; a global top-N fits the verification budget.
 * Here Markov(p) = E[p] . W, a rank-r stand-in for the drafter's head,
 * pi(.|u) = softmax over the vocabulary of z_d(u), s(root) = 0, depth 1 is
 * conditioned on the anchor, and the block has D = B - 1 drafted depths.
 * ------------------------------------------------------------------------ */
typedef struct {
  int32_t batch;        /* independent requests, >= 1                          */
  int32_t depth;        /* D, drafted depths (block size B = D + 1), 1..64      */
  int32_t vocab;        /* V, k..4194304 (2^22)                                  */
  int32_t rank;         /* r of E [V][r] and W [r][V], 1..256                   */
  int32_t k;            /* local top-k children per parent, 1..16              */
  int32_t beam;         /* frontier width kept per depth, 1..256, beam*k <= 1024 */
  int32_t n_nodes;      /* N, tree budget including the root, 1..4096;
                           depth * beam <= 4096                                 */
  int32_t logits_dtype; /* PCT_F32 or PCT_BF16, for L                           */
  int32_t markov_dtype; /* PCT_F32 or PCT_BF16, for E and W. BF16 runs on the
                           tcgen05 tensor cores and needs vocab % 8 == 0 (16-byte
                           rows for TMA); F32 runs on the FP32 pipes.           */
} pct_build_desc;

/* Workspace bytes pct_tree_build needs for `desc` on the current device;
 * 0 when desc is invalid. */
size_t pct_tree_build_workspace(const pct_build_desc* desc);

/* Build one PCTree per request.
 *   L          [batch][D][V] logits_dtype  drafter logits; row d-1 serves depth d
 *   anchor     [batch] int32               depth-0 token of each block
 *   E          [V][r] markov_dtype,  W [r][V] markov_dtype
 *   tok, parent, depth  [batch][N] int32;  score [batch][N] float (path log-prob)
 *   count      [batch] int32   nodes written, min(N, 1 + sum_d |F_d|)
 *   dev_status [batch] int32   0 or PCT_DEV_* bits
 * Ties between exactly equal scores follow the total order above. */
int32_t pct_tree_build(const pct_build_desc* desc, const void* L, const int32_t* anchor,
                       const void* E, const void* W, int32_t* tok, int32_t* parent,
                       int32_t* depth, float* score, int32_t* count, int32_t* dev_status,
                       void* workspace, size_t ws_bytes, void* cuda_stream);

/* pct_tree_build with the columns that seed each row's top-k gate given by
 * the caller instead of found by a pass over L (the tensor-core path keeps a
 * parent's value at or above a gate taken from the exact values at k columns
 * of the row; any columns give a valid gate, large L_d columns a tight one).
 *   Wt       NULL, or [V][r_pad] bf16: W transposed by pct_markov_transpose;
 *            with it each seed's W column is one contiguous read instead of r
 *            scattered ones (markov_dtype PCT_BF16, 16-byte aligned)
 *   seed_tok [batch][D][k] int32  columns for row d-1 of request b; entries
 *            outside [0, V) and repeats within a row are ignored (-1 = none)
 * The result is identical to pct_tree_build's whatever the seeds; only the
 * speed depends on them. With markov_dtype PCT_F32 the seeds are unused.
 * Same workspace as pct_tree_build. PCT_EINVAL when seed_tok is NULL. A use:
 * the top-k tokens cadd_tree_grow_topk writes for the same L (one pass over L
 * then serves both trees). */
int32_t pct_tree_build_seeded(const pct_build_desc* desc, const void* L, const int32_t* anchor,
                              const void* E, const void* W, const void* Wt,
                              const int32_t* seed_tok, int32_t* tok, int32_t* parent,
                              int32_t* depth, float* score, int32_t* count, int32_t* dev_status,
                              void* workspace, size_t ws_bytes, void* cuda_stream);

/* r_pad of a Markov rank: rank rounded up to a multiple of 64 (0 if rank is
 * outside 1..256). */
int32_t pct_markov_rank_pad(int32_t rank);

/* Wt [vocab][r_pad] bf16 = W [rank][vocab] bf16 transposed, zero in columns
 * rank..r_pad-1 (r_pad = pct_markov_rank_pad(rank)). W is a model constant,
 * so this runs once per model, not per round; the caller owns Wt
 * (vocab * r_pad * 2 bytes, 16-byte aligned). vocab % 8 == 0, <= 2^22. */
int32_t pct_markov_transpose(int32_t vocab, int32_t rank, const void* W, void* Wt,
                             void* cuda_stream);

/* One depth of PCTree's batched parent scoring (the step inside
 * pct_tree_build before the beam): for request b and each of its n_par
 * parents p with token parent_tok[b][p],
 *   z = L_row[b] + E[parent_tok] . W,  lse = log sum_v exp z,
 *   top_tok[b][p][j], top_logpi[b][p][j] = the k best (z desc, token asc)
 *   children and their log pi = z - lse.
 * Uses desc->vocab, rank, k, logits_dtype, markov_dtype; desc->batch is the
 * number of requests and n_par <= 1024 the parents per request.
 *   L_row [batch][V], parent_tok [batch][n_par] int32, lse [batch][n_par] float,
 *   top_tok [batch][n_par][k] int32, top_logpi [batch][n_par][k] float. */
size_t pct_score_parents_workspace(const pct_build_desc* desc, int32_t n_par);
int32_t pct_score_parents(const pct_build_desc* desc, int32_t n_par, const void* L_row,
                          const int32_t* parent_tok, const void* E, const void* W,
                          float* lse, int32_t* top_tok, float* top_logpi,
                          int32_t* dev_status, void* workspace, size_t ws_bytes,
                          void* cuda_stream);

/* ------------------------------------------------------------------------ *
 * CaDDTree: cost-aware best-first draft tree.
 * Source: "Cost-Aware Diffusion Draft Trees for Speculative Decoding"
 * (gist.science summary), technical summary, "Method: CaDDTree": a round
 * costs C(T; l) = C_d + C_v(|T|; l); the tree maximises (1 + Phi(T)) / C;
 * for a fixed size the best tree is greedy best-first by prefix probability;
 * with convex C_v the objective is unimodal, so nodes are added one at a time
 * until the marginal gain is non-positive.
 * Here q_d = softmax(L_d) are per-position marginals, a node's prefix
 * probability is prod_j q_j(v_j), Phi(T) sums it over non-root nodes, |T|
 * counts the root, C_v(n; l) = a + b l + c n + e n^2, and growth stops at the
 * first n with f(n + 1) <= f(n), f(n) = (1 + Phi_n) / C(n), at n = n_max, or
 * when no candidate is left.
 * ------------------------------------------------------------------------ */
typedef struct {
  int32_t batch;        /* requests, >= 1                                   */
  int32_t depth;        /* D, 1..63                                         */
  int32_t vocab;        /* V, 1..2^24                                       */
  int32_t n_max;        /* node cap including the root, 1..1024             */
  int32_t logits_dtype; /* PCT_F32 or PCT_BF16                              */
  float C_d;            /* draft cost                                       */
  float a, b, c, e;     /* C_v coefficients; c >= 0 and e >= 0 (convex)     */
} cadd_desc;

size_t cadd_tree_grow_workspace(const cadd_desc* desc);

/* Grow one CaDDTree per request.
 *   L       [batch][D][V] logits_dtype   marginal logits, row d-1 for depth d
 *   anchor  [batch] int32;  ctx_len [batch] int64 (context length l)
 *   tok, parent, depth [batch][n_max] int32; score [batch][n_max] float (log prefix prob)
 *   count   [batch] int32  n*;  phi [batch] float  Phi(T)
 *   dev_status [batch] int32
 * Fixed-budget (DDTree) trees: c = e = 0 with C_d + a + b l > 0 makes
 * dC(n) = 0, so the stop never fires and every request grows to n_max nodes,
 * or until its candidates run out. Since growth is best-first, Phi_n for every
 * n is then the sum of the n - 1 largest exp(score). */
int32_t cadd_tree_grow(const cadd_desc* desc, const void* L, const int32_t* anchor,
                       const int64_t* ctx_len, int32_t* tok, int32_t* parent, int32_t* depth,
                       float* score, int32_t* count, float* phi, int32_t* dev_status,
                       void* workspace, size_t ws_bytes, void* cuda_stream);

/* cadd_tree_grow, and in the same pass over L each row's top_k tokens:
 *   top_k    1..32
 *   top_tok  [batch][D][top_k] int32  the top_k largest logits of row d-1 of
 *            request b, value descending, ties to the lower token id; -1 past V.
 * The row pass already keeps every value above the row's CaDDTree threshold,
 * sorted, and writes the head of that list; only rows with fewer than top_k
 * such values are read again, by one more kernel that selects their top_k
 * exactly. That kernel runs beside the best-first growth on a second stream
 * the library keeps per device (forked from and joined back into cuda_stream
 * with events inside the call, so the call stays ordered on cuda_stream and
 * can be captured in a graph; the stream is created by the first call in a
 * context, which should come before any capture). Values order as IEEE floats except that -0.0 ranks below +0.0.
 * Same workspace as cadd_tree_grow. PCT_EINVAL when top_k is outside 1..32 or
 * top_tok is NULL. */
int32_t cadd_tree_grow_topk(const cadd_desc* desc, const void* L, const int32_t* anchor,
                            const int64_t* ctx_len, int32_t top_k, int32_t* tok, int32_t* parent,
                            int32_t* depth, float* score, int32_t* count, float* phi,
                            int32_t* top_tok, int32_t* dev_status, void* workspace,
                            size_t ws_bytes, void* cuda_stream);

/* ------------------------------------------------------------------------ *
 * Ancestor bitmask for tree attention: bit j of row i (word j / 32, bit
 * j % 32, least significant first) is set iff j == i or j is an ancestor of
 * i. Rows at or past count[b] are zero.
 *   parent [batch][n_stride] int32 (parent[i] < i), count [batch] int32
 *   mask   [batch][n_stride][ceil(n_stride / 32)] uint32
 * n_stride in 1..4096. No workspace.
 * ------------------------------------------------------------------------ */
int32_t tree_ancestor_mask(int32_t batch, int32_t n_stride, const int32_t* parent,
                           const int32_t* count, uint32_t* mask, int32_t* dev_status,
                           void* cuda_stream);

/* ------------------------------------------------------------------------ *
 * Greedy tree verification.
 * Source: DSpark explainer (xiaohu-jiedu), section on one round from drafting
 * to confirmation: drafts are checked from the head, consecutive matches are
 * kept, checking stops at the first miss, and the target adds its own token
 * there (four matches give five tokens for one verification).
 * Here, per node u < count: argmax[u] = argmax_v target[u][v] on the raw
 * values, ties toward the lower v. From the root, move to the child whose
 * token equals argmax[u] (the lowest-index such child), stop when none does;
 * accept_len = nodes moved to, correction = argmax at the last node reached.
 *   tok, parent [batch][n_stride] int32; count [batch] int32
 *   target [batch][n_stride][V] target_dtype (rows >= count are not read)
 *   argmax [batch][n_stride] int32 (-1 at rows >= count)
 *   accept_len [batch]; accept_path [batch][max_depth] node ids (-1 padded);
 *   correction [batch]; dev_status [batch]
 * n_stride in 1..4096, max_depth in 1..4096 (a walk longer than max_depth
 * stops there and sets PCT_DEV_DEPTH_OVERFLOW).
 * ------------------------------------------------------------------------ */
size_t tree_verify_accept_workspace(int32_t batch, int32_t n_stride);
int32_t tree_verify_accept(int32_t batch, int32_t n_stride, int32_t vocab, int32_t max_depth,
                           const int32_t* tok, const int32_t* parent, const int32_t* count,
                           const void* target, int32_t target_dtype, int32_t* argmax,
                           int32_t* accept_len, int32_t* accept_path, int32_t* correction,
                           int32_t* dev_status, void* workspace, size_t ws_bytes,
                           void* cuda_stream);

/* ------------------------------------------------------------------------ *
 * Lazy greedy verification: the same acceptance as tree_verify_accept, with
 * the argmax taken only where the walk goes.
 * Source: DSpark explainer (xiaohu-jiedu), section on one round from drafting
 * to confirmation: the drafts are compared from the head and the comparison
 * stops at the first miss, so only the rows of the nodes the walk reaches (the
 * root and each accepted node: at most max_depth + 1 rows per request) decide
 * the round; no other row is read.
 * Arguments, layouts, errors, accept_len, accept_path and correction are those
 * of tree_verify_accept (identical results). argmax [batch][n_stride] holds the
 * argmax of every row the walk reached and -1 in every other slot. No
 * workspace; one launch. The rows of one request are read one after another,
 * so the call is bound by latency rather than bandwidth.
 * ------------------------------------------------------------------------ */
int32_t tree_verify_walk(int32_t batch, int32_t n_stride, int32_t vocab, int32_t max_depth,
                         const int32_t* tok, const int32_t* parent, const int32_t* count,
                         const void* target, int32_t target_dtype, int32_t* argmax,
                         int32_t* accept_len, int32_t* accept_path, int32_t* correction,
                         int32_t* dev_status, void* cuda_stream);

/* ------------------------------------------------------------------------ *
 * Monte Carlo acceptance length of a batch of trees (tau = accepted + 1).
 * Source: DSpark explainer (xiaohu-jiedu), section on one round from drafting
 * to confirmation (checked from the head, the first miss ends the round, the
 * target adds its own token); PCTree article (qiita), numbers table (tau,
 * tokens accepted per round).
 * A walk starts at the root; at node u it draws one uniform x and moves to the
 * first child c of u, in index order, whose running sum of p_child exceeds x;
 * it stops when none does or after max_depth moves. p_child[b][c] is the
 * probability that the target's token at c's position equals c's token, given
 * that the target agreed with the path to c's parent (for a target equal to
 * the drafter: exp(score[c] - score[parent[c]])); the p_child of one node's
 * children must sum to at most 1.
 * Random numbers: Philox4x32-10 with counter (trial, request, step, 0) and key
 * (seed low 32 bits, seed high 32 bits); x = (first word >> 8) * 2^-24. Sums
 * and comparisons are fp32 in child index order (reproducible on a host).
 *   parent, p_child [batch][n_stride]; count [batch]
 *   hist [batch][max_depth + 1] int64: walks per accepted length (written)
 *   dev_status [batch]: PCT_DEV_BAD_PARENT / PCT_DEV_BAD_COUNT (that request's
 *   histogram stays zero)
 * n_stride in 1..4096, max_depth in 1..4096, trials in 1..2^31 - 1.
 * ------------------------------------------------------------------------ */
int32_t tree_accept_sim(int32_t batch, int32_t n_stride, int32_t max_depth, const int32_t* parent,
                        const int32_t* count, const float* p_child, int64_t trials, uint64_t seed,
                        int64_t* hist, int32_t* dev_status, void* cuda_stream);

/* ------------------------------------------------------------------------ *
 * cadd_cost_fit -- the verification cost model from latency samples.
 * "Cost-Aware Diffusion Draft Trees for Speculative Decoding" (gist.science
 * summary), "Method: CaDDTree": C_v is profiled offline as a convex function
 * of the tree size n that does not decrease as n grows, and grows with the
 * context length l. With C_v(n; l) = a + b l + c n + e n^2 that is the
 * non-negative least-squares fit
 *   min || X beta - t ||^2, beta = (a, b, c, e) >= 0, X = [1, l, n, n^2].
 * One launch on the stream, fp64 arithmetic: the normal equations over the
 * samples, then the least squares of each of the 16 free sets on unit-norm
 * columns (a free set whose columns are linearly dependent is skipped), the
 * feasible one with the smallest residual kept.
 *   n, ell, lat: device float32 [m], the samples (tree size, context length,
 *                measured latency)
 *   out:         device float64 [5], written: a, b, c, e and the root mean
 *                square residual
 *   dev_status:  device int32 [1], PCT_DEV_BAD_COST when a sample is not finite
 * m in 1..2^31 - 1; PCT_EINVAL for a null pointer or m out of range.
 * ------------------------------------------------------------------------ */
int32_t cadd_cost_fit(int64_t m, const float* n, const float* ell, const float* lat,
                      double* out, int32_t* dev_status, void* cuda_stream);

/* ------------------------------------------------------------------------ *
 * Allocation-free variant of tree_verify_accept. The pages have no
 * counterpart to this call: it exists for users of the library whose code
 * cannot allocate device memory -- for example a component inside a serving
 * runtime that reserves all device memory up front and hands its parts only
 * their input and output buffers, or code on a latency-critical path where a
 * cudaMalloc (which may synchronise the device) is not acceptable.
 *
 * Same arguments, results and errors as tree_verify_accept, minus the
 * workspace. The scratch it needs (one 32-bit arrival counter per request)
 * lives in a file-scope device array of PCT_NOALLOC_MAX_BATCH counters
 * (16 KB), which every GPU that loads the library holds until the process
 * exits. batch > PCT_NOALLOC_MAX_BATCH returns PCT_EUNSUPPORTED before
 * anything is launched. The call allocates nothing; it clears the counters it
 * uses on its stream before the kernel runs.
 *   - The first call in each CUDA context (per device, and again after
 *     cudaDeviceReset or when another context is made current) looks up the
 *     array's device address (cudaGetSymbolAddress); make that first call
 *     before any stream capture.
 *   - All calls share the one array: two calls that can run at the same time on
 *     the GPU (for example on different streams) race on it and give undefined
 *     results. Order them on one stream or with events.
 * ------------------------------------------------------------------------ */
#define PCT_NOALLOC_MAX_BATCH 4096
int32_t tree_verify_accept_noalloc(int32_t batch, int32_t n_stride, int32_t vocab,
                                   int32_t max_depth, const int32_t* tok, const int32_t* parent,
                                   const int32_t* count, const void* target, int32_t target_dtype,
                                   int32_t* argmax, int32_t* accept_len, int32_t* accept_path,
                                   int32_t* correction, int32_t* dev_status, void* cuda_stream);

/* ------------------------------------------------------------------------ *
 * Kernel trace (off by default; host-side bookkeeping only). While on, every
 * kernel the library launches is bracketed by two CUDA events on its stream
 * and the elapsed time is accumulated per kernel name. Not for use inside
 * CUDA-graph capture.
 * ------------------------------------------------------------------------ */
/* Enabling creates a pool of 16384 events up front, so a traced region spends
 * no host time creating them (a region that records more creates the rest). */
int32_t pct_trace_enable(int32_t on);   /* returns the previous setting */
int32_t pct_trace_reset(void);
/* Waits for the recorded events, then writes up to max_entries rows: a
 * NUL-terminated kernel name in names[i * name_stride], the launch count and
 * the summed device milliseconds. Returns the number of rows written, or -1. */
int32_t pct_trace_read(char* names, int32_t name_stride, int64_t* launches,
                       double* total_ms, int32_t max_entries);

/* Library version string (static storage). */
const char* pct_version(void);

#ifdef __cplusplus
}
#endif
#endif /* PCTREE_H */
