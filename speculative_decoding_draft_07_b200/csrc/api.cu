// C ABI of libpctree: argument checks, workspace planning and the launch
// sequence of each call. Everything here runs on the host and only enqueues
// work on the caller's stream; no call synchronises or allocates device memory.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "internal.h"

namespace pct {

size_t score_smem_bytes();

// ---------------------------------------------------------------------------
// device queries
int num_sms() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 1;
  if (dev >= 0 && dev < 64 && cache[dev] > 0) return cache[dev];
  int n = 0;
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  n = std::max(n, 1);
  if (dev >= 0 && dev < 64) cache[dev] = n;
  return n;
}

bool device_ok() {
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return false;
  return major == 10;
}

// ---------------------------------------------------------------------------
// auxiliary stream, per device and context
namespace {
typedef CUresult (*CurCtxFn)(CUcontext*);
CurCtxFn cur_ctx_fn() {
  static CurCtxFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CurCtxFn>(p);
  }
  return fn;
}
struct AuxSlot {
  CUcontext ctx;   // the context the handles belong to
  cudaStream_t s;
  cudaEvent_t fork, join;
};
std::mutex g_aux_mu;          // the slots
AuxSlot g_aux[64] = {};
std::mutex g_aux_use[64];     // one call's fork ... join on a device
}  // namespace

int aux_stream(AuxStream* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PCT_ECUDA;
  if (dev < 0 || dev >= 64) return PCT_EUNSUPPORTED;
  CurCtxFn cur = cur_ctx_fn();
  if (!cur) return PCT_ECUDA;
  std::lock_guard<std::mutex> lk(g_aux_mu);
  CUcontext ctx = nullptr;
  if (cur(&ctx) != CUDA_SUCCESS) return PCT_ECUDA;
  AuxSlot& a = g_aux[dev];
  if (ctx == nullptr || a.s == nullptr || a.ctx != ctx) {
    // a new context (first use, or the old one was reset): new handles; the
    // old ones went with their context
    AuxSlot n{};
    if (cudaStreamCreateWithFlags(&n.s, cudaStreamNonBlocking) != cudaSuccess) return PCT_ECUDA;
    if (cudaEventCreateWithFlags(&n.fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&n.join, cudaEventDisableTiming) != cudaSuccess)
      return PCT_ECUDA;
    if (cur(&ctx) != CUDA_SUCCESS || ctx == nullptr) return PCT_ECUDA;
    n.ctx = ctx;
    a = n;
  }
  out->s = a.s;
  out->fork = a.fork;
  out->join = a.join;
  out->mu = &g_aux_use[dev];
  return PCT_OK;
}
void aux_lock(const AuxStream& a) { static_cast<std::mutex*>(a.mu)->lock(); }
void aux_unlock(const AuxStream& a) { static_cast<std::mutex*>(a.mu)->unlock(); }

// ---------------------------------------------------------------------------
// kernel trace
namespace {
std::mutex g_mu;
volatile bool g_on = false;
struct Rec {
  int name;
  cudaEvent_t a, b;
};
std::vector<Rec> g_recs;
std::vector<std::string> g_names;
std::vector<cudaEvent_t> g_pool;
constexpr size_t kTracePool = 16384;   // events kept ready while tracing is on

cudaEvent_t take_event() {
  if (!g_pool.empty()) {
    cudaEvent_t e = g_pool.back();
    g_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}
int name_id(const char* n) {
  for (size_t i = 0; i < g_names.size(); ++i)
    if (g_names[i] == n) return (int)i;
  g_names.emplace_back(n);
  return (int)g_names.size() - 1;
}
}  // namespace

TraceScope::TraceScope(cudaStream_t s, const char* name) : stream(s), slot(-1) {
  if (!g_on) return;
  std::lock_guard<std::mutex> lk(g_mu);
  Rec r;
  r.name = name_id(name);
  r.a = take_event();
  r.b = take_event();
  if (!r.a || !r.b) return;
  cudaEventRecord(r.a, s);
  g_recs.push_back(r);
  slot = (int)g_recs.size() - 1;
}

TraceScope::~TraceScope() {
  if (slot < 0) return;
  std::lock_guard<std::mutex> lk(g_mu);
  if (slot < (int)g_recs.size()) cudaEventRecord(g_recs[slot].b, stream);
}

namespace {

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }
size_t esize(int dt) { return dt == PCT_BF16 ? 2 : 4; }
bool dtype_ok(int dt) { return dt == PCT_F32 || dt == PCT_BF16; }
bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// ---------------------------------------------------------------------------
// PCTree plan: frontier sizes per depth, V-slices per depth, workspace layout.
struct PctPlan {
  int batch, D, V, r, r_pad, k, beam, N, ldt, mdt;
  int F[66];
  int S[66];
  int Mmax, M_pad;
  size_t max_ps;
  size_t o_eg, o_ms, o_val, o_idx, o_ltok, o_lppos, o_ls, o_err, o_thr, o_scol, o_slval, o_swmax, o_swcol, o_sdk, total;
  bool chain;             // small frontiers: one persistent launch (pct_chain.cu)
  size_t o_chain;
};

ChainShape chain_shape(const PctPlan& P) {
  return ChainShape{P.batch, P.D, P.V, P.r, P.r_pad, P.k, P.beam, P.ldt, P.mdt};
}

int check_build_desc(const pct_build_desc* d) {
  if (!d) return PCT_EINVAL;
  if (d->batch < 1 || d->batch > 65535) return PCT_EINVAL;
  if (d->depth < 1 || d->depth > 64) return PCT_EINVAL;
  if (d->vocab < 1 || d->k < 1 || d->k > 16 || d->k > d->vocab) return PCT_EINVAL;
  if (d->rank < 1 || d->rank > 256) return PCT_EINVAL;
  if (d->beam < 1 || d->beam > 256 || d->beam * d->k > 1024) return PCT_EINVAL;
  if (d->n_nodes < 1 || d->n_nodes > 4096 || d->depth * d->beam > 4096) return PCT_EINVAL;
  if (!dtype_ok(d->logits_dtype) || !dtype_ok(d->markov_dtype)) return PCT_EINVAL;
  if (d->markov_dtype == PCT_BF16 && d->vocab % 8 != 0) return PCT_EUNSUPPORTED;
  if (d->vocab > (1 << 22)) return PCT_EUNSUPPORTED;   // token ids packed into 22-bit key fields
  return PCT_OK;
}

int make_plan(const pct_build_desc* d, PctPlan* P) {
  const int st = check_build_desc(d);
  if (st != PCT_OK) return st;
  P->batch = d->batch; P->D = d->depth; P->V = d->vocab; P->r = d->rank; P->k = d->k;
  P->beam = d->beam; P->N = d->n_nodes; P->ldt = d->logits_dtype; P->mdt = d->markov_dtype;
  P->r_pad = P->mdt == PCT_BF16 ? (P->r + 63) / 64 * 64 : P->r;
  P->F[0] = 1;
  P->Mmax = 0;
  P->max_ps = 0;
  for (int dd = 1; dd <= P->D; ++dd) {
    P->F[dd] = std::min(P->beam, P->F[dd - 1] * P->k);
    const int M = P->batch * P->F[dd - 1];
    P->Mmax = std::max(P->Mmax, M);
    P->S[dd] = score_slices(M, P->V, P->mdt);
    P->max_ps = std::max(P->max_ps, (size_t)M * P->S[dd]);
  }
  P->M_pad = (P->Mmax + 127) / 128 * 128;
  const size_t lvl = (size_t)P->D * P->batch * P->beam;
  size_t o = 0;
  P->o_eg = o;    o += align_up((size_t)P->M_pad * P->r_pad * esize(P->mdt));
  P->o_ms = o;    o += align_up(P->max_ps * sizeof(float2));
  P->o_val = o;   o += align_up(P->max_ps * P->k * sizeof(float));
  P->o_idx = o;   o += align_up(P->max_ps * P->k * sizeof(int32_t));
  P->o_ltok = o;  o += align_up(lvl * sizeof(int32_t));
  P->o_lppos = o; o += align_up(lvl * sizeof(int32_t));
  P->o_ls = o;    o += align_up(lvl * sizeof(float));
  P->o_err = o;   o += align_up(sizeof(int32_t));
  P->o_thr = o;   o += align_up((size_t)P->Mmax * sizeof(uint32_t));
  const size_t seeds = (size_t)P->batch * P->D * P->k;   // seed entries (request, depth, column)
  P->o_scol = o;  o += align_up(seeds * sizeof(int32_t));
  P->o_slval = o; o += align_up(seeds * sizeof(float));
  P->o_swmax = o; o += align_up(seeds * sizeof(float));
  P->o_swcol = o; o += P->mdt == PCT_BF16 ? align_up(seeds * P->r_pad * 2) : 0;
  P->o_sdk = o;   o += P->mdt == PCT_BF16 ? align_up(drafter_topk_scratch(P->batch * P->D)) : 0;
  P->chain = chain_eligible(chain_shape(*P));
  P->o_chain = o; o += P->chain ? align_up(chain_workspace(chain_shape(*P))) : 0;
  P->total = o;
  return PCT_OK;
}

int ws_check(const void* ws, size_t have, size_t need) {
  if (need == 0) return PCT_OK;
  if (!ws || !aligned(ws, kAlign) || have < need) return PCT_EWORKSPACE;
  return PCT_OK;
}

#define PCT_CU(x)                               \
  do {                                          \
    if ((x) != cudaSuccess) return PCT_ECUDA;   \
  } while (0)

// ---------------------------------------------------------------------------
// CaDDTree plan
int check_cadd(const cadd_desc* d) {
  if (!d) return PCT_EINVAL;
  if (d->batch < 1 || d->batch > 65535 || d->depth < 1 || d->depth > 63) return PCT_EINVAL;
  if (d->vocab < 1 || d->vocab > (1 << 24)) return PCT_EINVAL;
  if (d->n_max < 1 || d->n_max > 1024) return PCT_EINVAL;
  if (!dtype_ok(d->logits_dtype)) return PCT_EINVAL;
  if (!(d->c >= 0.f) || !(d->e >= 0.f)) return PCT_EINVAL;   // convex, monotone C_v
  if (!std::isfinite(d->C_d) || !std::isfinite(d->a) || !std::isfinite(d->b) ||
      !std::isfinite(d->c) || !std::isfinite(d->e))
    return PCT_EINVAL;
  return PCT_OK;
}
struct CaddPlan {
  size_t o_lse, o_cnt, o_q, o_tok, o_seg, seg_bytes, o_topk, total;
};
void cadd_plan(const cadd_desc* d, CaddPlan* P) {
  const size_t rows = (size_t)d->batch * d->depth;
  const size_t K1 = (size_t)std::max(d->n_max - 1, 1);
  size_t o = 0;
  P->o_lse = o; o += align_up(rows * sizeof(float));
  P->o_cnt = o; o += align_up(rows * sizeof(int32_t));
  P->o_q = o;   o += align_up(rows * K1 * sizeof(float));
  P->o_tok = o; o += align_up(rows * K1 * sizeof(int32_t));
  P->seg_bytes = cadd_seg_workspace(d->batch, d->depth, d->vocab, d->logits_dtype);
  P->o_seg = o; o += align_up(P->seg_bytes);
  P->o_topk = o; o += align_up(cadd_topk_workspace(rows));   // cadd_tree_grow_topk only
  P->total = o;
}

}  // namespace
}  // namespace pct

using namespace pct;

extern "C" {

const char* pct_version(void) { return "pctree-b200 0.1 (sm_100a)"; }

int32_t pct_trace_enable(int32_t on) {
  std::lock_guard<std::mutex> lk(g_mu);
  const int32_t prev = g_on ? 1 : 0;
  g_on = on != 0;
  // events are created here, not while a traced region launches: creating
  // them there costs host time that delays the launches being timed
  while (g_on && g_pool.size() + 2 * g_recs.size() < kTracePool) {
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) break;
    g_pool.push_back(e);
  }
  return prev;
}

int32_t pct_trace_reset(void) {
  std::lock_guard<std::mutex> lk(g_mu);
  for (auto& r : g_recs) {
    cudaEventSynchronize(r.b);
    g_pool.push_back(r.a);
    g_pool.push_back(r.b);
  }
  g_recs.clear();
  return PCT_OK;
}

int32_t pct_trace_read(char* names, int32_t name_stride, int64_t* launches, double* total_ms,
                       int32_t max_entries) {
  std::lock_guard<std::mutex> lk(g_mu);
  std::vector<int64_t> cnt(g_names.size(), 0);
  std::vector<double> ms(g_names.size(), 0.0);
  for (auto& r : g_recs) {
    if (cudaEventSynchronize(r.b) != cudaSuccess) return -1;
    float t = 0.f;
    if (cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess) return -1;
    cnt[r.name] += 1;
    ms[r.name] += t;
  }
  int32_t n = 0;
  for (size_t i = 0; i < g_names.size() && n < max_entries; ++i) {
    if (cnt[i] == 0) continue;
    if (names && name_stride > 0) {
      std::strncpy(names + (size_t)n * name_stride, g_names[i].c_str(), name_stride - 1);
      names[(size_t)n * name_stride + name_stride - 1] = '\0';
    }
    if (launches) launches[n] = cnt[i];
    if (total_ms) total_ms[n] = ms[i];
    ++n;
  }
  return n;
}

// ---------------------------------------------------------------------------
size_t pct_tree_build_workspace(const pct_build_desc* desc) {
  PctPlan P;
  if (make_plan(desc, &P) != PCT_OK) return 0;
  return P.total;
}

// seed_tok: null, or [batch][depth][k] columns that seed each row's top-k gate
// in place of the drafter top-k pass; Wt: null, or W transposed (their W columns).
static int32_t pct_build_impl(const pct_build_desc* desc, const void* L, const int32_t* anchor,
                              const void* E, const void* W, const void* Wt,
                              const int32_t* seed_tok, int32_t* tok,
                              int32_t* parent, int32_t* depth, float* score, int32_t* count,
                              int32_t* dev_status, void* workspace, size_t ws_bytes,
                              void* cuda_stream) {
  PctPlan P;
  const int st = make_plan(desc, &P);
  if (st != PCT_OK) return st;
  if (!L || !anchor || !E || !W || !tok || !parent || !depth || !score || !count || !dev_status)
    return PCT_EINVAL;
  if (P.mdt == PCT_BF16 && (!aligned(W, 16) || !aligned(L, 16))) return PCT_EINVAL;
  if (!device_ok()) return PCT_EDEVICE;
  const int wst = ws_check(workspace, ws_bytes, P.total);
  if (wst != PCT_OK) return wst;
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  char* ws = static_cast<char*>(workspace);
  void* Eg = ws + P.o_eg;
  Partials part{reinterpret_cast<float2*>(ws + P.o_ms), reinterpret_cast<float*>(ws + P.o_val),
                reinterpret_cast<int32_t*>(ws + P.o_idx)};
  int32_t* ltok = reinterpret_cast<int32_t*>(ws + P.o_ltok);
  int32_t* lppos = reinterpret_cast<int32_t*>(ws + P.o_lppos);
  float* ls = reinterpret_cast<float*>(ws + P.o_ls);
  int32_t* err = reinterpret_cast<int32_t*>(ws + P.o_err);
  const size_t lvl = (size_t)P.batch * P.beam;

  PCT_CU(cudaMemsetAsync(dev_status, 0, sizeof(int32_t) * P.batch, s));
  if (P.chain && aligned(E, 16) && aligned(W, 16) && aligned(L, 16)) {
    // every depth in one persistent launch, then the global top-N
    int32_t* cerr = nullptr;
    int32_t* ccol = reinterpret_cast<int32_t*>(ws + P.o_scol);
    float* clval = reinterpret_cast<float*>(ws + P.o_slval);
    float* cwmax = reinterpret_cast<float*>(ws + P.o_swmax);
    if (seed_tok)
      PCT_CU(launch_seed_columns(P.batch * P.D, P.V, P.k, P.ldt, L, W, Wt, P.r, P.r_pad,
                                 seed_tok, ccol, clval, cwmax, ws + P.o_swcol, s));
    else
      PCT_CU(launch_drafter_topk(P.batch * P.D, P.V, P.k, P.ldt, L, W, P.r, P.r_pad, ccol, clval,
                                 cwmax, ws + P.o_swcol, ws + P.o_sdk, s));
    PCT_CU(launch_chain(chain_shape(P), L, anchor, E, W, ws + P.o_chain, ltok, lppos, ls, &cerr,
                        dev_status, ccol, clval, cwmax, ws + P.o_swcol, s));
    FinalArgs f;
    f.batch = P.batch; f.D = P.D; f.beam = P.beam; f.N = P.N;
    for (int d = 0; d <= P.D; ++d) f.F[d] = P.F[d];
    f.anchor = anchor; f.lvl_tok = ltok; f.lvl_ppos = lppos; f.lvl_s = ls;
    f.tok = tok; f.parent = parent; f.depth = depth; f.count = count; f.score = score;
    f.status = dev_status;
    f.err = cerr;
    PCT_CU(launch_final(f, s));
    return PCT_OK;
  }
  PCT_CU(cudaMemsetAsync(err, 0, sizeof(int32_t), s));
  // tensor-core scoring: every row's top-k gate starts from a seed (k exact
  // values of the row at the request's best drafter columns of that depth)
  const bool seeded = P.mdt == PCT_BF16;
  uint32_t* row_thr = reinterpret_cast<uint32_t*>(ws + P.o_thr);
  int32_t* scol = reinterpret_cast<int32_t*>(ws + P.o_scol);
  float* slval = reinterpret_cast<float*>(ws + P.o_slval);
  float* swmax = reinterpret_cast<float*>(ws + P.o_swmax);
  char* swcol = ws + P.o_swcol;
  auto seed_for = [&](int di) {   // seeds of the rows scored against L index di
    SeedArgs sd{};
    if (!seeded || di >= P.D) return sd;
    const size_t e = (size_t)di * P.k;
    sd.cols = scol + e;
    sd.lval = slval + e;
    sd.wmax = swmax + e;
    sd.wcol = swcol + e * P.r_pad * 2;
    sd.req_stride = (long long)P.D * P.k;
    sd.ks = P.k;
    sd.thr = row_thr;
    return sd;
  };
  if (seeded && seed_tok)
    PCT_CU(launch_seed_columns(P.batch * P.D, P.V, P.k, P.ldt, L, W, Wt, P.r, P.r_pad, seed_tok,
                               scol, slval, swmax, swcol, s));
  else if (seeded)
    PCT_CU(launch_drafter_topk(P.batch * P.D, P.V, P.k, P.ldt, L, W, P.r, P.r_pad, scol, slval,
                               swmax, swcol, ws + P.o_sdk, s));
  PCT_CU(launch_gather_rows(P.batch, anchor, P.V, P.r, P.r_pad, P.mdt, E, Eg, dev_status, 1,
                            seed_for(0), s));
  for (int d = 1; d <= P.D; ++d) {
    ScoreArgs a;
    a.n_req = P.batch; a.n_par = P.F[d - 1]; a.V = P.V; a.r = P.r; a.r_pad = P.r_pad; a.k = P.k;
    a.logits_dtype = P.ldt; a.markov_dtype = P.mdt;
    a.L = static_cast<const char*>(L) + (size_t)(d - 1) * P.V * esize(P.ldt);
    a.L_req_stride = (long long)P.D * P.V;
    a.Eg = Eg; a.M_pad = P.M_pad; a.W = W; a.Wt = Wt; a.part = part; a.S = P.S[d]; a.err = err;
    a.row_thr = row_thr;
    a.thr_seeded = seeded;
    PCT_CU(launch_score(a, s));
    MergeArgs m;
    m.batch = P.batch; m.F_prev = P.F[d - 1]; m.F_new = P.F[d]; m.k = P.k; m.beam = P.beam;
    m.S = P.S[d]; m.V = P.V; m.r = P.r; m.r_pad = P.r_pad; m.markov_dtype = P.mdt; m.depth = d;
    m.part = part;
    m.prev_tok = nullptr;
    m.prev_s = d == 1 ? nullptr : ls + (size_t)(d - 2) * lvl;
    m.prev_stride = P.beam;
    m.lvl_tok = ltok + (size_t)(d - 1) * lvl;
    m.lvl_ppos = lppos + (size_t)(d - 1) * lvl;
    m.lvl_s = ls + (size_t)(d - 1) * lvl;
    m.E = E;
    m.Eg_next = d < P.D ? Eg : nullptr;
    m.err = err;
    m.status = dev_status;
    m.seed = seed_for(d);
    PCT_CU(launch_merge(m, s));
  }
  FinalArgs f;
  f.batch = P.batch; f.D = P.D; f.beam = P.beam; f.N = P.N;
  for (int d = 0; d <= P.D; ++d) f.F[d] = P.F[d];
  f.anchor = anchor; f.lvl_tok = ltok; f.lvl_ppos = lppos; f.lvl_s = ls;
  f.tok = tok; f.parent = parent; f.depth = depth; f.count = count; f.score = score;
  f.status = dev_status;
  f.err = err;
  PCT_CU(launch_final(f, s));
  return PCT_OK;
}

int32_t pct_tree_build(const pct_build_desc* desc, const void* L, const int32_t* anchor,
                       const void* E, const void* W, int32_t* tok, int32_t* parent,
                       int32_t* depth, float* score, int32_t* count, int32_t* dev_status,
                       void* workspace, size_t ws_bytes, void* cuda_stream) {
  return pct_build_impl(desc, L, anchor, E, W, nullptr, nullptr, tok, parent, depth, score,
                        count, dev_status, workspace, ws_bytes, cuda_stream);
}

int32_t pct_tree_build_seeded(const pct_build_desc* desc, const void* L, const int32_t* anchor,
                              const void* E, const void* W, const void* Wt,
                              const int32_t* seed_tok, int32_t* tok, int32_t* parent,
                              int32_t* depth, float* score, int32_t* count, int32_t* dev_status,
                              void* workspace, size_t ws_bytes, void* cuda_stream) {
  if (!seed_tok) return PCT_EINVAL;
  if (Wt && (!aligned(Wt, 16) || !desc || desc->markov_dtype != PCT_BF16)) return PCT_EINVAL;
  return pct_build_impl(desc, L, anchor, E, W, Wt, seed_tok, tok, parent, depth, score, count,
                        dev_status, workspace, ws_bytes, cuda_stream);
}

int32_t pct_markov_rank_pad(int32_t rank) {
  return (rank < 1 || rank > 256) ? 0 : (rank + 63) / 64 * 64;
}

int32_t pct_markov_transpose(int32_t vocab, int32_t rank, const void* W, void* Wt,
                             void* cuda_stream) {
  const int r_pad = pct_markov_rank_pad(rank);
  if (r_pad == 0 || vocab < 8 || vocab % 8 != 0 || vocab > (1 << 22) || !W || !Wt)
    return PCT_EINVAL;
  if (!aligned(W, 16) || !aligned(Wt, 16)) return PCT_EINVAL;
  if (!device_ok()) return PCT_EDEVICE;
  PCT_CU(launch_markov_transpose(vocab, rank, r_pad, W, Wt, static_cast<cudaStream_t>(cuda_stream)));
  return PCT_OK;
}

// ---------------------------------------------------------------------------
static int score_parents_plan(const pct_build_desc* d, int32_t n_par, PctPlan* P, size_t* o_eg,
                              size_t* o_ms, size_t* o_val, size_t* o_idx, size_t* o_err,
                              size_t* o_thr, size_t* total, int* S) {
  if (!d) return PCT_EINVAL;
  if (d->batch < 1 || d->batch > 65535 || n_par < 1 || n_par > 4096) return PCT_EINVAL;
  if (d->vocab < 1 || d->k < 1 || d->k > 16 || d->k > d->vocab) return PCT_EINVAL;
  if (d->rank < 1 || d->rank > 256) return PCT_EINVAL;
  if (!dtype_ok(d->logits_dtype) || !dtype_ok(d->markov_dtype)) return PCT_EINVAL;
  if (d->markov_dtype == PCT_BF16 && d->vocab % 8 != 0) return PCT_EUNSUPPORTED;
  P->batch = d->batch; P->V = d->vocab; P->r = d->rank; P->k = d->k;
  P->ldt = d->logits_dtype; P->mdt = d->markov_dtype;
  P->r_pad = P->mdt == PCT_BF16 ? (P->r + 63) / 64 * 64 : P->r;
  const int rows = d->batch * n_par;
  P->M_pad = (rows + 127) / 128 * 128;
  *S = score_slices(rows, P->V, P->mdt);
  const size_t ps = (size_t)rows * *S;
  size_t o = 0;
  *o_eg = o;  o += align_up((size_t)P->M_pad * P->r_pad * esize(P->mdt));
  *o_ms = o;  o += align_up(ps * sizeof(float2));
  *o_val = o; o += align_up(ps * P->k * sizeof(float));
  *o_idx = o; o += align_up(ps * P->k * sizeof(int32_t));
  *o_err = o; o += align_up(sizeof(int32_t));
  *o_thr = o; o += align_up((size_t)rows * sizeof(uint32_t));
  *total = o;
  return PCT_OK;
}

size_t pct_score_parents_workspace(const pct_build_desc* desc, int32_t n_par) {
  PctPlan P;
  size_t a, b, c, d, e, f, total;
  int S;
  if (score_parents_plan(desc, n_par, &P, &a, &b, &c, &d, &e, &f, &total, &S) != PCT_OK) return 0;
  return total;
}

int32_t pct_score_parents(const pct_build_desc* desc, int32_t n_par, const void* L_row,
                          const int32_t* parent_tok, const void* E, const void* W, float* lse,
                          int32_t* top_tok, float* top_logpi, int32_t* dev_status,
                          void* workspace, size_t ws_bytes, void* cuda_stream) {
  PctPlan P;
  size_t o_eg, o_ms, o_val, o_idx, o_err, o_thr, total;
  int S;
  const int st = score_parents_plan(desc, n_par, &P, &o_eg, &o_ms, &o_val, &o_idx, &o_err, &o_thr,
                                    &total, &S);
  if (st != PCT_OK) return st;
  if (!L_row || !parent_tok || !E || !W || !lse || !top_tok || !top_logpi || !dev_status)
    return PCT_EINVAL;
  if (P.mdt == PCT_BF16 && (!aligned(W, 16) || !aligned(L_row, 16))) return PCT_EINVAL;
  if (!device_ok()) return PCT_EDEVICE;
  const int wst = ws_check(workspace, ws_bytes, total);
  if (wst != PCT_OK) return wst;
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  char* ws = static_cast<char*>(workspace);
  Partials part{reinterpret_cast<float2*>(ws + o_ms), reinterpret_cast<float*>(ws + o_val),
                reinterpret_cast<int32_t*>(ws + o_idx)};
  int32_t* err = reinterpret_cast<int32_t*>(ws + o_err);
  const int rows = P.batch * n_par;
  PCT_CU(cudaMemsetAsync(dev_status, 0, sizeof(int32_t) * P.batch, s));
  PCT_CU(cudaMemsetAsync(err, 0, sizeof(int32_t), s));
  PCT_CU(launch_gather_rows(rows, parent_tok, P.V, P.r, P.r_pad, P.mdt, E, ws + o_eg, dev_status,
                            n_par, SeedArgs{}, s));
  ScoreArgs a;
  a.n_req = P.batch; a.n_par = n_par; a.V = P.V; a.r = P.r; a.r_pad = P.r_pad; a.k = P.k;
  a.logits_dtype = P.ldt; a.markov_dtype = P.mdt; a.L = L_row; a.L_req_stride = P.V;
  a.Eg = ws + o_eg; a.M_pad = P.M_pad; a.W = W; a.Wt = nullptr; a.part = part; a.S = S; a.err = err;
  a.row_thr = reinterpret_cast<uint32_t*>(ws + o_thr);
  a.thr_seeded = false;
  PCT_CU(launch_score(a, s));
  PCT_CU(launch_rows_finalize(rows, P.k, S, part, lse, top_tok, top_logpi, err, dev_status, n_par, s));
  return PCT_OK;
}

// ---------------------------------------------------------------------------
size_t cadd_tree_grow_workspace(const cadd_desc* desc) {
  if (check_cadd(desc) != PCT_OK) return 0;
  CaddPlan P;
  cadd_plan(desc, &P);
  return P.total;
}

static int32_t cadd_grow_impl(const cadd_desc* desc, const void* L, const int32_t* anchor,
                              const int64_t* ctx_len, int32_t top_k, int32_t* tok, int32_t* parent,
                              int32_t* depth, float* score, int32_t* count, float* phi,
                              int32_t* top_tok, int32_t* dev_status, void* workspace,
                              size_t ws_bytes, void* cuda_stream) {
  const int st = check_cadd(desc);
  if (st != PCT_OK) return st;
  if (!L || !anchor || !ctx_len || !tok || !parent || !depth || !score || !count || !phi || !dev_status)
    return PCT_EINVAL;
  if (top_k < 0 || top_k > 32 || (top_k > 0 && !top_tok)) return PCT_EINVAL;
  if (!device_ok()) return PCT_EDEVICE;
  CaddPlan P;
  cadd_plan(desc, &P);
  const int wst = ws_check(workspace, ws_bytes, P.total);
  if (wst != PCT_OK) return wst;
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  char* ws = static_cast<char*>(workspace);
  PCT_CU(cudaMemsetAsync(dev_status, 0, sizeof(int32_t) * desc->batch, s));
  CaddParams p{desc->batch, desc->depth, desc->vocab, desc->n_max, desc->logits_dtype,
               desc->C_d, desc->a, desc->b, desc->c, desc->e, top_k, top_tok};
  PCT_CU(launch_cadd(p, L, anchor, ctx_len, tok, parent, depth, score, count, phi, dev_status,
                     reinterpret_cast<float*>(ws + P.o_lse), reinterpret_cast<int32_t*>(ws + P.o_cnt),
                     reinterpret_cast<float*>(ws + P.o_q), reinterpret_cast<int32_t*>(ws + P.o_tok),
                     P.seg_bytes ? ws + P.o_seg : nullptr, ws + P.o_topk, s));
  return PCT_OK;
}

int32_t cadd_tree_grow(const cadd_desc* desc, const void* L, const int32_t* anchor,
                       const int64_t* ctx_len, int32_t* tok, int32_t* parent, int32_t* depth,
                       float* score, int32_t* count, float* phi, int32_t* dev_status,
                       void* workspace, size_t ws_bytes, void* cuda_stream) {
  return cadd_grow_impl(desc, L, anchor, ctx_len, 0, tok, parent, depth, score, count, phi,
                        nullptr, dev_status, workspace, ws_bytes, cuda_stream);
}

int32_t cadd_tree_grow_topk(const cadd_desc* desc, const void* L, const int32_t* anchor,
                            const int64_t* ctx_len, int32_t top_k, int32_t* tok, int32_t* parent,
                            int32_t* depth, float* score, int32_t* count, float* phi,
                            int32_t* top_tok, int32_t* dev_status, void* workspace,
                            size_t ws_bytes, void* cuda_stream) {
  if (top_k < 1) return PCT_EINVAL;
  return cadd_grow_impl(desc, L, anchor, ctx_len, top_k, tok, parent, depth, score, count, phi,
                        top_tok, dev_status, workspace, ws_bytes, cuda_stream);
}

// ---------------------------------------------------------------------------
int32_t tree_ancestor_mask(int32_t batch, int32_t n_stride, const int32_t* parent,
                           const int32_t* count, uint32_t* mask, int32_t* dev_status,
                           void* cuda_stream) {
  if (batch < 1 || batch > 65535 || n_stride < 1 || n_stride > 4096) return PCT_EINVAL;
  if (!parent || !count || !mask || !dev_status) return PCT_EINVAL;
  if (!device_ok()) return PCT_EDEVICE;
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  PCT_CU(cudaMemsetAsync(dev_status, 0, sizeof(int32_t) * batch, s));
  PCT_CU(launch_ancestor_mask(batch, n_stride, parent, count, mask, dev_status, s));
  return PCT_OK;
}

size_t tree_verify_accept_workspace(int32_t batch, int32_t n_stride) {
  if (batch < 1 || batch > 65535 || n_stride < 1 || n_stride > 4096) return 0;
  return align_up(sizeof(unsigned) * (size_t)batch);
}

int32_t tree_verify_accept(int32_t batch, int32_t n_stride, int32_t vocab, int32_t max_depth,
                           const int32_t* tok, const int32_t* parent, const int32_t* count,
                           const void* target, int32_t target_dtype, int32_t* argmax,
                           int32_t* accept_len, int32_t* accept_path, int32_t* correction,
                           int32_t* dev_status, void* workspace, size_t ws_bytes,
                           void* cuda_stream) {
  if (batch < 1 || batch > 65535 || n_stride < 1 || n_stride > 4096) return PCT_EINVAL;
  if (vocab < 1 || max_depth < 1 || max_depth > 4096 || !dtype_ok(target_dtype)) return PCT_EINVAL;
  if (!tok || !parent || !count || !target || !argmax || !accept_len || !accept_path ||
      !correction || !dev_status)
    return PCT_EINVAL;
  if (!device_ok()) return PCT_EDEVICE;
  const size_t need = tree_verify_accept_workspace(batch, n_stride);
  const int wst = ws_check(workspace, ws_bytes, need);
  if (wst != PCT_OK) return wst;
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  unsigned* arrive = static_cast<unsigned*>(workspace);
  PCT_CU(cudaMemsetAsync(dev_status, 0, sizeof(int32_t) * batch, s));
  PCT_CU(cudaMemsetAsync(arrive, 0, sizeof(unsigned) * batch, s));
  PCT_CU(launch_verify(batch, n_stride, vocab, max_depth, tok, parent, count, target, target_dtype,
                       argmax, accept_len, accept_path, correction, dev_status, arrive, s));
  return PCT_OK;
}

int32_t tree_verify_walk(int32_t batch, int32_t n_stride, int32_t vocab, int32_t max_depth,
                         const int32_t* tok, const int32_t* parent, const int32_t* count,
                         const void* target, int32_t target_dtype, int32_t* argmax,
                         int32_t* accept_len, int32_t* accept_path, int32_t* correction,
                         int32_t* dev_status, void* cuda_stream) {
  if (batch < 1 || batch > 65535 || n_stride < 1 || n_stride > 4096) return PCT_EINVAL;
  if (vocab < 1 || max_depth < 1 || max_depth > 4096 || !dtype_ok(target_dtype)) return PCT_EINVAL;
  if (!tok || !parent || !count || !target || !argmax || !accept_len || !accept_path ||
      !correction || !dev_status)
    return PCT_EINVAL;
  if (!device_ok()) return PCT_EDEVICE;
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  PCT_CU(cudaMemsetAsync(dev_status, 0, sizeof(int32_t) * batch, s));
  PCT_CU(launch_verify_walk(batch, n_stride, vocab, max_depth, tok, parent, count, target,
                            target_dtype, argmax, accept_len, accept_path, correction, dev_status,
                            s));
  return PCT_OK;
}

int32_t tree_accept_sim(int32_t batch, int32_t n_stride, int32_t max_depth, const int32_t* parent,
                        const int32_t* count, const float* p_child, int64_t trials, uint64_t seed,
                        int64_t* hist, int32_t* dev_status, void* cuda_stream) {
  if (batch < 1 || batch > 65535 || n_stride < 1 || n_stride > 4096) return PCT_EINVAL;
  if (max_depth < 1 || max_depth > 4096 || trials < 1 || trials > 2147483647LL) return PCT_EINVAL;
  if (!parent || !count || !p_child || !hist || !dev_status) return PCT_EINVAL;
  if (!device_ok()) return PCT_EDEVICE;
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  PCT_CU(cudaMemsetAsync(dev_status, 0, sizeof(int32_t) * batch, s));
  PCT_CU(cudaMemsetAsync(hist, 0, sizeof(int64_t) * (size_t)batch * (max_depth + 1), s));
  PCT_CU(launch_accept_sim(batch, n_stride, max_depth, parent, count, p_child, (long long)trials,
                           (unsigned long long)seed, reinterpret_cast<unsigned long long*>(hist),
                           dev_status, s));
  return PCT_OK;
}

int32_t cadd_cost_fit(int64_t m, const float* n, const float* ell, const float* lat,
                      double* out, int32_t* dev_status, void* cuda_stream) {
  if (m < 1 || m > 2147483647LL) return PCT_EINVAL;
  if (!n || !ell || !lat || !out || !dev_status) return PCT_EINVAL;
  if (!device_ok()) return PCT_EDEVICE;
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  PCT_CU(cudaMemsetAsync(dev_status, 0, sizeof(int32_t), s));
  PCT_CU(launch_cost_fit((long long)m, n, ell, lat, out, dev_status, s));
  return PCT_OK;
}

}  // extern "C"
