// Host runtime and C ABI of the causal IVF index (one handle = one request
// and layer).
//
// State follows the AttentionIndex explainer (paper-daily.com), section
// "索引怎么边算边建？": an append-only key store (insert), clusters appended
// per sealed window (seal), a periodic refit that replaces the clustered
// prefix (refit, side stream), and a version per seal / refit so that a
// query only uses clusters built from its own prefix (versions).
//
// Cluster arrays are double-buffered.  The published buffer holds
// [refit base clusters][clusters sealed after the base]; a refit writes the
// other buffer on the side stream while seals keep appending to the
// published one, and publication (next append, or ai_publish) makes the
// main stream wait on the refit's event, copies the clusters sealed after
// the refit watermark behind the new base, and swaps.
#include <cudaTypedefs.h>

#include <algorithm>
#include <chrono>
#include <cstring>
#include <string>
#include <thread>
#include <unordered_map>
#include <vector>

#include "../../include/ai_index.h"
#include "common.cuh"
#include "kernels.h"

#include <atomic>

using namespace aiidx;

namespace {
thread_local std::string g_err;
}  // namespace

namespace aiidx {
static std::atomic<long long> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
long long kernel_launches() { return g_launches.load(std::memory_order_relaxed); }
void set_last_error(const char* msg) { g_err = msg; }
}  // namespace aiidx

namespace {

int fail(int code, const std::string& msg) {
  g_err = msg;
  return code;
}

#define CK(call)                                                                            \
  do {                                                                                      \
    cudaError_t e_ = (call);                                                                \
    if (e_ != cudaSuccess)                                                                  \
      return fail(AI_ERR_CUDA, std::string(#call) + ": " + cudaGetErrorString(e_));         \
  } while (0)

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

bool get_encode() {
  if (g_encode) return true;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || fn == nullptr)
    return false;
  g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return true;
}

// 2-D bf16 map over rows of 128 elements (256 B), box = 64 x box_rows,
// 128-byte swizzle (the UMMA K-major layout), zero fill out of range.
bool make_map(CUtensorMap* m, const void* base, int64_t rows, int box_rows) {
  if (!get_encode()) return false;
  cuuint64_t dims[2] = {128, static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {256};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t es[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                        box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

uint64_t splitmix64(uint64_t seed, uint64_t ctr) {
  uint64_t z = seed + (ctr + 1) * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// n_seed distinct ids from [lo, hi) in draw order (partial Fisher-Yates;
// draw i swaps slot i with slot i + splitmix64(seed, (r << 32) | i) mod (n-i)).
std::vector<int64_t> seed_ids(uint64_t seed, uint64_t refit_index, int64_t lo, int64_t hi, int64_t n_seed) {
  const int64_t n = hi - lo;
  const int64_t s = std::min(n_seed, n);
  std::unordered_map<int64_t, int64_t> perm;
  std::vector<int64_t> out(static_cast<size_t>(std::max<int64_t>(s, 0)));
  for (int64_t i = 0; i < s; ++i) {
    const uint64_t r = splitmix64(seed, (refit_index << 32) | static_cast<uint64_t>(i));
    const int64_t j = i + static_cast<int64_t>(r % static_cast<uint64_t>(n - i));
    auto gi = perm.find(i);
    auto gj = perm.find(j);
    const int64_t vi = gi == perm.end() ? i : gi->second;
    const int64_t vj = gj == perm.end() ? j : gj->second;
    perm[i] = vj;
    perm[j] = vi;
    out[static_cast<size_t>(i)] = lo + vj;
  }
  return out;
}

__global__ void k_shift_offsets(const int32_t* src, int32_t* dst, int n, int32_t delta) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) dst[i] = src[i] + delta;
}

__global__ void k_fill(float* p, int64_t n, float v) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    p[i] = v;
}

struct Version {
  int64_t nC;
  int64_t n_v;
};

struct Buffer {
  int32_t* offsets = nullptr;   // [maxC + 1]
  int32_t* members = nullptr;   // [max_keys]
  double* centroids = nullptr;  // [maxC, d]
  uint16_t* reps = nullptr;     // [maxC_pad, d]
  int64_t nC = 0;               // clusters
  int64_t n_members = 0;        // offsets[nC]
  int64_t base_K = 0;           // refit-base clusters at the front
  int64_t base_n_r = 0;         // watermark of the base (0 = none)
  int64_t first_window = 0;     // first window sealed after the base
  std::vector<Version> versions;
};

struct ProfRec {
  int phase;
  cudaEvent_t a, b;
};

struct Checkpoint {
  bool valid = false;
  int64_t n_keys = 0, n_windows = 0, n_refits = 0, refit_n_old = 0, n_codes_bf16 = 0;
  int active = 0;
  Buffer meta[2];
};

}  // namespace

struct ai_index {
  ai_config cfg{};
  int cap = 0, iters = 10, n_seed_default = 0, seed_window_default = 0;
  int esize = 0;
  int num_sms = 148;
  cudaStream_t main = nullptr, side = nullptr;
  cudaEvent_t ev_main = nullptr, ev_refit = nullptr;
  // ev_main was recorded before this ai_seal call's seal kernels: a refit it
  // triggers needs only the appended keys and the published buffers, so it
  // may run beside the seal
  bool refit_ev_early = false;
  // key store
  void* keys = nullptr;
  float* scales = nullptr;
  int64_t n_keys = 0;
  uint16_t* codes_bf16 = nullptr;  // bf16 copy of fp8 codes (exhaustive GEMM)
  int64_t n_codes_bf16 = 0;
  // clusters
  int64_t maxC = 0, maxC_pad = 0;
  Buffer buf[2];
  int active = 0;
  int64_t n_windows = 0;
  int64_t n_refits = 0;
  int64_t refit_n_old = 0;  // keys [S, refit_n_old) carry bounds
  // pending refit
  bool pending = false;
  int pending_buf = 0;
  int64_t pending_n_r = 0, pending_K = 0;
  // refit scratch
  int32_t* assign = nullptr;
  float* ub = nullptr;
  float* lb = nullptr;
  double* cent_old = nullptr;
  float* cent32 = nullptr;
  double* drift = nullptr;
  float* seed_lb = nullptr;
  int32_t* counts = nullptr;
  int32_t* tile_counts = nullptr;
  int64_t max_tiles = 0;
  int32_t* scan_list = nullptr;
  int32_t* scan_words = nullptr;
  uint16_t* cent_hi = nullptr;  // tensor-core refit scan (bf16 keys, d = 128)
  uint16_t* cent_lo = nullptr;
  float* cent_cc = nullptr;
  int32_t* cand_scratch = nullptr;  // tensor-core refine: candidate lists, 4 per SM
  float* topk_scores = nullptr;      // tensor-core refine: scores for the output ordering [max_query_chunk, max_k]
  int32_t* split_ids = nullptr;      // split refine of small chunks: partial top-k [2 * num_sms, max_k]
  float* split_sc = nullptr;
  int refine_kernel = 0;             // tensor-core refine variant (0 = by occupancy)
  int refine_split = 0;              // parts per query of a small chunk (0 = by chunk size, 1 = none)
  int32_t* upd_chunk_off = nullptr;  // refit update chunks
  double* upd_part = nullptr;
  float* band_best = nullptr;  // near-tie bands of the tensor-core refit scan
  int32_t* band_ids = nullptr;
  int32_t* band_cnt = nullptr;
  int band_cap = 0;
  int64_t* seeds_dev = nullptr;
  int64_t* seeds_host = nullptr;   // pinned
  int32_t* nscan_host = nullptr;   // pinned [2]
  int64_t max_seeds = 0;
  // route / exhaustive scratch
  float* route = nullptr;          // [max_query_chunk, maxC_pad]
  uint32_t* route_kmin = nullptr;  // [max_query_chunk, 4] route score range partials (tensor-core route)
  uint32_t* route_kmax = nullptr;
  bool route_range = false;        // the last route call filled route_kmin / route_kmax
  float* exh = nullptr;            // [exh_rows, exh_ld]
  int64_t exh_rows = 0, exh_ld = 0;
  int* err_dev = nullptr;
  int* err_host = nullptr;         // pinned
  float* enc_wts = nullptr;
  double* phi = nullptr;           // [max_keys, d] encoder transform per key (encoder only)
  // phase timing (CUDA events on the launching stream)
  bool prof = false;
  std::vector<ProfRec> recs;
  std::vector<cudaEvent_t> ev_pool;
  double prof_ms[AI_N_PHASES] = {};
  int64_t prof_n[AI_N_PHASES] = {};
  // checkpoint copies of the per-key bounds
  Checkpoint ck;
  int32_t* ck_assign = nullptr;
  float* ck_ub = nullptr;
  float* ck_lb = nullptr;
  double* ck_drift = nullptr;  // the next refit's bounds read the last drifts
};

namespace {

int64_t round_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }

cudaEvent_t pool_event(ai_index* h) {
  if (!h->ev_pool.empty()) {
    cudaEvent_t e = h->ev_pool.back();
    h->ev_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

// Open / close a timed phase on stream st (no-op unless profiling is on).
int prof_begin(ai_index* h, int phase, cudaStream_t st) {
  if (!h->prof) return -1;
  ProfRec r{phase, pool_event(h), pool_event(h)};
  cudaEventRecord(r.a, st);
  h->recs.push_back(r);
  return static_cast<int>(h->recs.size()) - 1;
}
void prof_end(ai_index* h, int idx, cudaStream_t st) {
  if (idx >= 0) cudaEventRecord(h->recs[idx].b, st);
}

bool tc_route(const ai_index* h) {
  return h->cfg.q_dtype == AI_BF16 && h->cfg.d == 128 && (h->cfg.H == 32 || h->cfg.H == 64);
}
bool tc_keys(const ai_index* h) {
  return tc_route(h) && (h->cfg.key_dtype == AI_BF16 || h->cfg.key_dtype == AI_FP8E4M3);
}

template <class T>
cudaError_t dalloc(T** p, size_t count) {
  return cudaMalloc(reinterpret_cast<void**>(p), std::max<size_t>(count, 1) * sizeof(T));
}

// Route GEMM: cluster scores [T, nC] into h->route (ld maxC_pad).
int route_scores(ai_index* h, const void* q, const float* w, int T, int64_t nC) {
  const Buffer& b = h->buf[h->active];
  ScoreArgs sa{};
  sa.nA = static_cast<int>(nC);
  sa.T = T;
  sa.w = w;
  sa.row_scale = nullptr;
  sa.out = h->route;
  sa.ld_out = h->maxC_pad;
  sa.causal = 0;
  sa.err = h->err_dev;
  if (tc_route(h)) {
    CUtensorMap ma, mb;
    if (!make_map(&ma, b.reps, nC, 128) || !make_map(&mb, q, static_cast<int64_t>(T) * h->cfg.H, 256))
      return fail(AI_ERR_CUDA, "tensor map encoding failed (route)");
    const int apc = scores_tiles_per_item(nC, T, h->cfg.H, h->num_sms);
    // per-query score range, collected by the GEMM's epilogue (the candidate
    // build bins the scores over it)
    sa.row_kmin = h->route_kmin;
    sa.row_kmax = h->route_kmax;
    const int pi = prof_begin(h, AI_PHASE_ROUTE, h->main);
    if (apc < (nC + 127) / 128) {  // several items per query: atomic slots, pre-set
      CK(cudaMemsetAsync(h->route_kmin, 0xff, static_cast<size_t>(T) * 16, h->main));
      CK(cudaMemsetAsync(h->route_kmax, 0, static_cast<size_t>(T) * 16, h->main));
    }
    CK(launch_scores_tc(ma, mb, h->cfg.H, sa, static_cast<int>(apc), h->main));
    prof_end(h, pi, h->main);
    h->route_range = true;
  } else {
    h->route_range = false;
    const int pi = prof_begin(h, AI_PHASE_ROUTE, h->main);
    CK(launch_scores_simt(b.reps, KD_BF16, q, h->cfg.q_dtype == AI_BF16, h->cfg.d, h->cfg.H, sa, h->main));
    prof_end(h, pi, h->main);
  }
  return AI_OK;
}

int build_version_table(const ai_index* h, int64_t pos0, int T, VersionTable* vt) {
  const Buffer& b = h->buf[h->active];
  std::vector<VersionSeg> segs;
  segs.push_back(VersionSeg{INT64_MIN, h->cfg.n_sinks, 0, 0});
  for (const Version& v : b.versions) segs.push_back(VersionSeg{v.n_v - 1, v.n_v, static_cast<int32_t>(v.nC), 0});
  size_t first = 0;
  for (size_t i = 0; i < segs.size(); ++i)
    if (segs[i].first_pos <= pos0) first = i;
  size_t last = first;
  for (size_t i = first; i < segs.size(); ++i)
    if (segs[i].first_pos <= pos0 + T - 1) last = i;
  const size_t n = last - first + 1;
  if (n > static_cast<size_t>(kMaxSegs))
    return fail(AI_ERR_ARG, "too many index versions inside one query chunk; use a smaller T");
  vt->n = static_cast<int>(n);
  for (size_t i = 0; i < n; ++i) vt->seg[i] = segs[first + i];
  if (vt->n > 0) vt->seg[0].first_pos = INT64_MIN;
  return AI_OK;
}

int check_queries(const ai_index* h, const void* q, const float* w, int64_t pos0, int T, int k) {
  if (!q || !w) return fail(AI_ERR_ARG, "null query or weight pointer");
  if (tc_route(h) && (reinterpret_cast<uintptr_t>(q) % 16 != 0 || reinterpret_cast<uintptr_t>(w) % 16 != 0))
    return fail(AI_ERR_ARG, "q_dev and w_dev must be 16-byte aligned (bf16 queries)");
  if (T <= 0 || T > h->cfg.max_query_chunk) return fail(AI_ERR_ARG, "T out of range");
  if (k <= 0 || k > h->cfg.max_k) return fail(AI_ERR_ARG, "k out of range");
  if (pos0 < 0) return fail(AI_ERR_ARG, "negative pos0");
  if (pos0 + T > h->n_keys)
    return fail(AI_ERR_CAUSALITY, "query positions beyond the appended keys");
  return AI_OK;
}

int publish(ai_index* h) {
  if (!h->pending) return AI_OK;
  const int pp = prof_begin(h, AI_PHASE_PUBLISH, h->main);
  CK(cudaStreamWaitEvent(h->main, h->ev_refit, 0));
  Buffer& A = h->buf[h->active];
  Buffer& B = h->buf[h->pending_buf];
  const int64_t S = h->cfg.n_sinks, W = h->cfg.window, m = h->cfg.clusters_per_window;
  const int64_t n_r = h->pending_n_r;
  const int64_t K = h->pending_K;
  const int64_t w_r = (n_r - S) / W;  // windows covered by the refit
  const int64_t tail_w = h->n_windows - w_r;
  B.nC = K;
  B.n_members = n_r - S;
  B.base_K = K;
  B.base_n_r = n_r;
  B.first_window = w_r;
  B.versions.clear();
  B.versions.push_back(Version{K, n_r});
  if (tail_w > 0) {
    const int64_t c0 = A.base_K + (w_r - A.first_window) * m;
    const int64_t src_mem0 = (A.base_n_r > 0 ? A.base_n_r - S : 0) + (w_r - A.first_window) * W;
    const int64_t nc = tail_w * m;
    const int64_t d = h->cfg.d;
    if (c0 < 0 || c0 + nc > A.nC) return fail(AI_ERR_STATE, "internal: bad tail range at publish");
    CK(cudaMemcpyAsync(B.centroids + K * d, A.centroids + c0 * d, nc * d * sizeof(double),
                       cudaMemcpyDeviceToDevice, h->main));
    CK(cudaMemcpyAsync(B.reps + K * d, A.reps + c0 * d, nc * d * sizeof(uint16_t),
                       cudaMemcpyDeviceToDevice, h->main));
    CK(cudaMemcpyAsync(B.members + B.n_members, A.members + src_mem0, tail_w * W * sizeof(int32_t),
                       cudaMemcpyDeviceToDevice, h->main));
    const int n = static_cast<int>(nc + 1);
    count_launch();
    k_shift_offsets<<<(n + 255) / 256, 256, 0, h->main>>>(A.offsets + c0, B.offsets + K, n,
                                                           static_cast<int32_t>(B.n_members - src_mem0));
    CK(cudaGetLastError());
    for (int64_t w = w_r; w < h->n_windows; ++w)
      B.versions.push_back(Version{K + (w - w_r + 1) * m, S + (w + 1) * W});
    B.nC = K + nc;
    B.n_members += tail_w * W;
  }
  prof_end(h, pp, h->main);
  h->active = h->pending_buf;
  h->pending = false;
  return AI_OK;
}

// Refit over the keys of the first `windows_r` sealed windows (all sealed
// windows when negative).  Windows sealed beyond them stay in the published
// buffer and are carried behind the new base at publication.
int start_refit(ai_index* h, int64_t n_seed, int64_t seed_window, int64_t windows_r = -1) {
  const bool early = h->refit_ev_early && !h->pending;
  h->refit_ev_early = false;
  int rc = publish(h);
  if (rc) return rc;
  const int64_t S = h->cfg.n_sinks, W = h->cfg.window;
  const int64_t n_r = S + (windows_r >= 0 ? windows_r : h->n_windows) * W;
  if (n_r <= S) return AI_OK;
  Buffer& A = h->buf[h->active];
  const int target = 1 - h->active;
  Buffer& B = h->buf[target];
  const int64_t K_prev = A.base_K;
  const int64_t lo = std::max<int64_t>(S, n_r - seed_window);
  std::vector<int64_t> ids = seed_ids(h->cfg.seed, static_cast<uint64_t>(h->n_refits), lo, n_r, n_seed);
  const int64_t ns = static_cast<int64_t>(ids.size());
  const int64_t K = K_prev + ns;
  if (K > h->maxC) return fail(AI_ERR_OOM, "cluster capacity exceeded at refit");
  if (ns > h->max_seeds) return fail(AI_ERR_ARG, "too many refit seeds");
  cudaStream_t st = h->cfg.async_refit ? h->side : h->main;
  // the target buffer was last read by work on the main stream before the
  // event (route/refine of earlier chunks, the publish copy)
  if (!early) CK(cudaEventRecord(h->ev_main, h->main));
  CK(cudaStreamWaitEvent(st, h->ev_main, 0));
  if (ns > 0) {
    // the pinned staging buffer may still be read by an earlier refit's copy
    CK(cudaStreamSynchronize(st));
    std::memcpy(h->seeds_host, ids.data(), ns * sizeof(int64_t));
    CK(cudaMemcpyAsync(h->seeds_dev, h->seeds_host, ns * sizeof(int64_t), cudaMemcpyHostToDevice, st));
  }
  RefitArgs ra{};
  ra.keys = h->keys;
  ra.key_scale = h->scales;
  ra.key_dtype = h->cfg.key_dtype == AI_FP8E4M3 ? KD_FP8 : (h->cfg.key_dtype == AI_BF16 ? KD_BF16 : KD_FP32);
  ra.d = h->cfg.d;
  ra.S = S;
  ra.n_r = n_r;
  ra.n_old = h->refit_n_old;
  ra.K_prev = static_cast<int>(K_prev);
  ra.K = static_cast<int>(K);
  ra.seed_ids = h->seeds_dev;
  ra.prev_centroids = A.centroids;
  ra.cent = B.centroids;
  ra.cent32 = h->cent32;
  ra.cent_old = h->cent_old;
  ra.assign = h->assign;
  ra.ub = h->ub;
  ra.lb = h->lb;
  ra.counts = h->counts;
  ra.offsets = B.offsets;
  ra.members = B.members;
  ra.reps = B.reps;
  ra.drift = h->drift;
  ra.seed_lb = h->seed_lb;
  ra.tile_counts = h->tile_counts;
  ra.scan_list = h->scan_list;
  ra.n_scan = h->scan_words;
  ra.cent_hi = h->cent_hi;
  ra.cent_lo = h->cent_lo;
  ra.cent_cc = h->cent_cc;
  ra.upd_chunk_off = h->upd_chunk_off;
  ra.upd_part = h->upd_part;
  ra.band_best = h->band_best;
  ra.band_ids = h->band_ids;
  ra.band_cnt = h->band_cnt;
  ra.band_cap = h->band_cap;
  ra.err = h->err_dev;
  RefitTcMaps tcm{};
  const bool tc = h->cent_hi != nullptr;
  if (tc) {
    const int64_t K_pad = round_up(K, 128);
    // bf16 keys, or for fp8 keys the bf16 copy of the codes (kept current at append)
    const void* rows = h->cfg.key_dtype == AI_FP8E4M3 ? static_cast<const void*>(h->codes_bf16) : h->keys;
    if (!rows || !make_map(&tcm.keys, rows, n_r, 1) || !make_map(&tcm.hi, h->cent_hi, K_pad, 128) ||
        !make_map(&tcm.lo, h->cent_lo, K_pad, 128))
      return fail(AI_ERR_CUDA, "tensor map encoding failed (refit)");
    tcm.num_sms = h->num_sms;
  }
  const int pr = prof_begin(h, AI_PHASE_REFIT, st);
  CK(launch_refit(ra, h->max_tiles, st, h->nscan_host, tc ? &tcm : nullptr));
  if (h->enc_wts) {
    EncoderArgs ea{};
    ea.keys = h->keys;
    ea.key_scale = h->scales;
    ea.key_dtype = ra.key_dtype;
    ea.d = h->cfg.d;
    ea.offsets = B.offsets;
    ea.members = B.members;
    ea.centroids = B.centroids;
    ea.cl_begin = 0;
    ea.cl_end = static_cast<int>(K);
    ea.wts = h->enc_wts;
    ea.phi = h->phi;
    ea.reps = B.reps;
    ea.err = h->err_dev;
    CK(launch_encoder(ea, st));
  }
  prof_end(h, pr, st);
  CK(cudaEventRecord(h->ev_refit, st));
  h->pending = true;
  h->pending_buf = target;
  h->pending_n_r = n_r;
  h->pending_K = K;
  h->refit_n_old = n_r;
  h->n_refits += 1;
  return AI_OK;
}

int seal_group(ai_index* h, int64_t w0, int64_t nw) {
  Buffer& A = h->buf[h->active];
  const int64_t S = h->cfg.n_sinks, W = h->cfg.window, m = h->cfg.clusters_per_window;
  if (A.nC + nw * m > h->maxC) return fail(AI_ERR_OOM, "cluster capacity exceeded at seal");
  SealArgs sa{};
  sa.keys = h->keys;
  sa.key_scale = h->scales;
  sa.key_dtype = h->cfg.key_dtype == AI_FP8E4M3 ? KD_FP8 : (h->cfg.key_dtype == AI_BF16 ? KD_BF16 : KD_FP32);
  sa.d = h->cfg.d;
  sa.W = static_cast<int>(W);
  sa.m = static_cast<int>(m);
  sa.cap = h->cap;
  sa.iters = h->iters;
  sa.blocks = h->cfg.block_routing;
  sa.first_key = S + w0 * W;
  sa.n_windows = static_cast<int>(nw);
  sa.members = A.members;
  sa.mem_base = A.n_members;
  sa.offsets = A.offsets;
  sa.cl_base = A.nC;
  sa.centroids = A.centroids;
  sa.reps = A.reps;
  sa.err = h->err_dev;
  const int ps = prof_begin(h, AI_PHASE_SEAL, h->main);
  CK(launch_seal(sa, h->main));
  if (h->enc_wts) {
    EncoderArgs ea{};
    ea.keys = h->keys;
    ea.key_scale = h->scales;
    ea.key_dtype = sa.key_dtype;
    ea.d = h->cfg.d;
    ea.offsets = A.offsets;
    ea.members = A.members;
    ea.centroids = A.centroids;
    ea.cl_begin = static_cast<int>(A.nC);
    ea.cl_end = static_cast<int>(A.nC + nw * m);
    ea.wts = h->enc_wts;
    ea.phi = h->phi;
    ea.reps = A.reps;
    ea.err = h->err_dev;
    CK(launch_encoder(ea, h->main));
  }
  prof_end(h, ps, h->main);
  for (int64_t w = w0; w < w0 + nw; ++w) {
    A.nC += m;
    A.n_members += W;
    A.versions.push_back(Version{A.nC, S + (w + 1) * W});
  }
  h->n_windows += nw;
  return AI_OK;
}

int ensure_codes_bf16(ai_index* h) {
  if (h->cfg.key_dtype != AI_FP8E4M3) return AI_OK;
  if (!h->codes_bf16) CK(dalloc(&h->codes_bf16, static_cast<size_t>(h->cfg.max_keys) * h->cfg.d));
  if (h->n_codes_bf16 < h->n_keys) {
    const int64_t d = h->cfg.d;
    CK(launch_fp8_codes_to_bf16(static_cast<const uint8_t*>(h->keys) + h->n_codes_bf16 * d,
                                h->n_keys - h->n_codes_bf16, static_cast<int>(d),
                                h->codes_bf16 + h->n_codes_bf16 * d, h->main));
    h->n_codes_bf16 = h->n_keys;
  }
  return AI_OK;
}

// exhaustive score rows for queries [qoff, qoff+T) of the call into out
int exhaustive_scores(ai_index* h, const void* q, const float* w, int64_t pos0, int T, float* out,
                      int64_t ld) {
  const int64_t nA = std::min<int64_t>(pos0 + T, h->n_keys);
  ScoreArgs sa{};
  sa.nA = static_cast<int>(nA);
  sa.T = T;
  sa.w = w;
  sa.row_scale = h->cfg.key_dtype == AI_FP8E4M3 ? h->scales : nullptr;
  sa.out = out;
  sa.ld_out = ld;
  sa.causal = 1;
  sa.a_pos0 = 0;
  sa.q_pos0 = pos0;
  sa.err = h->err_dev;
  if (tc_keys(h)) {
    int rc = ensure_codes_bf16(h);
    if (rc) return rc;
    const void* A = h->cfg.key_dtype == AI_FP8E4M3 ? static_cast<const void*>(h->codes_bf16) : h->keys;
    CUtensorMap ma, mb;
    if (!make_map(&ma, A, nA, 128) || !make_map(&mb, q, static_cast<int64_t>(T) * h->cfg.H, 256))
      return fail(AI_ERR_CUDA, "tensor map encoding failed (exhaustive)");
    const int apc = scores_tiles_per_item(nA, T, h->cfg.H, h->num_sms);
    const int pe = prof_begin(h, AI_PHASE_EXH_SCORES, h->main);
    CK(launch_scores_tc(ma, mb, h->cfg.H, sa, static_cast<int>(apc), h->main));
    prof_end(h, pe, h->main);
  } else {
    const int pe = prof_begin(h, AI_PHASE_EXH_SCORES, h->main);
    const int kd = h->cfg.key_dtype == AI_FP8E4M3 ? KD_FP8 : (h->cfg.key_dtype == AI_BF16 ? KD_BF16 : KD_FP32);
    CK(launch_scores_simt(h->keys, kd, q, h->cfg.q_dtype == AI_BF16, h->cfg.d, h->cfg.H, sa, h->main));
    prof_end(h, pe, h->main);
  }
  return AI_OK;
}

}  // namespace

extern "C" {

const char* ai_last_error(void) { return g_err.c_str(); }

int ai_index_create(const ai_config* cfg, void* cuda_stream, ai_handle* out) {
  if (!cfg || !out) return fail(AI_ERR_ARG, "null config or output");
  const ai_config& c = *cfg;
  if (c.d <= 0 || c.d > 1024 || c.d % 8 != 0 || c.H <= 0 || c.H > 64)
    return fail(AI_ERR_ARG, "bad d (a multiple of 8 up to 1024) or H (1..64)");
  if (c.key_dtype < 0 || c.key_dtype > 2) return fail(AI_ERR_ARG, "bad key dtype");
  if (!(c.q_dtype == AI_BF16 || (c.q_dtype == AI_FP32 && c.key_dtype == AI_FP32)))
    return fail(AI_ERR_ARG, "queries must be bf16 (or fp32 with fp32 keys)");
  if (c.key_dtype != AI_FP32 && c.q_dtype == AI_BF16 && !(c.d == 128 && (c.H == 32 || c.H == 64)))
    return fail(AI_ERR_ARG, "bf16/fp8 keys need d = 128 and H in {32, 64}");
  if (c.n_sinks < 0 || c.window <= 0 || c.clusters_per_window <= 0 || c.clusters_per_window > 64)
    return fail(AI_ERR_ARG, "bad sinks / window / clusters per window");
  if (c.refit_period < 0 || (c.refit_period > 0 && c.refit_period % c.window != 0))
    return fail(AI_ERR_ARG, "refit period must be a multiple of the window");
  if (c.block_routing != 0 && c.block_routing != 1) return fail(AI_ERR_ARG, "block_routing must be 0 or 1");
  if (c.block_routing && (c.refit_period != 0 || c.encoder_weights_host))
    return fail(AI_ERR_ARG, "block routing takes no refit and no encoder");
  if ((c.refit_period > 0 || c.encoder_weights_host) && c.d > 128)
    return fail(AI_ERR_ARG, "refit and the correction encoder support d <= 128");
  if (c.max_keys <= 0 || c.max_keys >= (int64_t(1) << 31)) return fail(AI_ERR_ARG, "bad max_keys");
  if (c.max_query_chunk <= 0 || c.max_budget <= 0 || c.max_k <= 0) return fail(AI_ERR_ARG, "bad maxima");
  int cap = c.cluster_cap > 0 ? c.cluster_cap : (c.window + c.clusters_per_window - 1) / c.clusters_per_window;
  if (static_cast<int64_t>(cap) * c.clusters_per_window < c.window)
    return fail(AI_ERR_ARG, "cluster_cap * m < W: a window cannot be sealed");
  if (seal_smem_bytes(c.window, c.clusters_per_window, c.d) > 227 * 1024 ||
      static_cast<int64_t>(c.window) * c.clusters_per_window > 65535 || c.window > 32767 ||
      c.clusters_per_window > 64)
    return fail(AI_ERR_ARG, "window too large to seal in one CTA");
  const bool tcr = c.q_dtype == AI_BF16 && c.d == 128 && (c.H == 32 || c.H == 64);
  const bool tck = tcr && c.key_dtype != AI_FP32;
  if (refine_smem_bytes(c.max_budget, c.H, c.d, tck) > 227 * 1024)
    return fail(AI_ERR_ARG, "max_budget too large for the per-query kernel");
  if (tck && c.max_k > kTcMaxK) return fail(AI_ERR_ARG, "k above 2048 is not supported for bf16/fp8 keys");
  if (!tck && c.max_k > kRowTopkMaxK) return fail(AI_ERR_ARG, "k above 4096 is not supported for fp32 keys");

  ai_index* h = new ai_index();
  h->cfg = c;
  h->cap = cap;
  h->iters = c.seal_iters > 0 ? c.seal_iters : 10;
  h->n_seed_default = c.refit_new_seeds > 0 ? c.refit_new_seeds
                      : (c.refit_period > 0 ? static_cast<int>(static_cast<int64_t>(c.refit_period) * c.clusters_per_window / c.window) : 0);
  h->seed_window_default = c.refit_seed_window > 0 ? c.refit_seed_window : c.refit_period;
  h->esize = c.key_dtype == AI_FP32 ? 4 : (c.key_dtype == AI_BF16 ? 2 : 1);
  h->main = static_cast<cudaStream_t>(cuda_stream);
  auto bail = [&](int code, const std::string& msg) {
    ai_index_destroy(h);
    return fail(code, msg);
  };
#define CKC(call)                                                                     \
  do {                                                                                \
    cudaError_t e_ = (call);                                                          \
    if (e_ != cudaSuccess) return bail(e_ == cudaErrorMemoryAllocation ? AI_ERR_OOM : AI_ERR_CUDA, \
                                       std::string(#call) + ": " + cudaGetErrorString(e_)); \
  } while (0)
  int dev = 0;
  CKC(cudaGetDevice(&dev));
  CKC(cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, dev));
  CKC(cudaStreamCreateWithFlags(&h->side, cudaStreamNonBlocking));
  CKC(cudaEventCreateWithFlags(&h->ev_main, cudaEventDisableTiming));
  CKC(cudaEventCreateWithFlags(&h->ev_refit, cudaEventDisableTiming));
  const int64_t N = c.max_keys, d = c.d;
  CKC(cudaMalloc(&h->keys, static_cast<size_t>(N) * d * h->esize));
  if (c.key_dtype == AI_FP8E4M3) CKC(dalloc(&h->scales, N));
  const int64_t windows = N / c.window + 1;
  const int64_t refits = c.refit_period > 0 ? N / c.refit_period + 2 : 2;
  h->max_seeds = std::max<int64_t>(h->n_seed_default, 1024);
  h->maxC = windows * c.clusters_per_window + refits * std::max<int64_t>(h->n_seed_default, 1) + 4096;
  h->maxC_pad = round_up(h->maxC, 128);
  for (int i = 0; i < 2; ++i) {
    Buffer& b = h->buf[i];
    CKC(dalloc(&b.offsets, h->maxC + 1));
    CKC(dalloc(&b.members, N));
    CKC(dalloc(&b.centroids, static_cast<size_t>(h->maxC) * d));
    CKC(dalloc(&b.reps, static_cast<size_t>(h->maxC_pad) * d));
    CKC(cudaMemset(b.reps, 0, static_cast<size_t>(h->maxC_pad) * d * 2));
    CKC(cudaMemset(b.offsets, 0, (h->maxC + 1) * 4));
  }
  CKC(dalloc(&h->assign, N));
  CKC(dalloc(&h->ub, N));
  CKC(dalloc(&h->lb, N));
  CKC(dalloc(&h->cent_old, static_cast<size_t>(h->maxC) * d));
  CKC(dalloc(&h->cent32, static_cast<size_t>(h->maxC) * d));
  CKC(dalloc(&h->drift, h->maxC));
  CKC(dalloc(&h->seed_lb, h->maxC));
  CKC(dalloc(&h->counts, h->maxC));
  h->max_tiles = (N + refit_tile_size() - 1) / refit_tile_size();
  CKC(dalloc(&h->tile_counts, static_cast<size_t>(h->max_tiles) * h->maxC));
  CKC(dalloc(&h->scan_list, 2 * static_cast<size_t>(N)));
  CKC(dalloc(&h->scan_words, 16));
  // one candidate row per refine CTA (at most 4 per SM)
  if (tck) CKC(dalloc(&h->cand_scratch, static_cast<size_t>(h->num_sms) * 4 * c.max_budget));
  if (tck) CKC(dalloc(&h->topk_scores, static_cast<size_t>(c.max_query_chunk) * c.max_k));
  if (tck) CKC(dalloc(&h->split_ids, static_cast<size_t>(2 * h->num_sms) * c.max_k));
  if (tck) CKC(dalloc(&h->split_sc, static_cast<size_t>(2 * h->num_sms) * c.max_k));
  if (tcr) CKC(dalloc(&h->route_kmin, static_cast<size_t>(c.max_query_chunk) * 4));
  if (tcr) CKC(dalloc(&h->route_kmax, static_cast<size_t>(c.max_query_chunk) * 4));
  CKC(dalloc(&h->upd_chunk_off, h->maxC + 1));
  CKC(dalloc(&h->upd_part, static_cast<size_t>(N / refit_update_chunk() + h->maxC + 1) * d));
  if ((c.key_dtype == AI_BF16 || c.key_dtype == AI_FP8E4M3) && d == 128 && c.refit_period > 0) {
    CKC(dalloc(&h->cent_hi, static_cast<size_t>(h->maxC_pad) * 128));
    CKC(dalloc(&h->cent_lo, static_cast<size_t>(h->maxC_pad) * 128));
    CKC(dalloc(&h->cent_cc, h->maxC_pad));
    h->band_cap = static_cast<int>(std::max<int64_t>(4096, N / 16));
    CKC(dalloc(&h->band_best, h->band_cap));
    CKC(dalloc(&h->band_ids, static_cast<size_t>(h->band_cap) * 16));
    CKC(dalloc(&h->band_cnt, h->band_cap));
  }
  CKC(dalloc(&h->seeds_dev, h->max_seeds));
  CKC(cudaMallocHost(&h->seeds_host, h->max_seeds * sizeof(int64_t)));
  CKC(cudaMallocHost(&h->nscan_host, 2 * sizeof(int32_t)));
  h->nscan_host[0] = h->nscan_host[1] = 0;
  CKC(dalloc(&h->route, static_cast<size_t>(c.max_query_chunk) * h->maxC_pad));
  CKC(dalloc(&h->err_dev, 1));
  CKC(cudaMemset(h->err_dev, 0, 4));
  CKC(cudaMallocHost(&h->err_host, sizeof(int)));
  if (c.encoder_weights_host) {
    const size_t nw = static_cast<size_t>(d) * d + d + static_cast<size_t>(d) * (3 * d + 1) + d +
                      static_cast<size_t>(d) * d + d;
    CKC(dalloc(&h->enc_wts, nw));
    CKC(cudaMemcpy(h->enc_wts, c.encoder_weights_host, nw * sizeof(float), cudaMemcpyHostToDevice));
    CKC(dalloc(&h->phi, static_cast<size_t>(c.max_keys) * c.d));
    h->cfg.encoder_weights_host = nullptr;
  }
  CKC(cudaDeviceSynchronize());
#undef CKC
  *out = h;
  return AI_OK;
}

int ai_index_destroy(ai_handle h) {
  if (!h) return fail(AI_ERR_ARG, "null handle");
  if (h->main) cudaStreamSynchronize(h->main);
  if (h->side) cudaStreamSynchronize(h->side);
  cudaFree(h->keys);
  cudaFree(h->scales);
  cudaFree(h->codes_bf16);
  for (auto& b : h->buf) {
    cudaFree(b.offsets);
    cudaFree(b.members);
    cudaFree(b.centroids);
    cudaFree(b.reps);
  }
  cudaFree(h->assign);
  cudaFree(h->ub);
  cudaFree(h->lb);
  cudaFree(h->cent_old);
  cudaFree(h->cent32);
  cudaFree(h->cent_hi);
  cudaFree(h->cent_lo);
  cudaFree(h->cent_cc);
  cudaFree(h->cand_scratch);
  cudaFree(h->topk_scores);
  cudaFree(h->split_ids);
  cudaFree(h->split_sc);
  cudaFree(h->route_kmin);
  cudaFree(h->route_kmax);
  cudaFree(h->upd_chunk_off);
  cudaFree(h->upd_part);
  cudaFree(h->band_best);
  cudaFree(h->band_ids);
  cudaFree(h->band_cnt);
  cudaFree(h->drift);
  cudaFree(h->seed_lb);
  cudaFree(h->counts);
  cudaFree(h->tile_counts);
  cudaFree(h->scan_list);
  cudaFree(h->scan_words);
  cudaFree(h->seeds_dev);
  if (h->seeds_host) cudaFreeHost(h->seeds_host);
  if (h->nscan_host) cudaFreeHost(h->nscan_host);
  cudaFree(h->route);
  cudaFree(h->exh);
  cudaFree(h->err_dev);
  if (h->err_host) cudaFreeHost(h->err_host);
  cudaFree(h->enc_wts);
  cudaFree(h->phi);
  cudaFree(h->ck_assign);
  cudaFree(h->ck_ub);
  cudaFree(h->ck_lb);
  cudaFree(h->ck_drift);
  for (auto& r : h->recs) {
    cudaEventDestroy(r.a);
    cudaEventDestroy(r.b);
  }
  for (auto e : h->ev_pool) cudaEventDestroy(e);
  if (h->ev_main) cudaEventDestroy(h->ev_main);
  if (h->ev_refit) cudaEventDestroy(h->ev_refit);
  if (h->side) cudaStreamDestroy(h->side);
  delete h;
  return AI_OK;
}

int ai_append_keys(ai_handle h, const void* keys_dev, const float* scales_dev, int64_t n) {
  if (!h || (!keys_dev && n > 0) || n < 0) return fail(AI_ERR_ARG, "bad append arguments");
  if (h->cfg.key_dtype == AI_FP8E4M3 && !scales_dev && n > 0) return fail(AI_ERR_ARG, "fp8 keys need scales");
  if (h->n_keys + n > h->cfg.max_keys) return fail(AI_ERR_OOM, "key store full");
  int rc = publish(h);
  if (rc) return rc;
  if (n == 0) return AI_OK;
  const size_t row = static_cast<size_t>(h->cfg.d) * h->esize;
  CK(cudaMemcpyAsync(static_cast<uint8_t*>(h->keys) + h->n_keys * row, keys_dev, n * row,
                     cudaMemcpyDeviceToDevice, h->main));
  if (h->cfg.key_dtype == AI_FP8E4M3)
    CK(cudaMemcpyAsync(h->scales + h->n_keys, scales_dev, n * sizeof(float), cudaMemcpyDeviceToDevice, h->main));
  if (h->phi) {
    const int kd = h->cfg.key_dtype == AI_FP8E4M3 ? KD_FP8 : (h->cfg.key_dtype == AI_BF16 ? KD_BF16 : KD_FP32);
    CK(launch_phi(h->keys, h->scales, kd, h->cfg.d, h->enc_wts, h->n_keys, h->n_keys + n, h->phi, h->main));
  }
  h->n_keys += n;
  // the tensor-core refit screen reads fp8 keys through their bf16 copy
  if (h->cfg.key_dtype == AI_FP8E4M3 && h->cent_hi) return ensure_codes_bf16(h);
  return AI_OK;
}

int ai_seal(ai_handle h, int64_t* version_out) {
  if (!h) return fail(AI_ERR_ARG, "null handle");
  const int64_t S = h->cfg.n_sinks, W = h->cfg.window, R = h->cfg.refit_period;
  const int64_t complete = h->n_keys >= S ? (h->n_keys - S) / W : 0;
  h->refit_ev_early = false;
  if (R > 0 && h->cfg.async_refit && h->n_windows < complete &&
      R / W - (h->n_windows % (R / W)) <= complete - h->n_windows) {
    CK(cudaEventRecord(h->ev_main, h->main));
    h->refit_ev_early = true;
  }
  // every complete window in one launch (windows are independent); a refit
  // whose boundary falls among them reads only keys, so it starts after the
  // launch with the boundary's watermark
  const int64_t w0 = h->n_windows;
  if (complete > w0) {
    int rc = seal_group(h, w0, complete - w0);
    if (rc == AI_OK && R > 0) {
      const int64_t per = R / W;
      for (int64_t wb = (w0 / per + 1) * per; rc == AI_OK && wb <= complete; wb += per)
        rc = start_refit(h, h->n_seed_default, h->seed_window_default, wb);
    }
    if (rc) {
      h->refit_ev_early = false;
      return rc;
    }
  }
  h->refit_ev_early = false;
  if (version_out) *version_out = static_cast<int64_t>(h->buf[h->active].versions.size());
  return AI_OK;
}

int ai_refit(ai_handle h, int32_t n_new_seeds, int32_t seed_window, int64_t* version_out) {
  if (!h || n_new_seeds < 0 || seed_window < 0) return fail(AI_ERR_ARG, "bad refit arguments");
  h->refit_ev_early = false;
  int rc = start_refit(h, n_new_seeds > 0 ? n_new_seeds : h->n_seed_default,
                       seed_window > 0 ? seed_window : h->seed_window_default);
  if (rc) return rc;
  if (version_out) *version_out = static_cast<int64_t>(h->buf[h->active].versions.size());
  return AI_OK;
}

int ai_publish(ai_handle h) {
  if (!h) return fail(AI_ERR_ARG, "null handle");
  return publish(h);
}

// Parts per query of a chunk on the pipelined refine.  A chunk with at
// most half as many queries as the kernel's CTAs (two per SM) would leave
// most SMs idle, each query's 128-slot tiles gathered by one CTA; its list
// is divided instead among `split` CTAs (contiguous tile ranges, at least
// two tiles each, at most kMaxSplit parts) and their partial top-k merged.
// The tiles and so every score are the same as undivided.
constexpr int kMaxSplit = 8;
static int refine_split_for(const ai_index* h, int T, int C, int k) {
  const int cap = 2 * h->num_sms;
  if (h->refine_split == 1 || T <= 0 || 2 * T > cap) return 1;
  int S = h->refine_split > 1 ? h->refine_split : kMaxSplit;
  S = std::min(S, cap / T);
  S = std::min(S, ((C + 127) / 128) / 2);
  while (S > 1 && merge_smem_bytes(S, k) > 227 * 1024) --S;
  return S < 2 ? 1 : S;
}

static int route_refine_impl(ai_handle h, const void* q, const float* w, int64_t pos0, int T, int k,
                             int C, int32_t* out, float* out_scores, int32_t* cand_out,
                             float* cluster_scores_out, int shard = 0, int n_shards = 1) {
  int rc = check_queries(h, q, w, pos0, T, k);
  if (rc) return rc;
  if (C <= 0 || C > h->cfg.max_budget) return fail(AI_ERR_ARG, "C out of range");
  VersionTable vt;
  rc = build_version_table(h, pos0, T, &vt);
  if (rc) return rc;
  const Buffer& b = h->buf[h->active];
  const int64_t nC = b.nC;
  if (nC > 0) {
    rc = route_scores(h, q, w, T, nC);
    if (rc) return rc;
  }
  if (cluster_scores_out && nC > 0)
    CK(cudaMemcpy2DAsync(cluster_scores_out, nC * sizeof(float), h->route, h->maxC_pad * sizeof(float),
                         nC * sizeof(float), T, cudaMemcpyDeviceToDevice, h->main));
  RefineArgs ra{};
  ra.keys = h->keys;
  ra.key_scale = h->cfg.key_dtype == AI_FP8E4M3 ? h->scales : nullptr;
  ra.key_dtype = h->cfg.key_dtype == AI_FP8E4M3 ? KD_FP8 : (h->cfg.key_dtype == AI_BF16 ? KD_BF16 : KD_FP32);
  ra.q = q;
  ra.q_is_bf16 = h->cfg.q_dtype == AI_BF16;
  ra.w = w;
  ra.route = h->route;
  ra.ld_route = h->maxC_pad;
  ra.route_kmin = nC > 0 && h->route_range ? h->route_kmin : nullptr;
  ra.route_kmax = nC > 0 && h->route_range ? h->route_kmax : nullptr;
  ra.offsets = b.offsets;
  ra.members = b.members;
  ra.pos0 = pos0;
  ra.T = T;
  ra.H = h->cfg.H;
  ra.d = h->cfg.d;
  ra.k = k;
  ra.C = C;
  ra.n_sinks = h->cfg.n_sinks;
  ra.out = out;
  ra.out_scores = out_scores;
  ra.cand_out = cand_out;
  ra.cand_scratch = h->cand_scratch;
  ra.refine_kernel = h->refine_kernel;
  ra.shard = shard;
  ra.n_shards = n_shards;
  ra.err = h->err_dev;
  int32_t* tmp_out = nullptr;
  if (!out) {  // debug call: outputs still need a home
    CK(cudaMallocAsync(reinterpret_cast<void**>(&tmp_out), static_cast<size_t>(T) * k * 4, h->main));
    ra.out = tmp_out;
  }
  CUtensorMap kmap, qmap;
  const CUtensorMap* kmp = nullptr;
  const CUtensorMap* qmp = nullptr;
  if (tc_keys(h)) {
    // rows gathered by TMA (box 64 x 1): the bf16 key store, or for fp8
    // keys the bf16 copy of the codes (exact; the scale is applied to the
    // score)
    rc = ensure_codes_bf16(h);
    if (rc) return rc;
    const void* rows = h->cfg.key_dtype == AI_BF16 ? h->keys : static_cast<const void*>(h->codes_bf16);
    const bool ok_k = make_map(&kmap, rows, h->n_keys, 1);
    if (!ok_k || !make_map(&qmap, q, static_cast<int64_t>(T) * h->cfg.H, h->cfg.H))
      return fail(AI_ERR_CUDA, "tensor map encoding failed (key store / queries)");
    kmp = &kmap;
    qmp = &qmap;
  }
  // a small chunk on the pipelined refine: each query's list divided among
  // CTAs, the partial top-k merged into the output order
  int split = 1;
  if (tc_keys(h) && !cand_out && out && n_shards <= 1 && h->split_ids) {
    const int kind = h->refine_kernel == REFINE_AUTO
                         ? pick_refine_kernel(C, h->cfg.H, h->cand_scratch != nullptr)
                         : h->refine_kernel;
    if (kind == REFINE_PIPE || kind == REFINE_PIPE_1BUF) split = refine_split_for(h, T, C, k);
  }
  if (split > 1) {
    ra.split = split;
    ra.out = h->split_ids;
    ra.out_scores = h->split_sc;
    const int pf = prof_begin(h, AI_PHASE_REFINE, h->main);
    CK(launch_refine(ra, vt, kmp, qmp, h->num_sms, h->main));
    prof_end(h, pf, h->main);
    const int po = prof_begin(h, AI_PHASE_ORDER, h->main);
    CK(launch_merge_rows(h->split_ids, h->split_sc, split, T, k, out, out_scores, h->main));
    prof_end(h, po, h->main);
    return AI_OK;
  }
  // the tensor-core refine writes each row's ids (and scores) in slot
  // order; a second kernel puts them in the output order, reading the
  // scores from the caller's buffer or the handle's scratch
  const bool order = tc_keys(h) && !cand_out;
  float* sc_rows = out_scores;
  if (order && !sc_rows) sc_rows = h->topk_scores;
  ra.out_scores = order ? sc_rows : out_scores;
  const int pf = prof_begin(h, AI_PHASE_REFINE, h->main);
  CK(launch_refine(ra, vt, kmp, qmp, h->num_sms, h->main));
  prof_end(h, pf, h->main);
  if (order) {
    OrderRowsArgs oa{ra.out, sc_rows, ra.out, out_scores, T, k};
    const int po = prof_begin(h, AI_PHASE_ORDER, h->main);
    CK(launch_order_rows(oa, h->main));
    prof_end(h, po, h->main);
  }
  if (tmp_out) CK(cudaFreeAsync(tmp_out, h->main));
  return AI_OK;
}

int ai_route_refine(ai_handle h, const void* q_dev, const float* w_dev, int64_t pos0, int32_t T,
                    int32_t k, int32_t C, int32_t* out_dev, float* out_scores_dev) {
  if (!h || !out_dev) return fail(AI_ERR_ARG, "null handle or output");
  return route_refine_impl(h, q_dev, w_dev, pos0, T, k, C, out_dev, out_scores_dev, nullptr, nullptr);
}

int ai_route_refine_shard(ai_handle h, const void* q_dev, const float* w_dev, int64_t pos0, int32_t T,
                          int32_t k, int32_t C, int32_t shard, int32_t n_shards, int32_t* out_dev,
                          float* out_scores_dev) {
  if (!h || !out_dev || !out_scores_dev) return fail(AI_ERR_ARG, "null handle or output");
  if (n_shards < 1 || shard < 0 || shard >= n_shards) return fail(AI_ERR_ARG, "bad shard");
  if (n_shards > 1 && !tc_keys(h)) return fail(AI_ERR_ARG, "sharded rescore needs bf16 or fp8 keys");
  if (n_shards > 1 && h->refine_kernel != REFINE_AUTO && h->refine_kernel != REFINE_PIPE &&
      h->refine_kernel != REFINE_PIPE_1BUF)
    return fail(AI_ERR_ARG, "sharded rescore runs on the pipelined refine kernels only");
  return route_refine_impl(h, q_dev, w_dev, pos0, T, k, C, out_dev, out_scores_dev, nullptr, nullptr, shard,
                           n_shards);
}

int ai_debug_candidates(ai_handle h, const void* q_dev, const float* w_dev, int64_t pos0, int32_t T,
                        int32_t C, int32_t* cand_dev, float* cluster_scores_dev) {
  if (!h || !cand_dev) return fail(AI_ERR_ARG, "null handle or output");
  return route_refine_impl(h, q_dev, w_dev, pos0, T, 1, C, nullptr, nullptr, cand_dev, cluster_scores_dev);
}

int ai_select_exhaustive(ai_handle h, const void* q_dev, const float* w_dev, int64_t pos0, int32_t T,
                         int32_t k, int32_t* out_dev, float* out_scores_dev) {
  if (!h || !out_dev) return fail(AI_ERR_ARG, "null handle or output");
  int rc = check_queries(h, q_dev, w_dev, pos0, T, k);
  if (rc) return rc;
  if (!h->exh) {
    h->exh_ld = round_up(h->cfg.max_keys, 4);
    const int64_t budget = int64_t(4) << 30;  // bytes of score rows per sub-batch
    h->exh_rows = std::max<int64_t>(64, std::min<int64_t>(h->cfg.max_query_chunk, budget / (h->exh_ld * 4)));
    h->exh_rows = round_up(h->exh_rows, 8);
    CK(dalloc(&h->exh, static_cast<size_t>(h->exh_rows) * h->exh_ld));
  }
  const size_t qrow = static_cast<size_t>(h->cfg.H) * h->cfg.d * (h->cfg.q_dtype == AI_BF16 ? 2 : 4);
  for (int64_t b0 = 0; b0 < T; b0 += h->exh_rows) {
    const int tb = static_cast<int>(std::min<int64_t>(h->exh_rows, T - b0));
    const void* qb = static_cast<const uint8_t*>(q_dev) + b0 * qrow;
    const float* wb = w_dev + b0 * h->cfg.H;
    rc = exhaustive_scores(h, qb, wb, pos0 + b0, tb, h->exh, h->exh_ld);
    if (rc) return rc;
    RowTopkArgs ta{};
    ta.scores = h->exh;
    ta.ld = h->exh_ld;
    ta.T = tb;
    ta.q_pos0 = pos0 + b0;
    ta.n_keys = h->n_keys;
    ta.k = k;
    ta.out = out_dev + b0 * k;
    ta.out_scores = out_scores_dev ? out_scores_dev + b0 * k : nullptr;
    ta.err = h->err_dev;
    const int pt = prof_begin(h, AI_PHASE_EXH_TOPK, h->main);
    CK(launch_row_topk(ta, h->main));
    prof_end(h, pt, h->main);
  }
  return AI_OK;
}

int ai_debug_scores(ai_handle h, const void* q_dev, const float* w_dev, int64_t pos0, int32_t T,
                    float* out_dev) {
  if (!h || !out_dev) return fail(AI_ERR_ARG, "null handle or output");
  int rc = check_queries(h, q_dev, w_dev, pos0, T, 1);
  if (rc) return rc;
  const int64_t n = static_cast<int64_t>(T) * h->n_keys;
  count_launch();
  k_fill<<<static_cast<unsigned>(std::min<int64_t>((n + 255) / 256, 65535)), 256, 0, h->main>>>(out_dev, n, -INFINITY);
  CK(cudaGetLastError());
  return exhaustive_scores(h, q_dev, w_dev, pos0, T, out_dev, h->n_keys);
}

int ai_sync(ai_handle h) {
  if (!h) return fail(AI_ERR_ARG, "null handle");
  const auto t0 = std::chrono::steady_clock::now();
  for (cudaStream_t s : {h->main, h->side}) {
    for (;;) {
      cudaError_t e = cudaStreamQuery(s);
      if (e == cudaSuccess) break;
      if (e != cudaErrorNotReady) return fail(AI_ERR_CUDA, std::string("stream: ") + cudaGetErrorString(e));
      if (std::chrono::steady_clock::now() - t0 > std::chrono::seconds(120))
        return fail(AI_ERR_TIMEOUT, "device work did not finish within 120 s");
      std::this_thread::sleep_for(std::chrono::microseconds(50));
    }
  }
  CK(cudaMemcpy(h->err_host, h->err_dev, sizeof(int), cudaMemcpyDeviceToHost));
  const int e = *h->err_host;
  if (e) {
    CK(cudaMemset(h->err_dev, 0, sizeof(int)));
    if (e & DEV_ERR_TIMEOUT) return fail(AI_ERR_TIMEOUT, "a bounded device wait ran out");
    return fail(AI_ERR_DEVICE_CHECK, "device check failed (flags " + std::to_string(e) + ")");
  }
  return AI_OK;
}

int ai_get_stats(ai_handle h, ai_stats* out) {
  if (!h || !out) return fail(AI_ERR_ARG, "null handle or output");
  const Buffer& b = h->buf[h->active];
  out->n_keys = h->n_keys;
  out->n_sealed = h->n_windows;
  out->n_clusters = b.nC;
  out->n_versions = static_cast<int64_t>(b.versions.size());
  out->n_refits = h->n_refits;
  out->refit_pending = h->pending ? 1 : 0;
  out->base_watermark = b.base_n_r;
  out->last_refit_scanned = h->nscan_host ? h->nscan_host[0] : 0;
  out->last_refit_rechecked = h->nscan_host ? h->nscan_host[1] : 0;
  return AI_OK;
}

int ai_export_index(ai_handle h, int32_t* offsets_host, int32_t* members_host, uint16_t* reps_bf16_host,
                    double* centroids_host, int64_t* version_nc_host, int64_t* version_nv_host) {
  if (!h) return fail(AI_ERR_ARG, "null handle");
  CK(cudaStreamSynchronize(h->main));
  const Buffer& b = h->buf[h->active];
  const int64_t d = h->cfg.d;
  if (offsets_host) CK(cudaMemcpy(offsets_host, b.offsets, (b.nC + 1) * 4, cudaMemcpyDeviceToHost));
  if (members_host) CK(cudaMemcpy(members_host, b.members, b.n_members * 4, cudaMemcpyDeviceToHost));
  if (reps_bf16_host) CK(cudaMemcpy(reps_bf16_host, b.reps, b.nC * d * 2, cudaMemcpyDeviceToHost));
  if (centroids_host) CK(cudaMemcpy(centroids_host, b.centroids, b.nC * d * 8, cudaMemcpyDeviceToHost));
  for (size_t i = 0; i < b.versions.size(); ++i) {
    if (version_nc_host) version_nc_host[i] = b.versions[i].nC;
    if (version_nv_host) version_nv_host[i] = b.versions[i].n_v;
  }
  return AI_OK;
}

int ai_checkpoint(ai_handle h) {
  if (!h) return fail(AI_ERR_ARG, "null handle");
  if (h->pending) return fail(AI_ERR_STATE, "checkpoint while a refit is pending");
  const int64_t N = h->cfg.max_keys;
  if (!h->ck_assign) {
    CK(dalloc(&h->ck_assign, N));
    CK(dalloc(&h->ck_ub, N));
    CK(dalloc(&h->ck_lb, N));
    CK(dalloc(&h->ck_drift, h->maxC));
  }
  CK(cudaMemcpyAsync(h->ck_drift, h->drift, h->maxC * sizeof(double), cudaMemcpyDeviceToDevice, h->main));
  Checkpoint& c = h->ck;
  c.valid = true;
  c.n_keys = h->n_keys;
  c.n_windows = h->n_windows;
  c.n_refits = h->n_refits;
  c.refit_n_old = h->refit_n_old;
  c.n_codes_bf16 = h->n_codes_bf16;
  c.active = h->active;
  for (int i = 0; i < 2; ++i) c.meta[i] = h->buf[i];
  if (h->n_keys > 0) {
    CK(cudaMemcpyAsync(h->ck_assign, h->assign, h->n_keys * 4, cudaMemcpyDeviceToDevice, h->main));
    CK(cudaMemcpyAsync(h->ck_ub, h->ub, h->n_keys * 4, cudaMemcpyDeviceToDevice, h->main));
    CK(cudaMemcpyAsync(h->ck_lb, h->lb, h->n_keys * 4, cudaMemcpyDeviceToDevice, h->main));
  }
  return AI_OK;
}

int ai_rollback(ai_handle h) {
  if (!h) return fail(AI_ERR_ARG, "null handle");
  if (!h->ck.valid) return fail(AI_ERR_STATE, "no checkpoint");
  if (h->pending) {  // discard, after it finishes writing
    CK(cudaStreamWaitEvent(h->main, h->ev_refit, 0));
    h->pending = false;
  }
  const Checkpoint& c = h->ck;
  h->n_keys = c.n_keys;
  h->n_windows = c.n_windows;
  h->n_refits = c.n_refits;
  h->refit_n_old = c.refit_n_old;
  h->n_codes_bf16 = std::min(h->n_codes_bf16, c.n_codes_bf16);
  h->active = c.active;
  for (int i = 0; i < 2; ++i) {
    Buffer& b = h->buf[i];
    const Buffer& m = c.meta[i];
    b.nC = m.nC;
    b.n_members = m.n_members;
    b.base_K = m.base_K;
    b.base_n_r = m.base_n_r;
    b.first_window = m.first_window;
    b.versions = m.versions;
  }
  CK(cudaMemcpyAsync(h->drift, h->ck_drift, h->maxC * sizeof(double), cudaMemcpyDeviceToDevice, h->main));
  if (h->n_keys > 0) {
    CK(cudaMemcpyAsync(h->assign, h->ck_assign, h->n_keys * 4, cudaMemcpyDeviceToDevice, h->main));
    CK(cudaMemcpyAsync(h->ub, h->ck_ub, h->n_keys * 4, cudaMemcpyDeviceToDevice, h->main));
    CK(cudaMemcpyAsync(h->lb, h->ck_lb, h->n_keys * 4, cudaMemcpyDeviceToDevice, h->main));
  }
  // the side stream must not start the next refit before the restore lands
  CK(cudaEventRecord(h->ev_main, h->main));
  CK(cudaStreamWaitEvent(h->side, h->ev_main, 0));
  return AI_OK;
}

int ai_debug_refine_kernel(ai_handle h, int32_t kernel) {
  if (!h) return fail(AI_ERR_ARG, "null handle");
  if (kernel < 0 || kernel > 4) return fail(AI_ERR_ARG, "refine kernel must be 0..4");
  h->refine_kernel = kernel;
  return AI_OK;
}

int ai_debug_refine_split(ai_handle h, int32_t split) {
  if (!h) return fail(AI_ERR_ARG, "null handle");
  if (split < 0 || split > kMaxSplit) return fail(AI_ERR_ARG, "refine split must be 0..8");
  h->refine_split = split;
  return AI_OK;
}

int ai_refine_kernel_choice(ai_handle h, int32_t C, int32_t* kernel_out) {
  if (!h || !kernel_out) return fail(AI_ERR_ARG, "null handle or output");
  if (C <= 0 || C > h->cfg.max_budget) return fail(AI_ERR_ARG, "C out of range");
  if (!tc_keys(h)) {
    *kernel_out = 0;
  } else {
    *kernel_out = h->refine_kernel != REFINE_AUTO ? h->refine_kernel
                                                 : pick_refine_kernel(C, h->cfg.H, h->cand_scratch != nullptr);
  }
  return AI_OK;
}

int ai_profile_enable(ai_handle h, int enable) {
  if (!h) return fail(AI_ERR_ARG, "null handle");
  h->prof = enable != 0;
  return AI_OK;
}

int ai_profile_read(ai_handle h, double* ms_out, int64_t* launches_out) {
  if (!h) return fail(AI_ERR_ARG, "null handle");
  CK(cudaStreamSynchronize(h->main));
  CK(cudaStreamSynchronize(h->side));
  for (auto& r : h->recs) {
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, r.a, r.b) == cudaSuccess) {
      h->prof_ms[r.phase] += ms;
      h->prof_n[r.phase] += 1;
    }
    h->ev_pool.push_back(r.a);
    h->ev_pool.push_back(r.b);
  }
  h->recs.clear();
  for (int i = 0; i < AI_N_PHASES; ++i) {
    if (ms_out) ms_out[i] = h->prof_ms[i];
    if (launches_out) launches_out[i] = h->prof_n[i];
    h->prof_ms[i] = 0.0;
    h->prof_n[i] = 0;
  }
  return AI_OK;
}

long long ai_kernel_launches(void) { return aiidx::kernel_launches(); }

int ai_quantize_fp8(const uint16_t* keys_bf16_dev, int64_t n, int32_t d, uint8_t* codes_dev,
                    float* scales_dev, void* cuda_stream) {
  if (n < 0 || d <= 0 || d % 32 != 0 || (n > 0 && (!keys_bf16_dev || !codes_dev || !scales_dev)))
    return fail(AI_ERR_ARG, "bad quantize arguments");
  CK(launch_quantize_fp8(keys_bf16_dev, n, d, codes_dev, scales_dev, static_cast<cudaStream_t>(cuda_stream)));
  return AI_OK;
}

}  // extern "C"
