// Internal launchers of the causal IVF top-k library (not part of the C ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace aiidx {

// Kernel launches made by this library (all handles, all streams).
void count_launch();
long long kernel_launches();
// Message returned by ai_last_error() on this thread.
void set_last_error(const char* msg);

// ---------------------------------------------------------- score matrices
struct ScoreArgs {
  int nA;                  // rows of A
  int T;                   // queries
  const float* w;          // [T, H] head weights
  const float* row_scale;  // [nA] per-row positive scale or nullptr
  float* out;              // out[q * ld_out + a]
  uint32_t* row_kmin;      // [T, 4] per query and TMEM lane quarter: min / max of
  uint32_t* row_kmax;      //   f2key(out[q][a]) over the quarter's rows, or nullptr;
                           //   stored directly when one work item covers every A tile
                           //   (a_tiles_per_cta >= A tiles), else atomic (pre-set to
                           //   0xffffffff / 0)
  int64_t ld_out;
  int a_tiles_per_cta;      // A tiles per work item (tensor-core path)
  int causal;              // mask a_pos0 + a > q_pos0 + q to -inf
  int64_t a_pos0;
  int64_t q_pos0;
  int* err;
};
int scores_smem_bytes();
// A tiles per work item of launch_scores_tc for nA rows, T queries, H heads.
int scores_tiles_per_item(int64_t nA, int T, int H, int num_sms);
cudaError_t launch_scores_tc(const CUtensorMap& mapA, const CUtensorMap& mapB, int H,
                             const ScoreArgs& args, int a_tiles_per_cta, cudaStream_t st);
cudaError_t launch_scores_simt(const void* A, int a_dtype, const void* Q, int q_is_bf16, int d,
                               int H, const ScoreArgs& args, cudaStream_t st);

// --------------------------------------------------------- route + refine
constexpr int kMaxSegs = 64;
struct VersionSeg {
  int64_t first_pos;  // first query position that uses this version
  int64_t n_v;        // open-window start (clustered keys are [S, n_v))
  int32_t nC;         // visible clusters (a prefix of the cluster array)
  int32_t pad;
};
struct VersionTable {
  int n;
  int pad;
  VersionSeg seg[kMaxSegs];
};

struct RefineArgs {
  const void* keys;          // key store [N, d] (fp32 / bf16 / fp8 codes)
  const float* key_scale;    // fp8 per-key scale, else nullptr
  int key_dtype;
  const void* q;             // [T, H, d] (fp32 or bf16)
  int q_is_bf16;
  const float* w;            // [T, H]
  const float* route;        // [T, ld_route] cluster scores
  const uint32_t* route_kmin;  // [T, 4] partial order-preserving keys of the min / max route
  const uint32_t* route_kmax;  //   score over all clusters, or nullptr (then computed here)
  int64_t ld_route;
  const int32_t* offsets;    // CSR offsets [nC + 1]
  const int32_t* members;    // CSR members
  int64_t pos0;
  int T, H, d, k, C, n_sinks;
  int32_t* out;              // [T, k]
  float* out_scores;         // [T, k] or nullptr
  int32_t* cand_out;         // debug: [T, C] candidate lists or nullptr
  int32_t* cand_scratch;     // tensor-core path: candidate lists, [4 * num_sms, C]
  int refine_kernel;         // REFINE_* (tensor-core path; AUTO picks by occupancy)
  int shard, n_shards;       // rescore only this shard's tile range of each list (n_shards <= 1: all)
  int split;                 // pipelined kernels: > 1 divides each list's tiles among `split` work
                             // items; item sp of query i writes row sp * T + i of out / out_scores
                             // ([split, T, k]), to be merged
  int* err;
};
enum RefineKernel {
  REFINE_AUTO = 0,        // chosen by occupancy
  REFINE_SEQ_SMEM = 1,    // one query at a time per CTA, list in shared memory
  REFINE_SEQ_GLOBAL = 2,  // the same, list in global scratch
  REFINE_PIPE = 3,        // pipelined, two TMEM score buffers
  REFINE_PIPE_1BUF = 4    // pipelined, one TMEM score buffer (large budgets)
};
// The variant REFINE_AUTO launches for budget C and H heads (tensor-core path).
int pick_refine_kernel(int C, int H, bool has_scratch);
size_t refine_smem_bytes(int C, int H, int d, bool tc);
// kmap: TMA map of the bf16 key store (box 64 x 1); qmap: TMA map of the
// queries as [T*H, 128] bf16 rows (box 64 x H).  Both nullptr selects the
// SIMT kernel (fp32 keys).  For fp8 keys kmap covers the bf16 copy of the codes.
cudaError_t launch_refine(const RefineArgs& a, const VersionTable& vt, const CUtensorMap* kmap,
                          const CUtensorMap* qmap, int num_sms, cudaStream_t st);

// Largest k of every top-k that sorts its output in shared memory: the
// exhaustive row top-k and the fp32 (SIMT) route+refine.  The tensor-core
// route+refine allows 2048.
constexpr int kRowTopkMaxK = 4096;
constexpr int kTcMaxK = 2048;

// ------------------------------------------------ route+refine output order
// Sorts each row of [T, k] (ids, scores) -- valid entries a prefix, -1
// padding after -- by (score desc, id asc).  In place is allowed
// (ids_out == ids_in, scores_out == scores_in); scores_out may be nullptr.
struct OrderRowsArgs {
  const int32_t* ids_in;
  const float* scores_in;
  int32_t* ids_out;
  float* scores_out;
  int T, k;
};
cudaError_t launch_order_rows(const OrderRowsArgs& a, cudaStream_t st);
// Merge of P partial top-k lists per row, ids / scores [P, T, k] (valid
// entries id >= 0, disjoint ids across parts): the top k of their union by
// (score desc, id asc), written in that order to out / out_scores [T, k]
// and padded with -1 / -inf.  k <= kTcMaxK; shared memory merge_smem_bytes.
size_t merge_smem_bytes(int P, int k);
cudaError_t launch_merge_rows(const int32_t* ids, const float* scores, int P, int T, int k, int32_t* out,
                              float* out_scores, cudaStream_t st);

// ------------------------------------------------------- exhaustive top-k
struct RowTopkArgs {
  const float* scores;  // [T, ld]
  int64_t ld;
  int T;
  int64_t q_pos0;       // query i sees keys [0, q_pos0 + i]
  int64_t n_keys;       // keys in the store
  int k;
  int32_t* out;         // [T, k] (row stride k)
  float* out_scores;    // or nullptr
  int* err;
};
cudaError_t launch_row_topk(const RowTopkArgs& a, cudaStream_t st);

// ------------------------------------------------------------------ seal
struct SealArgs {
  const void* keys;
  const float* key_scale;
  int key_dtype;
  int d, W, m, cap, iters;
  int blocks;               // 1: contiguous blocks with mean representatives (no k-means)
  int64_t first_key;        // window j covers keys [first_key + j W, + W)
  int n_windows;
  int32_t* members;         // output: window j writes members[mem_base + j W ...]
  int64_t mem_base;
  int32_t* offsets;         // output: offsets[cl_base + j m + c] (start of each cluster)
  int64_t cl_base;
  double* centroids;        // [cl_base + j m + c][d]
  uint16_t* reps;           // bf16 [.., d]
  int* err;
};
size_t seal_smem_bytes(int W, int m, int d);
cudaError_t launch_seal(const SealArgs& a, cudaStream_t st);

// ----------------------------------------------------------------- refit
struct RefitArgs {
  const void* keys;
  const float* key_scale;
  int key_dtype;
  int d;
  int64_t S;             // first clustered key
  int64_t n_r;           // refit covers keys [S, n_r)
  int64_t n_old;         // keys [S, n_old) carry bounds from the previous refit
  int K_prev;            // centroids carried from the previous refit
  int K;                 // K_prev + seeds
  const int64_t* seed_ids;  // [K - K_prev] (device)
  const double* prev_centroids;  // [K_prev, d] (device, may alias nothing)
  double* cent;          // [K, d] working centroids (output: updated)
  float* cent32;         // [K, d] fp32 copy for screening
  double* cent_old;      // [K, d] centroids before update (for drift)
  int32_t* assign;       // [N] per key (index = key id)
  float* ub;             // [N] upper bound to own centre
  float* lb;             // [N] lower bound to every other centre
  int32_t* counts;       // [K]
  int32_t* offsets;      // [K + 1] output CSR
  int32_t* members;      // [n_r - S] output CSR members
  uint16_t* reps;        // [K, d] bf16
  double* drift;         // [K]
  float* seed_lb;        // [K_prev] min distance from old centre to any seed
  int32_t* tile_counts;  // scratch [ntiles * K]
  int32_t* scan_list;    // scratch [n_r - S] keys needing a full scan
  int32_t* n_scan;       // scratch [16]
  uint16_t* cent_hi;     // [K_pad, 128] bf16 high parts (tensor-core scan only)
  uint16_t* cent_lo;     // [K_pad, 128] bf16 residuals
  float* cent_cc;        // [K_pad] ||c||^2 (+inf for padding rows)
  int32_t* upd_chunk_off;  // scratch [K + 1] offsets of the update chunks
  double* upd_part;        // scratch [n / 128 + K, d] chunk sums
  float* band_best;        // scratch [band_cap] tensor-core scan: flagged keys' best d^2
  int32_t* band_ids;       // scratch [band_cap, 16] centres within the error band
  int32_t* band_cnt;       // scratch [band_cap]
  int band_cap;
  int* err;
};
// Tensor maps for the tensor-core full scan (bf16 keys, d = 128): keys with a
// one-row box (gather4), centre hi / lo parts with 128-row boxes.
struct RefitTcMaps {
  CUtensorMap keys, hi, lo;
  int num_sms;
};
cudaError_t launch_refit(const RefitArgs& a, int64_t max_tiles, cudaStream_t st,
                         int32_t* host_nscan /*nullable: read back count*/,
                         const RefitTcMaps* tc /*nullable: fp32 SIMT scan*/);
int64_t refit_tile_size();
int64_t refit_update_chunk();  // members per update chunk

// --------------------------------------------------------------- encoder
struct EncoderArgs {
  const void* keys;
  const float* key_scale;
  int key_dtype;
  int d;
  const int32_t* offsets;  // cluster c members offsets[c] .. offsets[c+1]
  const int32_t* members;
  const double* centroids; // [.., d]
  int cl_begin, cl_end;    // clusters to (re)compute
  const float* wts;        // packed A [d,d], a [d], B1 [d, 3d+1], b1 [d], B2 [d,d], b2 [d]
  const double* phi;       // [N, d] cached phi(k) per key (launch_phi), or nullptr
  uint16_t* reps;          // bf16 output
  int* err;
};
cudaError_t launch_encoder(const EncoderArgs& a, cudaStream_t st);
// phi(k_s) = ReLU(A k_s + a) (float64) for keys s in [s0, s1) into phi[s]:
// the per-key transform the encoder pools, computed once when keys arrive.
cudaError_t launch_phi(const void* keys, const float* key_scale, int key_dtype, int d, const float* wts,
                       int64_t s0, int64_t s1, double* phi, cudaStream_t st);

// ---------------------------------------------------------------- formats
cudaError_t launch_quantize_fp8(const uint16_t* keys_bf16, int64_t n, int d, uint8_t* codes,
                                float* scales, cudaStream_t st);
cudaError_t launch_fp8_codes_to_bf16(const uint8_t* codes, int64_t n, int d, uint16_t* out,
                                     cudaStream_t st);

}  // namespace aiidx
