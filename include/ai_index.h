/*
 * ai_index.h - C ABI of the causal IVF top-k key selection library
 * (libai_index.so, sm_100a).
 *
 * What it computes.  For every query of a chunked causal prefill, the top-k
 * keys under the DSA indexer score
 *     I(q, s) = sum_h w_h * ReLU(q_h . k_s),
 * selected through a causal inverted-file index over the indexer keys, as
 * described on the pages titled "AttentionIndex: Accelerating Learned Sparse
 * Attention with a Causal Inverted-File Index" (paper-daily.com explainer;
 * kurate.org review).  Sections cited below are those of the explainer.
 *
 * Conventions for every call.
 *  - Pointers named *_dev are CUDA device pointers owned by the caller; the
 *    library never frees them.  Pointers named *_host are host memory.
 *  - All work is enqueued on the handle's main stream (given at create time)
 *    and is asynchronous unless stated otherwise; call ai_sync() to wait
 *    and to collect device-side error flags.
 *  - Return value: AI_OK (0) or a negative AI_ERR_* code; ai_last_error()
 *    gives a message for the calling thread.  A call that fails leaves the
 *    index unchanged unless stated otherwise.
 *  - Layouts are row-major and dense: keys [n, d], queries [T, H, d],
 *    head weights [T, H] float32, outputs [T, k] int32.  With bf16 queries
 *    the query and head-weight pointers must be 16-byte aligned (they are
 *    read by bulk tensor copies); AI_ERR_ARG otherwise.
 *  - One handle is one (request, layer) index; handles are independent and
 *    must not be used from two threads at once.
 */
#ifndef AI_INDEX_H_
#define AI_INDEX_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ------------------------------------------------------------ errors */
#define AI_OK 0
#define AI_ERR_ARG (-1)          /* invalid argument, shape or dtype            */
#define AI_ERR_OOM (-2)          /* device allocation failed, or max_keys hit  */
#define AI_ERR_CAUSALITY (-3)    /* a query position beyond the appended keys  */
#define AI_ERR_DEVICE_CHECK (-4) /* a kernel flagged an out-of-range id/offset */
#define AI_ERR_TIMEOUT (-5)      /* a bounded device wait or host wait ran out */
#define AI_ERR_CUDA (-6)         /* a CUDA runtime call failed                 */
#define AI_ERR_STATE (-7)        /* call not valid in the current state        */

/* ------------------------------------------------------------ dtypes */
#define AI_FP32 0     /* float32                                              */
#define AI_BF16 1     /* bfloat16 bits (uint16)                               */
#define AI_FP8E4M3 2  /* OCP FP8 E4M3 codes (uint8) + one float32 scale per key */

typedef struct ai_index* ai_handle;

/* Index configuration.  Field names follow the pages' notation.           */
typedef struct ai_config {
  int32_t d;                   /* key / query head dimension                 */
  int32_t H;                   /* indexer heads                              */
  int32_t key_dtype;           /* AI_FP32 | AI_BF16 | AI_FP8E4M3             */
  int32_t q_dtype;             /* AI_FP32 (only with AI_FP32 keys) | AI_BF16 */
  int32_t n_sinks;             /* S: first keys, always candidates, never clustered */
  int32_t window;              /* W: open keys sealed together               */
  int32_t clusters_per_window; /* m                                          */
  int32_t cluster_cap;         /* size cap at seal; 0 -> ceil(W / m)         */
  int32_t refit_period;        /* R (multiple of W); 0 = never refit         */
  int32_t refit_new_seeds;     /* seeds per refit; 0 -> R * m / W            */
  int32_t refit_seed_window;   /* seeds come from the last keys; 0 -> R      */
  int32_t seal_iters;          /* k-means passes at seal; 0 -> 10            */
  int32_t async_refit;         /* 1: refit runs on an internal side stream   */
  int32_t max_query_chunk;     /* largest T passed to route/exhaustive calls */
  int32_t max_budget;          /* largest C passed to ai_route_refine        */
  int32_t max_k;               /* largest k: <= 2048 (bf16 / fp8 keys),      */
                               /* <= 4096 (fp32 keys)                        */
  int64_t max_keys;            /* capacity of the key store                  */
  uint64_t seed;               /* seed of the refit seed draws (SplitMix64)  */
  const float* encoder_weights_host; /* NULL: plain mean representatives.   */
  /* Else the correction encoder's float32 weights, packed in this order:
   * A [d,d], a [d], B1 [d, 3d+1], b1 [d], B2 [d,d], b2 [d] (copied at create). */
  int32_t block_routing;       /* 0: the inverted-file index (k-means seal,  */
  /* refit).  1: the contiguous-block baseline the explainer compares against
   * ("它到底在解决什么问题？", HiSA): a sealed window is cut into m blocks of
   * consecutive keys, block j = keys [lo + floor(jW/m), lo + floor((j+1)W/m)),
   * each represented by its member mean; no refit (refit_period must be 0),
   * no encoder.  Routing, candidate fill, rescore and top-k are unchanged.  */
} ai_config;

/* Create an index.  `cuda_stream` is the main stream (cudaStream_t, may be
 * NULL for the legacy default stream).  Allocates the key store and all
 * device scratch sized from the config.  Errors: AI_ERR_ARG, AI_ERR_OOM,
 * AI_ERR_CUDA.  On success *out is a new handle.                           */
int ai_index_create(const ai_config* cfg, void* cuda_stream, ai_handle* out);

/* Free a handle and everything it owns (waits for its streams first).     */
int ai_index_destroy(ai_handle h);

/* Insert (explainer, "索引怎么边算边建？" item 1).  Appends n keys to the
 * append-only store; they are candidates of every later query at once (the
 * open window).  keys_dev: [n, d] in the key dtype (fp8: codes);
 * scales_dev: [n] float32 per-key scales for AI_FP8E4M3, else NULL.
 * Also publishes a pending refit first (see ai_refit).  Errors: AI_ERR_ARG,
 * AI_ERR_OOM (store full).                                                */
int ai_append_keys(ai_handle h, const void* keys_dev, const float* scales_dev, int64_t n);

/* Seal (explainer, "索引怎么边算边建？" item 2).  Clusters every complete
 * W-window of open keys into m size-capped k-means clusters and appends
 * them; each seal creates a version whose open window starts after the
 * sealed keys.  Whenever the number of sealed keys reaches a multiple of R
 * a refit is started (see ai_refit).  *version_out (nullable) receives the
 * newest version number.                                                  */
int ai_seal(ai_handle h, int64_t* version_out);

/* Refit (explainer, "索引怎么边算边建？" item 3).  One warm-started assign +
 * update pass over all sealed keys [S, n_r): previous refit centres plus
 * new seeds drawn from the last keys, Hamerly bounds, member means.  Runs
 * on the side stream when async_refit = 1.  The result becomes the index
 * base at the next ai_append_keys or ai_publish call (a version with
 * watermark n_r).  n_new_seeds / seed_window: 0 -> config values.         */
int ai_refit(ai_handle h, int32_t n_new_seeds, int32_t seed_window, int64_t* version_out);

/* Make a pending refit the index base now (waits on the side stream from
 * the main stream, not from the host).  No-op without a pending refit.     */
int ai_publish(ai_handle h);

/* Route + refine (explainer, "查询时怎么挑候选？").  For the T queries at
 * positions pos0 .. pos0+T-1: each query t uses the newest version whose
 * keys all lie in its prefix, scores every visible cluster representative,
 * fills C candidate slots with the sinks, the open window [n_v, t] and
 * whole member lists in rank order (score desc, cluster id asc; the last
 * list is truncated), rescores the candidates exactly and writes the top k
 * ids to out_dev[T, k] sorted by score descending, ties by key id
 * ascending, then -1 padding (fewer than k candidates).  q_dev: [T, H, d]
 * in q_dtype; w_dev: [T, H] float32; out_scores_dev: [T, k] float32 (the
 * scores of those ids, -inf on padding) or NULL.
 * Limit: at most 2048 clusters of one query can reach its budget (the
 * clusters ranked in shared memory).  Clusters hold ~W/m keys after a seal,
 * so this binds only when C / (smallest cluster size) exceeds 2048; a
 * query over the limit ranks only 2048 of them and ai_sync then reports
 * AI_ERR_DEVICE_CHECK.
 * Errors: AI_ERR_ARG (T, k, C beyond the create-time maxima),
 * AI_ERR_CAUSALITY (pos0 + T - 1 >= appended keys).                        */
int ai_route_refine(ai_handle h, const void* q_dev, const float* w_dev, int64_t pos0,
                    int32_t T, int32_t k, int32_t C, int32_t* out_dev, float* out_scores_dev);

/* Sharded rescore for a cluster-sharded, several-GPU deployment (the
 * review's "tensor-parallel index ownership", Impact Assessment: Core
 * Contribution item 3; the explainer, 我认为它的局限 item 2, names the
 * cross-GPU synchronisation).  Every rank holds the same index (maintenance
 * is deterministic); for each query it builds the same candidate list and
 * rescores only its share: the contiguous range of the list's 128-slot
 * tiles with index shard of n_shards.  It writes that share's top k to
 * out_dev / out_scores_dev [T, k] (both required), in (score desc, id asc)
 * order, -1 / -inf padded.  The shards' lists hold disjoint ids and the
 * union of their top k holds the query's top k: gathering the n_shards
 * partial results and merging them with ai_merge_topk gives exactly
 * ai_route_refine's output.  bf16 / fp8 keys (pipelined refine kernels)
 * only; n_shards = 1 is ai_route_refine.  Errors as ai_route_refine, and
 * AI_ERR_ARG for a bad shard.                                              */
int ai_route_refine_shard(ai_handle h, const void* q_dev, const float* w_dev, int64_t pos0,
                          int32_t T, int32_t k, int32_t C, int32_t shard, int32_t n_shards,
                          int32_t* out_dev, float* out_scores_dev);

/* Merge n_parts partial top-k results per query: ids_dev / scores_dev are
 * [n_parts, T, k] (ids -1 where a part has fewer than k); writes the top k
 * of each query's union by (score desc, id asc) to out_dev [T, k] (and
 * out_scores_dev, nullable), -1 padded.  The parts must hold disjoint ids.
 * Enqueued on cuda_stream; needs no handle and allocates nothing.  Limits:
 * k <= 2048, n_parts * k <= 19,840 (AI_ERR_ARG).                          */
int ai_merge_topk(const int32_t* ids_dev, const float* scores_dev, int32_t n_parts, int32_t T,
                  int32_t k, int32_t* out_dev, float* out_scores_dev, void* cuda_stream);

/* Exhaustive selection (explainer, "它到底在解决什么问题？": the indexer
 * scores every key s <= t).  Same arguments and output order as
 * ai_route_refine (score descending, ties by id ascending, -1 padding).
 * The in-library baseline.                                                */
int ai_select_exhaustive(ai_handle h, const void* q_dev, const float* w_dev, int64_t pos0,
                         int32_t T, int32_t k, int32_t* out_dev, float* out_scores_dev);

/* Wait for all work of the handle (both streams) and report device-side
 * error flags: AI_ERR_DEVICE_CHECK or AI_ERR_TIMEOUT (flags are cleared).  */
int ai_sync(ai_handle h);

/* Message of the last error on this thread ("" if none).                  */
const char* ai_last_error(void);

/* -------------------------------------------------------- inspection */
typedef struct ai_stats {
  int64_t n_keys;        /* appended keys                                   */
  int64_t n_sealed;      /* sealed windows                                  */
  int64_t n_clusters;    /* clusters in the published array                 */
  int64_t n_versions;    /* versions in the published table                 */
  int64_t n_refits;      /* refits started                                  */
  int64_t refit_pending; /* 1 if a refit awaits publication                 */
  int64_t base_watermark;/* n_r of the published base (0 = none)            */
  int64_t last_refit_scanned; /* keys fully scanned by the last finished refit */
  int64_t last_refit_rechecked; /* of those, keys re-decided in float64 (near ties) */
} ai_stats;
int ai_get_stats(ai_handle h, ai_stats* out);

/* Copy the published index to host memory (synchronous).  Any pointer may
 * be NULL.  offsets_host [n_clusters + 1] (member offsets, relative),
 * members_host [offsets[n_clusters]], reps_bf16_host [n_clusters, d],
 * centroids_host [n_clusters, d] float64, version_nc_host / version_nv_host
 * [n_versions] (visible clusters, open-window start).                      */
int ai_export_index(ai_handle h, int32_t* offsets_host, int32_t* members_host,
                    uint16_t* reps_bf16_host, double* centroids_host, int64_t* version_nc_host,
                    int64_t* version_nv_host);

/* Debug: the candidate lists [T, C] (-1 padded) and cluster scores
 * [T, n_clusters] that ai_route_refine would use for these queries.        */
int ai_debug_candidates(ai_handle h, const void* q_dev, const float* w_dev, int64_t pos0,
                        int32_t T, int32_t C, int32_t* cand_dev, float* cluster_scores_dev);

/* Debug: the full indexer score matrix out_dev[T, n_keys] (float32, -inf
 * where key position > query position) computed by the exhaustive kernels. */
int ai_debug_scores(ai_handle h, const void* q_dev, const float* w_dev, int64_t pos0, int32_t T,
                    float* out_dev);

/* Checkpoint / rollback of the index state (host counters, version table,
 * active cluster buffer, per-key refit bounds and the last centre drifts).  Rollback forgets keys
 * appended after the checkpoint (they must be appended again).  Fails with
 * AI_ERR_STATE while a refit is pending at checkpoint time.               */
int ai_checkpoint(ai_handle h);
int ai_rollback(ai_handle h);

/* ----------------------------------------------------------- profiling */
/* Phase timing with CUDA events recorded on the stream each phase runs on
 * (refit: the side stream when async).  Off by default.                    */
#define AI_PHASE_ROUTE 0       /* cluster-score GEMM                          */
#define AI_PHASE_REFINE 1      /* candidate fill + rescore + top-k kernel     */
#define AI_PHASE_SEAL 2        /* seal k-means (+ encoder)                    */
#define AI_PHASE_REFIT 3       /* refit kernels (+ encoder)                   */
#define AI_PHASE_PUBLISH 4     /* wait for the refit + tail copy              */
#define AI_PHASE_EXH_SCORES 5  /* exhaustive score GEMM                       */
#define AI_PHASE_EXH_TOPK 6    /* exhaustive row top-k                        */
#define AI_PHASE_ORDER 7       /* route+refine output ordering (tensor core)  */
#define AI_N_PHASES 8
int ai_profile_enable(ai_handle h, int enable);
/* Waits for the handle's streams, then writes the summed milliseconds and
 * the number of timed launches per phase (arrays of AI_N_PHASES, nullable)
 * since the last read, and resets them.                                   */
int ai_profile_read(ai_handle h, double* ms_out, int64_t* launches_out);
/* Number of kernels this library has launched in the process.             */
long long ai_kernel_launches(void);

/* fp8 store helper: per-key scale = amax / 448 and E4M3 codes (round to
 * nearest even, saturating) from bf16 keys [n, d].  Enqueued on
 * cuda_stream.                                                            */
int ai_quantize_fp8(const uint16_t* keys_bf16_dev, int64_t n, int32_t d, uint8_t* codes_dev,
                    float* scales_dev, void* cuda_stream);

/* ----------------------------------------------- allocation-free variant */
/* Exhaustive selection for callers that cannot allocate device memory (for
 * example a server whose memory all comes from its own pre-reserved pool, or
 * a latency-critical path that must not hit the implicit synchronisation of
 * cudaMalloc / cudaFree).  No counterpart in the paper: it is a deployment
 * convenience with the same results as ai_select_exhaustive on the same
 * keys.  It needs no handle and calls no allocator: its only scratch is a
 * fixed 16 MiB device array inside the library, present on every device
 * that loads the library until the process exits.
 *   keys_dev: [n_keys, d] keys owned by the caller: AI_BF16 (d = 128,
 *     H in {32, 64}, bf16 queries) or AI_FP32 (fp32 queries); n_keys at
 *     most 1,048,576 (AI_ERR_ARG beyond); k at most 4096.
 *   q_dev [T, H, d], w_dev [T, H], pos0, T, k, out_dev [T, k],
 *   out_scores_dev [T, k] or NULL: as for ai_select_exhaustive (same
 *     output order).
 *   status_dev: NULL, or a device int32 that receives, in stream order
 *     after the call's kernels, the device flags they raised: 0 when clean,
 *     else an OR of AI_DEVFLAG_* (the handle-based calls report the same
 *     flags through ai_sync).  A nonzero status means the output is not
 *     valid.
 * Enqueued on cuda_stream.  The first call on a device looks up the
 * array's device address (make it before any stream capture).  All calls
 * share the array: calls whose work overlaps on the GPU (other streams,
 * other threads) race and must be serialised by the caller.              */
#define AI_DEVFLAG_TIMEOUT 1   /* a bounded wait inside a kernel ran out     */
#define AI_DEVFLAG_RANGE 2     /* an id or offset was out of range           */
#define AI_DEVFLAG_CAPACITY 4  /* a per-CTA buffer would have overflowed     */
int ai_select_exhaustive_noalloc(const void* keys_dev, int32_t key_dtype, int64_t n_keys,
                                 int32_t d, int32_t H, const void* q_dev, const float* w_dev,
                                 int64_t pos0, int32_t T, int32_t k, int32_t* out_dev,
                                 float* out_scores_dev, int32_t* status_dev, void* cuda_stream);

/* ------------------------------------------------ refine kernel variant */
/* Selects the kernel that runs route+refine on the tensor-core path (bf16
 * or fp8 keys) for later ai_route_refine / ai_debug_candidates calls on h.
 * All variants compute the same result; this exists so tests can cover
 * each one.  kernel: 0 = chosen by occupancy (the default), 1 = one query
 * at a time per CTA with the candidate list in shared memory, 2 = the same
 * with the list in global scratch, 3 = pipelined (the candidate build and
 * the top-k of neighbouring queries overlap the rescore of the current
 * one), 4 = pipelined with one TMEM score buffer (the epilogue's first
 * score store waits for the previous query's top-k; the default for
 * budgets where two buffers would cost the second CTA per SM).  A variant
 * whose shared memory or TMEM need does not fit the configuration makes
 * those calls fail with AI_ERR_CUDA.  Returns AI_OK, or AI_ERR_ARG for a
 * null handle or a kernel outside 0..4.                                   */
int ai_debug_refine_kernel(ai_handle h, int32_t kernel);

/* Parts per query for later ai_route_refine calls on h (tensor-core path,
 * pipelined refine kernels).  A chunk of T queries with 2 * T at most the
 * pipelined kernel's CTA count (two per SM) would leave most SMs idle, one
 * CTA gathering each query's whole candidate list; instead each list's
 * 128-slot tiles are divided among `split` CTAs (contiguous ranges, at
 * least two tiles each) and their partial top-k merged by a second kernel
 * into the documented output order.  Every tile, and so every score, is
 * the same as undivided: results are identical either way.  split: 0 =
 * chosen by chunk size (the default: up to 8 parts, and at most the CTA
 * count divided by T), 1 = never divide, 2..8 = at most that many parts.
 * Returns AI_OK, or AI_ERR_ARG for a null handle or split outside 0..8.   */
int ai_debug_refine_split(ai_handle h, int32_t split);

/* The refine kernel ai_route_refine launches on h for budget C:
 * *kernel_out = 0 for the fp32 (SIMT) path, else the tensor-core variant
 * as numbered for ai_debug_refine_kernel (1 to 4; the forced one if
 * set).  Host-only: launches nothing.  AI_ERR_ARG for a null argument or
 * C outside 1 .. max_budget.                                              */
int ai_refine_kernel_choice(ai_handle h, int32_t C, int32_t* kernel_out);

/* ------------------------------------------------- failure-path test hook */
/* Runs the library's bounded wait against a barrier that nothing completes
 * (the pages have no counterpart: this exists to test failure detection).
 * One thread polls an mbarrier phase at most spin_limit times (1 .. 2^26),
 * then records the timeout in a device status word and returns, exactly as
 * a kernel whose producer never arrives would.  Enqueued on cuda_stream and
 * waited for.  *status_out receives the device status flags (bit 0 =
 * timeout).  Returns AI_OK when the wait ran out and was reported,
 * AI_ERR_ARG for a bad limit or null output, AI_ERR_CUDA on a CUDA error.  */
int ai_debug_wait_timeout(int32_t spin_limit, int32_t* status_out, void* cuda_stream);

#ifdef __cplusplus
}
#endif

#endif /* AI_INDEX_H_ */
