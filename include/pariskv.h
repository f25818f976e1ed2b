/*
 * pariskv.h -- C-ABI of the B200 (sm_100a) ParisKV decode-time KV-cache
 * retrieval library (libpariskv.so).
 *
 * What the library computes (citations are to two public pages: the
 * "ParisKV" GitHub README of amy-77/ParisKV, called [readme] below, and the
 * slide deck "ParisKV: Fast and Drift-Robust KV-Cache Retrieval" reading of
 * arXiv 2602.07721v3, called [slides]):
 *
 *   pk_build_index  prefill: normalise + SRHT-rotate every key, split it into
 *                   B = D/m blocks, store the sign-pattern centre id of each
 *                   block (PolarANN codes) and the 4-bit RSQ-IP summary (1 sign
 *                   bit + 3-bit Lloyd-Max magnitude index per coordinate, one
 *                   fp32 weight per block) on the GPU; copy K/V into
 *                   index-owned storage in HBM or pinned host memory.
 *                   [readme] pipeline step 1 (prefill builds the compact
 *                   retrieval metadata); [slides] Eqs. (5)-(10).
 *   pk_append       index newly decoded keys with the same fixed codebook
 *                   ([slides] Sec. 4.1.2: the codebook is fixed, so new
 *                   keys are encoded without retraining centroids).
 *   pk_search       per (sequence, KV head): GQA-aggregate and rotate the
 *                   query, rank the sign-pattern buckets of every block, give
 *                   buckets inside the top-rho fraction one of six tier
 *                   bonuses 6..1, sum them into collision scores S_i
 *                   ([slides] Sec. 4.2.2, App. B.2.1 Eq. 15), keep the top
 *                   C = ceil(beta n) keys by S ([slides] Sec. 4.3), rerank
 *                   them with the 4-bit estimator ([slides] Eqs. 7-10) and
 *                   return the final Top-k indices.
 *   pk_attend       exact softmax attention of every query head over the
 *                   selected full-precision K/V rows, read from HBM or, for
 *                   host-resident K/V, over the host link through UVA
 *                   ([slides] Sec. 3 Eqs. (1)-(3); [readme] pipeline step 3:
 *                   only the selected K/V pairs are fetched).
 *
 * Conventions for every call:
 *   - D (head_dim) must be 128 and m (sub_dim) must be 8 (B = 16 blocks of
 *     256 sign-pattern centres).  Other values return PK_ERR_UNSUPPORTED.
 *   - Tensors are dense, row-major, and addressed by plain pointers that the
 *     GPU can dereference: device memory, or pinned/mapped host memory (UVA).
 *     Pageable host memory is rejected with PK_ERR_INVALID_ARG.
 *   - "BH" = batch * n_kv_heads; pair bh = b * n_kv_heads + h.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Every call only enqueues work on it and returns; nothing
 *     waits for the GPU except pk_last_device_error, pk_trace_read and the
 *     allocation/free calls.
 *   - Arguments are checked on the host before any launch; a bad argument
 *     returns an error status and launches nothing.  Kernels never trap: a
 *     device-side check that fails (e.g. an out-of-range index given to
 *     pk_attend) skips the access and records a code read by
 *     pk_last_device_error.
 *   - No C++ exception crosses this boundary.  Calls on one index must not
 *     run concurrently from several host threads or streams (they share the
 *     index's workspace).
 */
#ifndef PARISKV_H
#define PARISKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PK_OK = 0,
    PK_ERR_INVALID_ARG = 1,   /* null / misaligned / pageable pointer, bad value */
    PK_ERR_CAPACITY = 2,      /* n < topk, n + n_new > n_cap, n too large       */
    PK_ERR_OOM = 3,           /* device or pinned-host allocation failed        */
    PK_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed           */
    PK_ERR_TIMEOUT = 5,       /* reserved: a bounded device wait gave up        */
    PK_ERR_DEVICE_CHECK = 6,  /* a device-side check recorded a bad value       */
    PK_ERR_UNSUPPORTED = 7    /* head_dim != 128, sub_dim != 8, topk > 1024,
                                 batch * n_kv_heads * group > 65535             */
} pk_status;

typedef enum { PK_F32 = 0, PK_BF16 = 1 } pk_dtype;
typedef enum { PK_KV_DEVICE = 0, PK_KV_HOST_PINNED = 1 } pk_kv_location;

/* Index parameters.  [readme] parameter table: final_topk, enable_offload;
 * adaptive ratio table for beta (candidate ratio) and rho (collision ratio). */
typedef struct {
    int32_t batch;            /* sequences                                     */
    int32_t n_kv_heads;       /* H                                             */
    int32_t group;            /* G query heads per KV head (GQA); >= 1, <= 8   */
    int32_t head_dim;         /* D, must be 128                                */
    int32_t sub_dim;          /* m, must be 8                                  */
    int32_t topk;             /* largest k pk_search / pk_attend accept; <=1024 */
    int64_t n_cap;            /* keys per (sequence, KV head), appends included */
    int64_t cand_budget;      /* C; 0 = ceil(beta(n) n) from the ratio table   */
    float collision_ratio;    /* rho; 0 = ratio table                          */
    float attn_scale;         /* softmax scale; 0 = 1/sqrt(D)                  */
    uint64_t rot_seed;        /* seed of the SRHT sign diagonal                */
    int32_t kv_dtype;         /* pk_dtype of K, V and queries                  */
    int32_t kv_location;      /* pk_kv_location of the full K/V store          */
} pk_params;

typedef struct pk_index pk_index;

/* Facts about a built index (host struct filled by pk_get_info). */
typedef struct {
    int64_t n;                /* keys per (sequence, KV head) now              */
    int64_t n_cap;
    int32_t bh;               /* batch * n_kv_heads                            */
    int32_t nchunks;          /* key chunks per pair used by pk_search at n    */
    int64_t chunk;            /* keys per chunk                                */
    int64_t cand;             /* C at n                                        */
    int64_t coll;             /* R = ceil(rho n) at n                          */
    int64_t index_bytes;      /* codes + summaries + occupancy (device)        */
    int64_t kv_bytes;         /* full K/V store (device or pinned host)        */
    int32_t kv_location;
    int32_t num_sms;
    int64_t n_staged;         /* keys staged by pk_append_stage, not yet published */
} pk_info;

/* Optional intermediate outputs of pk_search_debug (device pointers; any may
 * be NULL).  Layouts: qt [BH][D] f32; qnorm [BH] f32; bonus [BH][16][256] u8;
 * S [BH][n] u8; hist [BH][97] u32 (count of S = s); sstar [BH] i32 (the S
 * threshold); cand [BH][C] i32 (candidate ids in ascending order); cand_est
 * [BH][C] f32 (the 4-bit estimate of cand[.]). */
typedef struct {
    float *qt;
    float *qnorm;
    uint8_t *bonus;
    uint8_t *S;
    uint32_t *hist;
    int32_t *sstar;
    int32_t *cand;
    float *cand_est;
} pk_debug_out;

/* Fill *p with defaults: batch 1, H 8, G 4, D 128, m 8, topk 100, n_cap 0,
 * ratio-table C and rho, scale 1/sqrt(D), seed 0, bf16, K/V in HBM. */
void pk_default_params(pk_params *p);

/* Build an index over n keys per pair.
 *   K, V   [BH][n][D] of kv_dtype (device or pinned host pointers; copied in).
 *   n      1 <= n <= n_cap (n_cap 0 means n).
 * On success *out owns: codes [BH][n_cap][16] u8, summary records
 * [BH][n_cap][128 B], occupancy [BH][16][256] u32, search workspace, and the
 * K/V store [BH][n_cap][2][D] (HBM, or cudaHostAlloc'd mapped host memory;
 * the K and V rows of a key are adjacent, so gathering a selected key's rows
 * touches one page of a host-resident store instead of two).
 * Errors: PK_ERR_INVALID_ARG, PK_ERR_UNSUPPORTED, PK_ERR_CAPACITY,
 * PK_ERR_OOM (nothing leaks), PK_ERR_CUDA. */
pk_status pk_build_index(const void *K, const void *V, int64_t n, const pk_params *params,
                         void *stream, pk_index **out);

/* Append n_new keys/values per pair: k_new, v_new [BH][n_new][D] kv_dtype.
 * Encodes them at positions n .. n+n_new-1 and updates the occupancy table.
 * PK_ERR_CAPACITY when n + n_new > n_cap (nothing is written). */
pk_status pk_append(pk_index *index, const void *k_new, const void *v_new, int64_t n_new,
                    void *stream);

/* Asynchronous re-indexing in two calls ([readme] section on long
 * generation: older tokens are indexed and offloaded in the background;
 * [slides] Fig. 5: a full update buffer is encoded and offloaded in one
 * batch).
 *
 * pk_append_stage encodes n_new keys per pair into the rows after the keys
 * already present or staged, copies their K/V rows into the store, and counts
 * their occupancy in a side table.  Searches and attention do not see staged
 * keys: they use n and the published occupancy only.  So the call may run on
 * a stream of its own, concurrently with pk_search / pk_attend on the decode
 * stream; the caller must not change the source rows until the staging work
 * is done (it is, for any stream, once that stream has passed
 * pk_append_publish).
 *   k_new, v_new  row 0 of pair 0 of a [BH][src_stride][D] kv_dtype array
 *                 (device or mapped host); rows 0..n_new-1 of each pair are
 *                 taken, so a window of a larger per-pair buffer can be staged
 *                 in place.  src_stride 0 means n_new.
 * PK_ERR_CAPACITY when n + staged + n_new > n_cap (nothing is written).
 * Two stage calls must not overlap on the GPU (use one staging stream).
 *
 * pk_append_publish makes every staged key visible to work enqueued on
 * `stream` after it: the stream waits (on the GPU) for the staging work, the
 * side counts are added into the occupancy table, and n grows by the staged
 * count.  Nothing to publish is not an error.  pk_append returns
 * PK_ERR_INVALID_ARG while keys are staged. */
pk_status pk_append_stage(pk_index *index, const void *k_new, const void *v_new, int64_t n_new,
                          int64_t src_stride, void *stream);
pk_status pk_append_publish(pk_index *index, void *stream);

/* Retrieve the Top-k keys of every pair for one decode step.
 *   q          [batch][H*G][D] kv_dtype; query head j belongs to KV head j/G.
 *   topk       1 <= topk <= params.topk and topk <= n.
 *   out_idx    [BH][topk] i32 device: key ids, best first (estimate desc, id asc).
 *   out_score  [BH][topk] f32 device or NULL: the 4-bit estimates.
 * Ties use one rule everywhere: higher score first, then lower key id. */
pk_status pk_search(pk_index *index, const void *q, int32_t topk, int32_t *out_idx,
                    float *out_score, void *stream);

/* pk_search that also writes the intermediates named in *dbg (may be NULL). */
pk_status pk_search_debug(pk_index *index, const void *q, int32_t topk, int32_t *out_idx,
                          float *out_score, const pk_debug_out *dbg, void *stream);

/* Exact attention over the selected rows.
 *   q        [batch][H*G][D] kv_dtype (the un-aggregated query heads).
 *   sel_idx  [BH][topk] i32 device; ids outside [0, n) are skipped and recorded
 *            as PK_ERR_DEVICE_CHECK (see pk_last_device_error).
 *   out      [batch][H*G][D] f32 device (or mapped host):
 *            o_g = sum_r softmax_r(scale <q_g, K[sel_r]>) V[sel_r]. */
pk_status pk_attend(pk_index *index, const void *q, const int32_t *sel_idx, int32_t topk,
                    float *out, void *stream);

/* Exact attention over the selected rows together with rows kept densely on
 * the GPU outside the index -- the sink tokens and the recent local window --
 * under one softmax (README, pipeline step 3: the sink, local and retrieved
 * tokens are attended together; slides, Fig. 5: sink and local tokens stay
 * on the GPU for dense attention while the retrieval region is searched).
 *   q, sel_idx, topk, out  as for pk_attend, except that topk may be 0
 *            (dense rows only; sel_idx may then be NULL).
 *   dense_K, dense_V  [BH][dense_stride][D] kv_dtype, device (or mapped host),
 *            16-byte aligned, owned by the caller; rows 0..dense_len-1 of every
 *            pair are attended (their order does not matter).
 *   dense_len  0 <= dense_len <= dense_stride; topk + dense_len >= 1.
 * o_g = sum over the topk selected rows and the dense rows of
 * softmax(scale <q_g, k>) v.  Errors: PK_ERR_INVALID_ARG for a bad pointer,
 * alignment or size; selected ids outside [0, n) as for pk_attend. */
pk_status pk_attend_dense(pk_index *index, const void *q, const int32_t *sel_idx, int32_t topk,
                          const void *dense_K, const void *dense_V, int64_t dense_stride,
                          int32_t dense_len, float *out, void *stream);

/* Per-query-head retrieval for GQA: every query head of a pair searches the
 * pair's index with its own query (no aggregation): its own bonus tables,
 * collision scores, candidates and Top-k.  The pages retrieve with one query
 * per KV head; this is the other reading of a GQA group, kept beside it to
 * compare recall and cost.
 *   q        [batch][H*G][D] kv_dtype.
 *   out_idx  [batch][H*G][topk] i32 device: key ids of the pair's index,
 *            best first for each query head; out_score likewise or NULL.
 * The first call allocates a workspace for batch*H*G query units (kept
 * until pk_free).  Errors as pk_search, and PK_ERR_OOM for that workspace. */
pk_status pk_search_heads(pk_index *index, const void *q, int32_t topk, int32_t *out_idx,
                          float *out_score, void *stream);

/* Attention of every query head over its own selected rows (as returned by
 * pk_search_heads): sel_idx [batch][H*G][topk] i32 device; out as for
 * pk_attend.  With K/V in pinned host memory and G x topk <= 1024, the rows
 * of a (sequence, KV head) pair cross the host link once: the union of its G
 * heads' lists, in order of first appearance, each id once; head g then
 * attends over the rows of its own list.  With K/V in HBM, or longer lists,
 * each query head's rows are gathered by its own CTAs.  A head's ids are
 * expected to be distinct (pk_search_heads' are): a repeated id counts once
 * on the union path and once per appearance on the per-head path.  Errors as
 * pk_attend. */
pk_status pk_attend_heads(pk_index *index, const void *q, const int32_t *sel_idx, int32_t topk,
                          float *out, void *stream);

/* Free everything the index owns (synchronises the device first). NULL is ok. */
void pk_free(pk_index *index);

/* Static description of a status code. */
const char *pk_status_str(pk_status s);

/* Wait for the device, then return and clear the index's device-check word:
 * PK_OK, or PK_ERR_DEVICE_CHECK with *detail (nullable) set to the first bad
 * value seen (e.g. the out-of-range key id). */
pk_status pk_last_device_error(pk_index *index, int64_t *detail);

pk_status pk_get_info(const pk_index *index, pk_info *info);

/* Copy the index's codes [BH][n][16] u8, records [BH][n][128] u8 and occupancy
 * [BH][16][256] u32 into caller device buffers (any may be NULL). */
pk_status pk_export_index(const pk_index *index, uint8_t *codes, uint8_t *records,
                          uint32_t *occ, void *stream);

/* The fp32 Lloyd-Max magnitude levels (L of them) and midpoints (L-1) of the
 * prior y = |u_j|, (u_j)^2 ~ Beta(1/2, (m-1)/2) ([slides] Prop. 4.1 /
 * App. B.1), computed on the host; the index uses m = 8, L = 8. */
pk_status pk_magnitude_levels(int32_t m, int32_t L, float *levels, float *thresholds);

/* Budgets for a retrieval zone of n keys ([readme] ratio table):
 * C = cand_budget or ceil(beta n), then min(max(C, topk), n);
 * R = ceil(rho n) clamped to [1, n], rho = collision_ratio or the table's. */
pk_status pk_resolve(int64_t n, int64_t cand_budget, float collision_ratio, int32_t topk,
                     int64_t *C, int64_t *R);

/* Candidate selection that allocates nothing.  (No counterpart on the pages:
 * it is a deployment aid for the candidate step of pk_search.)
 *
 * For callers that cannot allocate device memory at the moment they need a
 * candidate set -- code recorded into a CUDA graph (cudaMalloc cannot be
 * captured), serving runtimes whose memory pool is fully reserved up front,
 * or decode threads that must not take allocator locks -- this computes, from
 * one row of collision scores, the same Top-C candidate ids in the same
 * ascending order as the candidate step of pk_search (higher score first,
 * then lower id; ids written in ascending order).
 *   S     [n] u8 device (or pinned host) scores; scores from pk_search_debug
 *         lie in [0, 96]; any byte value is accepted.
 *   n     1 <= n <= 4,194,304 (PK_ERR_CAPACITY above that; nothing runs).
 *   C     1 <= C <= n.
 *   cand  [C] i32 device, 4-byte aligned: the candidate ids.
 * Scratch: a static device array of 266,496 bytes that every GPU loading the
 * library holds until the process exits; no cudaMalloc, cudaFree or other
 * allocating call is made.  The first call on a device looks up the array's
 * device address (cudaGetSymbolAddress) with that device current, so make it
 * once before any stream capture.  All calls share the array: calls whose
 * work overlaps on the GPU (different streams or host threads) race on it;
 * calls on one stream are ordered and safe.  Asynchronous on `stream`. */
pk_status pk_select_candidates_noalloc(const uint8_t *S, int64_t n, int64_t C, int32_t *cand,
                                       void *stream);

/* Per-kernel timing.  While tracing is on, the library records a CUDA event
 * pair on the launching stream around each of its kernels.  pk_trace_read
 * synchronises, then returns per kernel kind (0 encode, 1 query_prep,
 * 2 collision_scan, 3 compact, 4 rerank_topk, 5 topk_merge, 6 gather_attend)
 * the launch count and the summed event time in ms; it clears the record. */
enum { PK_K_ENCODE = 0, PK_K_QUERY_PREP = 1, PK_K_COLLISION_SCAN = 2, PK_K_COMPACT = 3,
       PK_K_RERANK_TOPK = 4, PK_K_TOPK_MERGE = 5, PK_K_GATHER_ATTEND = 6, PK_K_COUNT = 7 };
pk_status pk_trace_enable(pk_index *index, int32_t on);
pk_status pk_trace_read(pk_index *index, int64_t *launches, double *total_ms);

#ifdef __cplusplus
}
#endif
#endif /* PARISKV_H */
