/*
 * streamindex.h -- C ABI of the B200 (sm_100a) CSA lightning-indexer top-k library.
 *
 * The operation ("StreamIndex: Memory-Bounded Compressed Sparse Attention via
 * Streaming Top-k", Abstract): in Compressed Sparse Attention a lightning
 * indexer, a learned scoring projection over compressed keys, scores the keys
 * each query can see and the top-k keys are kept per query; StreamIndex does
 * this with a chunked partition-merge top-k driver that never materialises the
 * [B,S,H_I,T] fp32 score tensor.  The abstract prints no formula; this library
 * computes, for every batch b and query position t,
 *
 *     I[b,t,j] = sum_h w[b,t,h] * max(0, q[b,t,h,:] . kc[b,j,:])      (h < H_I)
 *
 * over the compressed keys j visible to t, i.e. (j+1)*m - 1 <= t, which is the
 * first V_t = min(T, floor((t+1)/m)) keys (T = S/m, m the compression ratio,
 * m = 4 for V4-Flash per the abstract).  It returns the min(topk, V_t) best
 * keys per query, sorted by score descending with ties broken by the lower
 * index (-0 and +0 are equal scores), followed by padding (index -1, score
 * -inf).
 *
 * Conventions for every call:
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    never frees them.  Layouts are dense row-major with the last named
 *    dimension fastest.  bf16 is passed as 16-bit storage, E4M3 as bytes.
 *  - Calls are asynchronous and ordered on `stream` (a cudaStream_t; NULL is
 *    the legacy default stream) unless stated otherwise.
 *  - The return value is a status: SI_OK (0) or a negative SI_ERR_* code.
 *    Argument errors are detected on the host before anything is launched.
 *    After a non-zero status the outputs are undefined.
 *  - Device-side waits are bounded; a kernel that gives up records a device
 *    error word, read back by si_get_last_device_error().
 *  - Limits: B >= 1; S >= 1 with S % m == 0; H_I in {8, 16, 32, 64};
 *    d_I in {64, 128}; 1 <= topk <= 2048; B*S*H_I < 2^31; pointers 16-byte
 *    aligned.  The selection keeps a candidate pool per query of a query
 *    tile in shared memory, so with few heads (many queries per tile) the
 *    largest topk is lower: bf16 H_I=8: 1056 (d_I=128), 1312 (d_I=64);
 *    FP8 H_I=8: 1280 (d_I=128), 1408 (d_I=64); 2048 otherwise.  A larger
 *    topk returns SI_ERR_TOPK.
 */
#ifndef STREAMINDEX_H
#define STREAMINDEX_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ---------------------------------------------------- */
#define SI_OK 0
#define SI_ERR_NULL -1           /* a required pointer is NULL */
#define SI_ERR_DIM -2            /* a dimension is out of range (see limits above) */
#define SI_ERR_TOPK -3           /* topk < 1, > 2048, or above the shape's limit */
#define SI_ERR_ALIGN -4          /* a pointer is not 16-byte aligned */
#define SI_ERR_WORKSPACE -5      /* caller workspace too small */
#define SI_ERR_CUDA -6           /* a CUDA runtime/driver call or launch failed */
#define SI_ERR_DEVICE_TIMEOUT -7 /* a kernel gave up on a bounded wait */
#define SI_ERR_OPTIONS -8        /* an si_options field is out of range */
#define SI_ERR_UNSUPPORTED -9    /* no sm_100 device, or the device is not a B200-class part */

#define SI_MAX_TOPK 2048

/* Tuning and debug knobs.  Pass NULL for the defaults. */
typedef struct si_options {
  int key_chunk;        /* keys per chunk of the partition-merge driver, a
                           multiple of 128; 0 = one chunk spans all keys of a
                           query.  Default 0. */
  int scratch_mb;       /* bound on partial-list scratch (MiB) used to size the
                           query blocks of the chunked driver.  Default 512. */
  int grid_ctas;        /* persistent CTAs; 0 = one per SM.  Default 0. */
  int timeout_ms;       /* limit of any single device-side wait.  Default 2000. */
  int debug_flags;      /* bit 0: the producer never issues its first load, so
                           the first consumer wait must expire (tests the
                           timeout path).  Default 0. */
  void* score_events[2];/* optional cudaEvent_t pair (NULL = none): the call
                           records [0] on `stream` just before its first
                           score-kernel launch and [1] just after its last
                           one, so cudaEventElapsedTime gives the fused score
                           kernel's own device time.  With several query
                           blocks, the finishing launches between them fall
                           inside the interval.  The events stay owned by
                           the caller. */
  int row_finish;       /* where a query's exact top-k row is finished when
                           one chunk spans all its keys: 1 = by the fused
                           kernel's selection warps (no partial lists, no
                           merge launch), 2 = by the merge kernel from the
                           fused kernel's pruned candidate lists, 0 = the
                           library's choice.  With several chunks the merge
                           kernel always finishes.  Default 0. */
  int key_tile;         /* keys per score strip handed from the tensor-core
                           epilogue to the selection warps: 128, 256, 512 or
                           1024 (one to eight 128-key MMA tiles), or 32 or 64
                           (a quarter or half of a tile: each tile's 32-key
                           lane quadrants are handed over in strips of their
                           own); 0 = the library's choice.  Default 0. */
  int strip_slots;      /* score strips in flight between the epilogue and
                           the selection warps: 2 to 4, a multiple of
                           128/key_tile for strips shorter than a tile (4 for
                           32, 2 or 4 for 64), else SI_ERR_OPTIONS; 0 = the
                           library's choice.  Default 0. */
  void** score_event_list; /* optional array of score_event_count
                           cudaEvent_t (NULL = none): the call records
                           [2i] on `stream` just before the score-kernel
                           launch of query block i and [2i+1] just after it,
                           for i < score_event_count / 2, so the score
                           kernel's own device time excludes the finishing
                           launches between query blocks (si_plan_info
                           .query_blocks gives the count needed).  The
                           events stay owned by the caller. */
  int score_event_count;
  int plan_heads;       /* si_topk_scores only: when > 0, select with the
                           fused score kernel's plan for H_I = plan_heads,
                           d_I = plan_dim and the bf16 (plan_fp8 = 0) or FP8
                           (1) path (queries per tile, keys per strip, pool
                           room, partial-list length), so the bit-exact test
                           entry runs exactly the selection the indexer runs
                           for that shape.  0 = the test entry's own plan
                           (4 queries, 1024-key strips).  Default 0. */
  int plan_dim;
  int plan_fp8;
} si_options;

/* The plan of one indexer call, as the library would run it. */
typedef struct si_plan_info {
  int queries_per_tile;   /* queries of one tensor-core tile (mma_n / H_I) */
  int mma_n;              /* MMA N: (query, head) columns of a tile, 128 or 256 */
  int key_tile;           /* keys per score strip handed to the selection warps */
  int stages;             /* key-tile pipeline stages in shared memory */
  int strip_slots;        /* score strips in flight */
  int pool_keys;          /* candidate-pool entries per query */
  int partial_len;        /* candidates per query and key chunk in the scratch lists */
  int key_chunks;         /* key chunks of the longest query tile */
  int query_blocks;       /* query blocks, i.e. score-kernel launches of one call */
  int launches;           /* kernel launches of one call */
  size_t workspace_bytes; /* device workspace of si_indexer_topk_ex for this plan */
  size_t smem_bytes;      /* dynamic shared memory of one score-kernel CTA */
} si_plan_info;

/* ---- the indexer step ------------------------------------------------ */

/*
 * si_indexer_topk: score, mask and select in one pass (bf16 inputs).
 *   q         bf16 [B,S,H_I,d_I]   indexer queries
 *   w         fp32 [B,S,H_I]       per-head weights (signed)
 *   kc        bf16 [B,T,d_I]       compressed keys, T = S/m
 *   out_idx   int32 [B,S,topk]     selected key indices, -1 padding
 *   out_score fp32  [B,S,topk]     their scores (fp32 accumulation), -inf padding
 * Uses an internal workspace allocated with cudaMallocAsync on `stream` and
 * released on the same stream before returning.
 */
int si_indexer_topk(const void* q, const float* w, const void* kc, int B, int S, int H_I, int d_I,
                    int m, int topk, int32_t* out_idx, float* out_score, void* stream);

/* Bytes of device workspace si_indexer_topk_ex needs for this problem. */
int si_indexer_topk_workspace_size(int B, int S, int H_I, int d_I, int m, int topk,
                                   const si_options* opt, size_t* bytes);

/*
 * si_indexer_topk_plan: the plan si_indexer_topk_ex (fp8 = 0) or
 * si_indexer_topk_fp8 (fp8 = 1) would run for this problem and these options:
 * tile shape, shared-memory plan, key chunks, query blocks and the number of
 * kernel launches of one call (the FP8 quantiser launches, which are separate
 * calls, are not counted).  Host only, nothing is launched.  The plan is made
 * for the current device; on a host with no usable CUDA device it is made for
 * the sm_100 limits (227 KB of shared memory per CTA).  Errors as the
 * workspace-size query, plus SI_ERR_TOPK when the selection pools of this
 * topk do not fit the shape's tile and SI_ERR_OPTIONS for a key_tile above
 * the largest strip the tile allows.
 */
int si_indexer_topk_plan(int B, int S, int H_I, int d_I, int m, int topk, int fp8,
                         const si_options* opt, si_plan_info* out);

/* As si_indexer_topk, with options and a caller-provided device workspace of
 * ws_bytes (at least what si_indexer_topk_workspace_size reports). */
int si_indexer_topk_ex(const void* q, const float* w, const void* kc, int B, int S, int H_I,
                       int d_I, int m, int topk, int32_t* out_idx, float* out_score,
                       const si_options* opt, void* workspace, size_t ws_bytes, void* stream);

/*
 * si_indexer_topk_fp8: the same step with E4M3 operands and per-row scales.
 *   q8  e4m3 [B,S,H_I,d_I] with s_q fp32 [B,S,H_I];  k8 e4m3 [B,T,d_I] with
 *   s_k fp32 [B,T]; the score is sum_h w * max(0, s_q*s_k*(q8 . k8)), the
 *   codes decoded exactly and the dot product accumulated in fp32.
 * Scales must be positive.  Workspace as in si_indexer_topk_ex (the size query
 * is the same call).
 */
int si_indexer_topk_fp8(const void* q8, const float* s_q, const float* w, const void* k8,
                        const float* s_k, int B, int S, int H_I, int d_I, int m, int topk,
                        int32_t* out_idx, float* out_score, const si_options* opt,
                        void* workspace, size_t ws_bytes, void* stream);

/*
 * si_quantize_fp8_rows: per-row E4M3 quantisation of a bf16 matrix.
 *   x [rows, cols] bf16 -> x8 [rows, cols] e4m3 and scale [rows] fp32, with
 *   scale = max|x_row| / 448 (1 for an all-zero row) and
 *   x8 = E4M3 round-to-nearest-even, saturating, of x / scale (fp32 division).
 * (The reference list of the abstract cites "FP8 Formats for Deep Learning"
 * for the format; the per-row scaling is this library's reading.)
 * cols must be a multiple of 8 and at most 4096.
 */
int si_quantize_fp8_rows(const void* x, int64_t rows, int cols, void* x8, float* scale,
                         void* stream);

/*
 * si_topk_scores: the selection stage alone on a given fp32 score tensor.
 *   scores [B,S,T] fp32; keys j >= V_t are ignored (never read).
 *   Output as si_indexer_topk; selected scores keep their input bit patterns.
 * Bit-exact: the same indices and bits as a plain sort of each row's visible
 * scores under the order above.  Workspace: internal (cudaMallocAsync).
 */
int si_topk_scores(const float* scores, int B, int S, int T, int m, int topk, int32_t* out_idx,
                   float* out_score, const si_options* opt, void* stream);

/*
 * si_indexer_topk_noalloc: si_indexer_topk for callers that cannot allocate
 * device memory.  The StreamIndex paper has no counterpart; this entry point
 * exists for callers embedded in a runtime that owns every device allocation
 * (a serving engine with a fixed memory pool, a plugin inside another
 * framework) or that cannot afford an allocator call in a latency-critical
 * loop, where an allocation may block on the allocator or fail when memory is
 * fragmented.
 *   Arguments, layouts and results are those of si_indexer_topk.  The call
 *   makes no cudaMalloc, cudaMallocAsync or cudaFree: its scratch is a fixed
 *   64 MiB device array inside the library (SI_NOALLOC_SCRATCH_BYTES), which
 *   every GPU that loads the library holds until the process exits.  Query
 *   tiles are processed in blocks sized to that array; a problem whose single
 *   query tile needs more returns SI_ERR_WORKSPACE.  That size check comes
 *   before the pointer checks, so it can be queried with NULL tensors.
 *   The first call on each device looks up the array's device address (once
 *   per device, with that device current); make that first call before any
 *   stream capture.
 *   All calls share the one array and each leaves its contents behind; the
 *   call clears what must start at zero (its work counter) on `stream` before
 *   use.  Calls whose work overlaps on the GPU (different streams, or other
 *   threads) race on the array and give undefined results: serialise them.
 */
#define SI_NOALLOC_SCRATCH_BYTES (64u << 20)
int si_indexer_topk_noalloc(const void* q, const float* w, const void* kc, int B, int S, int H_I,
                            int d_I, int m, int topk, int32_t* out_idx, float* out_score,
                            void* stream);

/* ---- decode ------------------------------------------------------------ */

/*
 * si_indexer_decode: the indexer step for the newest queries of sequences
 * whose compressed keys so far are given.  The abstract describes the step
 * for a whole sequence (every query against the keys it can see); decoding
 * scores only the queries of the tokens just produced, against the keys
 * compressed so far, so the result is the same formula with each query's
 * sequence position in place of t:
 *   query i of batch b sits at position t = t0 + i (0 <= i < S_q, the same
 *   t0 in every batch) and sees the first V = min(T, floor((t+1)/m)) keys.
 * A query row of a decode call therefore equals row t0 + i of si_indexer_topk
 * on a sequence whose keys are kc: a caller that appends one compressed key
 * per m tokens passes the grown kc and the new position each step.
 *   q         bf16 [B,S_q,H_I,d_I]   queries at positions t0 .. t0+S_q-1
 *   w         fp32 [B,S_q,H_I]       their head weights
 *   kc        bf16 [B,T,d_I]         compressed keys; keys past a query's V
 *                                    are never used (kc may be a buffer with
 *                                    room for more keys)
 *   out_idx   int32 [B,S_q,topk], out_score fp32 [B,S_q,topk]: as si_indexer_topk.
 * Limits: B, S_q, T, m >= 1; t0 >= 0 and t0 + S_q < 2^31; B*T < 2^31; H_I,
 * d_I, topk and alignment as si_indexer_topk (S need not be a multiple of m).
 * With few query tiles the keys of a tile are split into chunks so that the
 * work spreads over every SM (options.key_chunk > 0 fixes the chunk), and the
 * chunks' candidate lists are merged.  Workspace: caller-provided, at least
 * si_indexer_decode_workspace_size bytes.  bf16 operands only.
 */
int si_indexer_decode(const void* q, const float* w, const void* kc, int B, int S_q, int t0, int T,
                      int H_I, int d_I, int m, int topk, int32_t* out_idx, float* out_score,
                      const si_options* opt, void* workspace, size_t ws_bytes, void* stream);

/* Bytes of device workspace si_indexer_decode needs. */
int si_indexer_decode_workspace_size(int B, int S_q, int t0, int T, int H_I, int d_I, int m,
                                     int topk, const si_options* opt, size_t* bytes);

/* The plan si_indexer_decode would run (see si_indexer_topk_plan). */
int si_indexer_decode_plan(int B, int S_q, int t0, int T, int H_I, int d_I, int m, int topk,
                           const si_options* opt, si_plan_info* out);

/* ---- query-group candidate scan ---------------------------------------- */

/*
 * si_indexer_pivot: an approximate indexer step after the PIVOT news page
 * (nearby queries select nearly the same keys, so a group of queries shares
 * one scan).  The queries of each batch form groups of G consecutive
 * positions.  The group's last position scans every key it can see (the
 * step of si_indexer_topk for that query) and keeps its C best; each query of
 * the group then scores only those candidates it can see and keeps its topk
 * best, in the order and with the padding of si_indexer_topk.  The group's
 * last query gets its exact row (C >= topk); G = 1 is the exact step, and so
 * is C >= T.  Work: S/G full scans plus S*C candidate scores.
 *   Arguments as si_indexer_topk, plus G (S % G == 0) and C (topk <= C <= 2048).
 *   Workspace: caller-provided, at least si_indexer_pivot_workspace_size
 *   bytes (the representatives, their candidate rows and the gathered key
 *   rows: about B*S/G*C*(2*d_I + 12) bytes, plus an indexer workspace).
 * Errors as si_indexer_topk; SI_ERR_OPTIONS for a bad G or C.
 */
int si_indexer_pivot(const void* q, const float* w, const void* kc, int B, int S, int H_I,
                     int d_I, int m, int topk, int G, int C, int32_t* out_idx, float* out_score,
                     const si_options* opt, void* workspace, size_t ws_bytes, void* stream);

/* Bytes of device workspace si_indexer_pivot needs. */
int si_indexer_pivot_workspace_size(int B, int S, int H_I, int d_I, int m, int topk, int G, int C,
                                    const si_options* opt, size_t* bytes);

/* ---- sparse attention over the selected entries -------------------------- */

/*
 * si_sparse_attention: the consumer of the indexer's rows.  The abstract
 * describes it only as a sparse attention kernel that reads the selected
 * keys; this call computes multi-query attention over the entries a row
 * lists, all query heads sharing one key row and one value row per entry:
 *   J(b,t) = { idx[b,t,r] : 0 <= r < topk, 0 <= idx[b,t,r] < T }
 *   out[b,t,h,:] = sum_{j in J} softmax_j(scale * qa[b,t,h,:] . ka[b,j,:]) * va[b,j,:]
 * (entries count as listed; -1 padding and out-of-range entries are skipped;
 * a row that lists none gives zeros).
 *   qa   bf16 [B,S,H_a,d_a]   query heads (H_a = 128, d_a = 128)
 *   ka   bf16 [B,T,d_a]       key rows of the compressed entries
 *   va   bf16 [B,T,d_a]       value rows
 *   idx  int32 [B,S,topk]     the entries of each query (si_indexer_topk's out_idx)
 *   out  fp32 [B,S,H_a,d_a]
 * Arithmetic: q.k in fp32 from bf16 products on the tensor cores, softmax
 * in fp32, the probabilities rounded to bf16 for the weighted sum of the
 * value rows (accumulated in fp32).  Limits: 1 <= topk <= 2048; B*S*H_a <
 * 2^31; qa, ka, va, out 16-byte aligned, idx 4-byte aligned; scale finite and
 * >= 0 (SI_ERR_OPTIONS otherwise).
 * Options: grid_ctas and timeout_ms are used.  No workspace.
 */
int si_sparse_attention(const void* qa, const void* ka, const void* va, const int32_t* idx, int B,
                        int S, int T, int H_a, int d_a, int topk, float scale, float* out,
                        const si_options* opt, void* stream);

/* ---- diagnostics ------------------------------------------------------ */

/* Text for a status code (static storage). */
const char* si_status_string(int status);

/* Synchronises `stream`, then returns SI_OK, SI_ERR_DEVICE_TIMEOUT if a kernel
 * since the previous call gave up on a bounded wait, or SI_ERR_CUDA; clears
 * the device error word of the current device. */
int si_get_last_device_error(void* stream);

/*
 * si_role_cycles: per-CTA role counters of the profiling build of the library
 * (compiled with SI_ROLE_CLOCKS): for each CTA of the fused score kernel, 32
 * unsigned 64-bit words accumulated over every launch since the last reset --
 * cycles each warp role spends in total, waiting on each of its barriers and
 * in each selection phase, and event counts (units, key tiles, strips,
 * appended keys, prunes, radix selects); the slot order is the RoleSlot enum
 * of the library's device code.  Synchronises the device, copies the first
 * n_words words ([CTA][32], at most 1024 CTAs) to host memory `out`, and
 * zeroes them when `reset` is non-zero.  The normal build keeps no counters
 * and returns SI_ERR_UNSUPPORTED.
 */
int si_role_cycles(uint64_t* out, int n_words, int reset);

/* Library version as an integer, major*10000 + minor*100 + patch. */
int si_version(void);

#ifdef __cplusplus
}
#endif

#endif /* STREAMINDEX_H */
