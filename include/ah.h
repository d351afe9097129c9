/*
 * ah.h: C ABI of the B200 anisotropic-AH maximum inner product search library.
 *
 * The search path is the one the ScaNN blog post describes in "Three stages of
 * a search" (ScaNN: Anisotropic Vector Quantization for Maximum Inner Product
 * Search):
 *   partitioning  -> q . c for every centroid c; the num_leaves_to_search
 *                    highest-scoring leaves are the ones searched;
 *   asymmetric hashing (AH) -> a per-query lookup table of q . center for each
 *                    block's 16 centers; each point's 4-bit codes pick one
 *                    entry per block, and those entries add up to its
 *                    approximate score;
 *   reordering    -> exact dot products replace the approximate scores of
 *                    the top candidates (a few hundred), and the best k by
 *                    exact score are returned.
 * The search-time knobs follow the post's "Using the library" section
 * (search_batched with leaves_to_search and pre_reorder_num_neighbors, and
 * final_num_neighbors).  Besides the search the library provides the steps
 * that build an index (anisotropic code assignment, k-means partition
 * training: ah_encode, ah_kmeans_assign, ah_kmeans_update), index directories
 * (ah_save, ah_inspect, ah_load) and the exact merge of a leaf-partitioned
 * search (ah_merge_shards).
 *
 * Conventions for every entry point:
 *  - Status codes only: no exceptions cross the ABI, nothing calls exit/abort.
 *  - Device pointers are CUDA device memory on the current device; the library
 *    never frees memory it did not allocate.  An index belongs to the device
 *    that was current when it was built: ah_search, ah_search_traced,
 *    ah_search_host, ah_reserve and ah_search_leaves_noalloc need that device
 *    current (AH_ERR_INVALID_ARG otherwise, before anything is enqueued).
 *  - Every array must hold at least the elements that its documented shape
 *    and the sizes passed with it give.  The library checks the sizes, but it
 *    cannot see the allocation behind a pointer: a shorter buffer is read or
 *    written out of bounds.  (The Python binding checks tensor extents before
 *    it calls.)
 *  - Work is enqueued on the given stream (a cudaStream_t passed as void*; NULL
 *    means the legacy default stream) and is asynchronous unless stated
 *    otherwise: outputs are valid once that stream has been synchronised.
 *  - Errors a kernel detects are recorded in a per-index device error word;
 *    ah_sync_status() reports (and clears) them.
 *  - Ordering everywhere is (score descending, then lower id).  Results shorter
 *    than k are padded with id -1 and score -INFINITY.
 *  - Ids are the original datapoint ids (int32).
 *  - An index may be searched from one stream at a time (it owns one
 *    workspace, and a side stream for stages that do not depend on the
 *    partition stage, joined back before the results are written); different
 *    indexes are independent.
 */
#ifndef AH_H_
#define AH_H_

#include <stdint.h>

#if defined(__GNUC__)
#define AH_API __attribute__((visibility("default")))
#else
#define AH_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    AH_OK = 0,
    AH_ERR_INVALID_ARG = 1,  /* a null pointer, an out-of-range size or knob   */
    AH_ERR_UNSUPPORTED = 2,  /* valid request beyond the library's AH_MAX_*    */
    AH_ERR_OOM = 3,          /* device allocation failed                       */
    AH_ERR_CUDA = 4,         /* a CUDA runtime call failed                     */
    AH_ERR_DEVICE = 5,       /* a kernel reported an error (see ah_sync_status) */
    AH_ERR_TIMEOUT = 6       /* a bounded device wait gave up (ah_sync_status) */
} ah_status;

/* reorder_dtype values */
enum { AH_F32 = 0, AH_BF16 = 1 };
/* lut_mode values */
enum { AH_LUT_F32 = 0, AH_LUT_U8 = 1 };

/* Library limits (AH_ERR_UNSUPPORTED beyond them). */
#define AH_MAX_K 1024            /* final neighbours per query                 */
#define AH_MAX_R 4096            /* max(reorder_num, k)                        */
#define AH_MAX_LEAVES_SEARCHED 4096
#define AH_MAX_D 8192
#define AH_MAX_BLOCKS 1024       /* d / dims_per_block                         */
/* A search with fp32 tables (AH_LUT_F32) keeps eight queries' tables in one
 * scan CTA's shared memory when B = d / dims_per_block is above 400: 512 * B
 * bytes, which the 227 KB per-CTA limit of a B200 bounds at B <= 452 (with
 * 1 KB kept for the kernel's own arrays).  Above that a search with fp32
 * tables returns AH_ERR_UNSUPPORTED before any work is enqueued; uint8 tables
 * (AH_LUT_U8) serve every B up to AH_MAX_BLOCKS. */

/*
 * Index arrays, all in device memory and BORROWED: they must stay allocated
 * and unchanged until ah_destroy().  Source: ScaNN blog, "Three stages of a
 * search" (leaves, 16 centers per block, 4-bit codes) and "Worked example"
 * (64 blocks of 4 bits = 32 B per point at d = 128, dims_per_block = 2).
 *   n               points; 0 < n < 2^31 - 64
 *   d               dimension; divisible by 2 * dims_per_block
 *   num_leaves      NL >= 1 partitions
 *   dims_per_block  dimensions per AH block; B = d / dims_per_block blocks
 *   centroids       float [NL][d]
 *   leaf_offsets    int64 [NL+1]: leaf c holds slots leaf_offsets[c] ..
 *                   leaf_offsets[c+1]-1; non-decreasing, 0 .. n
 *   slot_ids        int32 [n]: original id of the point in each slot
 *   codes           uint8 [n][B/2], slot order; block 2i in the low nibble and
 *                   block 2i+1 in the high nibble of byte i
 *   codebook        float [B][16][dims_per_block]
 *   reorder_vecs    [n][d] slot order, float (AH_F32) or bfloat16 (AH_BF16);
 *                   may be NULL if the index is only searched with
 *                   reorder_num = 0
 *   residual        0: codes quantise each point; 1: codes quantise the
 *                   point minus its leaf's centroid (one codebook for all
 *                   leaves), so the approximate score of a point is the query's
 *                   centroid score of that leaf plus its table sum (added
 *                   after the sum, in fp32).  Residual indexes support fp32
 *                   tables only (AH_LUT_U8 is AH_ERR_UNSUPPORTED).
 */
typedef struct {
    int64_t n;
    int32_t d;
    int32_t num_leaves;
    int32_t dims_per_block;
    const float *centroids;
    const int64_t *leaf_offsets;
    const int32_t *slot_ids;
    const uint8_t *codes;
    const float *codebook;
    const void *reorder_vecs;
    int32_t reorder_dtype;
    int32_t residual;
} ah_index_views;

typedef struct ah_index ah_index;

/*
 * Validate the views and build the derived device state on cuda_stream:
 * int32 leaf offsets and a re-laid-out copy of the codes (32-point tiles of
 * 32-bit words, so a warp reads each code word of 32 consecutive slots with
 * one coalesced 128-byte access).  The copy is owned by the index.  This call
 * synchronises cuda_stream before returning.
 * Errors: AH_ERR_INVALID_ARG (null pointer, bad sizes), AH_ERR_UNSUPPORTED
 * (sizes beyond the limits), AH_ERR_OOM, AH_ERR_CUDA.  *out is NULL on error.
 */
AH_API ah_status ah_build_index_views(const ah_index_views *views, void *cuda_stream, ah_index **out);

/*
 * Search a batch (ScaNN blog, "Three stages of a search"; knobs as in
 * "Using the library": num_leaves_to_search = leaves_to_search, reorder_num =
 * pre_reorder_num_neighbors, k = final_num_neighbors).
 *   queries      float [nq][d], device
 *   nq           >= 0 (0 returns AH_OK with nothing enqueued)
 *   k            1 .. AH_MAX_K
 *   num_leaves_to_search  1 .. min(num_leaves, AH_MAX_LEAVES_SEARCHED)
 *   reorder_num  0 (no exact rescoring: scores are approximate) or >= k;
 *                the R = max(reorder_num, k) best candidates by approximate
 *                score are kept, then rescored exactly ("reorder not above k"
 *                in the post's failure modes); R <= AH_MAX_R
 *   lut_mode     AH_LUT_F32: fp32 table and fp32 sums;
 *                AH_LUT_U8: uint8 table, integer sums; the table is
 *                lut = q0*c0 then fmaf(q_t, c_t, lut), m_b = min_j lut,
 *                delta = max_b(max_j lut - m_b)/255 (1 if 0),
 *                u = min(255, rint((lut - m_b)/delta)), bias = sum_b m_b in
 *                fp32 in block order; approximate score = fmaf(delta, sum, bias).
 *   out_ids      int32 [nq][k], device
 *   out_scores   float [nq][k], device: exact fp32 dot products when
 *                reorder_num > 0, otherwise approximate scores
 * Errors: AH_ERR_INVALID_ARG, AH_ERR_UNSUPPORTED (a size above an AH_MAX_*
 * limit; uint8 tables with residual codes; fp32 tables beyond B = 452, see
 * AH_MAX_BLOCKS), AH_ERR_OOM (workspace growth), AH_ERR_CUDA (launch
 * failure).  Device-side errors of this call are reported by a later
 * ah_sync_status().
 */
AH_API ah_status ah_search(ah_index *ix, const float *queries, int32_t nq, int32_t k,
                    int32_t num_leaves_to_search, int32_t reorder_num, int32_t lut_mode,
                    int32_t *out_ids, float *out_scores, void *cuda_stream);

/*
 * Intermediate results of one search, for inspection and testing.  Every
 * pointer is device memory and optional (NULL to skip).
 *   leaf_ids, leaf_scores  [nq][L]  kept leaves and their fp32 centroid scores
 *   cand_ids, cand_scores  [nq][R]  best R by approximate score (padded -1/-inf)
 *   cand_sums              [nq][R]  uint8 mode: integer sums (0 otherwise)
 *   ncand                  [nq]     candidates kept (<= R)
 *   scanned                [nq]     points whose codes the query scanned
 *   passed                 [nq]     points whose approximate score reached the
 *                                   query's filter bound in the first scan pass
 *   rescans                [1]      queries rescanned after a buffer overflow
 *   cand_exact             [nq][R]  with reorder_num > 0: the exact score of
 *                                   each of cand_ids (same order; padded -inf)
 */
typedef struct {
    int32_t *leaf_ids;
    float *leaf_scores;
    int32_t *cand_ids;
    float *cand_scores;
    uint32_t *cand_sums;
    int32_t *ncand;
    int64_t *scanned;
    int32_t *passed;
    int32_t *rescans;
    float *cand_exact;
} ah_search_trace;

/* ah_search plus the intermediate results named in *trace (may be NULL). */
AH_API ah_status ah_search_traced(ah_index *ix, const float *queries, int32_t nq, int32_t k,
                           int32_t num_leaves_to_search, int32_t reorder_num, int32_t lut_mode,
                           int32_t *out_ids, float *out_scores, const ah_search_trace *trace,
                           void *cuda_stream);

/*
 * ah_search on HOST buffers: host_queries [nq][d], host_ids [nq][k] and
 * host_scores [nq][k] are host memory (pinned memory gives asynchronous
 * copies).  The queries are copied to the device, searched, and the results
 * copied back, all on cuda_stream; the call synchronises cuda_stream and
 * returns with the results in place, including any device-side error.
 */
AH_API ah_status ah_search_host(ah_index *ix, const float *host_queries, int32_t nq, int32_t k,
                         int32_t num_leaves_to_search, int32_t reorder_num, int32_t lut_mode,
                         int32_t *host_ids, float *host_scores, void *cuda_stream);

/*
 * Reserve workspace for searches up to max_nq queries with the given knobs,
 * so later searches allocate nothing.  Synchronous.
 */
AH_API ah_status ah_reserve(ah_index *ix, int32_t max_nq, int32_t k, int32_t num_leaves_to_search,
                     int32_t reorder_num, int32_t lut_mode);

/*
 * Search tuning knobs (they never change results, only speed).
 *   AH_OPT_THRESHOLD_SAMPLE  points scored per query, from its best leaves, to
 *                            bound its R-th best approximate score before the
 *                            scan (default 1024; the bound uses
 *                            max(value, 2 R) points, at most 4096; batches of
 *                            fewer than 1,024 queries use more, up to 4096,
 *                            when the bound would otherwise keep many points)
 *   AH_OPT_THRESHOLD_LEAVES  how many of the best leaves that sample is spread
 *                            over, evenly; the rest of the sample follows
 *                            rank order (default 1: a prefix in rank order)
 *   AH_OPT_PROGRESSIVE_LEAVES  scan each query's best L1 leaves first, raise its
 *                            bound to the R-th best point they kept, then scan
 *                            up to 8x as many leaves at a time the same way:
 *                            0 = automatic (batches of 1,024 or more queries:
 *                            several phases when the sample's bound is
 *                            expected to keep many points; smaller batches:
 *                            one pass with a larger sample), -1 = one pass,
 *                            n = L1
 *   AH_OPT_SCAN_CHUNK_TILES  32-point code tiles per scan work item (0 =
 *                            automatic, the default)
 *   AH_OPT_UINT8_TENSOR_CORES  how the scan sums uint8 tables: 0 = table
 *                            lookups in shared memory (the default); 1 = on
 *                            the int8 tensor cores (each point's codes
 *                            expanded one-hot and multiplied by the queries'
 *                            tables, summed exactly in int32).  The integer
 *                            sums, and so the results, are the same either way.
 *   AH_OPT_QUERY_MAJOR_SCAN  how the scan splits its work: 0 = automatic (the
 *                            default): query-major when on average at most one
 *                            query of the batch searches a leaf (nq x L <= NL)
 *                            and each scan phase covers at most 1,024 leaf
 *                            ranks, leaf-major (queries sharing a leaf share
 *                            its code reads) otherwise; 1 = query-major
 *                            whenever a phase covers at most 1,024 leaf
 *                            ranks; -1 = always leaf-major
 * Errors: AH_ERR_INVALID_ARG for an unknown option or a value out of range.
 */
enum {
    AH_OPT_THRESHOLD_SAMPLE = 1,
    AH_OPT_SCAN_CHUNK_TILES = 2,
    AH_OPT_THRESHOLD_LEAVES = 3,
    AH_OPT_PROGRESSIVE_LEAVES = 4,
    AH_OPT_UINT8_TENSOR_CORES = 5,
    AH_OPT_QUERY_MAJOR_SCAN = 6
};
AH_API ah_status ah_set_option(ah_index *ix, int32_t option, int64_t value);

/*
 * Synchronise cuda_stream, then report and clear the index's device error
 * word: AH_OK, or AH_ERR_DEVICE with ah_last_error() describing it.
 */
AH_API ah_status ah_sync_status(ah_index *ix, void *cuda_stream);

/*
 * Stage timing.  With profiling on, each search records CUDA events around its
 * stages on the search stream; ah_stage_times() synchronises on the last
 * event and writes up to max_stages durations in milliseconds (stage order as
 * ah_stage_name(i)), setting *n_stages.  Synchronous.  on: 0 off, 1 every
 * stage, 2 the scan phases only (the other stages read 0; the kernels before
 * and after the scan then keep their overlapped launches).  Other values:
 * AH_ERR_INVALID_ARG.
 */
AH_API ah_status ah_set_profiling(ah_index *ix, int32_t on);
AH_API ah_status ah_stage_times(ah_index *ix, float *ms, int32_t max_stages, int32_t *n_stages);
AH_API const char *ah_stage_name(int32_t stage);

/*
 * Counters of the last search: kernels launched (*launches) and the points
 * whose codes were scanned, summed over its queries (*points_scanned; asking
 * for it synchronises the device).  Either pointer may be NULL.
 */
AH_API ah_status ah_last_search_info(ah_index *ix, int32_t *launches, int64_t *points_scanned);

/* Device bytes owned by the index (derived state + workspace). */
AH_API ah_status ah_index_memory(ah_index *ix, int64_t *bytes);

/*
 * Partition stage without any device allocation (no counterpart in the
 * paper: it exists for callers that cannot allocate).  Some callers must not
 * allocate device memory on the call path: a serving process whose device
 * memory is reserved up front by another allocator, or a latency-critical
 * loop that cannot afford cudaMalloc's implicit device synchronisation.  For
 * them this call scores the queries against every centroid and keeps the best
 * num_leaves_to_search leaves, the first stage of ah_search, using a scratch
 * area that lives in the library itself: a device array of
 * AH_NOALLOC_SCRATCH_BYTES that every GPU loading the library holds until the
 * process exits.
 *   queries          float [nq][d], device
 *   out_leaf_ids     int32 [nq][num_leaves_to_search], device
 *   out_leaf_scores  float [nq][num_leaves_to_search], device (fp32 q . c)
 * The scratch must hold nq * num_leaves scores plus small counters; larger
 * batches are rejected with AH_ERR_UNSUPPORTED before anything is enqueued
 * (split the batch).  The index's device must be current.  The scratch's
 * device address is looked up when the index is built (ah_build_index_views,
 * ah_load): the first such lookup on a device loads the library's device
 * module that holds the array, which is when the array's memory is placed, so
 * this call itself neither allocates nor loads anything.  The address belongs
 * to the index: after the device's primary context is reset
 * (cudaDeviceReset) indexes built before the reset, and this address with
 * them, are invalid.  All calls share the one scratch area: calls whose work
 * overlaps on the GPU (different streams, or different indexes on one device)
 * race and must be serialised by the caller.  Results equal the leaves
 * ah_search_traced reports.
 */
#define AH_NOALLOC_SCRATCH_BYTES (8u << 20)
AH_API ah_status ah_search_leaves_noalloc(ah_index *ix, const float *queries, int32_t nq,
                                          int32_t num_leaves_to_search, int32_t *out_leaf_ids,
                                          float *out_leaf_scores, void *cuda_stream);

/*
 * Index directories (ScaNN blog, "Using the library": a built searcher is
 * written to a directory and loaded back later).  ah_save writes the index's
 * arrays into the existing directory `dir` as NumPy .npy files (format 1.0,
 * little endian, C order; numpy.load reads each one), overwriting them:
 *   centroids.npy     <f4 [num_leaves, d]
 *   leaf_offsets.npy  <i8 [num_leaves + 1]
 *   slot_ids.npy      <i4 [n]
 *   codes.npy         |u1 [n, d / dims_per_block / 2]
 *   codebook.npy      <f4 [d / dims_per_block, 16, dims_per_block]
 *   reorder_vecs.npy  <f4 [n, d], or <u2 [n, d] holding bfloat16 bit
 *                     patterns (absent when the index has no reorder copy)
 *   ah_index.txt      first line "ah-index 1", then "reorder_dtype f32",
 *                     "reorder_dtype bf16" or "reorder_dtype none", then
 *                     "residual 0" or "residual 1" (absent: 0)
 * Synchronous (device-to-host copies).  Errors: AH_ERR_INVALID_ARG (NULL
 * argument, a file that cannot be written: the message names it),
 * AH_ERR_CUDA.
 */
AH_API ah_status ah_save(ah_index *ix, const char *dir);

/*
 * Reads the sizes of an index directory without using the GPU: fills n, d,
 * num_leaves, dims_per_block and reorder_dtype of *out (-1 for no reorder
 * copy) and sets its pointers to NULL.  Every file's header is checked
 * against the others' and against the file's length.  Errors:
 * AH_ERR_INVALID_ARG (a missing or malformed file; the message names it).
 */
AH_API ah_status ah_inspect(const char *dir, ah_index_views *out);

/*
 * Loads an index directory onto the current device: the arrays are copied
 * into device memory that the index owns (counted by ah_index_memory, freed
 * by ah_destroy), then the index is built as by ah_build_index_views on
 * cuda_stream.  Synchronous.  Errors: those of ah_inspect, AH_ERR_OOM,
 * AH_ERR_CUDA, and those of ah_build_index_views.  *out is NULL on error.
 */
AH_API ah_status ah_load(const char *dir, void *cuda_stream, ah_index **out);

/*
 * Anisotropic code assignment, the index-build step before the search (ScaNN
 * blog, "Training an anisotropic codebook yourself": codes minimise the
 * anisotropic loss; blocks couple through r . u, so the assignment is refined
 * iteratively).  For each point x (row of X):
 *   eta = (d - 1) t / (1 - t), t = (T / ||x||)^2 ("The loss in one
 *   paragraph"); eta = 1 when T <= 0, ||x|| = 0 or t >= 1;
 *   loss(x~) = (eta - 1) ((x - x~) . x / ||x||)^2 + ||x - x~||^2;
 *   start from the nearest center of every block (ties: lower index), then up
 *   to `passes` passes over blocks 0..B-1, each replacing a block's center by
 *   the one of least loss with the other blocks fixed when that is strictly
 *   lower (ties: lower index); a pass without a change ends the descent.
 * fp64 arithmetic, each product and sum rounded separately, sums over a
 * block's coordinates in ascending order (the order is part of the result).
 *   X           [n][d] float, device
 *   codebook    [d/dims_per_block][16][dims_per_block] float, device
 *   codes       [n][d/dims_per_block/2] uint8 out, device: block 2i in the
 *               low nibble of byte i
 *   passes_used [n] int32 out, device, or NULL: passes run per point
 * Asynchronous on cuda_stream; nothing is allocated.  Errors:
 * AH_ERR_INVALID_ARG (NULL array, n < 0, d not divisible by
 * 2 * dims_per_block, passes outside [0, 1000]), AH_ERR_UNSUPPORTED (more
 * than AH_MAX_BLOCKS blocks), AH_ERR_CUDA.
 */
AH_API ah_status ah_encode(const float *X, int64_t n, int32_t d, int32_t dims_per_block, const float *codebook,
                           double T, int32_t passes, uint8_t *codes, int32_t *passes_used, void *cuda_stream);

/*
 * Partition training, the other index-build step (ScaNN blog, "Using the
 * library": the tree's leaves are k-means centroids trained on a sample, and
 * every point goes to its nearest leaf).  One Lloyd iteration is
 * ah_kmeans_assign followed by ah_kmeans_update.
 *
 * ah_kmeans_assign: assign[i] = argmin_c sum_t (X[i][t] - C[c][t])^2 over
 * c < nl, fp64 with every difference, square and sum rounded separately,
 * coordinates in ascending order, ties to the lower c; dist[i] (may be NULL)
 * = that minimum.  X [n][d], C [nl][d] float; assign [n] int32, dist [n]
 * double; all device memory.
 *
 * ah_kmeans_update: for every centroid c, its members i (assign[i] == c) in
 * ascending order are summed per coordinate in fp64 and C_new[c] = sum / m
 * (fp64 division, rounded to float); a centroid without members keeps
 * C_old[c]; counts[c] (may be NULL) = m.  Entries of assign outside [0, nl)
 * belong to no centroid.  C_new must not overlap C_old.
 *
 * Both asynchronous on cuda_stream; nothing is allocated.  Errors:
 * AH_ERR_INVALID_ARG (NULL array, n < 0, d < 1, nl < 1), AH_ERR_UNSUPPORTED
 * (d above AH_MAX_D; for the update, d above 6400), AH_ERR_CUDA.
 */
AH_API ah_status ah_kmeans_assign(const float *X, int64_t n, int32_t d, const float *C, int32_t nl, int32_t *assign,
                                  double *dist, void *cuda_stream);
AH_API ah_status ah_kmeans_update(const float *X, int64_t n, int32_t d, const int32_t *assign, int32_t nl,
                                  const float *C_old, float *C_new, int64_t *counts, void *cuda_stream);

/*
 * Anisotropic center update, the closed-form step of anisotropic k-means
 * (ScaNN blog, "Training an anisotropic codebook yourself", Theorem 4.2 form;
 * loss from "The loss in one paragraph" with h_perp = 1).  For every center c
 * with members i (assign[i] == c), in ascending point order:
 *   eta_i = (d - 1) t / (1 - t), t = (T / ||x_i||)^2 (eta_i = 1 when T <= 0,
 *   ||x_i|| = 0 or t >= 1), u_i = x_i / ||x_i||;
 *   C_new[c] solves (m I + sum_i (eta_i - 1) u_i u_i^T) c = sum_i eta_i x_i,
 * the minimiser of sum_i (eta_i - 1) ((x_i - c) . u_i)^2 + ||x_i - c||^2 (the
 * plain mean when every eta_i = 1).  A center without members keeps C_old[c].
 * The system matrix is never formed: conjugate gradients in fp64 from c = 0,
 * each step applying it as m p + sum_i (eta_i - 1) (u_i . p) u_i, stop when
 * the residual norm is at most tol times ||sum_i eta_i x_i|| or after
 * max_iters steps (the matrix is symmetric positive definite whenever every
 * eta_i > 0, with condition number at most max(eta) / min(eta, 1), so a few
 * tens of steps reach tol = 1e-14).  Every reduction runs in a fixed order, so
 * the result does not depend on scheduling; it is rounded to float at the end.
 *   X [n][d] float, assign [n] int32 (entries outside [0, nl) belong to no
 *   center), C_old [nl][d] float, C_new [nl][d] float out (must not overlap
 *   C_old), counts [nl] int64 out or NULL (members), iters [nl] int32 out or
 *   NULL (steps taken); all device memory.
 * Asynchronous on cuda_stream; a temporary workspace of about 28 n + 12 nl
 * bytes is taken from the device's stream-ordered memory pool on cuda_stream
 * and returned to it on the same stream (no device synchronisation).  Errors:
 * AH_ERR_INVALID_ARG (NULL array, n < 0, d < 1, nl < 1, max_iters outside
 * [0, 100000], tol outside [0, 1)), AH_ERR_UNSUPPORTED (d above 6400, n of
 * 2^31 or more), AH_ERR_OOM, AH_ERR_CUDA.
 */
AH_API ah_status ah_avq_update(const float *X, int64_t n, int32_t d, const int32_t *assign, int32_t nl,
                               const float *C_old, double T, int32_t max_iters, double tol, float *C_new,
                               int64_t *counts, int32_t *iters, void *cuda_stream);

/*
 * Exact merge for a leaf-partitioned search.  G shards hold the same
 * centroids and codebook and disjoint sets of leaves' points (the other
 * leaves empty), so every shard picks the same L leaves and scans its own
 * points of them; the union of the shards' best R by approximate score holds
 * the best R of all points.  Per query this keeps the best R of the G * R
 * entries by (approx desc, id asc) and returns the best k of those by
 * (exact desc, id asc): the result one index over all points gives.
 *   cand_ids     [G][nq][R] int32 (id < 0: padding)    device
 *   cand_approx  [G][nq][R] float: descending order = approximate ranking
 *                (ah_search_trace.cand_scores with fp32 tables; the integer
 *                sums converted to float with uint8 tables)
 *   cand_exact   [G][nq][R] float (ah_search_trace.cand_exact), or NULL when
 *                searched without reorder: the best k by approx are returned
 *   out_ids [nq][k] int32, out_scores [nq][k] float (exact, or approx without
 *                reorder; padding -1 / -inf)            device
 * Asynchronous on cuda_stream.  Errors: AH_ERR_INVALID_ARG (NULL array,
 * G < 1, nq < 0, k < 1, R < k), AH_ERR_UNSUPPORTED (R above AH_MAX_R,
 * G * R above 65536), AH_ERR_CUDA.
 */
AH_API ah_status ah_merge_shards(int32_t G, int32_t nq, int32_t R, int32_t k, const int32_t *cand_ids,
                                 const float *cand_approx, const float *cand_exact, int32_t *out_ids,
                                 float *out_scores, void *cuda_stream);

/* Release everything the index owns.  Does not touch the borrowed views. */
AH_API void ah_destroy(ah_index *ix);

/* Static text for a status code. */
AH_API const char *ah_status_string(ah_status s);

/* Detail of the last error on the calling thread ("" if none). */
AH_API const char *ah_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* AH_H_ */
