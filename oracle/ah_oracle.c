/*
 * Oracle for the anisotropic-AH maximum inner product search path.
 *
 * TEST INFRASTRUCTURE ONLY.  This is a plain, slow, obviously-correct CPU
 * restatement of what a search computes.  Only the test suite, the smoke
 * entry point and the CPU-baseline leg of the benchmark may load it.  It shares
 * no code, header, table or helper with the CUDA library, and the CUDA library
 * never calls it.
 *
 * Source: "ScaNN: Anisotropic Vector Quantization for Maximum Inner Product
 * Search" (blog post), section "Three stages of a search" for the steps, and
 * section "Worked example: cost of one query" for the sizes.  Steps, per query:
 *   1. score every partition centroid, s[c] = q . c  (metric "dot_product");
 *      keep the best num_leaves_to_search leaves;
 *   2. build the lookup table lut[b][j] = q_b . center[b][j] for every block b
 *      and each of its 16 centers j;
 *   3. for every point in the kept leaves, approximate score = sum over blocks
 *      of its table entries lut[b][code_b];
 *   4. keep the best R = max(reorder_num, k) points by approximate score;
 *   5. with reorder_num > 0, rescore those R with exact dot products against
 *      the stored vectors and return the best k; otherwise return the best k
 *      by approximate score ("reorder not above k" failure mode).
 * Orderings are (score descending, then lower id) everywhere; the pages fix no
 * tie-break.  Arithmetic is fp64 on the fp32 inputs, except the optional
 * uint8 lookup-table mode, whose table is defined in fp32 (see lut_u8).
 * Results shorter than k are padded with id -1 and score -infinity.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -fno-fast-math -shared -fPIC.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_CENTERS 16

typedef struct {
    int64_t n;
    int32_t d, num_leaves, dims_per_block;
    const float *centroids;       /* [num_leaves][d] */
    const int64_t *leaf_offsets;  /* [num_leaves + 1] */
    const int32_t *slot_ids;      /* [n] original id of each slot */
    const uint8_t *codes;         /* [n][B/2], block 2i low nibble, 2i+1 high */
    const float *codebook;        /* [B][16][dims_per_block] */
    const void *reorder_vecs;     /* [n][d], float32 or bfloat16 bits */
    int32_t reorder_is_bf16;
    int32_t residual;             /* codes quantise x - centroid of its leaf */
} orc_index;

typedef struct {
    double score;
    int32_t id;     /* tie-break key (original datapoint id, or leaf id) */
    int32_t slot;   /* slot (or leaf) the item refers to */
} orc_item;

typedef struct {
    uint32_t sum;
    int32_t id;
    int32_t slot;
} orc_uitem;

static int by_score_then_id(const void *pa, const void *pb) {
    const orc_item *a = (const orc_item *)pa, *b = (const orc_item *)pb;
    if (a->score > b->score) return -1;
    if (a->score < b->score) return 1;
    return (a->id > b->id) - (a->id < b->id);
}

static int by_sum_then_id(const void *pa, const void *pb) {
    const orc_uitem *a = (const orc_uitem *)pa, *b = (const orc_uitem *)pb;
    if (a->sum > b->sum) return -1;
    if (a->sum < b->sum) return 1;
    return (a->id > b->id) - (a->id < b->id);
}

static int blocks_of(const orc_index *ix) { return ix->d / ix->dims_per_block; }

/* 4-bit center index of block b in one point's code row. */
static int code_of(const uint8_t *row, int b) {
    uint8_t byte = row[b / 2];
    return (b % 2 == 0) ? (byte & 0x0F) : (byte >> 4);
}

/* Stored reorder vector coordinate, upcast to float then double. */
static double stored_coord(const orc_index *ix, int64_t slot, int t) {
    if (ix->reorder_is_bf16) {
        uint16_t h = ((const uint16_t *)ix->reorder_vecs)[slot * ix->d + t];
        uint32_t bits = (uint32_t)h << 16;
        float f;
        memcpy(&f, &bits, sizeof f);
        return (double)f;
    }
    return (double)((const float *)ix->reorder_vecs)[slot * ix->d + t];
}

/* Step 1: s[c] = sum_t q[t] * centroid[c][t]. */
static void centroid_scores(const orc_index *ix, const float *q, double *s) {
    for (int c = 0; c < ix->num_leaves; ++c) {
        double acc = 0.0;
        for (int t = 0; t < ix->d; ++t)
            acc += (double)q[t] * (double)ix->centroids[(int64_t)c * ix->d + t];
        s[c] = acc;
    }
}

/* Step 2 (fp64): lut[b][j] = sum over the block's dims of q * center. */
static void lut_f64(const orc_index *ix, const float *q, double *lut) {
    int B = blocks_of(ix), P = ix->dims_per_block;
    for (int b = 0; b < B; ++b)
        for (int j = 0; j < ORC_CENTERS; ++j) {
            double acc = 0.0;
            for (int t = 0; t < P; ++t)
                acc += (double)q[b * P + t] *
                       (double)ix->codebook[((int64_t)b * ORC_CENTERS + j) * P + t];
            lut[b * ORC_CENTERS + j] = acc;
        }
}

/*
 * Step 2, uint8 mode.  The pages describe no quantised table; this mode is
 * defined here in fp32 with IEEE round-to-nearest operations so that any
 * implementation following the same steps gets identical bits:
 *   (i)   lut = q0*c0, then lut = fmaf(q_t, c_t, lut) for t = 1..dpb-1;
 *   (ii)  m_b = min_j lut[b][j]; delta = max_b (max_j lut[b][j] - m_b) / 255
 *         (delta = 1 when that maximum is 0);
 *   (iii) u = min(255, rint((lut - m_b) / delta)) as uint8;
 *   (iv)  bias = sum_b m_b accumulated in b order in fp32.
 * A point's sum is the uint32 sum of its u entries; its score is
 * fmaf(delta, (float)sum, bias).
 */
static void lut_u8(const orc_index *ix, const float *q, uint8_t *lut8, float *delta_out,
                   float *bias_out) {
    int B = blocks_of(ix), P = ix->dims_per_block;
    float *lut = (float *)malloc(sizeof(float) * (size_t)B * ORC_CENTERS);
    float *mins = (float *)malloc(sizeof(float) * (size_t)B);
    float range_max = 0.0f;
    for (int b = 0; b < B; ++b) {
        float lo = INFINITY, hi = -INFINITY;
        for (int j = 0; j < ORC_CENTERS; ++j) {
            const float *c = &ix->codebook[((int64_t)b * ORC_CENTERS + j) * P];
            float v = q[b * P] * c[0];
            for (int t = 1; t < P; ++t) v = fmaf(q[b * P + t], c[t], v);
            lut[b * ORC_CENTERS + j] = v;
            if (v < lo) lo = v;
            if (v > hi) hi = v;
        }
        mins[b] = lo;
        float r = hi - lo;
        if (r > range_max) range_max = r;
    }
    float delta = range_max / 255.0f;
    if (delta == 0.0f) delta = 1.0f;
    float bias = 0.0f;
    for (int b = 0; b < B; ++b) {
        bias = bias + mins[b];
        for (int j = 0; j < ORC_CENTERS; ++j) {
            float qv = rintf((lut[b * ORC_CENTERS + j] - mins[b]) / delta);
            if (qv > 255.0f) qv = 255.0f;
            lut8[b * ORC_CENTERS + j] = (uint8_t)qv;
        }
    }
    *delta_out = delta;
    *bias_out = bias;
    free(lut);
    free(mins);
}

/* Step 3: sum of a point's table entries. */
static double ah_score_f64(const orc_index *ix, const double *lut, int64_t slot) {
    int B = blocks_of(ix);
    const uint8_t *row = ix->codes + slot * (B / 2);
    double acc = 0.0;
    for (int b = 0; b < B; ++b) acc += lut[b * ORC_CENTERS + code_of(row, b)];
    return acc;
}

static uint32_t ah_sum_u8(const orc_index *ix, const uint8_t *lut8, int64_t slot) {
    int B = blocks_of(ix);
    const uint8_t *row = ix->codes + slot * (B / 2);
    uint32_t acc = 0;
    for (int b = 0; b < B; ++b) acc += lut8[b * ORC_CENTERS + code_of(row, b)];
    return acc;
}

/* Step 5: exact inner product with the stored vector. */
static double exact_score(const orc_index *ix, const float *q, int64_t slot) {
    double acc = 0.0;
    for (int t = 0; t < ix->d; ++t) acc += (double)q[t] * stored_coord(ix, slot, t);
    return acc;
}

/*
 * Steps 2-5 for one query over a given list of L leaves (the order of the list
 * does not matter: every point of the listed leaves is scored, then ranked by
 * (score, id)).  s: the query's fp64 centroid scores (read only for residual
 * codes).  Outputs as for orc_search, for this query's row (NULL to skip).
 */
static void search_in_leaves(const orc_index *ix, const float *q, const double *s, const int32_t *leaf_list,
                             int32_t L, int32_t k, int32_t R, int32_t reorder_num, int32_t lut_mode,
                             int32_t *out_ids, double *out_scores, int32_t *out_cand_ids,
                             double *out_cand_scores, uint32_t *out_cand_sums, int32_t *out_ncand,
                             int64_t *out_scanned) {
    const int B = blocks_of(ix);

    /* 2. lookup table */
    double *lut = NULL;
    uint8_t *lut8 = NULL;
    float delta = 0.0f, bias = 0.0f;
    if (lut_mode == 0) {
        lut = (double *)malloc(sizeof(double) * (size_t)B * ORC_CENTERS);
        lut_f64(ix, q, lut);
    } else {
        lut8 = (uint8_t *)malloc((size_t)B * ORC_CENTERS);
        lut_u8(ix, q, lut8, &delta, &bias);
    }

    /* 3. approximate score of every point in the kept leaves */
    int64_t total = 0;
    for (int i = 0; i < L; ++i) {
        int c = leaf_list[i];
        total += ix->leaf_offsets[c + 1] - ix->leaf_offsets[c];
    }
    orc_item *cand = NULL;
    orc_uitem *ucand = NULL;
    if (lut_mode == 0) cand = (orc_item *)malloc(sizeof(orc_item) * (total > 0 ? total : 1));
    else ucand = (orc_uitem *)malloc(sizeof(orc_uitem) * (total > 0 ? total : 1));
    int64_t m = 0;
    for (int i = 0; i < L; ++i) {
        int c = leaf_list[i];
        for (int64_t p = ix->leaf_offsets[c]; p < ix->leaf_offsets[c + 1]; ++p, ++m) {
            if (lut_mode == 0) {
                /* residual codes: q . x~ = q . centroid + table sum */
                cand[m].score = ix->residual ? ah_score_f64(ix, lut, p) + s[c] : ah_score_f64(ix, lut, p);
                cand[m].id = ix->slot_ids[p];
                cand[m].slot = (int32_t)p;
            } else {
                ucand[m].sum = ah_sum_u8(ix, lut8, p);
                ucand[m].id = ix->slot_ids[p];
                ucand[m].slot = (int32_t)p;
            }
        }
    }
    if (out_scanned) *out_scanned = total;

    /* 4. best R by approximate score */
    if (lut_mode == 0) qsort(cand, total, sizeof(orc_item), by_score_then_id);
    else qsort(ucand, total, sizeof(orc_uitem), by_sum_then_id);
    int32_t nc = total < R ? (int32_t)total : R;
    if (out_ncand) *out_ncand = nc;
    for (int32_t i = 0; i < R; ++i) {
        if (i < nc) {
            if (out_cand_ids) out_cand_ids[i] = lut_mode == 0 ? cand[i].id : ucand[i].id;
            if (out_cand_scores)
                out_cand_scores[i] = lut_mode == 0 ? cand[i].score : (double)fmaf(delta, (float)ucand[i].sum, bias);
            if (out_cand_sums) out_cand_sums[i] = lut_mode == 0 ? 0u : ucand[i].sum;
        } else {
            if (out_cand_ids) out_cand_ids[i] = -1;
            if (out_cand_scores) out_cand_scores[i] = -INFINITY;
            if (out_cand_sums) out_cand_sums[i] = 0u;
        }
    }

    /* 5. reorder (exact rescoring) or pure approximate ranking */
    orc_item *fin = (orc_item *)malloc(sizeof(orc_item) * (nc > 0 ? nc : 1));
    for (int32_t i = 0; i < nc; ++i) {
        int32_t slot = lut_mode == 0 ? cand[i].slot : ucand[i].slot;
        fin[i].id = ix->slot_ids[slot];
        fin[i].slot = slot;
        if (reorder_num > 0) fin[i].score = exact_score(ix, q, slot);
        else if (lut_mode == 0) fin[i].score = cand[i].score;
        else fin[i].score = (double)fmaf(delta, (float)ucand[i].sum, bias);
    }
    if (reorder_num > 0) qsort(fin, nc, sizeof(orc_item), by_score_then_id);
    for (int32_t i = 0; i < k; ++i) {
        if (i < nc) {
            out_ids[i] = fin[i].id;
            out_scores[i] = fin[i].score;
        } else {
            out_ids[i] = -1;
            out_scores[i] = -INFINITY;
        }
    }
    free(fin);
    free(cand);
    free(ucand);
    free(lut);
    free(lut8);
}

static int bad_search_args(const orc_index *ix, const float *Q, int32_t nq, int32_t k, int32_t L,
                           int32_t reorder_num, int32_t lut_mode, const int32_t *out_ids,
                           const double *out_scores) {
    return !ix || !Q || !out_ids || !out_scores || nq < 0 || k <= 0 || L < 1 || L > ix->num_leaves ||
           reorder_num < 0 || (reorder_num > 0 && reorder_num < k) || (lut_mode != 0 && lut_mode != 1) ||
           (lut_mode == 1 && ix->residual);
}

/* Optional per-query output row (NULL stays NULL). */
#define ORC_ROW(ptr, qi, w) ((ptr) ? (ptr) + (int64_t)(qi) * (w) : NULL)

/*
 * Full search.  Required outputs: out_ids/out_scores [nq][k].  Optional (NULL
 * to skip): out_leaves/out_leaf_scores [nq][L]; out_cand_ids, out_cand_scores,
 * out_cand_sums [nq][R]; out_ncand [nq] (candidates kept, <= R);
 * out_scanned [nq] (points whose codes were scanned).
 * lut_mode 0 = fp64 table, 1 = uint8 table.  Returns 0, or -1 on bad arguments.
 */
int orc_search(const orc_index *ix, const float *Q, int32_t nq, int32_t k, int32_t L,
               int32_t reorder_num, int32_t lut_mode, int32_t nthreads,
               int32_t *out_ids, double *out_scores,
               int32_t *out_leaves, double *out_leaf_scores,
               int32_t *out_cand_ids, double *out_cand_scores, uint32_t *out_cand_sums,
               int32_t *out_ncand, int64_t *out_scanned) {
    if (bad_search_args(ix, Q, nq, k, L, reorder_num, lut_mode, out_ids, out_scores)) return -1;
    const int32_t R = reorder_num > k ? reorder_num : k;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int32_t qi = 0; qi < nq; ++qi) {
        const float *q = Q + (int64_t)qi * ix->d;

        /* 1. partition: best L leaves */
        double *s = (double *)malloc(sizeof(double) * ix->num_leaves);
        orc_item *leaves = (orc_item *)malloc(sizeof(orc_item) * ix->num_leaves);
        int32_t *leaf_list = (int32_t *)malloc(sizeof(int32_t) * L);
        centroid_scores(ix, q, s);
        for (int c = 0; c < ix->num_leaves; ++c) {
            leaves[c].score = s[c];
            leaves[c].id = c;
            leaves[c].slot = c;
        }
        qsort(leaves, ix->num_leaves, sizeof(orc_item), by_score_then_id);
        for (int i = 0; i < L; ++i) leaf_list[i] = leaves[i].id;
        if (out_leaves)
            for (int i = 0; i < L; ++i) out_leaves[(int64_t)qi * L + i] = leaves[i].id;
        if (out_leaf_scores)
            for (int i = 0; i < L; ++i) out_leaf_scores[(int64_t)qi * L + i] = leaves[i].score;

        /* 2-5 over those leaves */
        search_in_leaves(ix, q, s, leaf_list, L, k, R, reorder_num, lut_mode, ORC_ROW(out_ids, qi, k),
                         ORC_ROW(out_scores, qi, k), ORC_ROW(out_cand_ids, qi, R), ORC_ROW(out_cand_scores, qi, R),
                         ORC_ROW(out_cand_sums, qi, R), ORC_ROW(out_ncand, qi, 1), ORC_ROW(out_scanned, qi, 1));
        free(leaf_list);
        free(leaves);
        free(s);
    }
    return 0;
}

/*
 * Steps 2-5 only, over caller-given leaves: leaves [nq][L] (each row L
 * distinct leaf ids in [0, num_leaves)) replace step 1's choice; everything
 * after it is the arithmetic of orc_search.  Used to check the downstream
 * stages of a query whose searched leaf set differs from the oracle's own by a
 * near-tie at the L-th leaf.  Outputs as for orc_search (no leaf outputs).
 * Returns 0, or -1 on bad arguments (including a leaf id out of range).
 */
int orc_search_leaves(const orc_index *ix, const float *Q, int32_t nq, int32_t k, int32_t L,
                      const int32_t *leaves, int32_t reorder_num, int32_t lut_mode, int32_t nthreads,
                      int32_t *out_ids, double *out_scores, int32_t *out_cand_ids, double *out_cand_scores,
                      uint32_t *out_cand_sums, int32_t *out_ncand, int64_t *out_scanned) {
    if (bad_search_args(ix, Q, nq, k, L, reorder_num, lut_mode, out_ids, out_scores) || !leaves) return -1;
    for (int64_t i = 0; i < (int64_t)nq * L; ++i)
        if (leaves[i] < 0 || leaves[i] >= ix->num_leaves) return -1;
    const int32_t R = reorder_num > k ? reorder_num : k;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int32_t qi = 0; qi < nq; ++qi) {
        const float *q = Q + (int64_t)qi * ix->d;
        double *s = (double *)malloc(sizeof(double) * ix->num_leaves);
        centroid_scores(ix, q, s);
        search_in_leaves(ix, q, s, leaves + (int64_t)qi * L, L, k, R, reorder_num, lut_mode,
                         ORC_ROW(out_ids, qi, k), ORC_ROW(out_scores, qi, k), ORC_ROW(out_cand_ids, qi, R),
                         ORC_ROW(out_cand_scores, qi, R), ORC_ROW(out_cand_sums, qi, R), ORC_ROW(out_ncand, qi, 1),
                         ORC_ROW(out_scanned, qi, 1));
        free(s);
    }
    return 0;
}

/* Centroid scores of one query (step 1), [num_leaves]. */
void orc_centroid_scores(const orc_index *ix, const float *q, double *out) {
    centroid_scores(ix, q, out);
}

/* Per-slot scores of one query: approximate (fp64 table) and exact. */
void orc_point_scores(const orc_index *ix, const float *q, int64_t nslots, const int64_t *slots,
                      double *out_ah, double *out_exact) {
    int B = blocks_of(ix);
    double *lut = (double *)malloc(sizeof(double) * (size_t)B * ORC_CENTERS);
    lut_f64(ix, q, lut);
    double *s = ix->residual ? (double *)malloc(sizeof(double) * ix->num_leaves) : NULL;
    if (s) centroid_scores(ix, q, s);
    for (int64_t i = 0; i < nslots; ++i) {
        if (out_ah) {
            out_ah[i] = ah_score_f64(ix, lut, slots[i]);
            if (s) {
                /* the slot's leaf: the last c with leaf_offsets[c] <= slot */
                int lo = 0, hi = ix->num_leaves - 1;
                while (lo < hi) {
                    int mid = (lo + hi + 1) / 2;
                    if (ix->leaf_offsets[mid] <= slots[i]) lo = mid; else hi = mid - 1;
                }
                out_ah[i] = out_ah[i] + s[lo];
            }
        }
        if (out_exact) out_exact[i] = exact_score(ix, q, slots[i]);
    }
    free(s);
    free(lut);
}

/* uint8 table of one query (step 2, uint8 mode): lut8 [B][16], delta, bias. */
void orc_u8_table(const orc_index *ix, const float *q, uint8_t *lut8, float *delta, float *bias) {
    lut_u8(ix, q, lut8, delta, bias);
}

/* uint8-mode sums of one query for given slots. */
void orc_u8_sums(const orc_index *ix, const float *q, int64_t nslots, const int64_t *slots,
                 uint32_t *out_sums) {
    int B = blocks_of(ix);
    uint8_t *lut8 = (uint8_t *)malloc((size_t)B * ORC_CENTERS);
    float delta, bias;
    lut_u8(ix, q, lut8, &delta, &bias);
    for (int64_t i = 0; i < nslots; ++i) out_sums[i] = ah_sum_u8(ix, lut8, slots[i]);
    free(lut8);
}

int orc_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------
 * Anisotropic code assignment (index build; ScaNN blog, "Training an
 * anisotropic codebook yourself": codes minimise the anisotropic loss, and
 * since blocks couple through r . u the assignment is refined iteratively).
 *
 * Reading used (one point x, B = d / dpb blocks of 16 centers):
 *   norm = sqrt(sum_t x_t^2); u_t = x_t / norm; t_ = (T / norm)^2 and
 *   eta = (d - 1) t_ / (1 - t_) ("The loss in one paragraph"), or eta = 1
 *   when T <= 0, norm = 0 or t_ >= 1 (no valid anisotropic weight).
 *   Loss of a reconstruction x~: (eta - 1) (r . u)^2 + ||r||^2, r = x - x~.
 *   Start: per block the center of least squared error (ties: lower index).
 *   Then up to `passes` passes over b = 0..B-1; per block, with the other
 *   blocks fixed, the center of least loss (ties: lower index) replaces the
 *   current one only if its loss is strictly lower; a pass without a change
 *   ends the descent.
 * Arithmetic in fp64, every sum over a block's coordinates in ascending
 * order, multiplications and additions rounded separately (no fused
 * multiply-add), in this order:
 *   rpar = sum_t (x_t - x~_t) u_t, rn2 = sum_t (x_t - x~_t)^2 over all t;
 *   per block: wp = rpar - sum_s (x_s - c_cur,s) u_s, wn = rn2 - sum_s
 *   (x_s - c_cur,s)^2; per center j: p_j = wp + sum_s (x_s - c_j,s) u_s,
 *   n_j = wn + sum_s (x_s - c_j,s)^2, loss_j = (eta - 1) (p_j p_j) + n_j;
 *   on a change rpar = p_best, rn2 = n_best.
 * Output: codes [n][B/2] nibble-packed (block 2i low nibble of byte i);
 * passes_used[i] = passes run for point i (0 when none was needed).
 * ------------------------------------------------------------------------ */
void orc_encode(const float *X, int64_t n, int d, int dpb, const float *codebook, double T, int passes,
                uint8_t *codes, int32_t *passes_used) {
    const int B = d / dpb;
#pragma omp parallel for schedule(dynamic, 64)
    for (int64_t i = 0; i < n; ++i) {
        const float *xr = X + i * (int64_t)d;
        int code[4096];
        double nrm2 = 0.0;
        for (int t = 0; t < d; ++t) nrm2 = nrm2 + (double)xr[t] * (double)xr[t];
        const double norm = sqrt(nrm2);
        double eta = 1.0;
        if (T > 0.0 && norm > 0.0) {
            const double tt = (T / norm) * (T / norm);
            if (tt < 1.0) eta = ((double)(d - 1) * tt) / (1.0 - tt);
        }
        const double e1 = eta - 1.0;
        /* L2 start */
        for (int b = 0; b < B; ++b) {
            int best = 0;
            double bestv = 0.0;
            for (int j = 0; j < 16; ++j) {
                double e = 0.0;
                for (int s = 0; s < dpb; ++s) {
                    const double df = (double)xr[b * dpb + s] - (double)codebook[((int64_t)b * 16 + j) * dpb + s];
                    e = e + df * df;
                }
                if (j == 0 || e < bestv) {
                    bestv = e;
                    best = j;
                }
            }
            code[b] = best;
        }
        double rpar = 0.0, rn2 = 0.0;
        for (int b = 0; b < B; ++b)
            for (int s = 0; s < dpb; ++s) {
                const int t = b * dpb + s;
                const double x = (double)xr[t];
                const double u = norm > 0.0 ? x / norm : 0.0;
                const double r = x - (double)codebook[((int64_t)b * 16 + code[b]) * dpb + s];
                rpar = rpar + r * u;
                rn2 = rn2 + r * r;
            }
        int used = 0;
        for (int p = 0; p < passes; ++p) {
            int changed = 0;
            for (int b = 0; b < B; ++b) {
                const float *cb = codebook + (int64_t)b * 16 * dpb;
                const int cur = code[b];
                double wp = rpar, wn = rn2;
                {
                    double sp = 0.0, sn = 0.0;
                    for (int s = 0; s < dpb; ++s) {
                        const double x = (double)xr[b * dpb + s];
                        const double u = norm > 0.0 ? x / norm : 0.0;
                        const double r = x - (double)cb[cur * dpb + s];
                        sp = sp + r * u;
                        sn = sn + r * r;
                    }
                    wp = wp - sp;
                    wn = wn - sn;
                }
                int best = 0;
                double bl = 0.0, bp = 0.0, bn = 0.0, lcur = 0.0;
                for (int j = 0; j < 16; ++j) {
                    double sp = 0.0, sn = 0.0;
                    for (int s = 0; s < dpb; ++s) {
                        const double x = (double)xr[b * dpb + s];
                        const double u = norm > 0.0 ? x / norm : 0.0;
                        const double r = x - (double)cb[j * dpb + s];
                        sp = sp + r * u;
                        sn = sn + r * r;
                    }
                    const double pj = wp + sp, nj = wn + sn;
                    const double l = e1 * (pj * pj) + nj;
                    if (j == cur) lcur = l;
                    if (j == 0 || l < bl) {
                        bl = l;
                        best = j;
                        bp = pj;
                        bn = nj;
                    }
                }
                if (bl < lcur) {
                    code[b] = best;
                    rpar = bp;
                    rn2 = bn;
                    ++changed;
                }
            }
            used = p + 1;
            if (changed == 0) break;
        }
        if (passes_used) passes_used[i] = used;
        uint8_t *out = codes + i * (int64_t)(B / 2);
        for (int b = 0; b < B; b += 2) out[b / 2] = (uint8_t)(code[b] | (code[b + 1] << 4));
    }
}

/* ------------------------------------------------------------------------
 * Partition training (index build; ScaNN blog, "Using the library": the
 * tree's leaves are trained by k-means on a sample of the data, and every
 * point goes to its nearest leaf).
 *
 * Reading used:
 *   assignment  a_i = argmin_c sum_t (x_it - c_t)^2, fp64, t ascending, each
 *               difference, square and sum rounded separately; ties go to
 *               the lower centroid index; dist_i = that minimum.
 *   update      for each centroid c with members (a_i = c, i ascending):
 *               s_t = sum_i x_it in fp64 in ascending i, new c_t = s_t / m
 *               (fp64 division) rounded to float; a centroid without
 *               members keeps its value; counts_c = m.
 * ------------------------------------------------------------------------ */
void orc_kmeans_assign(const float *X, int64_t n, int d, const float *C, int nl, int32_t *assign, double *dist) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        const float *x = X + i * (int64_t)d;
        int best = 0;
        double bd = 0.0;
        for (int c = 0; c < nl; ++c) {
            const float *cr = C + (int64_t)c * d;
            double acc = 0.0;
            for (int t = 0; t < d; ++t) {
                const double df = (double)x[t] - (double)cr[t];
                acc = acc + df * df;
            }
            if (c == 0 || acc < bd) {
                bd = acc;
                best = c;
            }
        }
        assign[i] = best;
        if (dist) dist[i] = bd;
    }
}

void orc_kmeans_update(const float *X, int64_t n, int d, const int32_t *assign, int nl, const float *C_old,
                       float *C_new, int64_t *counts) {
#pragma omp parallel for schedule(dynamic, 4)
    for (int c = 0; c < nl; ++c) {
        double *s = (double *)calloc((size_t)d, sizeof(double));
        int64_t m = 0;
        for (int64_t i = 0; i < n; ++i) {
            if (assign[i] != c) continue;
            const float *x = X + i * (int64_t)d;
            for (int t = 0; t < d; ++t) s[t] = s[t] + (double)x[t];
            ++m;
        }
        for (int t = 0; t < d; ++t)
            C_new[(int64_t)c * d + t] = m ? (float)(s[t] / (double)m) : C_old[(int64_t)c * d + t];
        if (counts) counts[c] = m;
        free(s);
    }
}
