// Host-side launchers of the search kernels (implemented in kernels.cu).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "common.cuh"

namespace ah {

// Queries per scan work item (leaf, query group, slot chunk).
constexpr int kGroupF32 = 8;
constexpr int kGroupU8 = 8;
constexpr int kScanThreads = 256;
#ifndef AH_SAMPLE_MULT
#define AH_SAMPLE_MULT 2
#endif
constexpr int kSampleMult = AH_SAMPLE_MULT;       // the threshold sample holds at least this many times R slots
constexpr int kMaxThresholdSample = 4096;   // slots scored per query for the threshold

// Slots sampled per query for the filter bound: the requested sample, at
// least kSampleMult R (so a small share of them passes), at most
// kMaxThresholdSample.
__host__ __device__ __forceinline__ int threshold_sample(int R, int requested) {
    const int m = (R > requested ? R : requested);
    const int want = m > kSampleMult * R ? m : kSampleMult * R;
    return want < kMaxThresholdSample ? want : kMaxThresholdSample;
}

struct DeviceIndex {
    int64_t n;
    int d, nl, dpb, B, W;                 // W: 32-bit code words per point
    int V;                                // words per lane per vector load of the code copy (4, 2 or 1)
    const float* centroids;               // [NL][d]
    const int32_t* offs;                  // [NL+1] int32 leaf offsets (owned copy)
    const int32_t* ptile;                 // [NL+1] first code tile of each leaf (leaf-padded copy)
    const int32_t* slot_ids;              // [n]
    const uint32_t* codes_il;             // [ptile[NL]][W/V][32][V] leaf-padded tiles (owned)
    const float* codebook;                // [B][16][dpb]
    const float* c_hi;                    // [NL][d] centroids split for the tensor cores (owned; or null)
    const float* c_lo;                    // [NL][d]
    const void* reorder_vecs;             // [n][d]
    int reorder_bf16;
    int residual;                         // codes quantise x - its leaf's centroid: scores add q . centroid
};

struct SearchBuffers {
    // per query
    float* cscore;          // [nq][NL]
    float* q_hi;            // [nq][d] queries split for the tensor cores (or null: SIMT tiles)
    float* q_lo;            // [nq][d]
    uint64_t* topl_tmp;     // [nq][16 L] split top-L survivors (batches of at most 64; or null)
    int32_t* leaves;        // [nq][L]
    float* leaf_scores;     // [nq][L]
    int64_t* scanned;       // [nq]
    float* lut_f32;         // [nq][B][16]
    uint8_t* lut_u8;        // [nq][B][16]
    float* lut_delta;       // [nq]
    float* lut_bias;        // [nq]
    uint64_t* tau;          // [nq] lower bound on the R-th best (score key, id) key
    uint64_t* ckey;         // [nq][cap] kept candidates: (score key, id) keys
    int32_t* cslot;         // [nq][cap] and their slots
    int32_t* count;         // [nq]          (zeroed per search)
    int32_t* tdone;         // [nq]          (zeroed per search) threshold CTAs of the query done
    int32_t* redo;          // [2][nq]       queries to rescan after rounds 0 and 1
    int32_t* order;         // [nq]          finish order: queries with many kept candidates first
    int32_t* counters;      // [8]           (zeroed per search): 0 scan work (first phase), 1..2 redo
                            //               list sizes, 3..4 rescan work of rounds 1..2, 5 scan work
                            //               (second phase)
    // per leaf
    int32_t* qcount;        // [NL]          (zeroed per search)
    int32_t* qcursor;       // [NL]          (zeroed per search)
    int32_t* qoff;          // [NL+1]
    int32_t* item_off;      // [NL+1]
    int32_t* qlist;         // [nq*L]
    int* err;               // device error word
    int cap;                // candidate capacity per query
};

struct SearchArgs {
    const float* queries;
    int nq, k, L, reorder_num, R, lut_mode;
    int chunk;                  // code tiles (32 slots each) per scan work item
    int32_t* out_ids;
    float* out_scores;
    // optional trace outputs
    int32_t* tr_leaf_ids;
    float* tr_leaf_scores;
    int32_t* tr_cand_ids;
    float* tr_cand_scores;
    uint32_t* tr_cand_sums;
    int32_t* tr_ncand;
    int64_t* tr_scanned;
    int32_t* tr_passed;
    float* tr_cand_exact;       // [nq][R] exact scores of the traced candidates
    int32_t* tr_rescans;
    int scan_item_off_smem;     // set by the scan launcher
    int topl_row_smem;          // set by the top-leaves launcher
    int reorder_vec4;           // set by the finish launcher: 16-byte vector loads of 4 floats (1) or
                                // of 8 bfloat16 values (2) allowed
    int reorder_lanes;          // set by the finish launcher: lanes per rescored candidate
    int threshold_sample;       // slots sampled per query for the filter bound (requested)
    int threshold_leaves;       // best leaves the sample is spread over
    int scan_counter;           // index into counters[] of the scan's work counter
    int count_ranks;            // top-L kernel counts queries per leaf for ranks below this
    int topl_seg;               // split top-L: scores per segment (set by the top-L launcher)
    int topl_stride;            // split top-L: keys per query in topl_tmp
    int scan_tc;                // uint8 tables: scan on the int8 tensor cores (items of up to 128
                                // queries x 256 points) instead of table lookups
    int threshold_parts;        // CTAs per query scoring the threshold sample (1: one CTA does all)
};

// Build-time: the leaf-padded tiled code copy; V = code_vector_words(W).
int code_vector_words(int W);
cudaError_t launch_prepare_index(const int32_t* offs32, const int32_t* ptile, int nl, const uint8_t* codes, int cb,
                                 int W, int64_t ntiles, uint32_t* codes_il, cudaStream_t s);

cudaError_t launch_centroid_scores(const DeviceIndex& ix, const SearchArgs& a, const SearchBuffers& b, cudaStream_t s);
cudaError_t launch_top_leaves(const DeviceIndex& ix, SearchArgs a, const SearchBuffers& b, cudaStream_t s);
cudaError_t launch_invert(const DeviceIndex& ix, const SearchArgs& a, const SearchBuffers& b, int r0, int r1,
                          bool counted, cudaStream_t s);
cudaError_t launch_tau_update(const DeviceIndex& ix, const SearchArgs& a, const SearchBuffers& b, cudaStream_t s);
cudaError_t launch_lut(const DeviceIndex& ix, const SearchArgs& a, const SearchBuffers& b, cudaStream_t s);
cudaError_t launch_threshold(const DeviceIndex& ix, const SearchArgs& a, const SearchBuffers& b, cudaStream_t s);
cudaError_t launch_scan(const DeviceIndex& ix, const SearchArgs& a, const SearchBuffers& b, int num_sms, cudaStream_t s);
// Query-major scan of leaf ranks [r0, r1) of every query (r1 - r0 at most
// kQScanMaxLeaves), for batches whose queries seldom share a leaf: no leaf
// inversion needed.
constexpr int kQScanThreads = 256;
constexpr int kQScanMaxLeaves = 1024;
size_t scan_query_smem_bytes(int mode, int B, int leaves);
cudaError_t launch_scan_query(const DeviceIndex& ix, const SearchArgs& a, const SearchBuffers& b, int r0, int r1,
                              int num_sms, cudaStream_t s);
// best R, exact reorder, best k.  round 0: all queries; rounds 1..2: the
// redo list of the previous round
cudaError_t launch_finish(const DeviceIndex& ix, SearchArgs a, const SearchBuffers& b, int round, int num_sms,
                          cudaStream_t s);
cudaError_t launch_redo_scan(const DeviceIndex& ix, const SearchArgs& a, const SearchBuffers& b, int round,
                             int num_sms, cudaStream_t s);

int scan_group(const DeviceIndex& ix, int lut_mode);
// Shared memory the scan needs for one query group's tables (its launch adds
// at most the leaf item offsets when they fit, and 144 B of static arrays).
size_t scan_table_bytes(const DeviceIndex& ix, int lut_mode);
constexpr size_t kMaxSmemPerCta = 227 * 1024;   // sm_100 opt-in shared memory per CTA
size_t finish_smem_bytes(int R, int d);

// anisotropic code assignment (encode.cu)
size_t encode_smem_bytes(int d, int dpb, bool* cb_in_smem, bool* use_u);
cudaError_t launch_encode(const float* X, int64_t n, int d, int dpb, const float* codebook, double T, int passes,
                          uint8_t* codes, int32_t* passes_used, int num_sms, cudaStream_t s);

// partition training (kmeans.cu)
cudaError_t launch_kmeans_assign(const float* X, int64_t n, int d, const float* C, int nl, int32_t* assign,
                                 double* dist, cudaStream_t s);
size_t kmeans_update_smem_bytes(int d);
cudaError_t launch_kmeans_update(const float* X, int64_t n, int d, const int32_t* assign, int nl, const float* C_old,
                                 float* C_new, int64_t* counts, cudaStream_t s);

// closed-form anisotropic center update (avq.cu)
size_t avq_solve_smem_bytes(int d);
size_t avq_workspace_bytes(int64_t n, int nl);
cudaError_t launch_avq_update(const float* X, int64_t n, int d, const int32_t* assign, int nl, const float* C_old,
                              double T, float* C_new, int64_t* counts, int32_t* iters, int max_iters, double tol,
                              void* workspace, cudaStream_t s);

// uint8-table scan on the int8 tensor cores (scan_tc.cu)
int scan_tc_group();
int scan_tc_chunk_tiles();
size_t scan_tc_smem_bytes();
cudaError_t launch_scan_tc(const DeviceIndex& ix, const SearchArgs& a, const SearchBuffers& b, int num_sms,
                           cudaStream_t s);

// centroid scores on the tensor cores (centroid_tc.cu)
bool centroid_tc_usable(int nq, int nl, int d);
size_t centroid_tc_smem_bytes();
cudaError_t launch_split_tf32(const float* x, int64_t n, float* hi, float* lo, cudaStream_t s);
cudaError_t launch_centroid_scores_tc(const float* q_hi, const float* q_lo, const float* c_hi, const float* c_lo,
                                      float* S, int nq, int nl, int d, int* err, cudaStream_t s);

// exact merge of per-shard candidates (merge.cu)
cudaError_t launch_merge_shards(int G, int nq, int R, int k, const int32_t* ids, const float* approx,
                                const float* exact, int32_t* out_ids, float* out_scores, cudaStream_t s);

}  // namespace ah
