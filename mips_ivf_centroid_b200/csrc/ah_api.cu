// C ABI of the B200 anisotropic-AH MIPS search library (declared in include/ah.h).
//
// Host-side orchestration only: argument validation, the index's owned device
// state, workspace management and the launch sequence of the search kernels
// (kernels.cu) on the caller's stream.  No search arithmetic happens here.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <new>
#include <string>
#include <vector>

#include "ah.h"
#include "kernels.h"
#include "npy_io.h"

namespace {

thread_local std::string g_last_error;

ah_status fail(ah_status s, const std::string& msg) {
    g_last_error = msg;
    return s;
}

ah_status cuda_fail(cudaError_t e, const char* what) {
    g_last_error = std::string(what) + ": " + cudaGetErrorString(e);
    // The status carries the error; clear the runtime's per-thread last error
    // so that a non-sticky failure (a refused launch attribute, an allocation)
    // is not reported again by the caller's or the next call's error check.
    (void)cudaGetLastError();
    return e == cudaErrorMemoryAllocation ? AH_ERR_OOM : AH_ERR_CUDA;
}

constexpr int kStages = 10;
const char* kStageNames[kStages] = {"centroid_scores", "top_leaves", "invert", "lut", "threshold",
                                    "scan", "refine", "scan_rest", "finish", "rescan"};

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct Workspace {
    void* base = nullptr;
    size_t bytes = 0;
    // capacity this carving was made for
    int nq = 0, L = 0, R = 0, lut_mode = -1;
    ah::SearchBuffers buf{};
    // host-call staging
    float* dq = nullptr;
    int32_t* dids = nullptr;
    float* dscores = nullptr;
    int k = 0;
};

int cap_for(int R) { return std::max(8192, 16 * R); }



}  // namespace

// Scratch of ah_search_leaves_noalloc: the centroid score matrix and the
// per-leaf counters of the partition stage, in a file-scope device array so
// that the call never allocates.  On the host this name is only a stand-in for
// the array, not its device address: host code obtains the address with
// cudaGetSymbolAddress (on the current device) and passes that to kernels.
static __device__ __align__(256) unsigned char g_noalloc_scratch[AH_NOALLOC_SCRATCH_BYTES];

namespace {
// Device address of the scratch array on the current device.  The first
// lookup on a device loads this file's device module, which places the array
// in device memory; it is done when an index is built, so the search-time
// call itself neither allocates nor loads anything.
ah_status lookup_noalloc_scratch(void** out) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "scratch address lookup");
    *out = p;
    return AH_OK;
}
}  // namespace

struct ah_index {
    ah_index_views views{};
    ah::DeviceIndex dix{};
    int device = 0;
    int num_sms = 0;
    int32_t* offs32 = nullptr;
    int32_t* ptile = nullptr;
    uint32_t* codes_il = nullptr;
    float* c_split = nullptr;        // [2][NL][d] centroids split for the tensor-core scores (or null)
    int* err = nullptr;
    size_t owned_bytes = 0;
    Workspace ws;
    int profiling = 0;               // 0 off, 1 every stage, 2 scan phases only
    static constexpr int kMaxMarks = 64;
    cudaEvent_t ev[kMaxMarks]{};
    int mark_stage[kMaxMarks]{};      // stage ending at mark i (-1: none)
    int n_marks = 0;
    bool ev_ready = false;
    bool ev_recorded = false;
    int last_launches = 0;
    int last_nq = 0;
    int opt_threshold_sample = 1024;
    int opt_threshold_leaves = 1;
    int opt_progressive_leaves = 0;
    int opt_chunk_tiles = 0;
    int opt_u8_tensor = 0;           // uint8 scan: 0 table lookups (default), 1 int8 tensor cores
    int opt_query_scan = 0;          // query-major scan: 0 automatic, 1 whenever it applies, -1 never
    void* loaded[6] = {};            // index arrays owned by an index from ah_load
    void* noalloc_scratch = nullptr; // device address of the library's fixed scratch on this device
    // side stream for the stages that do not depend on the partition stage
    // (lookup tables; the query->leaf inversion once top-L is known)
    cudaStream_t side = nullptr;
    cudaEvent_t ev_fork = nullptr, ev_tl = nullptr, ev_lut = nullptr, ev_inv = nullptr;
};

namespace {

ah_status carve(ah_index* ix, int nq, int L, int R, int lut_mode, int k, bool host_staging) {
    Workspace& w = ix->ws;
    const bool fits = w.base && nq <= w.nq && L <= w.L && R <= w.R && (lut_mode == w.lut_mode || w.lut_mode == 2) &&
                      (!host_staging || (w.dq && k <= w.k));
    if (fits) return AH_OK;
    // grow: keep the larger of old and new needs
    int cnq = std::max(nq, w.nq), cL = std::max(L, w.L), cR = std::max(R, w.R);
    int mode = (w.lut_mode >= 0 && w.lut_mode != lut_mode) ? 2 : lut_mode;
    int ck = std::max(k, w.k);
    bool stage = host_staging || w.dq;
    const int NL = ix->dix.nl, B = ix->dix.B, d = ix->dix.d;
    const int cap = cap_for(cR);
    size_t sz[32];
    int n = 0;
    auto add = [&](size_t bytes) { sz[n++] = align_up(bytes, 256); };
    add(sizeof(float) * (size_t)cnq * NL);                      // 0 cscore
    add(sizeof(int32_t) * (size_t)cnq * cL);                    // 1 leaves
    add(sizeof(float) * (size_t)cnq * cL);                      // 2 leaf_scores
    add(sizeof(int64_t) * (size_t)cnq);                         // 3 scanned
    add((mode == 0 || mode == 2) ? sizeof(float) * (size_t)cnq * B * 16 : 0);   // 4 lut_f32
    add((mode == 1 || mode == 2) ? (size_t)cnq * B * 16 : 0);                   // 5 lut_u8
    add(sizeof(float) * (size_t)cnq);                           // 6 delta
    add(sizeof(float) * (size_t)cnq);                           // 7 bias
    add(sizeof(uint64_t) * (size_t)cnq);                        // 8 tau
    add(sizeof(uint64_t) * (size_t)cnq * cap);                  // 9 candidate keys
    add(sizeof(int32_t) * (size_t)(2 * NL + 2 * cnq + 8));      // 10 zero region: qcount, qcursor, count, counters, tdone
    add(sizeof(int32_t) * (size_t)2 * cnq);                     // 11 redo
    add(sizeof(int32_t) * (size_t)(NL + 1));                    // 12 qoff
    add(sizeof(int32_t) * (size_t)(NL + 1));                    // 13 item_off
    add(sizeof(int32_t) * (size_t)cnq * cL);                    // 14 qlist
    add(stage ? sizeof(float) * (size_t)cnq * d : 0);           // 15 dq
    add(stage ? sizeof(int32_t) * (size_t)cnq * ck : 0);        // 16 dids
    add(stage ? sizeof(float) * (size_t)cnq * ck : 0);          // 17 dscores
    add(sizeof(int32_t) * (size_t)cnq * cap);                   // 18 candidate slots
    add(sizeof(int32_t) * (size_t)cnq);                         // 19 finish order
    add(ix->c_split ? 2 * sizeof(float) * (size_t)cnq * d : 0);  // 20 queries split for the tensor cores
    const bool split_topl = NL > 4096 && cL <= 256;
    add(split_topl ? sizeof(uint64_t) * (size_t)std::min(cnq, 64) * 16 * cL : 0);   // 21 split top-L survivors
    size_t total = 0;
    for (int i = 0; i < n; ++i) total += sz[i];
    if (w.base) {
        cudaError_t e = cudaDeviceSynchronize();   // the old workspace may still be in use
        if (e != cudaSuccess) return cuda_fail(e, "workspace growth sync");
        cudaFree(w.base);
        ix->owned_bytes -= w.bytes;
        w.base = nullptr;
        w.bytes = 0;
    }
    void* base = nullptr;
    cudaError_t e = cudaMalloc(&base, total);
    if (e != cudaSuccess) return cuda_fail(e, "workspace allocation");
    w.base = base;
    w.bytes = total;
    ix->owned_bytes += total;
    char* p = static_cast<char*>(base);
    char* part[32];
    for (int i = 0; i < n; ++i) {
        part[i] = p;
        p += sz[i];
    }
    ah::SearchBuffers& b = w.buf;
    b.cscore = reinterpret_cast<float*>(part[0]);
    b.leaves = reinterpret_cast<int32_t*>(part[1]);
    b.leaf_scores = reinterpret_cast<float*>(part[2]);
    b.scanned = reinterpret_cast<int64_t*>(part[3]);
    b.lut_f32 = reinterpret_cast<float*>(part[4]);
    b.lut_u8 = reinterpret_cast<uint8_t*>(part[5]);
    b.lut_delta = reinterpret_cast<float*>(part[6]);
    b.lut_bias = reinterpret_cast<float*>(part[7]);
    b.tau = reinterpret_cast<uint64_t*>(part[8]);
    b.ckey = reinterpret_cast<uint64_t*>(part[9]);
    b.cslot = reinterpret_cast<int32_t*>(part[18]);
    b.order = reinterpret_cast<int32_t*>(part[19]);
    b.q_hi = ix->c_split ? reinterpret_cast<float*>(part[20]) : nullptr;
    b.q_lo = ix->c_split ? b.q_hi + (size_t)cnq * d : nullptr;
    b.topl_tmp = split_topl ? reinterpret_cast<uint64_t*>(part[21]) : nullptr;
    int32_t* zr = reinterpret_cast<int32_t*>(part[10]);
    b.qcount = zr;
    b.qcursor = zr + NL;
    b.count = zr + 2 * NL;
    b.counters = zr + 2 * NL + cnq;
    b.tdone = zr + 2 * NL + cnq + 8;
    b.redo = reinterpret_cast<int32_t*>(part[11]);
    b.qoff = reinterpret_cast<int32_t*>(part[12]);
    b.item_off = reinterpret_cast<int32_t*>(part[13]);
    b.qlist = reinterpret_cast<int32_t*>(part[14]);
    b.err = ix->err;
    b.cap = cap;
    w.dq = stage ? reinterpret_cast<float*>(part[15]) : nullptr;
    w.dids = stage ? reinterpret_cast<int32_t*>(part[16]) : nullptr;
    w.dscores = stage ? reinterpret_cast<float*>(part[17]) : nullptr;
    w.nq = cnq;
    w.L = cL;
    w.R = cR;
    w.lut_mode = mode;
    w.k = stage ? ck : 0;
    return AH_OK;
}

// The index's pointers and workspace belong to the device it was built on; a
// call made with another device current would allocate and launch there.
ah_status check_current_device(const ah_index* ix) {
    int device = -1;
    cudaError_t e = cudaGetDevice(&device);
    if (e != cudaSuccess) return cuda_fail(e, "device query");
    if (device != ix->device)
        return fail(AH_ERR_INVALID_ARG, "the index's device (" + std::to_string(ix->device) +
                                            ") is not the current device (" + std::to_string(device) + ")");
    return AH_OK;
}

ah_status validate_search(ah_index* ix, const void* queries, int32_t nq, int32_t k, int32_t L, int32_t reorder_num,
                          int32_t lut_mode, const void* out_ids, const void* out_scores) {
    if (!ix) return fail(AH_ERR_INVALID_ARG, "index is NULL");
    if (ah_status st = check_current_device(ix); st != AH_OK) return st;
    if (nq < 0) return fail(AH_ERR_INVALID_ARG, "nq < 0");
    if (nq > 0 && (!queries || !out_ids || !out_scores)) return fail(AH_ERR_INVALID_ARG, "NULL queries or outputs");
    if (k <= 0) return fail(AH_ERR_INVALID_ARG, "k must be >= 1");
    if (k > AH_MAX_K) return fail(AH_ERR_UNSUPPORTED, "k above AH_MAX_K");
    if (L < 1 || L > ix->dix.nl) return fail(AH_ERR_INVALID_ARG, "num_leaves_to_search outside [1, num_leaves]");
    if (L > AH_MAX_LEAVES_SEARCHED) return fail(AH_ERR_UNSUPPORTED, "num_leaves_to_search above AH_MAX_LEAVES_SEARCHED");
    if (reorder_num < 0 || (reorder_num > 0 && reorder_num < k))
        return fail(AH_ERR_INVALID_ARG, "reorder_num must be 0 or >= k");
    if (std::max(reorder_num, k) > AH_MAX_R) return fail(AH_ERR_UNSUPPORTED, "max(reorder_num, k) above AH_MAX_R");
    if (reorder_num > 0 && !ix->views.reorder_vecs)
        return fail(AH_ERR_INVALID_ARG, "reorder_num > 0 but the index has no reorder vectors");
    if (lut_mode != AH_LUT_F32 && lut_mode != AH_LUT_U8) return fail(AH_ERR_INVALID_ARG, "unknown lut_mode");
    if (lut_mode == AH_LUT_U8 && ix->views.residual)
        return fail(AH_ERR_UNSUPPORTED, "uint8 tables need codes of the points, not residuals");
    if (ah::scan_table_bytes(ix->dix, lut_mode) + 1024 > ah::kMaxSmemPerCta)
        return fail(AH_ERR_UNSUPPORTED, "a query group's fp32 tables exceed the scan's shared memory at this many "
                                        "blocks (d / dims_per_block above 452); use uint8 tables");
    const int64_t per_query_cand = static_cast<int64_t>(cap_for(std::max(reorder_num, k)));
    if (static_cast<int64_t>(nq) * per_query_cand > (int64_t(1) << 40)) return fail(AH_ERR_UNSUPPORTED, "batch too large");
    return AH_OK;
}

ah_status run_search(ah_index* ix, const float* queries, int32_t nq, int32_t k, int32_t L, int32_t reorder_num,
                     int32_t lut_mode, int32_t* out_ids, float* out_scores, const ah_search_trace* tr,
                     cudaStream_t s) {
    const int R = std::max(reorder_num, k);
    ah_status st = carve(ix, nq, L, R, lut_mode, 0, false);
    if (st != AH_OK) return st;
    ah::SearchBuffers b = ix->ws.buf;
    ah::SearchArgs a{};
    a.queries = queries;
    a.nq = nq;
    a.k = k;
    a.L = L;
    a.reorder_num = reorder_num;
    a.R = R;
    a.lut_mode = lut_mode;
    // uint8 tables: the int8 tensor-core scan only when asked for (on the
    // benchmarked batches it ran 1.1-2.9x slower than the table lookups)
    a.scan_tc = (lut_mode == AH_LUT_U8 && ix->opt_u8_tensor == 1) ? 1 : 0;
    // code tiles per scan item: up to 128 (each item stages its group's
    // tables, so long items stage less), fewer (multiples of 8, one tile per
    // warp of a 256-thread CTA) when the batch's tiles, estimated from the
    // average leaf, would give scan CTAs (about 6 per SM) fewer than about 32
    // items each, which leaves a ragged end on small batches
    {
        const double est_tiles = static_cast<double>(nq) * L * std::max(1.0, static_cast<double>(ix->dix.n) / ix->dix.nl / 32.0);
        const double ctas = static_cast<double>(ix->num_sms) * 6;
        const int c = 8 * static_cast<int>(std::ceil(est_tiles / ctas / 32.0 / 8.0));
        a.chunk = ix->opt_chunk_tiles > 0 ? ix->opt_chunk_tiles : std::min(128, std::max(8, c));
        if (a.scan_tc) a.chunk = ah::scan_tc_chunk_tiles();
    }
    a.threshold_sample = ix->opt_threshold_sample;
    a.threshold_parts = 1;
    a.threshold_leaves = ix->opt_threshold_leaves;
    a.out_ids = out_ids;
    a.out_scores = out_scores;
    if (tr) {
        a.tr_leaf_ids = tr->leaf_ids;
        a.tr_leaf_scores = tr->leaf_scores;
        a.tr_cand_ids = tr->cand_ids;
        a.tr_cand_scores = tr->cand_scores;
        a.tr_cand_sums = tr->cand_sums;
        a.tr_ncand = tr->ncand;
        a.tr_scanned = tr->scanned;
        a.tr_passed = tr->passed;
        a.tr_cand_exact = tr->cand_exact;
        a.tr_rescans = tr->rescans;
    }
    const ah::DeviceIndex& dix = ix->dix;
    const bool prof = ix->profiling && ix->ev_ready;
    int launches = 0;
    cudaError_t e;
    // mark(stage): the interval since the previous mark belongs to `stage`
    ix->n_marks = 0;
    // level 2 marks only the scan phases (stages 4..7: the first such mark
    // opens the interval), so the rest of the kernel chain runs unbroken
    auto mark = [&](int stage) {
        if (prof && ix->n_marks < ah_index::kMaxMarks && (ix->profiling == 1 || (stage >= 4 && stage <= 7))) {
            ix->mark_stage[ix->n_marks] = stage;
            cudaEventRecord(ix->ev[ix->n_marks++], s);
        }
    };
    e = cudaMemsetAsync(b.qcount, 0, sizeof(int32_t) * (size_t)(2 * dix.nl + 2 * ix->ws.nq + 8), s);
    if (e != cudaSuccess) return cuda_fail(e, "memset");
    // With per-stage profiling everything runs in order on s (clean stage
    // times); otherwise the tables and the inversion run on the side stream,
    // joined back before the threshold and the scan.
    const bool fork = ix->profiling != 1;
    if (fork && !ix->side) {
        if ((e = cudaStreamCreateWithFlags(&ix->side, cudaStreamNonBlocking)) != cudaSuccess)
            return cuda_fail(e, "side stream");
        for (cudaEvent_t* ev : {&ix->ev_fork, &ix->ev_tl, &ix->ev_lut, &ix->ev_inv})
            if ((e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming)) != cudaSuccess)
                return cuda_fail(e, "side stream events");
    }
    const cudaStream_t s2 = fork ? ix->side : s;
    if (fork) {
        if ((e = cudaEventRecord(ix->ev_fork, s)) != cudaSuccess || (e = cudaStreamWaitEvent(s2, ix->ev_fork, 0)) != cudaSuccess)
            return cuda_fail(e, "fork");
        if ((e = ah::launch_lut(dix, a, b, s2)) != cudaSuccess) return cuda_fail(e, "lut");
        if ((e = cudaEventRecord(ix->ev_lut, s2)) != cudaSuccess) return cuda_fail(e, "fork");
    }
    mark(-1);
    if ((e = ah::launch_centroid_scores(dix, a, b, s)) != cudaSuccess) return cuda_fail(e, "centroid scores");
    launches += 1;
    // Scan phases over leaf ranks [bounds[p], bounds[p+1]).  One phase when
    // the bound from the sample is expected to keep few points; otherwise the
    // first phase is small enough for that bound, each later phase covers up
    // to 8x the leaves scanned so far, and between phases every query's bound
    // is raised to the R-th best point kept (and its buffer compacted).
    std::vector<int> bounds{0};
    {
        const double avg_leaf = static_cast<double>(dix.n) / dix.nl;
        // points the sample's bound is expected to keep: about 0.25 R of
        // every M scanned (the sample comes from the best leaves)
        auto expect = [&](int M) { return 0.25 * a.R * L * avg_leaf / M; };
        // batches under 1,024 queries: the sample grows (up to 4,096 points)
        // until the expected kept set is an eighth of the buffer, and the scan
        // runs in one pass; on the 50M-point sweep index this beat scan
        // phases at every batch of 16-256 queries (phase boundaries cost more
        // there than the larger sample)
        const bool small = nq < 1024;
        if (small && ix->opt_progressive_leaves == 0) {
            const double need = 0.25 * a.R * L * avg_leaf / (b.cap / 8);
            a.threshold_sample = std::max(ix->opt_threshold_sample,
                                          static_cast<int>(std::min<double>(ah::kMaxThresholdSample, std::ceil(need))));
        }
        const int M = ah::threshold_sample(a.R, a.threshold_sample);
        // batches too small to give every SM a query: several CTAs per query
        // score the sample (256 points or more each; the last to finish
        // selects the bound)
        if (nq < ix->num_sms)
            a.threshold_parts = std::max(1, std::min((2 * ix->num_sms + nq - 1) / nq, M / 256));
        int first = L;
        if (ix->opt_progressive_leaves > 0) first = std::min(L, ix->opt_progressive_leaves);
        else if (ix->opt_progressive_leaves == 0 && !small && expect(M) > b.cap / 8)
            first = std::max(1, std::min(L, static_cast<int>(4.0 * M / avg_leaf)));
        for (int e2 = first; ; e2 = std::min(L, 8 * e2)) {
            bounds.push_back(e2);
            if (e2 >= L) break;
        }
    }
    // Query-major scan when the batch's queries seldom share a leaf (on
    // average at most one query per leaf over the searched ranks): the
    // leaf-major groups would almost all be lone queries, each item staging
    // its table again.  It needs no leaf inversion.
    bool qmajor = false;
    if (!a.scan_tc && ix->opt_query_scan >= 0) {
        int widest = 0;
        for (size_t p = 0; p + 1 < bounds.size(); ++p) widest = std::max(widest, bounds[p + 1] - bounds[p]);
        const bool fits = widest <= ah::kQScanMaxLeaves &&
                          ah::scan_query_smem_bytes(lut_mode, dix.B, widest) <= ah::kMaxSmemPerCta;
        qmajor = fits && (ix->opt_query_scan == 1 || static_cast<double>(nq) * L <= static_cast<double>(dix.nl));
    }
    mark(0);
    a.count_ranks = bounds[1];
    if ((e = ah::launch_top_leaves(dix, a, b, s)) != cudaSuccess) return cuda_fail(e, "top leaves");
    launches += 1;
    mark(1);
    if (fork) {
        if ((e = cudaEventRecord(ix->ev_tl, s)) != cudaSuccess || (e = cudaStreamWaitEvent(s2, ix->ev_tl, 0)) != cudaSuccess)
            return cuda_fail(e, "fork");
    }
    if (!qmajor) {
        if ((e = ah::launch_invert(dix, a, b, bounds[0], bounds[1], true, s2)) != cudaSuccess) return cuda_fail(e, "invert");
        launches += 2;
    }
    mark(2);
    if (fork) {
        if ((e = cudaEventRecord(ix->ev_inv, s2)) != cudaSuccess || (e = cudaStreamWaitEvent(s, ix->ev_lut, 0)) != cudaSuccess)
            return cuda_fail(e, "join");
    } else if ((e = ah::launch_lut(dix, a, b, s)) != cudaSuccess) {
        return cuda_fail(e, "lut");
    }
    launches += 1;
    mark(3);
    if ((e = ah::launch_threshold(dix, a, b, s)) != cudaSuccess) return cuda_fail(e, "threshold");
    launches += 1;
    if (fork && (e = cudaStreamWaitEvent(s, ix->ev_inv, 0)) != cudaSuccess) return cuda_fail(e, "join");
    mark(4);
    for (size_t p = 0; p + 1 < bounds.size(); ++p) {
        if (p > 0) {
            if ((e = ah::launch_tau_update(dix, a, b, s)) != cudaSuccess) return cuda_fail(e, "bound refinement");
            launches += 1;
            if (!qmajor) {
                if ((e = ah::launch_invert(dix, a, b, bounds[p], bounds[p + 1], false, s)) != cudaSuccess)
                    return cuda_fail(e, "invert");
                launches += 3;
            }
            mark(6);
        }
        if (qmajor) {
            if ((e = ah::launch_scan_query(dix, a, b, bounds[p], bounds[p + 1], ix->num_sms, s)) != cudaSuccess)
                return cuda_fail(e, "scan");
        } else {
            a.scan_counter = 0;
            if ((e = cudaMemsetAsync(b.counters, 0, sizeof(int32_t), s)) != cudaSuccess) return cuda_fail(e, "memset");
            if ((e = ah::launch_scan(dix, a, b, ix->num_sms, s)) != cudaSuccess) return cuda_fail(e, "scan");
        }
        launches += 1;
        mark(p == 0 ? 5 : 7);
    }
    if ((e = ah::launch_finish(dix, a, b, 0, ix->num_sms, s)) != cudaSuccess) return cuda_fail(e, "finish");
    launches += 2;                                           // the finish order and the finish
    mark(8);
    for (int round = 1; round <= 2; ++round) {
        if ((e = ah::launch_redo_scan(dix, a, b, round, ix->num_sms, s)) != cudaSuccess) return cuda_fail(e, "rescan");
        if ((e = ah::launch_finish(dix, a, b, round, ix->num_sms, s)) != cudaSuccess) return cuda_fail(e, "finish after rescan");
        launches += 2;
    }
    mark(9);
    if (prof) ix->ev_recorded = true;
    if (tr) {
        const size_t nL = (size_t)nq * L;
        if (tr->leaf_ids && (e = cudaMemcpyAsync(tr->leaf_ids, b.leaves, nL * 4, cudaMemcpyDeviceToDevice, s)) != cudaSuccess)
            return cuda_fail(e, "trace copy");
        if (tr->leaf_scores &&
            (e = cudaMemcpyAsync(tr->leaf_scores, b.leaf_scores, nL * 4, cudaMemcpyDeviceToDevice, s)) != cudaSuccess)
            return cuda_fail(e, "trace copy");
        if (tr->scanned &&
            (e = cudaMemcpyAsync(tr->scanned, b.scanned, (size_t)nq * 8, cudaMemcpyDeviceToDevice, s)) != cudaSuccess)
            return cuda_fail(e, "trace copy");
        if (tr->rescans &&
            (e = cudaMemcpyAsync(tr->rescans, b.counters + 1, 4, cudaMemcpyDeviceToDevice, s)) != cudaSuccess)
            return cuda_fail(e, "trace copy");
    }
    ix->last_launches = launches;
    ix->last_nq = nq;
    return AH_OK;
}

}  // namespace

extern "C" {

const char* ah_status_string(ah_status s) {
    switch (s) {
        case AH_OK: return "ok";
        case AH_ERR_INVALID_ARG: return "invalid argument";
        case AH_ERR_UNSUPPORTED: return "unsupported";
        case AH_ERR_OOM: return "out of device memory";
        case AH_ERR_CUDA: return "CUDA error";
        case AH_ERR_DEVICE: return "device-side error";
        case AH_ERR_TIMEOUT: return "timeout";
    }
    return "unknown status";
}

const char* ah_last_error(void) { return g_last_error.c_str(); }

ah_status ah_build_index_views(const ah_index_views* v, void* cuda_stream, ah_index** out) {
    if (!out) return fail(AH_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    if (!v) return fail(AH_ERR_INVALID_ARG, "views is NULL");
    if (v->n <= 0 || v->n >= (int64_t(1) << 31) - 64) return fail(AH_ERR_INVALID_ARG, "n outside (0, 2^31 - 64)");
    if (v->d <= 0 || v->dims_per_block <= 0 || v->num_leaves <= 0) return fail(AH_ERR_INVALID_ARG, "non-positive size");
    if (v->d % (2 * v->dims_per_block) != 0) return fail(AH_ERR_INVALID_ARG, "d not divisible by 2 * dims_per_block");
    if (v->d > AH_MAX_D) return fail(AH_ERR_UNSUPPORTED, "d above AH_MAX_D");
    if (v->d / v->dims_per_block > AH_MAX_BLOCKS) return fail(AH_ERR_UNSUPPORTED, "blocks above AH_MAX_BLOCKS");
    if (!v->centroids || !v->leaf_offsets || !v->slot_ids || !v->codes || !v->codebook)
        return fail(AH_ERR_INVALID_ARG, "NULL index array");
    if (v->reorder_dtype != AH_F32 && v->reorder_dtype != AH_BF16) return fail(AH_ERR_INVALID_ARG, "unknown reorder_dtype");
    cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
    ah_index* ix = new (std::nothrow) ah_index();
    if (!ix) return fail(AH_ERR_OOM, "host allocation");
    if (v->residual != 0 && v->residual != 1) {
        delete ix;
        return fail(AH_ERR_INVALID_ARG, "residual must be 0 or 1");
    }
    ix->views = *v;
    cudaError_t e = cudaGetDevice(&ix->device);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&ix->num_sms, cudaDevAttrMultiProcessorCount, ix->device);
    if (e != cudaSuccess) {
        delete ix;
        return cuda_fail(e, "device query");
    }
    if (ah_status st = lookup_noalloc_scratch(&ix->noalloc_scratch); st != AH_OK) {
        delete ix;
        return st;
    }
    const int B = v->d / v->dims_per_block;
    const int cb = B / 2;
    const int W = (cb + 3) / 4;
    const int NL = v->num_leaves;
    // leaf offsets: validated on the host, then int32 offsets and the first
    // code tile of each leaf in the leaf-padded code copy
    std::vector<int64_t> o64(NL + 1);
    if ((e = cudaMemcpy(o64.data(), v->leaf_offsets, sizeof(int64_t) * (NL + 1), cudaMemcpyDeviceToHost)) != cudaSuccess) {
        delete ix;
        return cuda_fail(e, "leaf offsets read");
    }
    std::vector<int32_t> o32(NL + 1), pt(NL + 1);
    if (o64[0] != 0 || o64[NL] != v->n) {
        delete ix;
        return fail(AH_ERR_INVALID_ARG, "leaf_offsets must start at 0 and end at n");
    }
    int64_t tiles = 0;
    for (int c = 0; c <= NL; ++c) {
        if (c < NL && o64[c + 1] < o64[c]) {
            delete ix;
            return fail(AH_ERR_INVALID_ARG, "leaf_offsets must be non-decreasing");
        }
        o32[c] = static_cast<int32_t>(o64[c]);
        pt[c] = static_cast<int32_t>(tiles);
        if (c < NL) tiles += (o64[c + 1] - o64[c] + 31) / 32;
    }
    if (tiles * 32 >= (int64_t(1) << 31)) {
        delete ix;
        return fail(AH_ERR_UNSUPPORTED, "padded code copy beyond 2^31 slots");
    }
    const size_t il_bytes = (size_t)std::max<int64_t>(tiles, 1) * W * 32 * sizeof(uint32_t);
    const size_t offs_bytes = sizeof(int32_t) * (size_t)(NL + 1);
    if ((e = cudaMalloc(&ix->codes_il, il_bytes)) != cudaSuccess ||
        (e = cudaMalloc(&ix->offs32, offs_bytes)) != cudaSuccess ||
        (e = cudaMalloc(&ix->ptile, offs_bytes)) != cudaSuccess ||
        (e = cudaMalloc(&ix->err, sizeof(int))) != cudaSuccess) {
        ah_destroy(ix);
        return cuda_fail(e, "index allocation");
    }
    ix->owned_bytes = il_bytes + 2 * offs_bytes + sizeof(int);
    // centroids split into tf32 halves for the tensor-core scores (when their
    // rows suit the tensor maps and there are enough of them)
    const bool tc = ah::centroid_tc_usable(1 << 20, NL, v->d);
    if (tc) {
        const size_t cs_bytes = 2 * sizeof(float) * (size_t)NL * v->d;
        if ((e = cudaMalloc(&ix->c_split, cs_bytes)) != cudaSuccess) {
            ah_destroy(ix);
            return cuda_fail(e, "index allocation");
        }
        ix->owned_bytes += cs_bytes;
        if ((e = ah::launch_split_tf32(v->centroids, (int64_t)NL * v->d, ix->c_split, ix->c_split + (size_t)NL * v->d,
                                       s)) != cudaSuccess) {
            ah_destroy(ix);
            return cuda_fail(e, "centroid split");
        }
    }
    if ((e = cudaMemcpy(ix->offs32, o32.data(), offs_bytes, cudaMemcpyHostToDevice)) != cudaSuccess ||
        (e = cudaMemcpy(ix->ptile, pt.data(), offs_bytes, cudaMemcpyHostToDevice)) != cudaSuccess ||
        (e = cudaMemsetAsync(ix->err, 0, sizeof(int), s)) != cudaSuccess ||
        (e = ah::launch_prepare_index(ix->offs32, ix->ptile, NL, v->codes, cb, W, tiles, ix->codes_il, s)) != cudaSuccess ||
        (e = cudaStreamSynchronize(s)) != cudaSuccess) {
        ah_destroy(ix);
        return cuda_fail(e, "index preparation");
    }
    ah::DeviceIndex& d = ix->dix;
    d.n = v->n;
    d.d = v->d;
    d.nl = v->num_leaves;
    d.dpb = v->dims_per_block;
    d.B = B;
    d.W = W;
    d.V = ah::code_vector_words(W);
    d.centroids = v->centroids;
    d.offs = ix->offs32;
    d.ptile = ix->ptile;
    d.slot_ids = v->slot_ids;
    d.codes_il = ix->codes_il;
    d.codebook = v->codebook;
    d.c_hi = ix->c_split;
    d.c_lo = ix->c_split ? ix->c_split + (size_t)NL * v->d : nullptr;
    d.reorder_vecs = v->reorder_vecs;
    d.reorder_bf16 = v->reorder_dtype == AH_BF16 ? 1 : 0;
    d.residual = v->residual;
    *out = ix;
    return AH_OK;
}

ah_status ah_reserve(ah_index* ix, int32_t max_nq, int32_t k, int32_t L, int32_t reorder_num, int32_t lut_mode) {
    ah_status st = validate_search(ix, reinterpret_cast<void*>(1), max_nq, k, L, reorder_num, lut_mode,
                                   reinterpret_cast<void*>(1), reinterpret_cast<void*>(1));
    if (st != AH_OK) return st;
    return carve(ix, std::max(max_nq, 1), L, std::max(reorder_num, k), lut_mode, k, false);
}

ah_status ah_search_traced(ah_index* ix, const float* queries, int32_t nq, int32_t k, int32_t L, int32_t reorder_num,
                           int32_t lut_mode, int32_t* out_ids, float* out_scores, const ah_search_trace* trace,
                           void* cuda_stream) {
    ah_status st = validate_search(ix, queries, nq, k, L, reorder_num, lut_mode, out_ids, out_scores);
    if (st != AH_OK || nq == 0) return st;
    return run_search(ix, queries, nq, k, L, reorder_num, lut_mode, out_ids, out_scores, trace,
                      static_cast<cudaStream_t>(cuda_stream));
}

ah_status ah_search(ah_index* ix, const float* queries, int32_t nq, int32_t k, int32_t L, int32_t reorder_num,
                    int32_t lut_mode, int32_t* out_ids, float* out_scores, void* cuda_stream) {
    return ah_search_traced(ix, queries, nq, k, L, reorder_num, lut_mode, out_ids, out_scores, nullptr, cuda_stream);
}

ah_status ah_search_host(ah_index* ix, const float* host_queries, int32_t nq, int32_t k, int32_t L,
                         int32_t reorder_num, int32_t lut_mode, int32_t* host_ids, float* host_scores,
                         void* cuda_stream) {
    ah_status st = validate_search(ix, host_queries, nq, k, L, reorder_num, lut_mode, host_ids, host_scores);
    if (st != AH_OK || nq == 0) return st;
    const int R = std::max(reorder_num, k);
    st = carve(ix, nq, L, R, lut_mode, k, true);
    if (st != AH_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
    Workspace& w = ix->ws;
    cudaError_t e = cudaMemcpyAsync(w.dq, host_queries, sizeof(float) * (size_t)nq * ix->dix.d, cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return cuda_fail(e, "query upload");
    st = run_search(ix, w.dq, nq, k, L, reorder_num, lut_mode, w.dids, w.dscores, nullptr, s);
    if (st != AH_OK) return st;
    if ((e = cudaMemcpyAsync(host_ids, w.dids, sizeof(int32_t) * (size_t)nq * k, cudaMemcpyDeviceToHost, s)) != cudaSuccess ||
        (e = cudaMemcpyAsync(host_scores, w.dscores, sizeof(float) * (size_t)nq * k, cudaMemcpyDeviceToHost, s)) !=
            cudaSuccess)
        return cuda_fail(e, "result download");
    return ah_sync_status(ix, cuda_stream);
}

ah_status ah_sync_status(ah_index* ix, void* cuda_stream) {
    if (!ix) return fail(AH_ERR_INVALID_ARG, "index is NULL");
    cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
    cudaError_t e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
    int code = 0;
    if ((e = cudaMemcpy(&code, ix->err, sizeof(int), cudaMemcpyDeviceToHost)) != cudaSuccess)
        return cuda_fail(e, "error word read");
    if (code == 0) return AH_OK;
    int zero = 0;
    cudaMemcpy(ix->err, &zero, sizeof(int), cudaMemcpyHostToDevice);
    switch (code) {
        case ah::kDevCandOverflow: return fail(AH_ERR_DEVICE, "candidate buffer overflow after the last rescan round");
        case ah::kDevBadLeaf: return fail(AH_ERR_DEVICE, "leaf id out of range");
        case ah::kDevSelectSize: return fail(AH_ERR_DEVICE, "selection size mismatch (duplicate keys)");
        case ah::kDevTimeout: return fail(AH_ERR_TIMEOUT, "a bounded wait in the tensor-core centroid scores gave up");
        default: return fail(AH_ERR_DEVICE, "device error " + std::to_string(code));
    }
}

ah_status ah_set_option(ah_index* ix, int32_t option, int64_t value) {
    if (!ix) return fail(AH_ERR_INVALID_ARG, "index is NULL");
    switch (option) {
        case AH_OPT_THRESHOLD_SAMPLE:
            if (value < 1 || value > 4096) return fail(AH_ERR_INVALID_ARG, "threshold sample outside [1, 4096]");
            ix->opt_threshold_sample = static_cast<int>(value);
            return AH_OK;
        case AH_OPT_THRESHOLD_LEAVES:
            if (value < 1 || value > 4096) return fail(AH_ERR_INVALID_ARG, "threshold leaves outside [1, 4096]");
            ix->opt_threshold_leaves = static_cast<int>(value);
            return AH_OK;
        case AH_OPT_PROGRESSIVE_LEAVES:
            if (value < -1 || value > AH_MAX_LEAVES_SEARCHED) return fail(AH_ERR_INVALID_ARG, "progressive leaves outside [-1, 4096]");
            ix->opt_progressive_leaves = static_cast<int>(value);
            return AH_OK;
        case AH_OPT_UINT8_TENSOR_CORES:
            if (value < 0 || value > 1) return fail(AH_ERR_INVALID_ARG, "uint8 tensor-core scan option outside [0, 1]");
            ix->opt_u8_tensor = static_cast<int>(value);
            return AH_OK;
        case AH_OPT_SCAN_CHUNK_TILES:
            if (value < 0 || value > 1024) return fail(AH_ERR_INVALID_ARG, "scan chunk outside [0, 1024] tiles");
            ix->opt_chunk_tiles = static_cast<int>(value);
            return AH_OK;
        case AH_OPT_QUERY_MAJOR_SCAN:
            if (value < -1 || value > 1) return fail(AH_ERR_INVALID_ARG, "query-major scan option outside [-1, 1]");
            ix->opt_query_scan = static_cast<int>(value);
            return AH_OK;
        default:
            return fail(AH_ERR_INVALID_ARG, "unknown option");
    }
}

ah_status ah_set_profiling(ah_index* ix, int32_t on) {
    if (!ix) return fail(AH_ERR_INVALID_ARG, "index is NULL");
    if (on && !ix->ev_ready) {
        for (int i = 0; i < ah_index::kMaxMarks; ++i) {
            cudaError_t e = cudaEventCreate(&ix->ev[i]);
            if (e != cudaSuccess) return cuda_fail(e, "event create");
        }
        ix->ev_ready = true;
    }
    if (on < 0 || on > 2) return fail(AH_ERR_INVALID_ARG, "profiling level must be 0, 1 or 2");
    ix->profiling = on;
    ix->ev_recorded = false;
    return AH_OK;
}

ah_status ah_stage_times(ah_index* ix, float* ms, int32_t max_stages, int32_t* n_stages) {
    if (!ix || !ms || !n_stages) return fail(AH_ERR_INVALID_ARG, "NULL argument");
    if (!ix->ev_recorded || ix->n_marks < 2) return fail(AH_ERR_INVALID_ARG, "no profiled search recorded");
    cudaError_t e = cudaEventSynchronize(ix->ev[ix->n_marks - 1]);
    if (e != cudaSuccess) return cuda_fail(e, "event synchronize");
    int n = std::min<int>(kStages, max_stages);
    for (int i = 0; i < n; ++i) ms[i] = 0.0f;
    for (int m = 1; m < ix->n_marks; ++m) {
        const int st = ix->mark_stage[m];
        if (st < 0 || st >= n) continue;
        float t = 0.0f;
        e = cudaEventElapsedTime(&t, ix->ev[m - 1], ix->ev[m]);
        if (e != cudaSuccess) return cuda_fail(e, "event elapsed");
        ms[st] += t;
    }
    *n_stages = n;
    return AH_OK;
}

const char* ah_stage_name(int32_t stage) {
    if (stage < 0 || stage >= kStages) return "";
    return kStageNames[stage];
}

ah_status ah_last_search_info(ah_index* ix, int32_t* launches, int64_t* points_scanned) {
    if (!ix) return fail(AH_ERR_INVALID_ARG, "index is NULL");
    if (launches) *launches = ix->last_launches;
    if (points_scanned) {
        *points_scanned = 0;
        if (ix->last_nq > 0) {
            cudaError_t e = cudaDeviceSynchronize();
            if (e != cudaSuccess) return cuda_fail(e, "synchronize");
            std::vector<int64_t> h(ix->last_nq);
            e = cudaMemcpy(h.data(), ix->ws.buf.scanned, sizeof(int64_t) * h.size(), cudaMemcpyDeviceToHost);
            if (e != cudaSuccess) return cuda_fail(e, "scanned read");
            for (int64_t v : h) *points_scanned += v;
        }
    }
    return AH_OK;
}

ah_status ah_index_memory(ah_index* ix, int64_t* bytes) {
    if (!ix || !bytes) return fail(AH_ERR_INVALID_ARG, "NULL argument");
    *bytes = static_cast<int64_t>(ix->owned_bytes);
    return AH_OK;
}

void ah_destroy(ah_index* ix) {
    if (!ix) return;
    cudaDeviceSynchronize();
    if (ix->ws.base) cudaFree(ix->ws.base);
    if (ix->codes_il) cudaFree(ix->codes_il);
    if (ix->c_split) cudaFree(ix->c_split);
    if (ix->offs32) cudaFree(ix->offs32);
    if (ix->ptile) cudaFree(ix->ptile);
    if (ix->err) cudaFree(ix->err);
    for (void* p : ix->loaded)
        if (p) cudaFree(p);
    for (cudaEvent_t ev : {ix->ev_fork, ix->ev_tl, ix->ev_lut, ix->ev_inv})
        if (ev) cudaEventDestroy(ev);
    if (ix->side) cudaStreamDestroy(ix->side);
    if (ix->ev_ready)
        for (int i = 0; i < ah_index::kMaxMarks; ++i) cudaEventDestroy(ix->ev[i]);
    delete ix;
}

ah_status ah_search_leaves_noalloc(ah_index* ix, const float* queries, int32_t nq, int32_t L,
                                   int32_t* out_leaf_ids, float* out_leaf_scores, void* cuda_stream) {
    if (!ix) return fail(AH_ERR_INVALID_ARG, "index is NULL");
    if (nq < 0) return fail(AH_ERR_INVALID_ARG, "nq < 0");
    if (L < 1 || L > ix->dix.nl) return fail(AH_ERR_INVALID_ARG, "num_leaves_to_search outside [1, num_leaves]");
    if (L > AH_MAX_LEAVES_SEARCHED) return fail(AH_ERR_UNSUPPORTED, "num_leaves_to_search above AH_MAX_LEAVES_SEARCHED");
    if (nq == 0) return AH_OK;
    if (!queries || !out_leaf_ids || !out_leaf_scores) return fail(AH_ERR_INVALID_ARG, "NULL queries or outputs");
    const int NL = ix->dix.nl;
    const size_t score_bytes = align_up(sizeof(float) * (size_t)nq * NL, 256);
    const size_t count_bytes = align_up(sizeof(int32_t) * (size_t)NL, 256);
    const size_t scanned_bytes = align_up(sizeof(int64_t) * (size_t)nq, 256);
    if (score_bytes + count_bytes + scanned_bytes > AH_NOALLOC_SCRATCH_BYTES)
        return fail(AH_ERR_UNSUPPORTED, "nq * num_leaves scores exceed the library's fixed scratch "
                                        "(AH_NOALLOC_SCRATCH_BYTES); split the batch");
    if (ah_status st = check_current_device(ix); st != AH_OK) return st;
    cudaError_t e;
    cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
    char* p = static_cast<char*>(ix->noalloc_scratch);
    ah::SearchBuffers b{};
    b.cscore = reinterpret_cast<float*>(p);
    b.qcount = reinterpret_cast<int32_t*>(p + score_bytes);
    b.scanned = reinterpret_cast<int64_t*>(p + score_bytes + count_bytes);
    b.leaves = out_leaf_ids;
    b.leaf_scores = out_leaf_scores;
    b.err = ix->err;
    ah::SearchArgs a{};
    a.queries = queries;
    a.nq = nq;
    a.L = L;
    a.k = 1;
    a.R = 1;
    // the per-leaf counters are accumulated by the top-L kernel: start them at zero
    if ((e = cudaMemsetAsync(b.qcount, 0, sizeof(int32_t) * (size_t)NL, s)) != cudaSuccess) return cuda_fail(e, "memset");
    if ((e = ah::launch_centroid_scores(ix->dix, a, b, s)) != cudaSuccess) return cuda_fail(e, "centroid scores");
    if ((e = ah::launch_top_leaves(ix->dix, a, b, s)) != cudaSuccess) return cuda_fail(e, "top leaves");
    return AH_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// index directories
// ---------------------------------------------------------------------------

namespace {

const char* const kIndexFiles[6] = {"centroids.npy", "leaf_offsets.npy", "slot_ids.npy",
                                    "codes.npy",     "codebook.npy",     "reorder_vecs.npy"};
const char* const kMetaFile = "ah_index.txt";
constexpr size_t kStageBytes = size_t(64) << 20;      // host staging for the copies

std::string path_in(const char* dir, const char* file) {
    std::string s(dir);
    if (!s.empty() && s.back() != '/') s += '/';
    return s + file;
}

// array i of the views: device pointer, dtype text, shape
struct ArraySpec {
    const void* ptr;
    std::string descr;
    std::vector<int64_t> shape;
};

std::vector<ArraySpec> array_specs(const ah_index_views& v) {
    const int64_t B = v.d / v.dims_per_block;
    std::vector<ArraySpec> a(6);
    a[0] = {v.centroids, "<f4", {v.num_leaves, v.d}};
    a[1] = {v.leaf_offsets, "<i8", {int64_t(v.num_leaves) + 1}};
    a[2] = {v.slot_ids, "<i4", {v.n}};
    a[3] = {v.codes, "|u1", {v.n, B / 2}};
    a[4] = {v.codebook, "<f4", {B, 16, v.dims_per_block}};
    a[5] = {v.reorder_vecs, v.reorder_dtype == AH_BF16 ? "<u2" : "<f4", {v.n, v.d}};
    return a;
}

ah_status write_array(const std::string& path, const ArraySpec& a, std::vector<char>& stage) {
    FILE* f = std::fopen(path.c_str(), "wb");
    if (!f) return fail(AH_ERR_INVALID_ARG, ("cannot write " + path).c_str());
    const std::string h = ah::npy::make_header(a.descr, a.shape);
    bool ok = std::fwrite(h.data(), 1, h.size(), f) == h.size();
    const int64_t bytes = ah::npy::count(a.shape) * ah::npy::item_size(a.descr);
    for (int64_t off = 0; ok && off < bytes; off += static_cast<int64_t>(stage.size())) {
        const size_t len = static_cast<size_t>(std::min<int64_t>(bytes - off, static_cast<int64_t>(stage.size())));
        cudaError_t e = cudaMemcpy(stage.data(), static_cast<const char*>(a.ptr) + off, len, cudaMemcpyDeviceToHost);
        if (e != cudaSuccess) {
            std::fclose(f);
            return cuda_fail(e, "index array read");
        }
        ok = std::fwrite(stage.data(), 1, len, f) == len;
    }
    ok = (std::fclose(f) == 0) && ok;
    return ok ? AH_OK : fail(AH_ERR_INVALID_ARG, ("short write to " + path).c_str());
}

}  // namespace

ah_status ah_save(ah_index* ix, const char* dir) {
    if (!ix || !dir) return fail(AH_ERR_INVALID_ARG, "NULL argument");
    const ah_index_views& v = ix->views;
    std::vector<ArraySpec> a = array_specs(v);
    std::vector<char> stage(kStageBytes);
    for (int i = 0; i < 6; ++i) {
        if (i == 5 && !v.reorder_vecs) continue;
        const ah_status st = write_array(path_in(dir, kIndexFiles[i]), a[i], stage);
        if (st != AH_OK) return st;
    }
    if (!v.reorder_vecs) std::remove(path_in(dir, kIndexFiles[5]).c_str());
    const std::string meta = path_in(dir, kMetaFile);
    FILE* f = std::fopen(meta.c_str(), "w");
    if (!f) return fail(AH_ERR_INVALID_ARG, ("cannot write " + meta).c_str());
    const char* dt = !v.reorder_vecs ? "none" : (v.reorder_dtype == AH_BF16 ? "bf16" : "f32");
    const bool ok = std::fprintf(f, "ah-index 1\nreorder_dtype %s\nresidual %d\n", dt, v.residual ? 1 : 0) > 0;
    if (std::fclose(f) != 0 || !ok) return fail(AH_ERR_INVALID_ARG, ("short write to " + meta).c_str());
    return AH_OK;
}

namespace {

ah_status inspect_dir(const char* dir, ah_index_views* out, ah::npy::Header hdr[6], bool* has_reorder) {
    // meta: version and the reorder copy's type
    const std::string meta = path_in(dir, kMetaFile);
    FILE* f = std::fopen(meta.c_str(), "r");
    if (!f) return fail(AH_ERR_INVALID_ARG, ("cannot open " + meta).c_str());
    char l1[64] = {0}, key[64] = {0}, val[64] = {0}, key2[64] = {0};
    int resid = 0;
    const bool ok = std::fgets(l1, sizeof(l1), f) && std::fscanf(f, "%63s %63s", key, val) == 2;
    const int got2 = ok ? std::fscanf(f, "%63s %d", key2, &resid) : 0;
    std::fclose(f);
    if (got2 == 2 && (std::strcmp(key2, "residual") != 0 || (resid != 0 && resid != 1)))
        return fail(AH_ERR_INVALID_ARG, (meta + ": third line must be \"residual 0\" or \"residual 1\"").c_str());
    if (got2 != 2) resid = 0;
    if (!ok || std::strncmp(l1, "ah-index 1", 10) != 0 || std::strcmp(key, "reorder_dtype") != 0)
        return fail(AH_ERR_INVALID_ARG, (meta + ": expected \"ah-index 1\" then \"reorder_dtype <f32|bf16|none>\"").c_str());
    int rdt;
    if (!std::strcmp(val, "f32")) rdt = AH_F32;
    else if (!std::strcmp(val, "bf16")) rdt = AH_BF16;
    else if (!std::strcmp(val, "none")) rdt = -1;
    else return fail(AH_ERR_INVALID_ARG, (meta + ": unknown reorder_dtype").c_str());
    *has_reorder = rdt >= 0;
    for (int i = 0; i < 6; ++i) {
        if (i == 5 && !*has_reorder) continue;
        const std::string p = path_in(dir, kIndexFiles[i]);
        const std::string why = ah::npy::read_header(p.c_str(), &hdr[i]);
        if (!why.empty()) return fail(AH_ERR_INVALID_ARG, (p + ": " + why).c_str());
    }
    auto bad = [&](int i, const char* what) { return fail(AH_ERR_INVALID_ARG, (path_in(dir, kIndexFiles[i]) + ": " + what).c_str()); };
    const auto& c = hdr[0].shape;
    if (hdr[0].descr != "<f4" || c.size() != 2) return bad(0, "need <f4 [num_leaves, d]");
    const int64_t NL = c[0], d = c[1];
    if (hdr[1].descr != "<i8" || hdr[1].shape != std::vector<int64_t>{NL + 1}) return bad(1, "need <i8 [num_leaves + 1]");
    if (hdr[2].descr != "<i4" || hdr[2].shape.size() != 1) return bad(2, "need <i4 [n]");
    const int64_t n = hdr[2].shape[0];
    const auto& cb = hdr[4].shape;
    if (hdr[4].descr != "<f4" || cb.size() != 3 || cb[1] != 16 || cb[0] <= 0 || cb[2] <= 0 || cb[0] * cb[2] != d || cb[0] % 2)
        return bad(4, "need <f4 [B, 16, dims_per_block] with B even and B * dims_per_block = d");
    const int64_t B = cb[0];
    if ((hdr[3].descr != "|u1" && hdr[3].descr != "<u1") || hdr[3].shape != std::vector<int64_t>{n, B / 2})
        return bad(3, "need |u1 [n, B / 2]");
    if (*has_reorder) {
        const char* want = rdt == AH_BF16 ? "<u2" : "<f4";
        if (hdr[5].descr != want || hdr[5].shape != std::vector<int64_t>{n, d})
            return bad(5, rdt == AH_BF16 ? "need <u2 [n, d] (bfloat16 bits)" : "need <f4 [n, d]");
    }
    if (NL <= 0 || NL > INT32_MAX || d <= 0 || d > INT32_MAX || n <= 0) return bad(0, "sizes out of range");
    *out = ah_index_views{};
    out->n = n;
    out->d = static_cast<int32_t>(d);
    out->num_leaves = static_cast<int32_t>(NL);
    out->dims_per_block = static_cast<int32_t>(cb[2]);
    out->reorder_dtype = rdt;
    out->residual = resid;
    return AH_OK;
}

}  // namespace

ah_status ah_inspect(const char* dir, ah_index_views* out) {
    if (!dir || !out) return fail(AH_ERR_INVALID_ARG, "NULL argument");
    ah::npy::Header hdr[6];
    bool has_reorder = false;
    return inspect_dir(dir, out, hdr, &has_reorder);
}

ah_status ah_load(const char* dir, void* cuda_stream, ah_index** out) {
    if (!out) return fail(AH_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    if (!dir) return fail(AH_ERR_INVALID_ARG, "dir is NULL");
    ah_index_views v;
    ah::npy::Header hdr[6];
    bool has_reorder = false;
    ah_status st = inspect_dir(dir, &v, hdr, &has_reorder);
    if (st != AH_OK) return st;
    void* dev[6] = {};
    size_t total = 0;
    auto release = [&]() {
        for (void*& p : dev)
            if (p) cudaFree(p);
    };
    std::vector<char> stage(kStageBytes);
    for (int i = 0; i < 6; ++i) {
        if (i == 5 && !has_reorder) continue;
        const int64_t bytes = ah::npy::count(hdr[i].shape) * ah::npy::item_size(hdr[i].descr);
        cudaError_t e = cudaMalloc(&dev[i], static_cast<size_t>(std::max<int64_t>(bytes, 1)));
        if (e != cudaSuccess) {
            release();
            return cuda_fail(e, "index arrays");      // AH_ERR_OOM for an allocation failure
        }
        total += static_cast<size_t>(bytes);
        const std::string p = path_in(dir, kIndexFiles[i]);
        FILE* f = std::fopen(p.c_str(), "rb");
        bool ok = f && std::fseek(f, static_cast<long>(hdr[i].data_offset), SEEK_SET) == 0;
        for (int64_t off = 0; ok && off < bytes; off += static_cast<int64_t>(stage.size())) {
            const size_t len = static_cast<size_t>(std::min<int64_t>(bytes - off, static_cast<int64_t>(stage.size())));
            ok = std::fread(stage.data(), 1, len, f) == len;
            if (ok && (e = cudaMemcpy(static_cast<char*>(dev[i]) + off, stage.data(), len, cudaMemcpyHostToDevice)) != cudaSuccess) {
                std::fclose(f);
                release();
                return cuda_fail(e, "index array copy");
            }
        }
        if (f) std::fclose(f);
        if (!ok) {
            release();
            return fail(AH_ERR_INVALID_ARG, ("cannot read " + p).c_str());
        }
    }
    v.centroids = static_cast<const float*>(dev[0]);
    v.leaf_offsets = static_cast<const int64_t*>(dev[1]);
    v.slot_ids = static_cast<const int32_t*>(dev[2]);
    v.codes = static_cast<const uint8_t*>(dev[3]);
    v.codebook = static_cast<const float*>(dev[4]);
    v.reorder_vecs = dev[5];
    if (!has_reorder) v.reorder_dtype = AH_F32;
    ah_index* ix = nullptr;
    st = ah_build_index_views(&v, cuda_stream, &ix);
    if (st != AH_OK) {
        release();
        return st;
    }
    for (int i = 0; i < 6; ++i) ix->loaded[i] = dev[i];
    ix->owned_bytes += total;
    *out = ix;
    return AH_OK;
}

// ---------------------------------------------------------------------------
// anisotropic code assignment
// ---------------------------------------------------------------------------

ah_status ah_encode(const float* X, int64_t n, int32_t d, int32_t dims_per_block, const float* codebook, double T,
                    int32_t passes, uint8_t* codes, int32_t* passes_used, void* cuda_stream) {
    if (n < 0) return fail(AH_ERR_INVALID_ARG, "n < 0");
    if (n == 0) return AH_OK;
    if (!X || !codebook || !codes) return fail(AH_ERR_INVALID_ARG, "NULL array");
    if (d <= 0 || dims_per_block <= 0 || d % (2 * dims_per_block) != 0)
        return fail(AH_ERR_INVALID_ARG, "d not a positive multiple of 2 * dims_per_block");
    if (d / dims_per_block > AH_MAX_BLOCKS) return fail(AH_ERR_UNSUPPORTED, "blocks above AH_MAX_BLOCKS");
    if (passes < 0 || passes > 1000) return fail(AH_ERR_INVALID_ARG, "passes outside [0, 1000]");
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess)
        e = ah::launch_encode(X, n, d, dims_per_block, codebook, T, passes, codes, passes_used, sms,
                              static_cast<cudaStream_t>(cuda_stream));
    return e == cudaSuccess ? AH_OK : cuda_fail(e, "encode");
}

// ---------------------------------------------------------------------------
// partition training
// ---------------------------------------------------------------------------

ah_status ah_kmeans_assign(const float* X, int64_t n, int32_t d, const float* C, int32_t nl, int32_t* assign,
                           double* dist, void* cuda_stream) {
    if (n < 0 || d < 1 || nl < 1) return fail(AH_ERR_INVALID_ARG, "n < 0, d < 1 or nl < 1");
    if (n == 0) return AH_OK;
    if (!X || !C || !assign) return fail(AH_ERR_INVALID_ARG, "NULL array");
    if (d > AH_MAX_D) return fail(AH_ERR_UNSUPPORTED, "d above AH_MAX_D");
    const cudaError_t e = ah::launch_kmeans_assign(X, n, d, C, nl, assign, dist, static_cast<cudaStream_t>(cuda_stream));
    return e == cudaSuccess ? AH_OK : cuda_fail(e, "k-means assignment");
}

ah_status ah_avq_update(const float* X, int64_t n, int32_t d, const int32_t* assign, int32_t nl, const float* C_old,
                        double T, int32_t max_iters, double tol, float* C_new, int64_t* counts, int32_t* iters,
                        void* cuda_stream) {
    if (n < 0 || d < 1 || nl < 1) return fail(AH_ERR_INVALID_ARG, "n < 0, d < 1 or nl < 1");
    if ((n > 0 && (!X || !assign)) || !C_old || !C_new) return fail(AH_ERR_INVALID_ARG, "NULL array");
    if (max_iters < 0 || max_iters > 100000) return fail(AH_ERR_INVALID_ARG, "max_iters outside [0, 100000]");
    if (!(tol >= 0.0 && tol < 1.0)) return fail(AH_ERR_INVALID_ARG, "tol outside [0, 1)");
    if (ah::avq_solve_smem_bytes(d) > 200 * 1024) return fail(AH_ERR_UNSUPPORTED, "d above 6400 for the update");
    if (n >= (int64_t(1) << 31)) return fail(AH_ERR_UNSUPPORTED, "n of 2^31 or more");
    cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
    void* ws = nullptr;
    cudaError_t e = cudaMallocAsync(&ws, ah::avq_workspace_bytes(n, nl), s);
    if (e != cudaSuccess) return cuda_fail(e, "center update workspace");
    e = ah::launch_avq_update(X, n, d, assign, nl, C_old, T, C_new, counts, iters, max_iters, tol, ws, s);
    const cudaError_t ef = cudaFreeAsync(ws, s);
    if (e != cudaSuccess) return cuda_fail(e, "anisotropic center update");
    return ef == cudaSuccess ? AH_OK : cuda_fail(ef, "center update workspace release");
}

ah_status ah_kmeans_update(const float* X, int64_t n, int32_t d, const int32_t* assign, int32_t nl, const float* C_old,
                           float* C_new, int64_t* counts, void* cuda_stream) {
    if (n < 0 || d < 1 || nl < 1) return fail(AH_ERR_INVALID_ARG, "n < 0, d < 1 or nl < 1");
    if ((n > 0 && (!X || !assign)) || !C_old || !C_new) return fail(AH_ERR_INVALID_ARG, "NULL array");
    if (ah::kmeans_update_smem_bytes(d) > 200 * 1024) return fail(AH_ERR_UNSUPPORTED, "d above 6400 for the update");
    const cudaError_t e = ah::launch_kmeans_update(X, n, d, assign, nl, C_old, C_new, counts,
                                                   static_cast<cudaStream_t>(cuda_stream));
    return e == cudaSuccess ? AH_OK : cuda_fail(e, "k-means update");
}

// ---------------------------------------------------------------------------
// leaf-partitioned search: exact merge of the shards' candidates
// ---------------------------------------------------------------------------

ah_status ah_merge_shards(int32_t G, int32_t nq, int32_t R, int32_t k, const int32_t* cand_ids,
                          const float* cand_approx, const float* cand_exact, int32_t* out_ids, float* out_scores,
                          void* cuda_stream) {
    if (G < 1 || nq < 0 || k < 1 || R < k) return fail(AH_ERR_INVALID_ARG, "need G >= 1, nq >= 0, 1 <= k <= R");
    if (R > AH_MAX_R) return fail(AH_ERR_UNSUPPORTED, "R above AH_MAX_R");
    if (static_cast<int64_t>(G) * R > 65536) return fail(AH_ERR_UNSUPPORTED, "G * R above 65536");
    if (nq == 0) return AH_OK;
    if (!cand_ids || !cand_approx || !out_ids || !out_scores) return fail(AH_ERR_INVALID_ARG, "NULL array");
    const cudaError_t e = ah::launch_merge_shards(G, nq, R, k, cand_ids, cand_approx, cand_exact, out_ids, out_scores,
                                                  static_cast<cudaStream_t>(cuda_stream));
    return e == cudaSuccess ? AH_OK : cuda_fail(e, "shard merge");
}
