// Exact merge for the leaf-partitioned search.  Shards hold the same
// centroids and codebook and disjoint leaves' points, so each scans its own
// points of the same L leaves; the union of their best R by approximate score
// contains the best R of all points.  Per query: the best R of the G * R
// entries by (approximate score desc, id asc), then the best k of those by
// (exact score desc, id asc), the order one index over all points uses.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "common.cuh"
#include "kernels.h"
#include "select.cuh"

namespace ah {

namespace {

constexpr int kMergeThreads = 256;

// One CTA per query.  Shared memory: the best R keys and their entry
// indices, then the best k keys.
__global__ void __launch_bounds__(kMergeThreads) merge_shards_kernel(int G, int nq, int R, int k,
                                                                   const int32_t* __restrict__ ids,
                                                                   const float* __restrict__ approx,
                                                                   const float* __restrict__ exact,
                                                                   int32_t* __restrict__ out_ids,
                                                                   float* __restrict__ out_scores, int* err) {
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ SelectScratch scr;
    const int q = blockIdx.x;
    const int PR = next_pow2(R), PK = next_pow2(k);
    uint64_t* rkeys = reinterpret_cast<uint64_t*>(smem);         // [PR]
    int32_t* ridx = reinterpret_cast<int32_t*>(rkeys + PR);        // [PR]
    uint64_t* fkeys = reinterpret_cast<uint64_t*>(smem) + PR + (PR + 1) / 2;   // [PK], after ridx
    const int n = G * R;
    // entry e = (shard g, rank r) of this query
    auto at = [&](int e) { return (static_cast<int64_t>(e / R) * nq + q) * R + e % R; };
    auto key1 = [&](int e) {
        const int64_t o = at(e);
        const int32_t id = ids[o];
        return id >= 0 ? make_key(float_key(approx[o]), id) : 0ull;    // padding ranks last
    };
    auto pay1 = [&](int e) { return e; };
    // count the real entries first: selecting min(R, real) keeps the cut
    // above the padding keys (0), so no padding can take a real entry's place
    if (threadIdx.x == 0) scr.count = 0;
    __syncthreads();
    int local = 0;
    for (int e = threadIdx.x; e < n; e += kMergeThreads) local += (ids[at(e)] >= 0) ? 1 : 0;
    atomicAdd(&scr.count, local);
    __syncthreads();
    const int nv = scr.count;
    __syncthreads();
    const int K1 = block_topk<kMergeThreads>(key1, pay1, n, min(R, nv), scr, rkeys, ridx, err, exact == nullptr);
    const int64_t oo = static_cast<int64_t>(q) * k;
    if (exact == nullptr) {
        // best R sorted by approximate key: its first k are the result
        for (int i = threadIdx.x; i < k; i += kMergeThreads) {
            const bool have = i < K1;
            out_ids[oo + i] = have ? key_id(rkeys[i]) : -1;
            out_scores[oo + i] = have ? key_float(key_score(rkeys[i])) : -INFINITY;
        }
        return;
    }
    // best k of the kept (all real) by exact score
    auto key2 = [&](int i) {
        const int64_t o = at(ridx[i]);
        return make_key(float_key(exact[o]), ids[o]);
    };
    auto pay2 = [&](int i) { return i; };
    const int K2 = block_topk<kMergeThreads>(key2, pay2, K1, k, scr, fkeys, static_cast<int32_t*>(nullptr), err, true);
    for (int i = threadIdx.x; i < k; i += kMergeThreads) {
        const bool have = i < K2;
        out_ids[oo + i] = have ? key_id(fkeys[i]) : -1;
        out_scores[oo + i] = have ? key_float(key_score(fkeys[i])) : -INFINITY;
    }
}

}  // namespace

cudaError_t launch_merge_shards(int G, int nq, int R, int k, const int32_t* ids, const float* approx,
                                const float* exact, int32_t* out_ids, float* out_scores, cudaStream_t s) {
    if (nq <= 0) return cudaSuccess;
    const size_t PR = static_cast<size_t>(next_pow2(R)), PK = static_cast<size_t>(next_pow2(k));
    const size_t smem = PR * sizeof(uint64_t) + ((PR + 1) / 2) * sizeof(uint64_t) + PK * sizeof(uint64_t);
    cudaError_t e = cudaFuncSetAttribute(merge_shards_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    merge_shards_kernel<<<nq, kMergeThreads, smem, s>>>(G, nq, R, k, ids, approx, exact, out_ids, out_scores, nullptr);
    return cudaGetLastError();
}

}  // namespace ah
