// Partition training (index build): nearest-centroid assignment and the
// centroid means of k-means (ScaNN blog, "Using the library": the tree's
// leaves are trained by k-means on a sample, every point goes to its nearest
// leaf).
//
// Both kernels fix their arithmetic order so that results do not depend on
// the launch: squared distances in fp64 over coordinates in ascending order
// (each difference, square and sum rounded separately; ties to the lower
// centroid), and each centroid's sum over its members in ascending point order.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "kernels.h"

namespace ah {

namespace {

constexpr int kAP = 64;     // points per assignment CTA
constexpr int kAC = 64;     // centroids per chunk
constexpr int kAK = 16;     // coordinates per step

// (d, c) is below (bd, bc) in (distance, centroid) order
__device__ __forceinline__ bool better(double d, int c, double bd, int bc) { return d < bd || (d == bd && c < bc); }

// CTA of 256 threads: 64 points x all centroids in chunks of 64; thread
// (tp, tc) accumulates points 4 tp .. 4 tp + 3 against centroids
// 4 tc .. 4 tc + 3 of the chunk.
__global__ void __launch_bounds__(256) kmeans_assign_kernel(const float* __restrict__ X, int64_t n, int d,
                                                            const float* __restrict__ C, int nl,
                                                            int32_t* __restrict__ assign, double* __restrict__ dist) {
    __shared__ float xs[kAK][kAP + 1];
    __shared__ float cs[kAK][kAC + 1];
    const int tid = threadIdx.x, tp = tid >> 4, tc = tid & 15;
    const int64_t p0 = static_cast<int64_t>(blockIdx.x) * kAP;
    double best_d[4];
    int best_c[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        best_d[i] = 0.0;
        best_c[i] = -1;
    }
    for (int c0 = 0; c0 < nl; c0 += kAC) {
        double acc[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = 0.0;
        for (int k0 = 0; k0 < d; k0 += kAK) {
            // stage 16 coordinates of the 64 points and of the 64 centroids
            for (int e = tid; e < kAK * kAP; e += 256) {
                const int r = e / kAK, k = e % kAK;
                const int64_t p = p0 + r;
                xs[k][r] = (p < n && k0 + k < d) ? X[p * d + k0 + k] : 0.0f;
                const int c = c0 + r;
                cs[k][r] = (c < nl && k0 + k < d) ? C[static_cast<int64_t>(c) * d + k0 + k] : 0.0f;
            }
            __syncthreads();
            const int kn = min(kAK, d - k0);
            for (int k = 0; k < kn; ++k) {
                double xv[4], cv[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) xv[i] = static_cast<double>(xs[k][4 * tp + i]);
#pragma unroll
                for (int j = 0; j < 4; ++j) cv[j] = static_cast<double>(cs[k][4 * tc + j]);
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const double df = __dadd_rn(xv[i], -cv[j]);
                        acc[i][j] = __dadd_rn(acc[i][j], __dmul_rn(df, df));
                    }
            }
            __syncthreads();
        }
        // best of this chunk per point, over the 16 threads sharing the point
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            double bd = 0.0;
            int bc = -1;                          // -1: no real centroid yet
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int c = c0 + 4 * tc + j;
                if (c < nl && (bc < 0 || better(acc[i][j], c, bd, bc))) {
                    bd = acc[i][j];
                    bc = c;
                }
            }
#pragma unroll
            for (int off = 8; off > 0; off >>= 1) {
                const double od = __shfl_xor_sync(0xFFFFFFFFu, bd, off, 16);
                const int oc = __shfl_xor_sync(0xFFFFFFFFu, bc, off, 16);
                if (oc >= 0 && (bc < 0 || better(od, oc, bd, bc))) {
                    bd = od;
                    bc = oc;
                }
            }
            if (bc >= 0 && (best_c[i] < 0 || better(bd, bc, best_d[i], best_c[i]))) {
                best_d[i] = bd;
                best_c[i] = bc;
            }
        }
    }
    if (tc == 0) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int64_t p = p0 + 4 * tp + i;
            if (p < n) {
                assign[p] = best_c[i];
                if (dist) dist[p] = best_d[i];
            }
        }
    }
}

constexpr int kUC = 4;        // centroids per update CTA
constexpr int kUT = 256;      // threads per update CTA
constexpr int kUChunk = 1024; // assignments scanned per step

// CTA of 256 threads owns centroids c0 .. c0 + 3.  It walks the assignment in
// ascending point order, 1024 entries at a time, compacts its members (order
// kept) and adds each member's row to its centroid's fp64 sums; thread t owns
// dimensions t, t + 256, ..., so every (centroid, dimension) sum is one
// thread's, in ascending member order.
__global__ void __launch_bounds__(kUT) kmeans_update_kernel(const float* __restrict__ X, int64_t n, int d,
                                                            const int32_t* __restrict__ assign, int nl,
                                                            const float* __restrict__ C_old,
                                                            float* __restrict__ C_new, int64_t* __restrict__ counts) {
    extern __shared__ __align__(16) unsigned char smem[];
    double* sums = reinterpret_cast<double*>(smem);                 // [kUC][d]
    __shared__ int mem_idx[kUChunk];
    __shared__ unsigned char mem_c[kUChunk];
    __shared__ int warp_n[kUT / 32];
    __shared__ int s_n;
    __shared__ long long s_cnt[kUC];
    const int c0 = blockIdx.x * kUC;
    const int cn = min(kUC, nl - c0);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int e = tid; e < kUC * d; e += kUT) sums[e] = 0.0;
    if (tid < kUC) s_cnt[tid] = 0;
    __syncthreads();
    for (int64_t base = 0; base < n; base += kUChunk) {
        // compact this chunk's members in point order: 4 entries per thread,
        // thread-major within a warp's 128 entries
        int loc[4], lc[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int64_t i = base + warp * 128 + u * 32 + lane;
            const int a = (i < n) ? assign[i] : -1;
            const bool mine = a >= c0 && a < c0 + cn;
            lc[u] = mine ? a - c0 : -1;
            loc[u] = static_cast<int>(i - base);
        }
        // per warp: count of members, then positions
        int wcount = 0;
#pragma unroll
        for (int u = 0; u < 4; ++u) wcount += __popc(__ballot_sync(0xFFFFFFFFu, lc[u] >= 0));
        if (lane == 0) warp_n[warp] = wcount;
        __syncthreads();
        int wbase = 0;
        for (int w = 0; w < warp; ++w) wbase += warp_n[w];
        int run = wbase;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const unsigned m = __ballot_sync(0xFFFFFFFFu, lc[u] >= 0);
            if (lc[u] >= 0) {
                const int pos = run + __popc(m & ((1u << lane) - 1u));
                mem_idx[pos] = loc[u];
                mem_c[pos] = static_cast<unsigned char>(lc[u]);
            }
            run += __popc(m);
        }
        if (tid == kUT - 1) s_n = run;
        __syncthreads();
        const int nm = s_n;
        // members four at a time: their rows are loaded together, then added
        // in member order
        for (int m0 = 0; m0 < nm; m0 += 4) {
            const int mn = min(4, nm - m0);
            for (int t = tid; t < d; t += kUT) {
                float v[4];
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    v[u] = (u < mn) ? X[(base + mem_idx[m0 + u]) * static_cast<int64_t>(d) + t] : 0.0f;
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    if (u < mn) {
                        const int c = mem_c[m0 + u];
                        sums[c * d + t] = __dadd_rn(sums[c * d + t], static_cast<double>(v[u]));
                    }
            }
            if (tid == 0)
                for (int u = 0; u < mn; ++u) s_cnt[mem_c[m0 + u]] += 1;
        }
        __syncthreads();
    }
    for (int c = 0; c < cn; ++c) {
        const long long m = s_cnt[c];
        for (int t = tid; t < d; t += kUT) {
            const int64_t o = static_cast<int64_t>(c0 + c) * d + t;
            C_new[o] = m ? __double2float_rn(__ddiv_rn(sums[c * d + t], static_cast<double>(m))) : C_old[o];
        }
        if (tid == 0 && counts) counts[c0 + c] = m;
    }
}

}  // namespace

cudaError_t launch_kmeans_assign(const float* X, int64_t n, int d, const float* C, int nl, int32_t* assign,
                                 double* dist, cudaStream_t s) {
    if (n <= 0) return cudaSuccess;
    const int64_t grid = (n + kAP - 1) / kAP;
    if (grid > 0x7FFFFFFF) return cudaErrorInvalidValue;
    kmeans_assign_kernel<<<static_cast<unsigned>(grid), 256, 0, s>>>(X, n, d, C, nl, assign, dist);
    return cudaGetLastError();
}

size_t kmeans_update_smem_bytes(int d) { return static_cast<size_t>(kUC) * d * sizeof(double); }

cudaError_t launch_kmeans_update(const float* X, int64_t n, int d, const int32_t* assign, int nl, const float* C_old,
                                 float* C_new, int64_t* counts, cudaStream_t s) {
    const size_t smem = kmeans_update_smem_bytes(d);
    cudaError_t e = cudaFuncSetAttribute(kmeans_update_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const int grid = (nl + kUC - 1) / kUC;
    kmeans_update_kernel<<<grid, kUT, smem, s>>>(X, n, d, assign, nl, C_old, C_new, counts);
    return cudaGetLastError();
}

}  // namespace ah
