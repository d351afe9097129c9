// Search kernels of the B200 anisotropic-AH MIPS library.
//
// Path (ScaNN blog post, "Three stages of a search"):
//   centroid_scores_kernel   s[q][c] = q . centroid_c                 (partitioning)
//   top_leaves_*_kernel      best L leaves per query
//   invert_*                 query->leaf lists become leaf->query lists, so a
//                            leaf's codes are read once per query group
//   lut_*_kernel             lut[q][b][j] = q_b . center[b][j]        (AH table)
//   threshold_kernel         a lower bound on each query's R-th best approximate
//                            score, from a prefix of its best leaves
//   scan_kernel              leaf-major 4-bit code scan: per slot, the sum of
//                            table entries for every query of the group;
//                            scores at or above the bound are kept
//   tau_update_kernel        between scan phases, raises each bound to the R-th
//                            best point kept so far
//   redo_scan_kernel         query-major rescan for the rare query whose kept
//                            set overflowed its buffer (with a tighter bound)
//   finish_kernel            best R by approximate score, exact fp32 dot
//                            products for them (reordering), best k
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <type_traits>
#include <mutex>
#include <unordered_map>
#include <utility>

#include "common.cuh"
#include "kernels.h"
#include "select.cuh"


namespace ah {

// cudaFuncSetAttribute costs host time on every call; each kernel's dynamic
// shared-memory limit and carveout are raised once per device and size.
namespace {
std::mutex g_attr_mu;
std::unordered_map<uint64_t, int> g_attr_smem;
}  // namespace

static cudaError_t ensure_smem(const void* kernel, size_t bytes, bool max_carveout) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t key = (reinterpret_cast<uint64_t>(kernel) << 6) ^ static_cast<uint64_t>(dev);
    std::lock_guard<std::mutex> lock(g_attr_mu);
    auto it = g_attr_smem.find(key);
    if (it != g_attr_smem.end() && it->second >= static_cast<int>(bytes)) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
    if (e == cudaSuccess && max_carveout)
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (e == cudaSuccess) g_attr_smem[key] = static_cast<int>(bytes);
    return e;
}


// Programmatic dependent launch.  The search kernels form one chain on a
// stream; each is launched with the programmatic-serialization attribute, so
// its CTAs may be scheduled while the previous kernel drains, and its first
// action is to wait until that kernel has finished and its writes are
// visible (a no-op when the previous operation was not a kernel launched
// this way).  Each kernel then lets the next one launch; that next kernel
// waits the same way before reading anything, so every kernel still sees all
// earlier results.
__device__ __forceinline__ void chain_entry() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
static cudaError_t launch_chained(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                                  Args&&... args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ---------------------------------------------------------------------------
// index preparation
// ---------------------------------------------------------------------------

// codes [n][cb] bytes -> il[tile][W/V][lane][V] 32-bit words.  Tiles are
// padded per leaf: leaf c owns tiles ptile[c] .. ptile[c+1]-1, and lane l of
// its tile t holds slot offs[c] + 32 (t - ptile[c]) + l (zero codes past the
// leaf's end).  Word w holds code bytes 4w..4w+3; a lane's words come in
// groups of V consecutive words (V = 4, 2 or 1, the largest dividing W), so it
// reads a group with one 16- or 8-byte load and a warp's load of a group is
// 128 V contiguous bytes.
__global__ void interleave_codes_kernel(const uint8_t* __restrict__ codes, const int32_t* __restrict__ offs,
                                        const int32_t* __restrict__ ptile, int nl, int cb, int W, int V,
                                        uint32_t* __restrict__ il, int64_t total_words) {
    int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (e >= total_words) return;
    const int per_tile = W * 32;
    const int tile = static_cast<int>(e / per_tile);
    const int r = static_cast<int>(e - static_cast<int64_t>(tile) * per_tile);
    const int grp = r / (32 * V), rem = r - grp * 32 * V;
    const int lane = rem / V;
    const int w = grp * V + (rem - lane * V);
    int lo = 0, hi = nl - 1;                   // leaf owning the tile: last c with ptile[c] <= tile
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (ptile[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    const int64_t slot = static_cast<int64_t>(offs[lo]) + 32ll * (tile - ptile[lo]) + lane;
    uint32_t v = 0;
    if (slot < offs[lo + 1]) {
        const uint8_t* row = codes + slot * cb;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            int byte = 4 * w + i;
            if (byte < cb) v |= static_cast<uint32_t>(row[byte]) << (8 * i);
        }
    }
    il[e] = v;
}

int code_vector_words(int W) { return (W % 4 == 0) ? 4 : (W % 2 == 0) ? 2 : 1; }

cudaError_t launch_prepare_index(const int32_t* offs32, const int32_t* ptile, int nl, const uint8_t* codes, int cb,
                                 int W, int64_t ntiles, uint32_t* codes_il, cudaStream_t s) {
    const int64_t total = ntiles * W * 32;
    if (total == 0) return cudaSuccess;
    const int64_t grid = (total + 255) / 256;
    interleave_codes_kernel<<<static_cast<unsigned>(grid), 256, 0, s>>>(codes, offs32, ptile, nl, cb, W,
                                                                          code_vector_words(W), codes_il, total);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// partitioning: centroid scores and top-L leaves
// ---------------------------------------------------------------------------

constexpr int kGemmBK = 16;

// S[q][c] = sum_t Q[q][t] * C[c][t]  (fp32, SIMT; TM x TM tile, 16x16 threads,
// (TM/16)^2 outputs per thread)
template <int TM>
__global__ void __launch_bounds__(256) centroid_scores_kernel(const float* __restrict__ Q, const float* __restrict__ C,
                                                              float* __restrict__ S, int nq, int nl, int d) {
    chain_entry();
    constexpr int PT = TM / 16;              // outputs per thread per dimension
    constexpr int LOADS = TM * kGemmBK / 256;
    __shared__ float As[2][kGemmBK][TM + 4];
    __shared__ float Bs[2][kGemmBK][TM + 4];
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    const int m0 = blockIdx.y * TM, n0 = blockIdx.x * TM;
    float acc[PT][PT];
#pragma unroll
    for (int i = 0; i < PT; ++i)
#pragma unroll
        for (int j = 0; j < PT; ++j) acc[i][j] = 0.0f;
    // the next k step's operands are loaded into registers while the current
    // one is multiplied (each output still accumulates over k in order)
    float ra[LOADS], rb[LOADS];
    auto gload = [&](int k0) {
#pragma unroll
        for (int r = 0; r < LOADS; ++r) {
            const int e = threadIdx.x + 256 * r;
            const int row = e >> 4, col = e & 15;
            const int gk = k0 + col, gm = m0 + row, gn = n0 + row;
            ra[r] = (gm < nq && gk < d) ? Q[static_cast<int64_t>(gm) * d + gk] : 0.0f;
            rb[r] = (gn < nl && gk < d) ? C[static_cast<int64_t>(gn) * d + gk] : 0.0f;
        }
    };
    auto sstore = [&](int buf) {
#pragma unroll
        for (int r = 0; r < LOADS; ++r) {
            const int e = threadIdx.x + 256 * r;
            const int row = e >> 4, col = e & 15;
            As[buf][col][row] = ra[r];
            Bs[buf][col][row] = rb[r];
        }
    };
    gload(0);
    sstore(0);
    __syncthreads();
    int buf = 0;
    for (int k0 = 0; k0 < d; k0 += kGemmBK) {
        const bool more = k0 + kGemmBK < d;
        if (more) gload(k0 + kGemmBK);
#pragma unroll
        for (int kk = 0; kk < kGemmBK; ++kk) {
            float av[PT], bv[PT];
#pragma unroll
            for (int i = 0; i < PT; ++i) av[i] = As[buf][kk][ty + 16 * i];
#pragma unroll
            for (int j = 0; j < PT; ++j) bv[j] = Bs[buf][kk][tx + 16 * j];
#pragma unroll
            for (int i = 0; i < PT; ++i)
#pragma unroll
                for (int j = 0; j < PT; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
        if (more) sstore(buf ^ 1);
        __syncthreads();
        buf ^= 1;
    }
#pragma unroll
    for (int i = 0; i < PT; ++i) {
        int gm = m0 + ty + 16 * i;
        if (gm >= nq) continue;
#pragma unroll
        for (int j = 0; j < PT; ++j) {
            int gn = n0 + tx + 16 * j;
            if (gn < nl) S[static_cast<int64_t>(gm) * nl + gn] = acc[i][j];
        }
    }
}

// 128x128 output tile per CTA of 256 threads, 8x8 outputs per thread (two
// 4-wide fragments per dimension, read as float4 from shared memory), k in
// steps of 8 with the next step's operands loaded from global memory while
// the current one is multiplied.  Each output accumulates over k in ascending
// order with fmaf, as the 64-wide kernel does, so both give identical scores.
// VEC: d % 4 == 0 and 16-byte aligned rows, so operands load as float4.
template <bool VEC>
__global__ void __launch_bounds__(256, 2) centroid_scores128_kernel(const float* __restrict__ Q,
                                                                    const float* __restrict__ C,
                                                                    float* __restrict__ S, int nq, int nl, int d) {
    chain_entry();
    constexpr int T = 128, BK = 8, P = T + 4;
    __shared__ __align__(16) float As[2][BK][P];
    __shared__ __align__(16) float Bs[2][BK][P];
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const int m0 = blockIdx.y * T, n0 = blockIdx.x * T;
    const int lrow = tid >> 1, lk = (tid & 1) * 4;      // operand row and first k this thread loads
    float ra[4], rb[4];
    auto gload = [&](int k0) {
        const int gk = k0 + lk, gm = m0 + lrow, gn = n0 + lrow;
        if (VEC) {
            float4 a = make_float4(0.f, 0.f, 0.f, 0.f), c = a;
            if (gm < nq && gk < d) a = *reinterpret_cast<const float4*>(Q + static_cast<int64_t>(gm) * d + gk);
            if (gn < nl && gk < d) c = *reinterpret_cast<const float4*>(C + static_cast<int64_t>(gn) * d + gk);
            ra[0] = a.x; ra[1] = a.y; ra[2] = a.z; ra[3] = a.w;
            rb[0] = c.x; rb[1] = c.y; rb[2] = c.z; rb[3] = c.w;
        } else {
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                ra[t] = (gm < nq && gk + t < d) ? Q[static_cast<int64_t>(gm) * d + gk + t] : 0.0f;
                rb[t] = (gn < nl && gk + t < d) ? C[static_cast<int64_t>(gn) * d + gk + t] : 0.0f;
            }
        }
    };
    auto sstore = [&](int buf) {
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            As[buf][lk + t][lrow] = ra[t];
            Bs[buf][lk + t][lrow] = rb[t];
        }
    };
    float acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.0f;
    gload(0);
    sstore(0);
    __syncthreads();
    int buf = 0;
    for (int k0 = 0; k0 < d; k0 += BK) {
        const bool more = k0 + BK < d;
        if (more) gload(k0 + BK);
#pragma unroll
        for (int kk = 0; kk < BK; ++kk) {
            const float4 a0 = *reinterpret_cast<const float4*>(&As[buf][kk][ty * 4]);
            const float4 a1 = *reinterpret_cast<const float4*>(&As[buf][kk][64 + ty * 4]);
            const float4 b0 = *reinterpret_cast<const float4*>(&Bs[buf][kk][tx * 4]);
            const float4 b1 = *reinterpret_cast<const float4*>(&Bs[buf][kk][64 + tx * 4]);
            const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
        if (more) sstore(buf ^ 1);
        __syncthreads();
        buf ^= 1;
    }
    const bool vstore = VEC && (nl % 4 == 0);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int gm = m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + (i - 4));
        if (gm >= nq) continue;
        float* row = S + static_cast<int64_t>(gm) * nl;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int gn = n0 + 64 * h + tx * 4;
            if (vstore && gn + 3 < nl) {
                *reinterpret_cast<float4*>(row + gn) =
                    make_float4(acc[i][4 * h], acc[i][4 * h + 1], acc[i][4 * h + 2], acc[i][4 * h + 3]);
            } else {
#pragma unroll
                for (int t = 0; t < 4; ++t)
                    if (gn + t < nl) row[gn + t] = acc[i][4 * h + t];
            }
        }
    }
}

// 128x128 tiles for large batches, 64x64 for mid-size ones, 32x32 for very
// small problems (more CTAs in flight).
cudaError_t launch_centroid_scores(const DeviceIndex& ix, const SearchArgs& a, const SearchBuffers& b, cudaStream_t s) {
    if (ix.c_hi && b.q_hi && centroid_tc_usable(a.nq, ix.nl, ix.d)) {
        // tensor cores: the queries split into tf32 halves, then the tiles
        cudaError_t e = launch_split_tf32(a.queries, static_cast<int64_t>(a.nq) * ix.d, b.q_hi, b.q_lo, s);
        if (e != cudaSuccess) return e;
        return launch_centroid_scores_tc(b.q_hi, b.q_lo, ix.c_hi, ix.c_lo, b.cscore, a.nq, ix.nl, ix.d, b.err, s);
    }
    const int64_t big = static_cast<int64_t>((ix.nl + 63) / 64) * ((a.nq + 63) / 64);
    const int64_t tiles128 = static_cast<int64_t>((ix.nl + 127) / 128) * ((a.nq + 127) / 128);
    if (tiles128 >= 256) {                   // enough 128-wide tiles to fill every SM twice
        dim3 grid((ix.nl + 127) / 128, (a.nq + 127) / 128);
        const bool vec = ix.d % 4 == 0 && reinterpret_cast<uintptr_t>(a.queries) % 16 == 0 &&
                         reinterpret_cast<uintptr_t>(ix.centroids) % 16 == 0;
        const cudaError_t le = vec ? launch_chained(centroid_scores128_kernel<true>, grid, dim3(256), 0, s, a.queries,
                                                    ix.centroids, b.cscore, a.nq, ix.nl, ix.d)
                                   : launch_chained(centroid_scores128_kernel<false>, grid, dim3(256), 0, s, a.queries,
                                                    ix.centroids, b.cscore, a.nq, ix.nl, ix.d);
        if (le != cudaSuccess) return le;
    } else if (big >= 64) {
        dim3 grid((ix.nl + 63) / 64, (a.nq + 63) / 64);
        if (const cudaError_t le = launch_chained(centroid_scores_kernel<64>, dim3(grid), dim3(256), 0, s, a.queries, ix.centroids, b.cscore, a.nq, ix.nl, ix.d); le != cudaSuccess) return le;
    } else {
        dim3 grid((ix.nl + 31) / 32, (a.nq + 31) / 32);
        if (const cudaError_t le = launch_chained(centroid_scores_kernel<32>, dim3(grid), dim3(256), 0, s, a.queries, ix.centroids, b.cscore, a.nq, ix.nl, ix.d); le != cudaSuccess) return le;
    }
    return cudaGetLastError();
}

#ifndef AH_REORDER_BATCH
#define AH_REORDER_BATCH 4
#endif
#ifndef AH_FINISH_MIN_BLOCKS
#define AH_FINISH_MIN_BLOCKS 6
#endif
constexpr int kSelThreads = 256;

// One CTA per query: best L leaves by (score desc, leaf id asc), the points
// the query will scan, and (for leaf ranks below count_ranks) the queries per
// leaf of the first scan phase.
__global__ void __launch_bounds__(kSelThreads) top_leaves_kernel(DeviceIndex ix, SearchArgs a, SearchBuffers b) {
    chain_entry();
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ SelectScratch scr;
    __shared__ long long s_scanned;
    const int q = blockIdx.x;
    const int L = a.L, nl = ix.nl;
    const int P2 = next_pow2(L);
    uint64_t* keys = reinterpret_cast<uint64_t*>(smem);
    const float* grow = b.cscore + static_cast<int64_t>(q) * nl;
    const float* row = grow;
    if (a.topl_row_smem) {                    // stage the score row once; the selection reads it several times
        float* srow = reinterpret_cast<float*>(keys + P2);
        for (int i = threadIdx.x; i < nl; i += kSelThreads) srow[i] = grow[i];
        __syncthreads();
        row = srow;
    }
    auto get = [&](int i) { return make_key(float_key(row[i]), i); };
    auto pay = [&](int i) { return i; };
    if (threadIdx.x == 0) s_scanned = 0;
    block_topk<kSelThreads>(get, pay, nl, L, scr, keys, nullptr, b.err);
    long long local = 0;
    for (int i = threadIdx.x; i < L; i += kSelThreads) {
        uint64_t key = keys[i];
        int leaf = key_id(key);
        b.leaves[static_cast<int64_t>(q) * L + i] = leaf;
        b.leaf_scores[static_cast<int64_t>(q) * L + i] = key_float(key_score(key));
        if (i < a.count_ranks) atomicAdd(&b.qcount[leaf], 1);     // queries per leaf, first scan phase
        local += ix.offs[leaf + 1] - ix.offs[leaf];
    }
    atomicAdd(reinterpret_cast<unsigned long long*>(&s_scanned), static_cast<unsigned long long>(local));
    __syncthreads();
    if (threadIdx.x == 0) b.scanned[q] = s_scanned;
}

static cudaError_t launch_top_leaves_block(const DeviceIndex& ix, SearchArgs a, const SearchBuffers& b, cudaStream_t s) {
    size_t smem = static_cast<size_t>(next_pow2(a.L)) * sizeof(uint64_t);
    const size_t row = static_cast<size_t>(ix.nl) * sizeof(float);
    a.topl_row_smem = (row <= 64 * 1024) ? 1 : 0;
    if (a.topl_row_smem) smem += row;
    cudaError_t e = ensure_smem(reinterpret_cast<const void*>(top_leaves_kernel), smem, true);
    if (e != cudaSuccess) return e;
    if (const cudaError_t le = launch_chained(top_leaves_kernel, dim3(a.nq), dim3(kSelThreads), smem, s, ix, a, b); le != cudaSuccess) return le;
    return cudaGetLastError();
}

constexpr int kWarpMaxK = 256;          // warp-cooperative selection up to this K

// The K = min(K, n) largest of n <= KPL*NT keys read by get(i) (payload
// pay(i)) through registers: block_kth_reg finds the K-th key, the keys at or
// above it are gathered (atomic positions; sorted descending when `sort`,
// padding key 0 up to next_pow2(K)).  Returns K on every thread.
template <int KPL, int NT, class GetKey, class GetVal>
__device__ int block_topk_reg(GetKey get, GetVal pay, int n, int K, RegSelectScratch<NT>& rs, int* counter,
                              uint64_t* out_k, int32_t* out_v, bool sort) {
    uint64_t kk[KPL];
    int32_t vv[KPL];
#pragma unroll
    for (int j = 0; j < KPL; ++j) {
        const int i = threadIdx.x + NT * j;
        kk[j] = (i < n) ? get(i) : 0ull;
        vv[j] = (i < n && out_v) ? pay(i) : -1;
    }
    if (K > n) K = n;
    if (K <= 0) return 0;
    if (threadIdx.x == 0) *counter = 0;
    const uint64_t thr = (K < n) ? block_kth_reg<KPL, NT>(kk, n, K, rs) : 1ull;
    if (K >= n) __syncthreads();
    const int P2 = next_pow2(K);
    for (int i = K + threadIdx.x; i < P2; i += NT) {
        out_k[i] = 0ull;
        if (out_v) out_v[i] = -1;
    }
#pragma unroll
    for (int j = 0; j < KPL; ++j) {
        if (kk[j] != 0ull && kk[j] >= thr) {
            const int pos = atomicAdd(counter, 1);
            out_k[pos] = kk[j];
            if (out_v) out_v[pos] = vv[j];
        }
    }
    __syncthreads();
    if (sort) block_sort_desc<NT>(out_k, out_v, P2);
    return K;
}

// One CTA of NT threads per query with the score row in registers (KPL per
// thread): for 1024 < centroids <= KPL * NT.
// MERGE: the keys are the survivors of top_leaves_seg_kernel's segments
// instead of the score row (the leaf id is inside each key).
template <int KPL, int NT, bool MERGE = false>
__global__ void __launch_bounds__(NT) top_leaves_reg_kernel(DeviceIndex ix, SearchArgs a, SearchBuffers b) {
    chain_entry();
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ RegSelectScratch<NT> rs;
    __shared__ int s_count;
    __shared__ long long s_scanned;
    const int q = blockIdx.x;
    const int L = a.L, nl = ix.nl;
    uint64_t* keys = reinterpret_cast<uint64_t*>(smem);
    const float* row = b.cscore + static_cast<int64_t>(q) * nl;
    int n = nl;
    const uint64_t* cand = nullptr;
    if (MERGE) {
        // segment s kept min(L, its size) keys, stored back to back
        const int seg = a.topl_seg, S = (nl + seg - 1) / seg;
        n = (S - 1) * min(L, seg) + min(L, nl - (S - 1) * seg);
        cand = b.topl_tmp + static_cast<int64_t>(q) * a.topl_stride;
    }
    auto get = [&](int i) { return MERGE ? cand[i] : make_key(float_key(row[i]), i); };
    auto pay = [&](int i) { return i; };
    if (threadIdx.x == 0) s_scanned = 0;
    block_topk_reg<KPL, NT>(get, pay, n, L, rs, &s_count, keys, static_cast<int32_t*>(nullptr), true);
    long long local = 0;
    for (int i = threadIdx.x; i < L; i += NT) {
        const uint64_t key = keys[i];
        const int leaf = key_id(key);
        b.leaves[static_cast<int64_t>(q) * L + i] = leaf;
        b.leaf_scores[static_cast<int64_t>(q) * L + i] = key_float(key_score(key));
        if (i < a.count_ranks) atomicAdd(&b.qcount[leaf], 1);
        local += ix.offs[leaf + 1] - ix.offs[leaf];
    }
    atomicAdd(reinterpret_cast<unsigned long long*>(&s_scanned), static_cast<unsigned long long>(local));
    __syncthreads();
    if (threadIdx.x == 0) b.scanned[q] = s_scanned;
}

constexpr int kReorderBatch = AH_REORDER_BATCH;
// One CTA per query, two warp-level stages: warp w keeps the best L of its
// slice of the score row (KPL keys per lane, in registers), then warp 0 keeps
// the best L of the 8 slices' survivors (at most 8 L <= 512 keys).  One
// barrier in all.  For 1024 < centroids <= 8 * 32 * KPL and L <= 64.
template <int KPL>
__global__ void __launch_bounds__(kSelThreads) top_leaves_2stage_kernel(DeviceIndex ix, SearchArgs a, SearchBuffers b) {
    chain_entry();
    __shared__ uint64_t cand[8 * 64];
    __shared__ uint64_t keys[64];
    __shared__ int s_count;
    const int q = blockIdx.x;
    const int L = a.L, nl = ix.nl;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float* row = b.cscore + static_cast<int64_t>(q) * nl;
    const int per = (nl + 7) / 8;
    const int lo = warp * per, n = max(0, min(per, nl - lo));
    if (threadIdx.x == 0) s_count = 0;
    __syncthreads();
    {
        uint64_t k[KPL];
#pragma unroll
        for (int j = 0; j < KPL; ++j) {
            const int i = lane + 32 * j;
            k[j] = (i < n) ? make_key(float_key(row[lo + i]), lo + i) : 0ull;
        }
        const int keep = min(L, n);
        if (keep > 0) {
            const uint64_t thr = (keep < n) ? warp_kth_reg<KPL>(k, n, keep) : 1ull;
            int base = 0;
            if (lane == 0) base = atomicAdd(&s_count, keep);
            base = __shfl_sync(0xFFFFFFFFu, base, 0);
#pragma unroll
            for (int j = 0; j < KPL; ++j) {
                const bool sel = k[j] != 0ull && k[j] >= thr;
                const unsigned m = __ballot_sync(0xFFFFFFFFu, sel);
                if (sel) cand[base + __popc(m & ((1u << lane) - 1u))] = k[j];
                base += __popc(m);
            }
        }
    }
    __syncthreads();
    if (warp == 0) {
        const int tot = s_count;
        warp_topk_src<16>(cand, static_cast<const int32_t*>(nullptr), tot, L, keys, static_cast<int32_t*>(nullptr), true);
        long long local = 0;
        for (int i = lane; i < L; i += 32) {
            const uint64_t key = keys[i];
            const int leaf = key_id(key);
            b.leaves[static_cast<int64_t>(q) * L + i] = leaf;
            b.leaf_scores[static_cast<int64_t>(q) * L + i] = key_float(key_score(key));
            if (i < a.count_ranks) atomicAdd(&b.qcount[leaf], 1);
            local += ix.offs[leaf + 1] - ix.offs[leaf];
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) local += __shfl_xor_sync(0xFFFFFFFFu, local, off);
        if (lane == 0) b.scanned[q] = local;
    }
}

constexpr int kTopWarps = 8;
constexpr int kTopRegWide = 1024;      // threads of the widest register top-L form
// split top-L (small batches, more than 4096 centroids): up to this many
// segments per query, batches up to kTopSplitMaxQ queries, L up to kTopSplitMaxL
constexpr int kTopSplitSegs = 16;
constexpr int kTopSplitMaxQ = 64;
constexpr int kTopSplitMaxL = 256;

// One warp per query when the centroids fit 32 per lane: the scores stay in
// registers and the selection needs no shared-memory passes.
__global__ void __launch_bounds__(kTopWarps * 32) top_leaves_warp_kernel(DeviceIndex ix, SearchArgs a, SearchBuffers b) {
    chain_entry();
    extern __shared__ __align__(16) unsigned char smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q = blockIdx.x * kTopWarps + warp;
    if (q >= a.nq) return;
    const int L = a.L, nl = ix.nl, P2 = next_pow2(L);
    uint64_t* keys = reinterpret_cast<uint64_t*>(smem) + static_cast<size_t>(warp) * P2;
    const float* row = b.cscore + static_cast<int64_t>(q) * nl;
    auto get = [&](int i) { return make_key(float_key(row[i]), i); };
    auto pay = [&](int i) { return i; };
    warp_topk_reg<32>(get, pay, nl, L, keys, nullptr, true);
    long long local = 0;
    for (int i = lane; i < L; i += 32) {
        const uint64_t key = keys[i];
        const int leaf = key_id(key);
        b.leaves[static_cast<int64_t>(q) * L + i] = leaf;
        b.leaf_scores[static_cast<int64_t>(q) * L + i] = key_float(key_score(key));
        if (i < a.count_ranks) atomicAdd(&b.qcount[leaf], 1);
        local += ix.offs[leaf + 1] - ix.offs[leaf];
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) local += __shfl_xor_sync(0xFFFFFFFFu, local, off);
    if (lane == 0) b.scanned[q] = local;
}

// Small batches over many centroids, first step: CTA (s, q) keeps the best
// min(L, size) keys of segment s of query q's score row (1,024 scores per
// segment at most, 4 per thread), unordered, at tmp[q][s * min(L, seg)].
// Any key of the row's best L is among its segment's best L, so the
// segments' survivors hold the row's best L; top_leaves_reg_kernel<...,
// true> keeps those.
__global__ void __launch_bounds__(kSelThreads) top_leaves_seg_kernel(DeviceIndex ix, SearchArgs a, SearchBuffers b) {
    chain_entry();
    __shared__ RegSelectScratch<kSelThreads> rs;
    __shared__ int s_count;
    __shared__ uint64_t keys[1024];
    const int sidx = blockIdx.x, q = blockIdx.y;
    const int seg = a.topl_seg, L = a.L;
    const int lo = sidx * seg, n = min(seg, ix.nl - lo);
    const float* row = b.cscore + static_cast<int64_t>(q) * ix.nl + lo;
    auto get = [&](int i) { return make_key(float_key(row[i]), lo + i); };
    auto pay = [&](int i) { return i; };
    const int K = block_topk_reg<4, kSelThreads>(get, pay, n, min(L, n), rs, &s_count, keys,
                                                 static_cast<int32_t*>(nullptr), false);
    uint64_t* out = b.topl_tmp + static_cast<int64_t>(q) * a.topl_stride + static_cast<int64_t>(sidx) * min(L, seg);
    for (int i = threadIdx.x; i < K; i += kSelThreads) out[i] = keys[i];
}

cudaError_t launch_top_leaves(const DeviceIndex& ix, SearchArgs a, const SearchBuffers& b, cudaStream_t s) {
    if (b.topl_tmp && ix.nl > 16 * kSelThreads && a.nq <= kTopSplitMaxQ && a.L <= kTopSplitMaxL) {
        // split form: segments of at most 1,024 scores in parallel, then one
        // CTA per query merges the survivors (at most 16 x 256 keys)
        a.topl_seg = (ix.nl + kTopSplitSegs - 1) / kTopSplitSegs;
        if (a.topl_seg > 1024) a.topl_seg = 1024;
        const int S = (ix.nl + a.topl_seg - 1) / a.topl_seg;
        a.topl_stride = S * a.L;
        if (S <= kTopSplitSegs) {
            if (const cudaError_t le = launch_chained(top_leaves_seg_kernel, dim3(S, a.nq), dim3(kSelThreads), 0, s, ix, a, b);
                le != cudaSuccess)
                return le;
            const size_t smem = static_cast<size_t>(next_pow2(a.L)) * sizeof(uint64_t);
            cudaError_t e = ensure_smem(reinterpret_cast<const void*>(top_leaves_reg_kernel<16, kSelThreads, true>), smem, false);
            if (e != cudaSuccess) return e;
            if (const cudaError_t le = launch_chained(top_leaves_reg_kernel<16, kSelThreads, true>, dim3(a.nq),
                                                      dim3(kSelThreads), smem, s, ix, a, b);
                le != cudaSuccess)
                return le;
            return cudaGetLastError();
        }
    }
    if (ix.nl <= 32 * 32 && a.L <= kWarpMaxK) {
        const size_t smem = static_cast<size_t>(kTopWarps) * next_pow2(a.L) * sizeof(uint64_t);
        cudaError_t e = ensure_smem(reinterpret_cast<const void*>(top_leaves_warp_kernel), smem, false);
        if (e != cudaSuccess) return e;
        if (const cudaError_t le = launch_chained(top_leaves_warp_kernel, dim3((a.nq + kTopWarps - 1) / kTopWarps), dim3(kTopWarps * 32), smem, s, ix, a, b); le != cudaSuccess) return le;
        return cudaGetLastError();
    }
    if (ix.nl <= 16 * kSelThreads && a.L <= 64) {
        const cudaError_t le = (ix.nl <= 8 * kSelThreads)
            ? launch_chained(top_leaves_2stage_kernel<8>, dim3(a.nq), dim3(kSelThreads), 0, s, ix, a, b)
            : launch_chained(top_leaves_2stage_kernel<16>, dim3(a.nq), dim3(kSelThreads), 0, s, ix, a, b);
        if (le != cudaSuccess) return le;
        return cudaGetLastError();
    }
    if (ix.nl <= 16 * kSelThreads || (ix.nl <= 16 * kTopRegWide && a.nq <= 512)) {
        // the score row in registers: 256 threads up to 4096 centroids, 1024
        // threads (16 keys each) up to 16384 for batches of at most 512
        // queries (larger batches of such rows ran faster in the
        // shared-memory radix form: its CTAs are lighter and more fit an SM)
        const size_t smem = static_cast<size_t>(next_pow2(a.L)) * sizeof(uint64_t);
        const int form = (ix.nl <= 8 * kSelThreads) ? 0 : (ix.nl <= 16 * kSelThreads) ? 1 : 2;
        const void* fn = form == 0 ? reinterpret_cast<const void*>(top_leaves_reg_kernel<8, kSelThreads>)
                       : form == 1 ? reinterpret_cast<const void*>(top_leaves_reg_kernel<16, kSelThreads>)
                                   : reinterpret_cast<const void*>(top_leaves_reg_kernel<16, kTopRegWide>);
        cudaError_t e = ensure_smem(fn, smem, false);
        if (e != cudaSuccess) return e;
        const cudaError_t le =
            form == 0 ? launch_chained(top_leaves_reg_kernel<8, kSelThreads>, dim3(a.nq), dim3(kSelThreads), smem, s, ix, a, b)
          : form == 1 ? launch_chained(top_leaves_reg_kernel<16, kSelThreads>, dim3(a.nq), dim3(kSelThreads), smem, s, ix, a, b)
                      : launch_chained(top_leaves_reg_kernel<16, kTopRegWide>, dim3(a.nq), dim3(kTopRegWide), smem, s, ix, a, b);
        if (le != cudaSuccess) return le;
        return cudaGetLastError();
    }
    return launch_top_leaves_block(ix, a, b, s);
}

// ---------------------------------------------------------------------------
// inversion: leaf -> query lists and the scan work items
// ---------------------------------------------------------------------------

constexpr int kScanBlock = 1024;

// Exclusive prefix sums of a pair of values over a 1,024-thread block; the
// block's totals in *total.
__device__ __forceinline__ int2 block_exclusive_scan2_1024(int2 v, int2* warp_sums, int2* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int2 x = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int yx = __shfl_up_sync(0xFFFFFFFFu, x.x, off), yy = __shfl_up_sync(0xFFFFFFFFu, x.y, off);
        if (lane >= off) { x.x += yx; x.y += yy; }
    }
    if (lane == 31) warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
        const int2 w = warp_sums[lane];
        int2 xs = w;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int yx = __shfl_up_sync(0xFFFFFFFFu, xs.x, off), yy = __shfl_up_sync(0xFFFFFFFFu, xs.y, off);
            if (lane >= off) { xs.x += yx; xs.y += yy; }
        }
        warp_sums[lane] = make_int2(xs.x - w.x, xs.y - w.y);   // exclusive prefix of warps
        if (lane == 31) *total = xs;
    }
    __syncthreads();
    const int2 r = make_int2(warp_sums[warp].x + x.x - v.x, warp_sums[warp].y + x.y - v.y);
    __syncthreads();
    return r;
}

// Single CTA: qoff = exclusive scan of queries per leaf; item_off = exclusive
// scan of work items per leaf (query groups x chunks of `chunk` code tiles).
// Each thread takes 8 consecutive leaves, so 8,192 leaves cost one block scan.
__global__ void __launch_bounds__(kScanBlock) invert_offsets_kernel(DeviceIndex ix, SearchBuffers b, int group, int chunk) {
    chain_entry();
    constexpr int E = 8;
    __shared__ int2 warp_sums[32];
    __shared__ int2 total;
    int carry_q = 0, carry_i = 0;
    for (int base = 0; base < ix.nl; base += kScanBlock * E) {
        const int c0 = base + threadIdx.x * E;
        int eq[E], ei[E];
        int sq = 0, si = 0;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const int c = c0 + e;
            int qc = 0, it = 0;
            if (c < ix.nl) {
                qc = b.qcount[c];
                const int tiles = ix.ptile[c + 1] - ix.ptile[c];
                it = (qc > 0 && tiles > 0) ? ((qc + group - 1) / group) * ((tiles + chunk - 1) / chunk) : 0;
            }
            eq[e] = sq;
            ei[e] = si;
            sq += qc;
            si += it;
        }
        const int2 ex = block_exclusive_scan2_1024(make_int2(sq, si), warp_sums, &total);
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const int c = c0 + e;
            if (c < ix.nl) {
                b.qoff[c] = carry_q + ex.x + eq[e];
                b.item_off[c] = carry_i + ex.y + ei[e];
            }
        }
        carry_q += total.x;
        carry_i += total.y;
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        b.qoff[ix.nl] = carry_q;
        b.item_off[ix.nl] = carry_i;
    }
}

// Queries per leaf over leaf ranks [r0, r1) of every query.
__global__ void invert_count_kernel(SearchArgs a, SearchBuffers b, int r0, int r1) {
    chain_entry();
    const int span = r1 - r0;
    int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (e >= static_cast<int64_t>(a.nq) * span) return;
    const int q = static_cast<int>(e / span), r = r0 + static_cast<int>(e - static_cast<int64_t>(q) * span);
    atomicAdd(&b.qcount[b.leaves[static_cast<int64_t>(q) * a.L + r]], 1);
}

__global__ void invert_scatter_kernel(SearchArgs a, SearchBuffers b, int r0, int r1) {
    chain_entry();
    const int span = r1 - r0;
    int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (e >= static_cast<int64_t>(a.nq) * span) return;
    const int q = static_cast<int>(e / span), r = r0 + static_cast<int>(e - static_cast<int64_t>(q) * span);
    const int leaf = b.leaves[static_cast<int64_t>(q) * a.L + r];
    const int pos = atomicAdd(&b.qcursor[leaf], 1);
    b.qlist[b.qoff[leaf] + pos] = q;
}

// leaf -> query lists (and scan work items) for the leaves of ranks [r0, r1)
// (counted: the queries per leaf are already in qcount and qcursor is zero)
cudaError_t launch_invert(const DeviceIndex& ix, const SearchArgs& a, const SearchBuffers& b, int r0, int r1,
                          bool counted, cudaStream_t s) {
    const int64_t total = static_cast<int64_t>(a.nq) * (r1 - r0);
    const unsigned grid = static_cast<unsigned>((total + 255) / 256);
    if (!counted) {
        cudaError_t e = cudaMemsetAsync(b.qcount, 0, sizeof(int32_t) * 2 * static_cast<size_t>(ix.nl), s);   // qcount, qcursor
        if (e != cudaSuccess) return e;
        if (const cudaError_t le = launch_chained(invert_count_kernel, dim3(grid), dim3(256), 0, s, a, b, r0, r1); le != cudaSuccess) return le;
    }
    const int group = a.scan_tc ? scan_tc_group() : scan_group(ix, a.lut_mode);
    if (const cudaError_t le = launch_chained(invert_offsets_kernel, dim3(1), dim3(kScanBlock), 0, s, ix, b, group, a.chunk); le != cudaSuccess) return le;
    if (const cudaError_t le = launch_chained(invert_scatter_kernel, dim3(grid), dim3(256), 0, s, a, b, r0, r1); le != cudaSuccess) return le;
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// lookup tables
// ---------------------------------------------------------------------------

// lut[q][b][j] = q[b*dpb] * c[0], then fmaf(q[b*dpb+t], c[t], lut) for t >= 1.
__device__ __forceinline__ float lut_entry(const float* __restrict__ q, const float* __restrict__ c, int dpb) {
    float v = __fmul_rn(q[0], c[0]);
    for (int t = 1; t < dpb; ++t) v = fmaf(q[t], c[t], v);
    return v;
}

// grid (queries, entries / 256): thread r of query blockIdx.x writes entry r
__global__ void lut_f32_kernel(DeviceIndex ix, SearchArgs a, SearchBuffers b) {
    chain_entry();
    const int per_q = ix.B * kCenters;
    const int q = blockIdx.x;
    const int r = blockIdx.y * blockDim.x + threadIdx.x;
    if (r >= per_q) return;
    b.lut_f32[static_cast<int64_t>(q) * per_q + r] =
        lut_entry(a.queries + static_cast<int64_t>(q) * ix.d + (r >> 4) * ix.dpb, ix.codebook + r * ix.dpb, ix.dpb);
}

// One CTA per query: the uint8 table, delta and bias, all in fp32 with
// round-to-nearest operations in a fixed order.
__global__ void __launch_bounds__(256) lut_u8_kernel(DeviceIndex ix, SearchArgs a, SearchBuffers b) {
    chain_entry();
    extern __shared__ __align__(16) unsigned char smem[];
    float* lut = reinterpret_cast<float*>(smem);          // [B*16]
    float* mins = lut + ix.B * kCenters;                  // [B]
    __shared__ unsigned int s_range_bits;
    const int q = blockIdx.x;
    const int per_q = ix.B * kCenters;
    const float* qv = a.queries + static_cast<int64_t>(q) * ix.d;
    if (threadIdx.x == 0) s_range_bits = 0u;
    for (int r = threadIdx.x; r < per_q; r += blockDim.x)
        lut[r] = lut_entry(qv + (r >> 4) * ix.dpb, ix.codebook + static_cast<int64_t>(r) * ix.dpb, ix.dpb);
    __syncthreads();
    for (int blk = threadIdx.x; blk < ix.B; blk += blockDim.x) {
        float lo = lut[blk * kCenters], hi = lo;
        for (int j = 1; j < kCenters; ++j) {
            lo = fminf(lo, lut[blk * kCenters + j]);
            hi = fmaxf(hi, lut[blk * kCenters + j]);
        }
        mins[blk] = lo;
        float range = __fsub_rn(hi, lo);                  // >= 0: bits order as floats
        atomicMax(&s_range_bits, __float_as_uint(range));
    }
    __syncthreads();
    float delta = __fdiv_rn(__uint_as_float(s_range_bits), 255.0f);
    if (delta == 0.0f) delta = 1.0f;
    uint8_t* out = b.lut_u8 + static_cast<int64_t>(q) * per_q;
    for (int r = threadIdx.x; r < per_q; r += blockDim.x) {
        float v = rintf(__fdiv_rn(__fsub_rn(lut[r], mins[r >> 4]), delta));
        out[r] = static_cast<uint8_t>(fminf(v, 255.0f));
    }
    if (threadIdx.x == 0) {
        float bias = 0.0f;
        for (int blk = 0; blk < ix.B; ++blk) bias = __fadd_rn(bias, mins[blk]);
        b.lut_delta[q] = delta;
        b.lut_bias[q] = bias;
    }
}

cudaError_t launch_lut(const DeviceIndex& ix, const SearchArgs& a, const SearchBuffers& b, cudaStream_t s) {
    if (a.lut_mode == 0) {
        const unsigned per_q = static_cast<unsigned>(ix.B) * kCenters;
        if (const cudaError_t le = launch_chained(lut_f32_kernel, dim3(static_cast<unsigned>(a.nq), (per_q + 255) / 256), dim3(256), 0, s, ix, a, b); le != cudaSuccess) return le;
    } else {
        size_t smem = (static_cast<size_t>(ix.B) * kCenters + ix.B) * sizeof(float);
        cudaError_t e = ensure_smem(reinterpret_cast<const void*>(lut_u8_kernel), smem, true);
        if (e != cudaSuccess) return e;
        if (const cudaError_t le = launch_chained(lut_u8_kernel, dim3(a.nq), dim3(256), smem, s, ix, a, b); le != cudaSuccess) return le;
    }
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// per-slot approximate score (query-major kernels): sum over blocks in order
// ---------------------------------------------------------------------------

// fp32: table in shared memory as [B][16] floats; returns the score key.
// uint8: table as [B][16] bytes; returns the integer sum.
// `pos` is the slot's position in the leaf-padded code copy.
// With residual codes the leaf's centroid score `off` is added after the sum.
// Offset of word w of lane `lane` within a tile of the code copy
// ([W/V][32][V] words, V a power of two up to 4).
__device__ __forceinline__ int code_word(int w, int lane, int V) {
    const int r = w & (V - 1);
    return (w - r) * 32 + lane * V + r;
}

// Words w .. w+3 of a lane (w a multiple of 4): one 16-byte load (V = 4), two
// 8-byte loads (V = 2) or four 4-byte loads.
__device__ __forceinline__ void code_words4(const uint32_t* __restrict__ tile, int lane, int w, int V, uint32_t& c0,
                                            uint32_t& c1, uint32_t& c2, uint32_t& c3) {
    if (V == 4) {
        const uint4 v = *reinterpret_cast<const uint4*>(tile + w * 32 + lane * 4);
        c0 = v.x; c1 = v.y; c2 = v.z; c3 = v.w;
    } else if (V == 2) {
        const uint2 a = *reinterpret_cast<const uint2*>(tile + w * 32 + lane * 2);
        const uint2 b = *reinterpret_cast<const uint2*>(tile + (w + 2) * 32 + lane * 2);
        c0 = a.x; c1 = a.y; c2 = b.x; c3 = b.y;
    } else {
        c0 = tile[w * 32 + lane]; c1 = tile[(w + 1) * 32 + lane];
        c2 = tile[(w + 2) * 32 + lane]; c3 = tile[(w + 3) * 32 + lane];
    }
}

// Shared loads by 32-bit shared-window address (the address arithmetic stays
// 32-bit; a constant offset folds into the load).
__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}
__device__ __forceinline__ uint32_t lds_u8(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u8 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}
__device__ __forceinline__ uint2 lds_u64(uint32_t addr) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
    return v;
}

template <int MODE>
__device__ __forceinline__ uint32_t slot_value(const uint32_t* __restrict__ codes_il, int W, int V, int B,
                                               const unsigned char* lut, int32_t pos, bool add_off, float off) {
    const uint32_t* tile = codes_il + (static_cast<int64_t>(pos >> 5) * W) * 32;
    const int lane = pos & 31;
    if (MODE == 0) {
        const float* lf = reinterpret_cast<const float*>(lut);
        float acc = 0.0f;
        for (int w = 0; w < W; ++w) {
            uint32_t c = tile[code_word(w, lane, V)];
            int nb = min(8, B - 8 * w);
            for (int i = 0; i < nb; ++i) acc = __fadd_rn(acc, lf[(8 * w + i) * kCenters + ((c >> (4 * i)) & 15u)]);
        }
        return float_key(add_off ? __fadd_rn(acc, off) : acc);
    } else {
        uint32_t acc = 0;
        for (int w = 0; w < W; ++w) {
            uint32_t c = tile[code_word(w, lane, V)];
            int nb = min(8, B - 8 * w);
            for (int i = 0; i < nb; ++i) acc += lut[(8 * w + i) * kCenters + ((c >> (4 * i)) & 15u)];
        }
        return acc;
    }
}

// Four slots at once (independent chains for latency hiding); each slot's sum
// still runs over blocks in order, identical to slot_value.  A slot's code
// words are read four at a time (one 16-byte load where the copy's vector
// width is 4), so a warp's loads for consecutive slots stay contiguous.
// fp32: `lut` starts 256-byte aligned in the shared window; a word's 8 blocks
// span 512 bytes, so an entry's address is the word's address with its low
// byte replaced by the nibble's byte offset (one byte permute per lookup).
template <int MODE>
__device__ __forceinline__ void slot_values4(const uint32_t* __restrict__ codes_il, int W, int V, int B,
                                             const unsigned char* lut, const int32_t* pos, const bool* valid,
                                             const float* off, uint32_t* out) {
    const uint32_t* cw[4];
    int ln[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int32_t sl = valid[u] ? pos[u] : 0;
        cw[u] = codes_il + (static_cast<int64_t>(sl >> 5) * W) * 32;
        ln[u] = sl & 31;
    }
    const int Wf = B >> 3, tail = B & 7;
    if (MODE == 0) {
        const float* lf = reinterpret_cast<const float*>(lut);
        const uint32_t tb = static_cast<uint32_t>(__cvta_generic_to_shared(lut));
        float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        auto word = [&](int u, uint32_t c, int w, int nb) {
            const float* base = lf + 8 * w * kCenters;
            for (int i = 0; i < nb; ++i) acc[u] = __fadd_rn(acc[u], base[i * kCenters + ((c >> (4 * i)) & 15u)]);
        };
        int w = 0;
        for (; w + 4 <= Wf; w += 4) {
            uint32_t c[4][4];
#pragma unroll
            for (int u = 0; u < 4; ++u) code_words4(cw[u], ln[u], w, V, c[u][0], c[u][1], c[u][2], c[u][3]);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                // byte offsets of the word's 8 entries: nibbles 0, 2, 4, 6 in
                // the bytes of ev, 1, 3, 5, 7 in those of od (times 4 bytes)
                const uint32_t xw = tb + static_cast<uint32_t>(w + k) * (8 * kCenters * 4);
                uint32_t ev[4], od[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    ev[u] = (c[u][k] & 0x0F0F0F0Fu) << 2;
                    od[u] = ((c[u][k] >> 4) & 0x0F0F0F0Fu) << 2;
                }
#pragma unroll
                for (int i = 0; i < 8; ++i)
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const uint32_t p = __byte_perm((i & 1) ? od[u] : ev[u], xw, 0x7650u | (i >> 1)) + i * 4 * kCenters;
                        acc[u] = __fadd_rn(acc[u], __uint_as_float(lds_u32(p)));
                    }
            }
        }
        for (; w < Wf; ++w)
#pragma unroll
            for (int u = 0; u < 4; ++u) word(u, cw[u][code_word(w, ln[u], V)], w, 8);
        if (tail)
#pragma unroll
            for (int u = 0; u < 4; ++u) word(u, cw[u][code_word(Wf, ln[u], V)], Wf, tail);
#pragma unroll
        for (int u = 0; u < 4; ++u) out[u] = float_key(off ? __fadd_rn(acc[u], off[u]) : acc[u]);
    } else {
        uint32_t acc[4] = {0u, 0u, 0u, 0u};
        auto word = [&](int u, uint32_t c, int w, int nb) {
            const unsigned char* base = lut + 8 * w * kCenters;
            for (int i = 0; i < nb; ++i) acc[u] += base[i * kCenters + ((c >> (4 * i)) & 15u)];
        };
        int w = 0;
        for (; w + 4 <= Wf; w += 4) {
            uint32_t c[4][4];
#pragma unroll
            for (int u = 0; u < 4; ++u) code_words4(cw[u], ln[u], w, V, c[u][0], c[u][1], c[u][2], c[u][3]);
#pragma unroll
            for (int k = 0; k < 4; ++k)
#pragma unroll
                for (int u = 0; u < 4; ++u) word(u, c[u][k], w + k, 8);
        }
        for (; w < Wf; ++w)
#pragma unroll
            for (int u = 0; u < 4; ++u) word(u, cw[u][code_word(w, ln[u], V)], w, 8);
        if (tail)
#pragma unroll
            for (int u = 0; u < 4; ++u) word(u, cw[u][code_word(Wf, ln[u], V)], Wf, tail);
#pragma unroll
        for (int u = 0; u < 4; ++u) out[u] = acc[u];
    }
}

// One query's table in shared memory for the query-major kernels, where each
// lane scores its own slot: fp32 [b][16] floats, uint8 [b][16] bytes.  (A
// conflict-free layout with every fp32 entry twice measured slower in the
// threshold kernel: the doubled table cost more in occupancy than the bank
// conflicts did.)
template <int MODE>
__device__ __forceinline__ void load_query_table(const DeviceIndex& ix, const SearchBuffers& b, int q, unsigned char* lut) {
    const int per_q = ix.B * kCenters;
    if (MODE == 0) {
        float* lf = reinterpret_cast<float*>(lut);
        const float* src = b.lut_f32 + static_cast<int64_t>(q) * per_q;
        for (int r = threadIdx.x; r < per_q; r += blockDim.x) lf[r] = src[r];
    } else {
        const uint8_t* src = b.lut_u8 + static_cast<int64_t>(q) * per_q;
        for (int r = threadIdx.x; r < per_q; r += blockDim.x) lut[r] = src[r];
    }
}

// Shared memory of one query's table in the query-major kernels.
__host__ __device__ __forceinline__ int table_bytes(int mode, int B) {
    return B * kCenters * (mode == 0 ? 4 : 1);
}

// ---------------------------------------------------------------------------
// threshold: R-th best approximate score over a prefix of the best leaves
// ---------------------------------------------------------------------------


constexpr int kThresholdSegs = 256;      // sample segments (leaves) per query at most
// samples above 2,048 keys (batches under 1,024 queries grow theirs up to
// 4,096): the bound by the register-held bitwise selection, 16 keys per
// thread, rather than the shared-memory radix (threshold stage at one query
// and L = 256: 20.6 us against 22.8 us; 16 queries: 24.7 against 35.0 us)
#ifndef AH_THR_REG16
#define AH_THR_REG16 1
#endif

// One CTA per query, or `threshold_parts` CTAs per query for batches too
// small to fill the GPU: each scores an even share of the sample into the
// query's candidate buffer (unused until the scan) and the last to finish
// copies all the keys to its shared memory and selects.  Scores a sample of M = min(points, threshold_sample)
// slots of the query's best leaves (an even share of the S best, topped up in
// rank order); the R-th largest (score, id) key among them
// is a lower bound on the R-th largest over all its leaves (a subset's R-th
// best can only be lower), so every point of the final top R has a key >= it.
// With fewer than R points in total the bound is 0 (keep everything).
template <int MODE>
__global__ void __launch_bounds__(kSelThreads, 5) threshold_kernel(DeviceIndex ix, SearchArgs a, SearchBuffers b) {
    chain_entry();
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ SelectScratch scr;
    __shared__ RegSelectScratch<kSelThreads> rs;
    __shared__ int seg_end[kThresholdSegs], seg_pos[kThresholdSegs], seg_slot[kThresholdSegs];
    __shared__ float seg_off[kThresholdSegs];       // residual codes: the leaf's centroid score
    __shared__ int s_nseg, s_taken, s_last;
    const int parts = a.threshold_parts;
    const int q = blockIdx.x / parts, part = blockIdx.x - q * parts;
    const int R = a.R;
    // the table starts 256-byte aligned in the shared window (slot_values4's
    // byte-permute addressing); the launch adds 256 bytes for this
    unsigned char* lut = smem + ((256u - (static_cast<uint32_t>(__cvta_generic_to_shared(smem)) & 255u)) & 255u);
    uint64_t* vals = reinterpret_cast<uint64_t*>(lut + ((table_bytes(MODE, ix.B) + 15) & ~15));
    uint64_t* top = nullptr;
    load_query_table<MODE>(ix, b, q, lut);
    __syncthreads();
    const int M = threshold_sample(R, a.threshold_sample);
    // The sample as segments (leaf, first slot, count) in order: the first
    // M/S slots of each of the S best leaves, then the remaining slots of the
    // leaves in rank order until M.  One warp builds the table with prefix
    // sums; every thread then scores its sample indices in one pass, so a
    // sample that spans several small leaves costs no extra passes.  A table
    // that would exceed kThresholdSegs entries ends the sample early (a smaller
    // subset still gives a valid bound).
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        const int64_t lrow = static_cast<int64_t>(q) * a.L;
        const int S = max(1, min(a.L, a.threshold_leaves));
        const int per = M / S;
        int nseg = 0, taken = 0;
        bool full = false;
        // append this warp round's segments (cnt > 0) in lane order
        auto append = [&](int cnt, int leaf, int start) {
            int incl = cnt;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int v = __shfl_up_sync(0xFFFFFFFFu, incl, off);
                if (lane >= off) incl += v;
            }
            const unsigned m = __ballot_sync(0xFFFFFFFFu, cnt > 0);
            const int idx = nseg + __popc(m & ((1u << lane) - 1u));
            if (cnt > 0 && idx < kThresholdSegs) {
                seg_end[idx] = taken + incl;
                seg_pos[idx] = ix.ptile[leaf] * 32 + start;
                seg_slot[idx] = ix.offs[leaf] + start;
                seg_off[idx] = ix.residual ? b.cscore[static_cast<int64_t>(q) * ix.nl + leaf] : 0.0f;
            }
            const int total = __shfl_sync(0xFFFFFFFFu, incl, 31);
            const int n = __popc(m);
            if (nseg + n >= kThresholdSegs) {
                // the table is full: keep its first kThresholdSegs segments and
                // stop.  nseg < kThresholdSegs on entry (a full table ends both
                // loops), so some lane holds index kThresholdSegs - 1 here
                const unsigned lm = __ballot_sync(0xFFFFFFFFu, cnt > 0 && idx == kThresholdSegs - 1);
                taken += __shfl_sync(0xFFFFFFFFu, incl, __ffs(lm) - 1);   // end of the last kept segment
                nseg = kThresholdSegs;
                full = true;
            } else {
                taken += total;
                nseg += n;
            }
        };
        for (int i0 = 0; i0 < S && !full; i0 += 32) {
            const int i = i0 + lane;
            int cnt = 0, leaf = 0;
            if (i < S) {
                leaf = b.leaves[lrow + i];
                cnt = min(ix.offs[leaf + 1] - ix.offs[leaf], per);
            }
            append(cnt, leaf, 0);
        }
        for (int i0 = 0; i0 < a.L && taken < M && !full; i0 += 32) {
            const int i = i0 + lane;
            int avail = 0, leaf = 0, start = 0;
            if (i < a.L) {
                leaf = b.leaves[lrow + i];
                const int size = ix.offs[leaf + 1] - ix.offs[leaf];
                start = (i < S) ? min(size, per) : 0;
                avail = size - start;
            }
            int excl = avail;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int v = __shfl_up_sync(0xFFFFFFFFu, excl, off);
                if (lane >= off) excl += v;
            }
            excl -= avail;
            const int cnt = max(0, min(avail, M - taken - excl));
            append(cnt, leaf, start);
        }
        if (lane == 0) {
            s_nseg = nseg;
            s_taken = taken;
        }
    }
    __syncthreads();
    const int nseg = s_nseg, taken = s_taken;
    // this CTA's share of the sample; with several CTAs per query the keys
    // go to the query's candidate buffer (unused until the scan)
    const int i_begin = static_cast<int>(static_cast<int64_t>(taken) * part / parts);
    const int i_end = static_cast<int>(static_cast<int64_t>(taken) * (part + 1) / parts);
    uint64_t* gk = b.ckey + static_cast<int64_t>(q) * b.cap;
    for (int t0 = i_begin; t0 < i_end; t0 += 4 * kSelThreads) {
        int32_t ps[4], sid[4];
        bool ok[4];
        uint32_t v[4];
        float off4[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = t0 + u * kSelThreads + threadIdx.x;
            ok[u] = i < i_end;
            int lo = 0, hi = nseg - 1;                 // first segment whose end is above i
            while (lo < hi) {
                const int mid = (lo + hi) >> 1;
                if (seg_end[mid] > i) hi = mid; else lo = mid + 1;
            }
            const int off = i - (lo > 0 ? seg_end[lo - 1] : 0);
            ps[u] = seg_pos[lo] + off;
            sid[u] = ok[u] ? ix.slot_ids[seg_slot[lo] + off] : 0;
            off4[u] = seg_off[lo];
        }
        slot_values4<MODE>(ix.codes_il, ix.W, ix.V, ix.B, lut, ps, ok, ix.residual ? off4 : nullptr, v);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = t0 + u * kSelThreads + threadIdx.x;
            if (ok[u]) {
                const uint64_t key = make_key(v[u], sid[u]);
                if (parts == 1) vals[i] = key;
                else gk[i] = key;
            }
        }
    }
    if (parts > 1) {
        // the query's last CTA to finish selects from all parts' keys
        __threadfence();
        __syncthreads();
        if (threadIdx.x == 0) s_last = atomicAdd(&b.tdone[q], 1) == parts - 1;
        __syncthreads();
        if (!s_last) return;
        __threadfence();
        for (int i = threadIdx.x; i < taken; i += kSelThreads) vals[i] = __ldcg(gk + i);
    }
    __syncthreads();
    if (taken <= 4 * kSelThreads) {
        uint64_t tau = 0ull;
        if (taken >= R) {
            uint64_t kk[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int i = threadIdx.x + kSelThreads * j;
                kk[j] = (i < taken) ? vals[i] : 0ull;
            }
            tau = block_kth_reg<4, kSelThreads>(kk, taken, R, rs);
        }
        if (threadIdx.x == 0) b.tau[q] = tau;
    } else if (taken <= 8 * kSelThreads) {
        uint64_t tau = 0ull;
        if (taken >= R) {
            uint64_t kk[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int i = threadIdx.x + kSelThreads * j;
                kk[j] = (i < taken) ? vals[i] : 0ull;
            }
            tau = block_kth_reg<8, kSelThreads>(kk, taken, R, rs);
        }
        if (threadIdx.x == 0) b.tau[q] = tau;
    } else if (AH_THR_REG16 && taken <= 16 * kSelThreads) {
        uint64_t tau = 0ull;
        if (taken >= R) {
            uint64_t kk[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int i = threadIdx.x + kSelThreads * j;
                kk[j] = (i < taken) ? vals[i] : 0ull;
            }
            tau = block_kth_reg<16, kSelThreads>(kk, taken, R, rs);
        }
        if (threadIdx.x == 0) b.tau[q] = tau;
    } else {
        auto get = [&](int i) { return vals[i]; };
        uint64_t tau = 0ull;
        if (taken >= R) tau = block_kth_largest<kSelThreads>(get, taken, R, scr);
        if (threadIdx.x == 0) b.tau[q] = tau;
    }
    (void)top;
}

cudaError_t launch_threshold(const DeviceIndex& ix, const SearchArgs& a, const SearchBuffers& b, cudaStream_t s) {
    cudaError_t e;
    size_t smem = 256 + ((table_bytes(a.lut_mode, ix.B) + 15) & ~15) + static_cast<size_t>(threshold_sample(a.R, a.threshold_sample)) * sizeof(uint64_t);
    if (a.lut_mode == 0) {
        e = ensure_smem(reinterpret_cast<const void*>(threshold_kernel<0>), smem, true);
        if (e != cudaSuccess) return e;
        if (const cudaError_t le = launch_chained(threshold_kernel<0>, dim3(a.nq * a.threshold_parts), dim3(kSelThreads), smem, s, ix, a, b); le != cudaSuccess) return le;
    } else {
        e = ensure_smem(reinterpret_cast<const void*>(threshold_kernel<1>), smem, true);
        if (e != cudaSuccess) return e;
        if (const cudaError_t le = launch_chained(threshold_kernel<1>, dim3(a.nq * a.threshold_parts), dim3(kSelThreads), smem, s, ix, a, b); le != cudaSuccess) return le;
    }
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// the code scan (leaf-major)
// ---------------------------------------------------------------------------

// Does (value, id of slot) reach the bound (th, tl)?  The id is only read for
// an exact tie on the score part.
__device__ __forceinline__ bool reaches(uint32_t v, uint32_t th, uint32_t tl, const int32_t* __restrict__ slot_ids,
                                        int32_t slot) {
    if (v != th) return v > th;
    return (0xFFFFFFFFu - static_cast<uint32_t>(slot_ids[slot])) >= tl;
}

// Warp-aggregated append of the lanes with `pass` set to query q's buffer, as
// full (score key, id) keys.  Entries past the capacity are counted, not stored.
__device__ __forceinline__ void append_candidates(bool pass, uint32_t key, int32_t slot, int q, const DeviceIndex& ix,
                                                  const SearchBuffers& b) {
    const unsigned m = __ballot_sync(0xFFFFFFFFu, pass);
    if (m == 0u) return;
    const int lane = threadIdx.x & 31;
    const int leader = __ffs(m) - 1;
    int base = 0;
    if (lane == leader) base = atomicAdd(&b.count[q], __popc(m));
    base = __shfl_sync(0xFFFFFFFFu, base, leader);
    if (pass) {
        int pos = base + __popc(m & ((1u << lane) - 1u));
        if (pos < b.cap) {
            const int64_t o = static_cast<int64_t>(q) * b.cap + pos;
            b.ckey[o] = make_key(key, ix.slot_ids[slot]);
            b.cslot[o] = slot;
        }
    }
}

// Keep (value, slot) for query qi of the group when it reaches the query's
// bound.  Only the bound's score word is read for every slot: its id word is
// read when some lane ties it exactly, and the query index when some lane
// passes (both rare), each behind a warp vote so that no lane reads them
// otherwise.
__device__ __forceinline__ void keep_if_reaches(bool valid, uint32_t v, int32_t slot, int qi, const int* s_q,
                                                const uint32_t* s_th, const uint32_t* s_tl, const DeviceIndex& ix,
                                                const SearchBuffers& b) {
    const uint32_t th = s_th[qi];
    bool pass = valid && v >= th;
    const bool tie = pass && v == th;
    if (__any_sync(0xFFFFFFFFu, tie)) {
        const uint32_t tl = s_tl[qi];
        if (tie) pass = (0xFFFFFFFFu - static_cast<uint32_t>(ix.slot_ids[slot])) >= tl;
    }
    if (__any_sync(0xFFFFFFFFu, pass)) append_candidates(pass, v, slot, s_q[qi], ix, b);
}

// One code word (8 blocks) for a group of G queries, fp32 tables staged as
// [b][G/2][16] float2: per nibble one 8-byte shared load per query pair, one
// packed add.  `base` points at block 8w's tables.
template <int G>
__device__ __forceinline__ void f32_word(uint32_t c, const float2* __restrict__ base, float2 (&acc)[G / 2]) {
    constexpr int BS = (G / 2) * kCenters;   // float2 per block
#pragma unroll
    for (int nib = 0; nib < 8; ++nib) {
        const float2* p = base + nib * BS + ((c >> (4 * nib)) & 15u);
#pragma unroll
        for (int pr = 0; pr < G / 2; ++pr) acc[pr] = __fadd2_rn(acc[pr], p[pr * kCenters]);
    }
}

template <int G>
__device__ __forceinline__ void f32_tail(uint32_t c, int nb, const float2* __restrict__ base, float2 (&acc)[G / 2]) {
    constexpr int BS = (G / 2) * kCenters;
    for (int nib = 0; nib < nb; ++nib) {
        const float2* p = base + nib * BS + ((c >> (4 * nib)) & 15u);
#pragma unroll
        for (int pr = 0; pr < G / 2; ++pr) acc[pr] = __fadd2_rn(acc[pr], p[pr * kCenters]);
    }
}

// uint8 tables, two staged layouts.
// SPLIT: [b][G/4][16] word pairs: for a quad of queries the entry's four bytes
// already spread into two words of 16-bit lanes (queries 4d+0/4d+2 in .x,
// 4d+1/4d+3 in .y), so a nibble costs one 8-byte load and two adds per quad;
// 16 entries x 8 B of a (block, quad) cover the 32 banks once (one wavefront
// per half-warp).  Used when a group's tables stay within 64 KB (B <= 256).
// Packed: [b][G/4][16] words (4 queries' bytes per word), spread into the
// 16-bit lanes after the load (mask and byte permute): half the shared memory,
// for wider tables.  Both accumulate queries 4d+0/4d+2 in ae and 4d+1/4d+3 in ao.
template <bool SPLIT>
struct U8Layout {
    using Entry = uint32_t;
    __device__ __forceinline__ static void add(const Entry* p, uint32_t& ae, uint32_t& ao) {
        const uint32_t v = *p;
        ae += v & 0x00FF00FFu;
        ao += __byte_perm(v, 0u, 0x4341);
    }
    __device__ __forceinline__ static Entry make(const uint32_t (&v)[4]) {
        return v[0] | (v[1] << 8) | (v[2] << 16) | (v[3] << 24);
    }
};
template <>
struct U8Layout<true> {
    using Entry = uint2;
    __device__ __forceinline__ static void add(const Entry* p, uint32_t& ae, uint32_t& ao) {
        const uint2 v = *p;
        ae += v.x;
        ao += v.y;
    }
    __device__ __forceinline__ static Entry make(const uint32_t (&v)[4]) {
        return make_uint2(v[0] | (v[2] << 16), v[1] | (v[3] << 16));
    }
};

// One code word (up to 8 blocks) for a group of G queries, uint8 tables.
// xw: shared address of the word's first block's entries, a multiple of 256
// (the staged tables start 256-byte aligned and a word's blocks span a
// multiple of 256 bytes), so an entry's address is xw with its low byte
// replaced by the nibble's byte offset (nibble x entry size < 256): one byte
// permute per nibble, the block and quad offsets folding into the loads.
template <int G, bool SPLIT>
__device__ __forceinline__ void u8_nibbles(uint32_t c, int nb, uint32_t xw, uint32_t (&ae)[G / 4],
                                           uint32_t (&ao)[G / 4]) {
    using Entry = typename U8Layout<SPLIT>::Entry;
    constexpr int E = static_cast<int>(sizeof(Entry));
    constexpr int BSB = (G / 4) * kCenters * E;   // bytes per block
    constexpr int SH = E == 8 ? 3 : 2;
    // byte offsets of the word's entries: nibbles 0, 2, 4, 6 in the bytes of
    // ev, 1, 3, 5, 7 in those of od
    const uint32_t ev = (c & 0x0F0F0F0Fu) << SH, od = ((c >> 4) & 0x0F0F0F0Fu) << SH;
    if (SPLIT) {
#pragma unroll
        for (int nib = 0; nib < 8; ++nib) {
            if (nib < nb) {
                const uint32_t p = __byte_perm((nib & 1) ? od : ev, xw, 0x7650u | (nib >> 1)) + nib * BSB;
#pragma unroll
                for (int qd = 0; qd < G / 4; ++qd) {
                    const uint2 v = lds_u64(p + qd * kCenters * E);
                    ae[qd] += v.x;
                    ao[qd] += v.y;
                }
            }
        }
    } else {
        // packed words: nibbles in pairs, so each 16-bit-lane accumulator
        // takes both nibbles' halves in one three-input add (the integer
        // pipe, at half the issue rate, bounds this loop)
#pragma unroll
        for (int n2 = 0; n2 < 8; n2 += 2) {
            if (n2 < nb) {
                const bool second = n2 + 1 < nb;
                const uint32_t p0 = __byte_perm(ev, xw, 0x7650u | (n2 >> 1)) + n2 * BSB;
                const uint32_t p1 = __byte_perm(od, xw, 0x7650u | (n2 >> 1)) + (n2 + 1) * BSB;
#pragma unroll
                for (int qd = 0; qd < G / 4; ++qd) {
                    const uint32_t v0 = lds_u32(p0 + qd * kCenters * E);
                    const uint32_t v1 = second ? lds_u32(p1 + qd * kCenters * E) : 0u;
                    ae[qd] += (v0 & 0x00FF00FFu) + (v1 & 0x00FF00FFu);
                    ao[qd] += __byte_perm(v0, 0u, 0x4341) + __byte_perm(v1, 0u, 0x4341);
                }
            }
        }
    }
}

template <int G>
__device__ __forceinline__ void u8_flush(uint32_t (&sums)[G], uint32_t (&ae)[G / 4], uint32_t (&ao)[G / 4]) {
#pragma unroll
    for (int qd = 0; qd < G / 4; ++qd) {
        sums[4 * qd + 0] += ae[qd] & 0xFFFFu;
        sums[4 * qd + 2] += ae[qd] >> 16;
        sums[4 * qd + 1] += ao[qd] & 0xFFFFu;
        sums[4 * qd + 3] += ao[qd] >> 16;
        ae[qd] = 0u;
        ao[qd] = 0u;
    }
}

// Shared-memory bytes per (query, block, center) of the scan's staged tables:
// fp32 4; uint8 2 (each quad's bytes spread into 16-bit lanes) or 1.
__host__ __device__ __forceinline__ int scan_entry_bytes(int mode, bool split) { return mode == 0 ? 4 : (split ? 2 : 1); }
// uint8 tables use the split layout when a group of 8 queries' tables stays
// within AH_U8_SPLIT_BYTES that way
#ifndef AH_U8_SPLIT_BYTES
#define AH_U8_SPLIT_BYTES (64 * 1024)
#endif
// uint8 tables of up to 100 KB per group of 8 (256 < B <= 400) in the split
// layout too, as two 512-thread CTAs per SM with groups kept at 8 (the
// OpenAI-shaped uint8 step: 15.14 ms against 15.61 ms with packed words)
#ifndef AH_U8_WIDE_SPLIT
#define AH_U8_WIDE_SPLIT 1
#endif
__host__ __device__ __forceinline__ bool u8_wide_split(int B) {
    return AH_U8_WIDE_SPLIT && B * kCenters * 2 * kGroupU8 > AH_U8_SPLIT_BYTES && B * kCenters * 2 * kGroupU8 <= 100 * 1024;
}
__host__ __device__ __forceinline__ bool u8_split(int B) {
    return B * kCenters * 2 * kGroupU8 <= AH_U8_SPLIT_BYTES || u8_wide_split(B);
}

struct TileJob {
    int t0, t1;          // code tiles [t0, t1) of one leaf
    int slot_base;       // slot of lane 0 of tile t is slot_base + 32 t
    int send;            // first slot past the leaf
    int gsize;           // real queries in the group (<= G)
};

// The warps of a CTA split the item's tiles; a lane owns one slot.  Blocks are
// summed in order 0..B-1 with IEEE fp32 adds (two queries per packed add), the
// order every kernel that scores a slot uses.
template <int G, int NT, bool RES>
__device__ __forceinline__ void scan_tiles_f32(const DeviceIndex& ix, const SearchBuffers& b, const unsigned char* smem,
                                               const TileJob& job, const int* s_q, const uint32_t* s_th,
                                               const uint32_t* s_tl, const float* s_off) {
    constexpr int BS = (G / 2) * kCenters;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int W = ix.W, V = ix.V, Wf = ix.B >> 3, tail = ix.B & 7;
    const float2* lut2 = reinterpret_cast<const float2*>(smem);
    for (int t = job.t0 + warp; t < job.t1; t += NT / 32) {
        const int slot = job.slot_base + 32 * t + lane;
        const bool valid = slot < job.send;
        const uint32_t* tw = ix.codes_il + static_cast<int64_t>(t) * W * 32;
        float2 acc[G / 2];
#pragma unroll
        for (int pr = 0; pr < G / 2; ++pr) acc[pr] = make_float2(0.0f, 0.0f);
        int w = 0;
        for (; w + 4 <= Wf; w += 4) {
            uint32_t c0, c1, c2, c3;
            code_words4(tw, lane, w, V, c0, c1, c2, c3);
            f32_word<G>(c0, lut2 + (8 * w + 0) * BS, acc);
            f32_word<G>(c1, lut2 + (8 * w + 8) * BS, acc);
            f32_word<G>(c2, lut2 + (8 * w + 16) * BS, acc);
            f32_word<G>(c3, lut2 + (8 * w + 24) * BS, acc);
        }
        for (; w < Wf; ++w) f32_word<G>(tw[code_word(w, lane, V)], lut2 + 8 * w * BS, acc);
        if (tail) f32_tail<G>(tw[code_word(Wf, lane, V)], tail, lut2 + 8 * Wf * BS, acc);
#pragma unroll
        for (int qi = 0; qi < G; ++qi) {
            if (qi < job.gsize) {
                const float sum = (qi & 1) ? acc[qi >> 1].y : acc[qi >> 1].x;
                const float sc = RES ? __fadd_rn(sum, s_off[qi]) : sum;
                const uint32_t key = float_key(sc);
                keep_if_reaches(valid, key, slot, qi, s_q, s_th, s_tl, ix, b);
            }
        }
    }
}

template <int G, int NT, bool SPLIT>
__device__ __forceinline__ void scan_tiles_u8(const DeviceIndex& ix, const SearchBuffers& b, const unsigned char* smem,
                                              const TileJob& job, const int* s_q, const uint32_t* s_th,
                                              const uint32_t* s_tl) {
    // bytes of one word's 8 blocks of entries (a multiple of 256)
    constexpr uint32_t WB = 8u * (G / 4) * kCenters * static_cast<uint32_t>(sizeof(typename U8Layout<SPLIT>::Entry));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int W = ix.W, V = ix.V, Wf = ix.B >> 3, tail = ix.B & 7;
    const uint32_t tbase = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    for (int t = job.t0 + warp; t < job.t1; t += NT / 32) {
        const int slot = job.slot_base + 32 * t + lane;
        const bool valid = slot < job.send;
        const uint32_t* tw = ix.codes_il + static_cast<int64_t>(t) * W * 32;
        uint32_t sums[G];
        uint32_t ae[G / 4], ao[G / 4];
#pragma unroll
        for (int qi = 0; qi < G; ++qi) sums[qi] = 0u;
#pragma unroll
        for (int qd = 0; qd < G / 4; ++qd) { ae[qd] = 0u; ao[qd] = 0u; }
        // 16-bit lanes hold 256 blocks of 255: flush every 32 words
        for (int w0 = 0; w0 < Wf; w0 += 32) {
            const int wend = min(Wf, w0 + 32);
            int w = w0;
            for (; w + 4 <= wend; w += 4) {
                uint32_t c0, c1, c2, c3;
                code_words4(tw, lane, w, V, c0, c1, c2, c3);
                const uint32_t xw = tbase + w * WB;
                u8_nibbles<G, SPLIT>(c0, 8, xw, ae, ao);
                u8_nibbles<G, SPLIT>(c1, 8, xw + WB, ae, ao);
                u8_nibbles<G, SPLIT>(c2, 8, xw + 2 * WB, ae, ao);
                u8_nibbles<G, SPLIT>(c3, 8, xw + 3 * WB, ae, ao);
            }
            for (; w < wend; ++w) u8_nibbles<G, SPLIT>(tw[code_word(w, lane, V)], 8, tbase + w * WB, ae, ao);
            u8_flush<G>(sums, ae, ao);
        }
        if (tail) {
            u8_nibbles<G, SPLIT>(tw[code_word(Wf, lane, V)], tail, tbase + Wf * WB, ae, ao);
            u8_flush<G>(sums, ae, ao);
        }
#pragma unroll
        for (int qi = 0; qi < G; ++qi) {
            if (qi < job.gsize)
                keep_if_reaches(valid, sums[qi], slot, qi, s_q, s_th, s_tl, ix, b);
        }
    }
}

// A group of one query (common when queries seldom share a leaf: small
// batches, or many leaves): its table staged once, entries twice as for the
// query-major kernels (fp32 [b][16][2], uint8 [b][16]), so each lookup is
// useful and a warp's 32 lookups take one wavefront, instead of padding the
// group to a pair (fp32) or a quad (uint8).  Blocks are summed in order.
template <int NT, bool RES>
__device__ __forceinline__ void scan_tiles_f32_single(const DeviceIndex& ix, const SearchBuffers& b,
                                                      const unsigned char* smem, const TileJob& job, const int* s_q,
                                                      const uint32_t* s_th, const uint32_t* s_tl, const float* s_off) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int W = ix.W, V = ix.V, Wf = ix.B >> 3, tail = ix.B & 7;
    const float* lut1 = reinterpret_cast<const float*>(smem) + ((lane >> 4) & 1);
    auto word = [&](uint32_t c, int nb, const float* base, float& acc) {
#pragma unroll
        for (int nib = 0; nib < 8; ++nib)
            if (nib < nb) acc = __fadd_rn(acc, base[2 * (nib * kCenters + ((c >> (4 * nib)) & 15u))]);
    };
    for (int t = job.t0 + warp; t < job.t1; t += NT / 32) {
        const int slot = job.slot_base + 32 * t + lane;
        const bool valid = slot < job.send;
        const uint32_t* tw = ix.codes_il + static_cast<int64_t>(t) * W * 32;
        float acc = 0.0f;
        int w = 0;
        for (; w + 4 <= Wf; w += 4) {
            uint32_t c0, c1, c2, c3;
            code_words4(tw, lane, w, V, c0, c1, c2, c3);
            word(c0, 8, lut1 + 2 * (8 * w + 0) * kCenters, acc);
            word(c1, 8, lut1 + 2 * (8 * w + 8) * kCenters, acc);
            word(c2, 8, lut1 + 2 * (8 * w + 16) * kCenters, acc);
            word(c3, 8, lut1 + 2 * (8 * w + 24) * kCenters, acc);
        }
        for (; w < Wf; ++w) word(tw[code_word(w, lane, V)], 8, lut1 + 2 * 8 * w * kCenters, acc);
        if (tail) word(tw[code_word(Wf, lane, V)], tail, lut1 + 2 * 8 * Wf * kCenters, acc);
        const float sc = RES ? __fadd_rn(acc, s_off[0]) : acc;
        keep_if_reaches(valid, float_key(sc), slot, 0, s_q, s_th, s_tl, ix, b);
    }
}

template <int NT>
__device__ __forceinline__ void scan_tiles_u8_single(const DeviceIndex& ix, const SearchBuffers& b,
                                                     const unsigned char* smem, const TileJob& job, const int* s_q,
                                                     const uint32_t* s_th, const uint32_t* s_tl) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int W = ix.W, V = ix.V, Wf = ix.B >> 3, tail = ix.B & 7;
    auto word = [&](uint32_t c, int nb, const unsigned char* base, uint32_t& acc) {
#pragma unroll
        for (int nib = 0; nib < 8; ++nib)
            if (nib < nb) acc += base[nib * kCenters + ((c >> (4 * nib)) & 15u)];
    };
    for (int t = job.t0 + warp; t < job.t1; t += NT / 32) {
        const int slot = job.slot_base + 32 * t + lane;
        const bool valid = slot < job.send;
        const uint32_t* tw = ix.codes_il + static_cast<int64_t>(t) * W * 32;
        uint32_t acc = 0u;
        int w = 0;
        for (; w + 4 <= Wf; w += 4) {
            uint32_t c0, c1, c2, c3;
            code_words4(tw, lane, w, V, c0, c1, c2, c3);
            word(c0, 8, smem + (8 * w + 0) * kCenters, acc);
            word(c1, 8, smem + (8 * w + 8) * kCenters, acc);
            word(c2, 8, smem + (8 * w + 16) * kCenters, acc);
            word(c3, 8, smem + (8 * w + 24) * kCenters, acc);
        }
        for (; w < Wf; ++w) word(tw[code_word(w, lane, V)], 8, smem + 8 * w * kCenters, acc);
        if (tail) word(tw[code_word(Wf, lane, V)], tail, smem + 8 * Wf * kCenters, acc);
        keep_if_reaches(valid, acc, slot, 0, s_q, s_th, s_tl, ix, b);
    }
}

// Persistent CTAs take work items (leaf, query group, chunk of code tiles) from
// an atomic counter.  A leaf's m queries form groups of GMAX, then one group of
// the remainder rounded up to GSTEP (a lone query stays a group of one), so
// at most GSTEP-1 table slots of a leaf are padding.  Per item the group's
// tables are staged in shared memory (fp32 pair-interleaved, uint8
// quad-interleaved and spread into 16-bit lanes) and the warps scan the
// chunk's tiles.  Only a leaf's last tile is partial (leaf-padded code copy).
#ifndef AH_SCAN_MIN_BLOCKS
#define AH_SCAN_MIN_BLOCKS 6
#endif
// uint8 scan: 5 CTAs per SM (48 registers: groups of 8 queries keep 12
// accumulator registers per lane plus 8-byte table loads; at 40 the compiler
// spills)
#ifndef AH_SCAN_MIN_BLOCKS_U8
#define AH_SCAN_MIN_BLOCKS_U8 5
#endif

// RES: residual codes (each query's centroid score of the leaf is added to its
// sums); a separate instantiation so plain indexes pay nothing for it.
template <int MODE, int NT, int GMAX, bool RES, bool SPLIT>
__global__ void __launch_bounds__(NT, (NT == 256 ? (MODE == 0 ? AH_SCAN_MIN_BLOCKS : AH_SCAN_MIN_BLOCKS_U8)
                                                 : (NT == 512 ? 2 : 1)))
    scan_kernel(DeviceIndex ix, SearchArgs a, SearchBuffers b) {
    chain_entry();
    constexpr int GSTEP = (MODE == 0) ? 2 : 4;
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ int s_item, s_leaf;
    __shared__ int s_q[GMAX];
    __shared__ uint32_t s_th[GMAX], s_tl[GMAX];
    __shared__ float s_off[GMAX];            // residual codes: each query's score of this leaf
    const int B = ix.B;
    const int total_items = b.item_off[ix.nl];
    const size_t lut_bytes = static_cast<size_t>(B) * GMAX * kCenters * scan_entry_bytes(MODE, SPLIT);
    // uint8 tables start 256-byte aligned in the shared window (u8_nibbles
    // builds entry addresses by replacing an address's low byte); the launch
    // adds 256 bytes for this
    unsigned char* tsm = smem;
    if (MODE == 1) tsm += (256u - (static_cast<uint32_t>(__cvta_generic_to_shared(smem)) & 255u)) & 255u;
    int* s_item_off = reinterpret_cast<int*>(tsm + lut_bytes);
    const bool off_in_smem = a.scan_item_off_smem != 0;
    if (off_in_smem)
        for (int i = threadIdx.x; i <= ix.nl; i += NT) s_item_off[i] = b.item_off[i];
    const int* item_off = off_in_smem ? s_item_off : b.item_off;

    // 256-thread form (short items): the next item's index is claimed while
    // the current one is scanned, so the atomic's latency is hidden (thread 0
    // holds it in `next`).  The wide forms' items are long; they claim items
    // as they go (the extra register would spill there).
    constexpr bool kPrefetch = NT == 256;
    int next = 0;
    if (kPrefetch && threadIdx.x == 0) next = atomicAdd(&b.counters[a.scan_counter], 1);
    for (;;) {
        __syncthreads();   // previous item's tables are no longer read
        if (threadIdx.x == 0) {
            const int item = kPrefetch ? next : atomicAdd(&b.counters[a.scan_counter], 1);
            s_item = item;
            if (item < total_items) {
                int lo = 0, hi = ix.nl;
                while (lo < hi) {
                    int mid = (lo + hi + 1) >> 1;
                    if (item_off[mid] <= item) lo = mid; else hi = mid - 1;
                }
                s_leaf = lo;
            }
        }
        __syncthreads();
        const int item = s_item;
        if (item >= total_items) break;
        if (kPrefetch && threadIdx.x == 0) next = atomicAdd(&b.counters[a.scan_counter], 1);
        const int leaf = s_leaf;
        const int pt0 = ix.ptile[leaf], ntile = ix.ptile[leaf + 1] - pt0;
        const int npc = (ntile + a.chunk - 1) / a.chunk;
        const int local = item - item_off[leaf];
        const int g = local / npc, c = local - g * npc;
        const int qcnt = b.qcount[leaf];
        TileJob job;
        job.gsize = min(GMAX, qcnt - g * GMAX);
        // table width of this group (a lone query is not padded)
        const int G = job.gsize == 1 ? 1 : ((job.gsize + GSTEP - 1) / GSTEP) * GSTEP;
        job.t0 = pt0 + c * a.chunk;
        job.t1 = min(pt0 + ntile, job.t0 + a.chunk);
        job.slot_base = ix.offs[leaf] - 32 * pt0;
        job.send = ix.offs[leaf + 1];
        if (threadIdx.x < GMAX) {
            int qq = (threadIdx.x < job.gsize) ? b.qlist[b.qoff[leaf] + g * GMAX + threadIdx.x] : -1;
            s_q[threadIdx.x] = qq;
            uint64_t t = (qq >= 0) ? b.tau[qq] : ~0ull;
            s_th[threadIdx.x] = static_cast<uint32_t>(t >> 32);
            s_tl[threadIdx.x] = static_cast<uint32_t>(t);
            if (RES) s_off[threadIdx.x] = (qq >= 0) ? b.cscore[static_cast<int64_t>(qq) * ix.nl + leaf] : 0.0f;
        }
        __syncthreads();
        // stage the group's tables
        const int per_q = B * kCenters;
        if (G == 1) {
            const int q0 = s_q[0];
            if (MODE == 0) {
                float2* lf = reinterpret_cast<float2*>(smem);
                const float* src = b.lut_f32 + static_cast<int64_t>(q0) * per_q;
                for (int r = threadIdx.x; r < per_q; r += NT) lf[r] = make_float2(src[r], src[r]);
            } else {
                const uint8_t* src = b.lut_u8 + static_cast<int64_t>(q0) * per_q;
                for (int r = threadIdx.x; r < per_q; r += NT) tsm[r] = src[r];
            }
        } else if (MODE == 0) {
            // one 8-byte store per (block, center) of each query pair
            float2* lf = reinterpret_cast<float2*>(smem);
            const int half = G / 2;
            for (int pr = 0; pr < half; ++pr) {
                const int qa = s_q[2 * pr], qb = s_q[2 * pr + 1];
                const float* la = b.lut_f32 + static_cast<int64_t>(qa < 0 ? 0 : qa) * per_q;
                const float* lb = b.lut_f32 + static_cast<int64_t>(qb < 0 ? 0 : qb) * per_q;
                for (int r = threadIdx.x; r < per_q; r += NT) {
                    const float va = (qa >= 0) ? la[r] : 0.0f;
                    const float vb = (qb >= 0) ? lb[r] : 0.0f;
                    lf[((r >> 4) * half + pr) * kCenters + (r & 15)] = make_float2(va, vb);
                }
            }
        } else {
            // one store per (block, center) of each query quad
            auto* lw = reinterpret_cast<typename U8Layout<SPLIT>::Entry*>(tsm);
            const int quads = G / 4;
            for (int qd = 0; qd < quads; ++qd) {
                const uint8_t* src[4];
                bool ok[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int qq = s_q[4 * qd + u];
                    ok[u] = qq >= 0;
                    src[u] = b.lut_u8 + static_cast<int64_t>(ok[u] ? qq : 0) * per_q;
                }
                for (int r = threadIdx.x; r < per_q; r += NT) {
                    uint32_t v[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) v[u] = ok[u] ? static_cast<uint32_t>(src[u][r]) : 0u;
                    lw[((r >> 4) * quads + qd) * kCenters + (r & 15)] = U8Layout<SPLIT>::make(v);
                }
            }
        }
        __syncthreads();
        if (G == 1) {
            if (MODE == 0) scan_tiles_f32_single<NT, RES>(ix, b, smem, job, s_q, s_th, s_tl, s_off);
            else scan_tiles_u8_single<NT>(ix, b, tsm, job, s_q, s_th, s_tl);
        } else if (MODE == 0) {
            switch (G) {
                case 8: scan_tiles_f32<8, NT, RES>(ix, b, smem, job, s_q, s_th, s_tl, s_off); break;
                case 6: scan_tiles_f32<6, NT, RES>(ix, b, smem, job, s_q, s_th, s_tl, s_off); break;
                case 4: scan_tiles_f32<4, NT, RES>(ix, b, smem, job, s_q, s_th, s_tl, s_off); break;
                default: scan_tiles_f32<2, NT, RES>(ix, b, smem, job, s_q, s_th, s_tl, s_off); break;
            }
        } else {
            if (GMAX >= 8 && G == 8) scan_tiles_u8<(GMAX >= 8 ? 8 : 4), NT, SPLIT>(ix, b, tsm, job, s_q, s_th, s_tl);
            else scan_tiles_u8<4, NT, SPLIT>(ix, b, tsm, job, s_q, s_th, s_tl);
        }
    }
}

// Scan CTA shape: threads per CTA and queries per group.  Narrow tables
// (a full group's tables within 64 KB): 256 threads, groups of 8 queries
// (fp32 and uint8), several CTAs per SM.  Wide tables (half a group within
// 100 KB): two CTAs of 512 threads per SM with half-size groups, so one
// CTA's table staging and item-end barrier overlap the other's scanning.
// Wider tables: one CTA of 1,024 threads, fp32 groups of 8 (B 401-452; the
// search refuses fp32 tables beyond that), uint8 groups of 4.
#ifndef AH_WIDE_SPLIT
#define AH_WIDE_SPLIT 1
#endif
void scan_shape(const DeviceIndex& ix, int lut_mode, int* nt, int* gmax) {
    const int g = lut_mode == 0 ? kGroupF32 : kGroupU8;
    const size_t table = static_cast<size_t>(ix.B) * kCenters * scan_entry_bytes(lut_mode, u8_split(ix.B)) * g;
    if (lut_mode == 1 && u8_wide_split(ix.B)) {
        *nt = 512;
        *gmax = g;
    } else if (table <= 64 * 1024) {
        *nt = 256;
        *gmax = g;
    } else if (AH_WIDE_SPLIT && table / 2 <= 100 * 1024) {
        *nt = 512;
        *gmax = g / 2;
    } else {
        // one CTA of 1,024 threads per SM: fp32 groups of 8 (B <= 452);
        // uint8 groups of 4, which fit every B up to AH_MAX_BLOCKS
        *nt = 1024;
        *gmax = lut_mode == 0 ? g : g / 2;
    }
}

int scan_group(const DeviceIndex& ix, int lut_mode) {
    int nt, g;
    scan_shape(ix, lut_mode, &nt, &g);
    return g;
}

size_t scan_table_bytes(const DeviceIndex& ix, int lut_mode) {
    int nt, g;
    scan_shape(ix, lut_mode, &nt, &g);
    return static_cast<size_t>(ix.B) * g * kCenters * scan_entry_bytes(lut_mode, u8_split(ix.B)) + (lut_mode == 1 ? 256 : 0);
}

template <int MODE, int NT, int GMAX, bool RES, bool SPLIT = false>
static cudaError_t launch_scan_t(const DeviceIndex& ix, SearchArgs a, const SearchBuffers& b, int num_sms,
                                 cudaStream_t s) {
    size_t smem = static_cast<size_t>(ix.B) * GMAX * kCenters * scan_entry_bytes(MODE, SPLIT) + (MODE == 1 ? 256 : 0);
    const size_t off_bytes = static_cast<size_t>(ix.nl + 1) * sizeof(int);
    const size_t room = (NT == 512) ? 110 * 1024 : 200 * 1024;
    a.scan_item_off_smem = (smem + off_bytes <= room && off_bytes <= 64 * 1024) ? 1 : 0;
    if (a.scan_item_off_smem) smem += off_bytes;
    cudaError_t e = ensure_smem(reinterpret_cast<const void*>(scan_kernel<MODE, NT, GMAX, RES, SPLIT>), smem, true);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, scan_kernel<MODE, NT, GMAX, RES, SPLIT>, NT, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    if (const cudaError_t le = launch_chained(scan_kernel<MODE, NT, GMAX, RES, SPLIT>, dim3(num_sms * per_sm), dim3(NT), smem, s, ix, a, b); le != cudaSuccess) return le;
    return cudaGetLastError();
}

cudaError_t launch_scan(const DeviceIndex& ix, const SearchArgs& a, const SearchBuffers& b, int num_sms, cudaStream_t s) {
    if (a.scan_tc) return launch_scan_tc(ix, a, b, num_sms, s);
    int nt, g;
    scan_shape(ix, a.lut_mode, &nt, &g);
    if (a.lut_mode == 0) {
        if (ix.residual) {
            if (nt == 256) return launch_scan_t<0, 256, kGroupF32, true>(ix, a, b, num_sms, s);
            if (nt == 512) return launch_scan_t<0, 512, kGroupF32 / 2, true>(ix, a, b, num_sms, s);
            return launch_scan_t<0, 1024, kGroupF32, true>(ix, a, b, num_sms, s);
        }
        if (nt == 256) return launch_scan_t<0, 256, kGroupF32, false>(ix, a, b, num_sms, s);
        if (nt == 512) return launch_scan_t<0, 512, kGroupF32 / 2, false>(ix, a, b, num_sms, s);
        return launch_scan_t<0, 1024, kGroupF32, false>(ix, a, b, num_sms, s);
    }
    // uint8 tables are refused for residual codes before any launch
    if (u8_split(ix.B)) {
        if (nt == 512) return launch_scan_t<1, 512, kGroupU8, false, true>(ix, a, b, num_sms, s);
        return launch_scan_t<1, 256, kGroupU8, false, true>(ix, a, b, num_sms, s);
    }
    if (nt == 256) return launch_scan_t<1, 256, kGroupU8, false>(ix, a, b, num_sms, s);
    if (nt == 512) return launch_scan_t<1, 512, kGroupU8 / 2, false>(ix, a, b, num_sms, s);
    return launch_scan_t<1, 1024, kGroupU8 / 2, false>(ix, a, b, num_sms, s);
}

// ---------------------------------------------------------------------------
// the code scan (query-major, for batches whose queries seldom share a leaf)
// ---------------------------------------------------------------------------

// The leaf-major scan forms groups per leaf; when queries seldom share a leaf
// nearly every group is a lone query whose table is staged again for every
// item.  Here CTA (q, part) takes an even share of query q's code tiles over
// its leaf ranks [r0, r1): the table is staged once, each leaf rank's tile
// count, first tile, slot range and (residual codes) centroid score are held
// in shared memory, and each warp scans two tiles at a time so that two
// tiles' code loads are in flight together.  The sums run over blocks in
// order, as in every other kernel that scores a slot.
// The table starts 256-byte aligned in the shared window and a block's 16
// entries take 64 bytes (fp32) or 32 bytes (uint8: 16 bytes and 16 of
// padding), so a code word's 8 blocks span a multiple of 256 bytes and each
// lookup's address is one byte permute of the word's address.

__host__ __device__ __forceinline__ size_t qscan_table_bytes(int mode, int B) {
    return 256 + static_cast<size_t>(B) * (mode == 0 ? kCenters * 4 : 32);
}

size_t scan_query_smem_bytes(int mode, int B, int leaves) {
    return qscan_table_bytes(mode, B) + sizeof(int32_t) * (5 * static_cast<size_t>(leaves) + 1);
}

// All W <= 8 code words of one lane's slot in a tile, V words per load (V
// divides W), zero past W: one round of loads for the whole tile.
template <int V>
__device__ __forceinline__ void tile_words8(const uint32_t* __restrict__ tw, int lane, int W, uint32_t (&cw)[8]) {
#pragma unroll
    for (int w = 0; w < 8; w += V) {
        if (w < W) {
            if (V == 4) {
                const uint4 v = *reinterpret_cast<const uint4*>(tw + w * 32 + lane * 4);
                cw[w] = v.x; cw[w + 1] = v.y; cw[w + 2] = v.z; cw[w + 3] = v.w;
            } else if (V == 2) {
                const uint2 v = *reinterpret_cast<const uint2*>(tw + w * 32 + lane * 2);
                cw[w] = v.x; cw[w + 1] = v.y;
            } else {
                cw[w] = tw[w * 32 + lane];
            }
        } else {
#pragma unroll
            for (int j = 0; j < V; ++j) cw[w + j] = 0u;
        }
    }
}

// VW: the code copy's words per vector load (ix.V), fixed per instantiation so
// the per-word index arithmetic folds (each word feeds only 8 lookups here).
template <int MODE, bool RES, int VW>
__global__ void __launch_bounds__(kQScanThreads) scan_query_kernel(DeviceIndex ix, SearchArgs a, SearchBuffers b,
                                                                   int r0, int r1, int parts) {
    chain_entry();
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ int s_q[1];
    __shared__ uint32_t s_th[1], s_tl[1];
    constexpr int NW = kQScanThreads / 32;
    const int q = blockIdx.x / parts, part = blockIdx.x - q * parts;
    const int nL = r1 - r0;
    const int B = ix.B, per_q = B * kCenters;
    unsigned char* tsm = smem + ((256u - (static_cast<uint32_t>(__cvta_generic_to_shared(smem)) & 255u)) & 255u);
    const uint32_t tbase = static_cast<uint32_t>(__cvta_generic_to_shared(tsm));
    int* s_pre = reinterpret_cast<int*>(smem + qscan_table_bytes(MODE, B));   // [nL + 1] tiles before rank i
    int* s_pt = s_pre + nL + 1;                                               // first tile of the rank's leaf
    int* s_os = s_pt + nL;                                                    // its first slot
    int* s_oe = s_os + nL;                                                    // one past its last slot
    float* s_lo = reinterpret_cast<float*>(s_oe + nL);                        // the query's score of the leaf
    if (MODE == 0) {
        float* lf = reinterpret_cast<float*>(tsm);
        const float* src = b.lut_f32 + static_cast<int64_t>(q) * per_q;
        for (int r = threadIdx.x; r < per_q; r += kQScanThreads) lf[r] = src[r];
    } else {
        const uint8_t* src = b.lut_u8 + static_cast<int64_t>(q) * per_q;
        for (int r = threadIdx.x; r < per_q; r += kQScanThreads) tsm[(r >> 4) * 32 + (r & 15)] = src[r];
    }
    // tile counts per leaf rank, and their prefix sums: every thread takes
    // ranks tid, tid + 256, ... (one round of loads for up to 256 ranks), then
    // warp scans and one pass over the warp totals per round
    __shared__ int s_wsum[kQScanThreads / 32];
    {
        const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
        int carry = 0;
        for (int i0 = 0; i0 < nL; i0 += kQScanThreads) {
            const int i = i0 + threadIdx.x;
            int cnt = 0;
            if (i < nL) {
                const int leaf = b.leaves[static_cast<int64_t>(q) * a.L + r0 + i];
                const int pt = ix.ptile[leaf];
                cnt = ix.ptile[leaf + 1] - pt;
                s_pt[i] = pt;
                s_os[i] = ix.offs[leaf];
                s_oe[i] = ix.offs[leaf + 1];
                if (RES) s_lo[i] = b.cscore[static_cast<int64_t>(q) * ix.nl + leaf];
            }
            int incl = cnt;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int v = __shfl_up_sync(0xFFFFFFFFu, incl, off);
                if (lane >= off) incl += v;
            }
            if (lane == 31) s_wsum[wid] = incl;
            __syncthreads();
            int before = carry, all = 0;
#pragma unroll
            for (int w2 = 0; w2 < kQScanThreads / 32; ++w2) {
                const int ws = s_wsum[w2];
                before += (w2 < wid) ? ws : 0;
                all += ws;
            }
            if (i < nL) s_pre[i + 1] = before + incl;
            carry += all;
            __syncthreads();                   // s_wsum is rewritten next round
        }
        if (threadIdx.x == 0) {
            s_pre[0] = 0;
            s_q[0] = q;
            const uint64_t t = b.tau[q];
            s_th[0] = static_cast<uint32_t>(t >> 32);
            s_tl[0] = static_cast<uint32_t>(t);
        }
    }
    __syncthreads();
    const int total = s_pre[nL];
    const int t_begin = static_cast<int>(static_cast<int64_t>(total) * part / parts);
    const int t_end = static_cast<int>(static_cast<int64_t>(total) * (part + 1) / parts);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int V = VW;
    const int W = ix.W, Wf = B >> 3, tail = B & 7;
    int ci = 0;                                    // leaf rank of the warp's latest tile (tiles only increase)
    // U tiles at a time (U = 2 while two remain), their code loads issued together
    auto run = [&](auto u_tag, int tt) {
        constexpr int U = decltype(u_tag)::value;
        int cr[U], slot[U];
        bool valid[U];
        const uint32_t* tw[U];
        uint32_t key[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int t = tt + u * NW;
            while (s_pre[ci + 1] <= t) ++ci;
            cr[u] = ci;
            const int l = t - s_pre[ci];
            tw[u] = ix.codes_il + static_cast<int64_t>(s_pt[ci] + l) * W * 32;
            slot[u] = s_os[ci] + 32 * l + lane;
            valid[u] = slot[u] < s_oe[ci];
        }
        if (MODE == 0) {
            constexpr uint32_t WB = 8 * kCenters * 4;      // bytes of a word's 8 blocks
            auto word = [&](uint32_t c, int nb, uint32_t xw, float& acc) {
                const uint32_t ev = (c & 0x0F0F0F0Fu) << 2, od = ((c >> 4) & 0x0F0F0F0Fu) << 2;
#pragma unroll
                for (int nib = 0; nib < 8; ++nib)
                    if (nib < nb) {
                        const uint32_t p = __byte_perm((nib & 1) ? od : ev, xw, 0x7650u | (nib >> 1)) + nib * kCenters * 4;
                        acc = __fadd_rn(acc, __uint_as_float(lds_u32(p)));
                    }
            };
            float acc[U];
#pragma unroll
            for (int u = 0; u < U; ++u) acc[u] = 0.0f;
            if (W <= 8) {
                // narrow codes (up to 64 blocks): both tiles' words in one round of loads
                uint32_t cw[U][8];
#pragma unroll
                for (int u = 0; u < U; ++u) tile_words8<V>(tw[u], lane, W, cw[u]);
#pragma unroll
                for (int w8 = 0; w8 < 8; ++w8)
                    if (w8 < Wf)
#pragma unroll
                        for (int u = 0; u < U; ++u) word(cw[u][w8], 8, tbase + w8 * WB, acc[u]);
                if (tail) {
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        uint32_t last = 0u;
#pragma unroll
                        for (int w8 = 0; w8 < 8; ++w8) last = (w8 == Wf) ? cw[u][w8] : last;
                        word(last, tail, tbase + Wf * WB, acc[u]);
                    }
                }
            } else {
            int w = 0;
            for (; w + 4 <= Wf; w += 4) {
                uint32_t cw[U][4];
#pragma unroll
                for (int u = 0; u < U; ++u) code_words4(tw[u], lane, w, V, cw[u][0], cw[u][1], cw[u][2], cw[u][3]);
                const uint32_t xw = tbase + w * WB;
#pragma unroll
                for (int k = 0; k < 4; ++k)
#pragma unroll
                    for (int u = 0; u < U; ++u) word(cw[u][k], 8, xw + k * WB, acc[u]);
            }
            for (; w < Wf; ++w) {
                uint32_t cw[U];
#pragma unroll
                for (int u = 0; u < U; ++u) cw[u] = tw[u][code_word(w, lane, V)];
#pragma unroll
                for (int u = 0; u < U; ++u) word(cw[u], 8, tbase + w * WB, acc[u]);
            }
            if (tail) {
                uint32_t cw[U];
#pragma unroll
                for (int u = 0; u < U; ++u) cw[u] = tw[u][code_word(Wf, lane, V)];
#pragma unroll
                for (int u = 0; u < U; ++u) word(cw[u], tail, tbase + Wf * WB, acc[u]);
            }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) key[u] = float_key(RES ? __fadd_rn(acc[u], s_lo[cr[u]]) : acc[u]);
        } else {
            constexpr uint32_t WB = 8 * 32;                // bytes of a word's 8 blocks
            auto word = [&](uint32_t c, int nb, uint32_t xw, uint32_t& acc) {
                const uint32_t ev = c & 0x0F0F0F0Fu, od = (c >> 4) & 0x0F0F0F0Fu;
#pragma unroll
                for (int nib = 0; nib < 8; ++nib)
                    if (nib < nb) acc += lds_u8(__byte_perm((nib & 1) ? od : ev, xw, 0x7650u | (nib >> 1)) + nib * 32);
            };
            uint32_t acc[U];
#pragma unroll
            for (int u = 0; u < U; ++u) acc[u] = 0u;
            if (W <= 8) {
                // narrow codes (up to 64 blocks): both tiles' words in one round of loads
                uint32_t cw[U][8];
#pragma unroll
                for (int u = 0; u < U; ++u) tile_words8<V>(tw[u], lane, W, cw[u]);
#pragma unroll
                for (int w8 = 0; w8 < 8; ++w8)
                    if (w8 < Wf)
#pragma unroll
                        for (int u = 0; u < U; ++u) word(cw[u][w8], 8, tbase + w8 * WB, acc[u]);
                if (tail) {
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        uint32_t last = 0u;
#pragma unroll
                        for (int w8 = 0; w8 < 8; ++w8) last = (w8 == Wf) ? cw[u][w8] : last;
                        word(last, tail, tbase + Wf * WB, acc[u]);
                    }
                }
            } else {
            int w = 0;
            for (; w + 4 <= Wf; w += 4) {
                uint32_t cw[U][4];
#pragma unroll
                for (int u = 0; u < U; ++u) code_words4(tw[u], lane, w, V, cw[u][0], cw[u][1], cw[u][2], cw[u][3]);
                const uint32_t xw = tbase + w * WB;
#pragma unroll
                for (int k = 0; k < 4; ++k)
#pragma unroll
                    for (int u = 0; u < U; ++u) word(cw[u][k], 8, xw + k * WB, acc[u]);
            }
            for (; w < Wf; ++w) {
                uint32_t cw[U];
#pragma unroll
                for (int u = 0; u < U; ++u) cw[u] = tw[u][code_word(w, lane, V)];
#pragma unroll
                for (int u = 0; u < U; ++u) word(cw[u], 8, tbase + w * WB, acc[u]);
            }
            if (tail) {
                uint32_t cw[U];
#pragma unroll
                for (int u = 0; u < U; ++u) cw[u] = tw[u][code_word(Wf, lane, V)];
#pragma unroll
                for (int u = 0; u < U; ++u) word(cw[u], tail, tbase + Wf * WB, acc[u]);
            }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) key[u] = acc[u];
        }
#pragma unroll
        for (int u = 0; u < U; ++u) keep_if_reaches(valid[u], key[u], slot[u], 0, s_q, s_th, s_tl, ix, b);
    };
    for (int tt = t_begin + warp; tt < t_end; tt += 2 * NW) {
        if (tt + NW < t_end) run(std::integral_constant<int, 2>{}, tt);   // the same for the whole warp
        else run(std::integral_constant<int, 1>{}, tt);
    }
}

cudaError_t launch_scan_query(const DeviceIndex& ix, const SearchArgs& a, const SearchBuffers& b, int r0, int r1,
                              int num_sms, cudaStream_t s) {
    const int nL = r1 - r0;
    if (nL < 1 || nL > kQScanMaxLeaves) return cudaErrorInvalidValue;
    const size_t smem = scan_query_smem_bytes(a.lut_mode, ix.B, nL);
    // CTAs per query: enough to fill the SMs, no more than about two tiles per warp
    // of the query's expected tiles (from the average leaf)
    const double avg_tiles = std::max(1.0, static_cast<double>(ix.n) / ix.nl / 32.0);
    const int max_parts = std::max(1, static_cast<int>(nL * avg_tiles / (2.0 * kQScanThreads / 32)));
    auto go = [&](auto kernel) -> cudaError_t {
        cudaError_t e = ensure_smem(reinterpret_cast<const void*>(kernel), smem, true);
        if (e != cudaSuccess) return e;
        int per_sm = 0;
        if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kQScanThreads, smem)) != cudaSuccess)
            return e;
        if (per_sm < 1) return cudaErrorInvalidConfiguration;
        const int want = (num_sms * per_sm + a.nq - 1) / a.nq;
        const int parts = std::max(1, std::min(want, max_parts));
        if (const cudaError_t le = launch_chained(kernel, dim3(static_cast<unsigned>(a.nq) * parts), dim3(kQScanThreads),
                                                  smem, s, ix, a, b, r0, r1, parts);
            le != cudaSuccess)
            return le;
        return cudaGetLastError();
    };
    auto by_v = [&](auto k4, auto k2, auto k1) { return ix.V == 4 ? go(k4) : ix.V == 2 ? go(k2) : go(k1); };
    if (a.lut_mode == 0) {
        if (ix.residual)
            return by_v(scan_query_kernel<0, true, 4>, scan_query_kernel<0, true, 2>, scan_query_kernel<0, true, 1>);
        return by_v(scan_query_kernel<0, false, 4>, scan_query_kernel<0, false, 2>, scan_query_kernel<0, false, 1>);
    }
    return by_v(scan_query_kernel<1, false, 4>, scan_query_kernel<1, false, 2>, scan_query_kernel<1, false, 1>);
}

// ---------------------------------------------------------------------------
// bound refinement between scan phases
// ---------------------------------------------------------------------------

// One CTA per query, between scan phases: every point of the leaves scanned so
// far whose key reaches the current bound is in the buffer, so when at least R
// are there, the R-th best of them is a tighter lower bound on the query's
// R-th best over all its leaves.  The buffer is then compacted in place to the
// keys that reach the new bound (order kept; writes only move entries left,
// and each chunk is read completely before any of it is written).
__global__ void __launch_bounds__(kSelThreads) tau_update_kernel(DeviceIndex ix, SearchArgs a, SearchBuffers b) {
    chain_entry();
    __shared__ SelectScratch scr;
    __shared__ RegSelectScratch<kSelThreads> rs;
    __shared__ int s_kept;
    __shared__ int s_warp[kSelThreads / 32];
    const int q = blockIdx.x;
    const int cnt = b.count[q];
    if (cnt < a.R || cnt > b.cap) return;       // too few to bound, or overflowed (handled after the scan)
    uint64_t* ck = b.ckey + static_cast<int64_t>(q) * b.cap;
    int32_t* cs = b.cslot + static_cast<int64_t>(q) * b.cap;
    auto get = [&](int i) { return ck[i]; };
    uint64_t t;
    if (cnt <= 4 * kSelThreads) {
        uint64_t kk[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int i = threadIdx.x + kSelThreads * j;
            kk[j] = (i < cnt) ? ck[i] : 0ull;
        }
        t = block_kth_reg<4, kSelThreads>(kk, cnt, a.R, rs);
    } else {
        t = block_kth_largest<kSelThreads>(get, cnt, a.R, scr);
    }
    const uint64_t old = b.tau[q];
    if (t < old) t = old;
    if (threadIdx.x == 0) {
        b.tau[q] = t;
        s_kept = 0;
    }
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int base = 0; base < cnt; base += kSelThreads) {
        const int i = base + threadIdx.x;
        const bool in = i < cnt;
        const uint64_t k = in ? ck[i] : 0ull;
        const int32_t sl = in ? cs[i] : 0;
        const bool keep = in && k >= t;
        const unsigned m = __ballot_sync(0xFFFFFFFFu, keep);
        if (lane == 0) s_warp[warp] = __popc(m);
        __syncthreads();
        int before = s_kept;
        for (int w = 0; w < warp; ++w) before += s_warp[w];
        if (keep) {
            const int pos = before + __popc(m & ((1u << lane) - 1u));
            ck[pos] = k;
            cs[pos] = sl;
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            int tot = 0;
            for (int w = 0; w < kSelThreads / 32; ++w) tot += s_warp[w];
            s_kept += tot;
        }
        __syncthreads();
    }
    if (threadIdx.x == 0) b.count[q] = s_kept;
}

cudaError_t launch_tau_update(const DeviceIndex& ix, const SearchArgs& a, const SearchBuffers& b, cudaStream_t s) {
    if (const cudaError_t le = launch_chained(tau_update_kernel, dim3(a.nq), dim3(kSelThreads), 0, s, ix, a, b); le != cudaSuccess) return le;
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// redo scan (query-major, rare): rescan a query's leaves with its tighter bound
// ---------------------------------------------------------------------------

// Persistent CTAs take (redo query, leaf rank) pairs from a counter; each pair
// rescans one leaf for one query with the query's tighter bound.  With no query
// to redo every CTA exits after one atomic.
template <int MODE>
__global__ void __launch_bounds__(kSelThreads) redo_scan_kernel(DeviceIndex ix, SearchArgs a, SearchBuffers b, int round) {
    chain_entry();
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ int s_item;
    const int* list = b.redo + static_cast<int64_t>(round - 1) * a.nq;
    const int total = b.counters[round] * a.L;
    int loaded_q = -1;
    for (;;) {
        __syncthreads();
        if (threadIdx.x == 0) s_item = atomicAdd(&b.counters[2 + round], 1);
        __syncthreads();
        const int item = s_item;
        if (item >= total) break;
        const int r = item / a.L, i = item - r * a.L;
        const int q = list[r];
        if (q != loaded_q) {
            load_query_table<MODE>(ix, b, q, smem);
            loaded_q = q;
            __syncthreads();
        }
        const uint64_t tau = b.tau[q];
        const uint32_t th = static_cast<uint32_t>(tau >> 32), tl = static_cast<uint32_t>(tau);
        const int leaf = b.leaves[static_cast<int64_t>(q) * a.L + i];
        const int s0 = ix.offs[leaf], s1 = ix.offs[leaf + 1];
        const int p0 = ix.ptile[leaf] * 32 - s0;            // padded position = slot + p0
        const float off = ix.residual ? b.cscore[static_cast<int64_t>(q) * ix.nl + leaf] : 0.0f;
        for (int base = s0; base < s1; base += kSelThreads) {
            const int slot = base + threadIdx.x;
            const bool in = slot < s1;
            const uint32_t v = in ? slot_value<MODE>(ix.codes_il, ix.W, ix.V, ix.B, smem, slot + p0, ix.residual != 0, off)
                                  : 0u;
            append_candidates(in && reaches(v, th, tl, ix.slot_ids, slot), v, slot, q, ix, b);
        }
    }
}

cudaError_t launch_redo_scan(const DeviceIndex& ix, const SearchArgs& a, const SearchBuffers& b, int round,
                             int num_sms, cudaStream_t s) {
    size_t smem = table_bytes(a.lut_mode, ix.B);
    cudaError_t e;
    const int grid = num_sms * 2;
    if (a.lut_mode == 0) {
        e = ensure_smem(reinterpret_cast<const void*>(redo_scan_kernel<0>), smem, true);
        if (e != cudaSuccess) return e;
        if (const cudaError_t le = launch_chained(redo_scan_kernel<0>, dim3(grid), dim3(kSelThreads), smem, s, ix, a, b, round); le != cudaSuccess) return le;
    } else {
        e = ensure_smem(reinterpret_cast<const void*>(redo_scan_kernel<1>), smem, true);
        if (e != cudaSuccess) return e;
        if (const cudaError_t le = launch_chained(redo_scan_kernel<1>, dim3(grid), dim3(kSelThreads), smem, s, ix, a, b, round); le != cudaSuccess) return le;
    }
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// finish: best R, exact reorder, best k (one CTA per query)
// ---------------------------------------------------------------------------

constexpr int kFinishThreads = 256;
constexpr int kStageCap = 1024;          // candidate keys staged in shared memory up to this count

size_t finish_smem_bytes(int R, int d) {
    const size_t p2 = static_cast<size_t>(next_pow2(R));
    return static_cast<size_t>(kStageCap) * (sizeof(uint64_t) + sizeof(int32_t)) +   // staged keys, slots
           p2 * (2 * sizeof(uint64_t) + sizeof(int32_t)) +                            // best R keys, slots; exact keys
           256 * sizeof(int) + static_cast<size_t>(d) * sizeof(float) + 64;            // warp histogram; query
}

// One CTA per query (round 0) or per entry of the previous round's redo list.
//  1. The best R of the query's kept candidates by (approximate score, id) key.
//     A query whose buffer overflowed instead gets a tighter bound (the R-th
//     best stored key: stored entries are real candidates, so it is still a
//     lower bound on the R-th best) and is queued for a rescan; on the last
//     round an overflow is reported through the error word and the stored
//     subset is used.
//  2. Without reorder, the best k of those are the result.  With reorder,
//     groups of 2..32 lanes (by d) compute the exact fp32 dot product of each
//     candidate's stored vector (float, or bfloat16 upcast) with the query,
//     and one warp keeps the best k by (exact score, id).
template <int MODE>
__device__ void finish_query(const DeviceIndex& ix, const SearchArgs& a, const SearchBuffers& b, int round, int q,
                             unsigned char* smem, SelectScratch& scr,
                             RegSelectScratch<kFinishThreads>& rs) {
    const int cap = b.cap, R = a.R, k = a.k, d = ix.d;
    const int P2 = next_pow2(R);
    uint64_t* skeys = reinterpret_cast<uint64_t*>(smem);            // [kStageCap]
    uint64_t* okeys = skeys + kStageCap;                            // [P2]
    uint64_t* ekeys = okeys + P2;                                   // [P2]
    int32_t* sslots = reinterpret_cast<int32_t*>(ekeys + P2);       // [kStageCap]
    int32_t* oslots = sslots + kStageCap;                           // [P2]
    int* whist = oslots + P2;                                       // [256]
    float* qv = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(whist + 256) + 15) & ~uintptr_t(15));  // [d], 16-B aligned
    const uint64_t* ck = b.ckey + static_cast<int64_t>(q) * cap;
    const int32_t* cs = b.cslot + static_cast<int64_t>(q) * cap;
    int cnt = b.count[q];
    if (round == 0 && a.tr_passed && threadIdx.x == 0) a.tr_passed[q] = cnt;
    if (cnt > cap) {
        if (round < 2) {
            auto get = [&](int i) { return ck[i]; };
            const uint64_t tau = block_kth_largest<kFinishThreads>(get, cap, R, scr);
            if (threadIdx.x == 0) {
                b.tau[q] = tau;
                b.count[q] = 0;
                int pos = atomicAdd(&b.counters[round + 1], 1);
                b.redo[static_cast<int64_t>(round) * a.nq + pos] = q;
            }
            return;
        }
        if (threadIdx.x == 0) raise_error(b.err, kDevCandOverflow);
        cnt = cap;
    }
    // the best R need an order only when they are reported (trace) or are the
    // result (no reorder); the reorder path reads them as a set
    const bool sorted = a.reorder_num == 0 || a.tr_cand_ids || a.tr_cand_scores || a.tr_cand_sums;
    int K;
    int staged = -1;                  // keys staged in shared memory, or -1: read from global
    if (cnt <= 8 * 32 && R <= kWarpMaxK) {
        // few kept candidates: one warp selects straight from global memory
        if (threadIdx.x < 32) {
            int kk;
            if (cnt <= 2 * 32)
                kk = warp_topk_src<2>(ck, cs, cnt, R, okeys, oslots, sorted);
            else if (cnt <= 4 * 32)
                kk = warp_topk_src<4>(ck, cs, cnt, R, okeys, oslots, sorted);
            else
                kk = warp_topk_src<8>(ck, cs, cnt, R, okeys, oslots, sorted);
            if (threadIdx.x == 0) scr.count = kk;
        }
        __syncthreads();
        staged = -2;
    } else if (cnt <= kStageCap) {
        for (int i = threadIdx.x; i < cnt; i += kFinishThreads) {
            skeys[i] = ck[i];
            sslots[i] = cs[i];
        }
        staged = cnt;
        __syncthreads();
    } else if (R < kStageCap) {
        // Many kept candidates: the R-th best of any subset is a lower bound on
        // the R-th best of all, so the largest such bound over kStageCap-key
        // chunks (keys below the running bound dropped first) lets one
        // batched pass keep only the keys that reach it.
        constexpr int CPT = kStageCap / kFinishThreads;
        uint64_t bound = 0ull;
        for (int c0 = 0; c0 < cnt; c0 += kStageCap) {
            uint64_t sk[CPT];
            int live = 0;
#pragma unroll
            for (int j = 0; j < CPT; ++j) {
                const int i = c0 + threadIdx.x + kFinishThreads * j;
                const uint64_t key = (i < cnt) ? ck[i] : 0ull;
                sk[j] = (key >= bound) ? key : 0ull;
                live += (sk[j] != 0ull) ? 1 : 0;
            }
            live = block_sum_parity<kFinishThreads>(live, rs, (c0 / kStageCap) & 1);
            if (live > R) bound = block_kth_reg<CPT, kFinishThreads>(sk, live, R, rs);
        }
        if (threadIdx.x == 0) scr.count = 0;
        __syncthreads();
        constexpr int U = 4;
        for (int i0 = 0; i0 < cnt; i0 += U * kFinishThreads) {
            uint64_t kk[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int i = i0 + u * kFinishThreads + threadIdx.x;
                kk[u] = (i < cnt) ? ck[i] : 0ull;
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int i = i0 + u * kFinishThreads + threadIdx.x;
                if (i < cnt && kk[u] >= bound) {
                    const int pos = atomicAdd(&scr.count, 1);
                    if (pos < kStageCap) {
                        skeys[pos] = kk[u];
                        sslots[pos] = cs[i];
                    }
                }
            }
        }
        __syncthreads();
        if (scr.count <= kStageCap) staged = scr.count;
        __syncthreads();
    }
    if (staged == -2) {
        K = scr.count;
    } else if (staged >= 0 && staged <= kStageCap) {
        auto get = [&](int i) { return skeys[i]; };
        auto pay = [&](int i) { return sslots[i]; };
        K = block_topk_reg<kStageCap / kFinishThreads, kFinishThreads>(get, pay, staged, R, rs, &scr.count, okeys,
                                                                       oslots, sorted);
    } else if (staged >= 0) {
        auto get = [&](int i) { return skeys[i]; };
        auto pay = [&](int i) { return sslots[i]; };
        K = block_topk<kFinishThreads>(get, pay, staged, R, scr, okeys, oslots, b.err, sorted);
    } else {
        auto get = [&](int i) { return ck[i]; };
        auto pay = [&](int i) { return cs[i]; };
        K = block_topk<kFinishThreads>(get, pay, cnt, R, scr, okeys, oslots, b.err, sorted);
    }
    const float delta = (MODE == 1) ? b.lut_delta[q] : 0.0f;
    const float bias = (MODE == 1) ? b.lut_bias[q] : 0.0f;
    auto approx_score = [&](uint32_t sk) {
        return (MODE == 0) ? key_float(sk) : fmaf(delta, static_cast<float>(sk), bias);
    };
    const int64_t ro = static_cast<int64_t>(q) * R;
    if (a.tr_cand_ids || a.tr_cand_scores || a.tr_cand_sums) {
        for (int i = threadIdx.x; i < R; i += kFinishThreads) {
            const bool have = i < K;
            if (a.tr_cand_ids) a.tr_cand_ids[ro + i] = have ? key_id(okeys[i]) : -1;
            if (a.tr_cand_scores) a.tr_cand_scores[ro + i] = have ? approx_score(key_score(okeys[i])) : -INFINITY;
            if (a.tr_cand_sums) a.tr_cand_sums[ro + i] = (have && MODE == 1) ? key_score(okeys[i]) : 0u;
        }
    }
    if (a.tr_ncand && threadIdx.x == 0) a.tr_ncand[q] = K;
    const int64_t oo = static_cast<int64_t>(q) * k;
    if (a.reorder_num == 0) {
        for (int i = threadIdx.x; i < k; i += kFinishThreads) {
            const bool have = i < K;
            a.out_ids[oo + i] = have ? key_id(okeys[i]) : -1;
            a.out_scores[oo + i] = have ? approx_score(key_score(okeys[i])) : -INFINITY;
        }
        return;
    }
    // exact reorder: groups of `lpc` lanes, one candidate per group per round.
    // For 8-value bfloat16 loads the query is staged as two halves, values
    // 8c..8c+3 at 4c and 8c+4..8c+7 at d/2 + 4c, so that the lanes' 16-byte
    // reads of their chunks are consecutive (no bank conflicts).
    const bool split_q = ix.reorder_bf16 && a.reorder_vec4 == 2;
    for (int t = threadIdx.x; t < d; t += kFinishThreads) {
        const int c = t >> 3, r = t & 7;
        const int dst = !split_q ? t : (r < 4 ? 4 * c + r : (d >> 1) + 4 * c + (r - 4));
        qv[dst] = a.queries[static_cast<int64_t>(q) * d + t];
    }
    __syncthreads();
    const int lpc = a.reorder_lanes;                  // power of two in [2, 32]
    const int groups = kFinishThreads / lpc;
    const int grp = threadIdx.x / lpc, gl = threadIdx.x & (lpc - 1);
    for (int base = 0; base < K; base += groups) {
        const int i = base + grp;
        float acc = 0.0f;
        if (i < K) {
            const int64_t slot = oslots[i];
            if (a.reorder_vec4) {        // d % 4 == 0 and 16-byte aligned rows (checked on the host)
                const float4* q4 = reinterpret_cast<const float4*>(qv);
                // The row loads are issued kReorderBatch at a time ahead of
                // the multiply-adds (same accumulation order), so a lane waits
                // for memory once per batch rather than once per load.
                const int n4 = d / 4;
                if (ix.reorder_bf16 && a.reorder_vec4 == 2) {
                    // bfloat16 rows, d % 8 == 0: 16-byte loads of 8 values
                    const uint4* v = reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(ix.reorder_vecs) + slot * d);
                    const int n8 = d / 8;
                    for (int t0 = gl; t0 < n8; t0 += kReorderBatch * lpc) {
                        uint4 h[kReorderBatch];
#pragma unroll
                        for (int u = 0; u < kReorderBatch; ++u) {
                            const int t = t0 + u * lpc;
                            h[u] = (t < n8) ? v[t] : make_uint4(0u, 0u, 0u, 0u);
                        }
#pragma unroll
                        for (int u = 0; u < kReorderBatch; ++u) {
                            const int t = t0 + u * lpc;
                            if (t < n8) {
                                const float4 x0 = q4[t], x1 = q4[n8 + t];
                                acc = fmaf(x0.x, __uint_as_float(h[u].x << 16), acc);
                                acc = fmaf(x0.y, __uint_as_float(h[u].x & 0xFFFF0000u), acc);
                                acc = fmaf(x0.z, __uint_as_float(h[u].y << 16), acc);
                                acc = fmaf(x0.w, __uint_as_float(h[u].y & 0xFFFF0000u), acc);
                                acc = fmaf(x1.x, __uint_as_float(h[u].z << 16), acc);
                                acc = fmaf(x1.y, __uint_as_float(h[u].z & 0xFFFF0000u), acc);
                                acc = fmaf(x1.z, __uint_as_float(h[u].w << 16), acc);
                                acc = fmaf(x1.w, __uint_as_float(h[u].w & 0xFFFF0000u), acc);
                            }
                        }
                    }
                } else if (ix.reorder_bf16) {
                    const uint2* v = reinterpret_cast<const uint2*>(reinterpret_cast<const uint16_t*>(ix.reorder_vecs) + slot * d);
                    for (int t0 = gl; t0 < n4; t0 += kReorderBatch * lpc) {
                        uint2 h[kReorderBatch];
#pragma unroll
                        for (int u = 0; u < kReorderBatch; ++u) {
                            const int t = t0 + u * lpc;
                            h[u] = (t < n4) ? v[t] : make_uint2(0u, 0u);
                        }
#pragma unroll
                        for (int u = 0; u < kReorderBatch; ++u) {
                            const int t = t0 + u * lpc;
                            if (t < n4) {
                                const float4 x = q4[t];
                                acc = fmaf(x.x, __uint_as_float(h[u].x << 16), acc);
                                acc = fmaf(x.y, __uint_as_float(h[u].x & 0xFFFF0000u), acc);
                                acc = fmaf(x.z, __uint_as_float(h[u].y << 16), acc);
                                acc = fmaf(x.w, __uint_as_float(h[u].y & 0xFFFF0000u), acc);
                            }
                        }
                    }
                } else {
                    const float4* v = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(ix.reorder_vecs) + slot * d);
                    for (int t0 = gl; t0 < n4; t0 += kReorderBatch * lpc) {
                        float4 h[kReorderBatch];
#pragma unroll
                        for (int u = 0; u < kReorderBatch; ++u) {
                            const int t = t0 + u * lpc;
                            h[u] = (t < n4) ? v[t] : make_float4(0.f, 0.f, 0.f, 0.f);
                        }
#pragma unroll
                        for (int u = 0; u < kReorderBatch; ++u) {
                            const int t = t0 + u * lpc;
                            if (t < n4) {
                                const float4 x = q4[t];
                                acc = fmaf(x.x, h[u].x, acc);
                                acc = fmaf(x.y, h[u].y, acc);
                                acc = fmaf(x.z, h[u].z, acc);
                                acc = fmaf(x.w, h[u].w, acc);
                            }
                        }
                    }
                }
            } else if (ix.reorder_bf16) {
                const uint16_t* v = reinterpret_cast<const uint16_t*>(ix.reorder_vecs) + slot * d;
                for (int t = gl; t < d; t += lpc) acc = fmaf(qv[t], __uint_as_float(static_cast<uint32_t>(v[t]) << 16), acc);
            } else {
                const float* v = reinterpret_cast<const float*>(ix.reorder_vecs) + slot * d;
                for (int t = gl; t < d; t += lpc) acc = fmaf(qv[t], v[t], acc);
            }
        }
        for (int off = lpc >> 1; off > 0; off >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, off);
        if (i < K && gl == 0) ekeys[i] = make_key(float_key(acc), key_id(okeys[i]));
    }
    __syncthreads();
    if (a.tr_cand_exact)
        for (int i = threadIdx.x; i < R; i += kFinishThreads)
            a.tr_cand_exact[ro + i] = (i < K) ? key_float(key_score(ekeys[i])) : -INFINITY;
    auto eget = [&](int i) { return ekeys[i]; };
    auto epay = [&](int i) { return i; };
    if (k <= kWarpMaxK) {
        if (threadIdx.x < 32) {
            const int Kk = (K <= 32 * 4) ? warp_topk_reg<4>(eget, epay, K, k, okeys, nullptr, true)
                                         : warp_topk(eget, epay, K, k, whist, okeys, nullptr);
            for (int i = threadIdx.x; i < k; i += 32) {
                const bool have = i < Kk;
                a.out_ids[oo + i] = have ? key_id(okeys[i]) : -1;
                a.out_scores[oo + i] = have ? key_float(key_score(okeys[i])) : -INFINITY;
            }
        }
    } else {
        const int Kk = block_topk<kFinishThreads>(eget, epay, K, k, scr, okeys, nullptr, b.err);
        for (int i = threadIdx.x; i < k; i += kFinishThreads) {
            const bool have = i < Kk;
            a.out_ids[oo + i] = have ? key_id(okeys[i]) : -1;
            a.out_scores[oo + i] = have ? key_float(key_score(okeys[i])) : -INFINITY;
        }
    }
}

// The finish's CTAs start in grid order, and a query with more than
// kStageCap kept candidates takes about twice as long as the rest; listing
// those first keeps them out of the grid's last, partial wave.  (Positions
// come from atomics; each query's result does not depend on them.)
__global__ void __launch_bounds__(256) finish_order_kernel(SearchArgs a, SearchBuffers b) {
    chain_entry();
    const int q = blockIdx.x * 256 + threadIdx.x;
    if (q >= a.nq) return;
    const bool heavy = b.count[q] > kStageCap;
    const int pos = heavy ? atomicAdd(&b.counters[5], 1) : a.nq - 1 - atomicAdd(&b.counters[6], 1);
    b.order[pos] = q;
}

template <int MODE>
__global__ void __launch_bounds__(kFinishThreads, AH_FINISH_MIN_BLOCKS) finish_kernel(DeviceIndex ix, SearchArgs a, SearchBuffers b, int round) {
    chain_entry();
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ SelectScratch scr;
    __shared__ RegSelectScratch<kFinishThreads> rs;
    if (round == 0) {
        finish_query<MODE>(ix, a, b, 0, b.order[blockIdx.x], smem, scr, rs);
        return;
    }
    // rescan rounds: a small grid walks the previous round's redo list
    const int n = b.counters[round];
    for (int e = blockIdx.x; e < n; e += gridDim.x) {
        finish_query<MODE>(ix, a, b, round, b.redo[static_cast<int64_t>(round - 1) * a.nq + e], smem, scr, rs);
        __syncthreads();
    }
}

static int lanes_per_candidate(int d) {
    const int vec = (d + 3) / 4;                 // 4-element loads per row
    int lpc = 2;
    while (lpc < 32 && lpc * 8 < vec) lpc <<= 1;  // about 8 loads per lane
    return lpc;
}

template <class Kernel>
static cudaError_t prefer_shared(Kernel k, size_t smem) {
    return ensure_smem(reinterpret_cast<const void*>(k), smem, true);
}

cudaError_t launch_finish(const DeviceIndex& ix, SearchArgs a, const SearchBuffers& b, int round, int num_sms,
                          cudaStream_t s) {
    const uintptr_t qa = reinterpret_cast<uintptr_t>(a.queries), va = reinterpret_cast<uintptr_t>(ix.reorder_vecs);
    a.reorder_vec4 = (ix.d % 4 == 0 && qa % 16 == 0 && va % 16 == 0) ? 1 : 0;
    if (a.reorder_vec4 && ix.reorder_bf16 && ix.d % 8 == 0) a.reorder_vec4 = 2;   // 16-byte bf16 loads
    a.reorder_lanes = lanes_per_candidate(a.reorder_vec4 == 2 ? ix.d / 2 : ix.d);
    const size_t smem = finish_smem_bytes(a.R, ix.d);
    const unsigned grid = (round == 0) ? static_cast<unsigned>(a.nq) : static_cast<unsigned>(std::min(a.nq, 2 * num_sms));
    cudaError_t e;
    if (round == 0) {
        if (const cudaError_t le = launch_chained(finish_order_kernel, dim3((a.nq + 255) / 256), dim3(256), 0, s, a, b);
            le != cudaSuccess)
            return le;
    }
    if (a.lut_mode == 0) {
        if ((e = prefer_shared(finish_kernel<0>, smem)) != cudaSuccess) return e;
        if (const cudaError_t le = launch_chained(finish_kernel<0>, dim3(grid), dim3(kFinishThreads), smem, s, ix, a, b, round); le != cudaSuccess) return le;
    } else {
        if ((e = prefer_shared(finish_kernel<1>, smem)) != cudaSuccess) return e;
        if (const cudaError_t le = launch_chained(finish_kernel<1>, dim3(grid), dim3(kFinishThreads), smem, s, ix, a, b, round); le != cudaSuccess) return le;
    }
    return cudaGetLastError();
}

}  // namespace ah
