// Anisotropic code assignment (index build), ScaNN blog, "Training an
// anisotropic codebook yourself": each point's codes minimise the anisotropic
// loss (eta - 1) (r . u)^2 + ||r||^2, r = x - x~, u = x / ||x||, with eta per
// point from the threshold T ("The loss in one paragraph").  Blocks couple
// through r . u, so the codes are refined block by block: start from the
// per-block nearest centers, then passes over the blocks in order, each
// taking the center of least loss with the other blocks fixed when it is
// strictly better (ties: lower center), until a pass changes nothing.
//
// Half a warp per point, lane j scoring center j of the current block; the
// point's scalars (norm, eta, r . u, ||r||^2) are computed redundantly by all
// 16 lanes in one fixed order.  fp64 throughout with every product and sum
// rounded on its own (__dmul_rn / __dadd_rn never fuse), sums over a block's
// coordinates in ascending order: the same arithmetic the oracle states, so
// the codes match it bit for bit.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstddef>

#include "kernels.h"

namespace ah {

namespace {

// (loss, center) minimum over the half-warp, ties to the lower center: the
// minimum value by a shuffle reduction, then the lowest lane holding it.
__device__ __forceinline__ void half_argmin(double& l, int& j, unsigned mask) {
    double m = l;
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) m = fmin(m, __shfl_xor_sync(mask, m, off, 16));
    const unsigned hit = __ballot_sync(mask, l == m) & mask;
    j = (__ffs(hit) - 1) & 15;
    l = m;
}

// USE_U: the point's unit vector u = x / ||x|| is computed once (each element
// by one lane, the same correctly rounded division) into shared memory;
// otherwise every use recomputes it, with identical values.
template <bool USE_U, int DPB>
__global__ void __launch_bounds__(256) encode_kernel(const float* __restrict__ X, int64_t n, int d, int dpb_rt,
                                                     const float* __restrict__ codebook, double T, int passes,
                                                     int cb_in_smem, uint8_t* __restrict__ codes,
                                                     int32_t* __restrict__ passes_used) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int dpb = DPB > 0 ? DPB : dpb_rt;      // compile-time for the common block widths
    const int B = d / dpb;
    float* scb = reinterpret_cast<float*>(smem);
    const int cb_elems = B * 16 * dpb;
    uint8_t* scode = smem + (cb_in_smem ? static_cast<size_t>(cb_elems) * sizeof(float) : 0);
    double* su_all = reinterpret_cast<double*>(
        (reinterpret_cast<uintptr_t>(scode + static_cast<size_t>(16) * B) + 15) & ~static_cast<uintptr_t>(15));
    if (cb_in_smem) {
        for (int e = threadIdx.x; e < cb_elems; e += blockDim.x) scb[e] = codebook[e];
        __syncthreads();
    }
    const float* cb = cb_in_smem ? scb : codebook;
    const int half = threadIdx.x >> 4, j = threadIdx.x & 15;
    const unsigned mask = (threadIdx.x & 16) ? 0xFFFF0000u : 0x0000FFFFu;
    uint8_t* code = scode + static_cast<size_t>(half) * B;
    const int64_t halves = static_cast<int64_t>(gridDim.x) * (blockDim.x / 16);
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * (blockDim.x / 16) + half; i < n; i += halves) {
        const float* xr = X + i * static_cast<int64_t>(d);
        double nrm2 = 0.0;
        for (int t = 0; t < d; ++t) {
            const double x = static_cast<double>(xr[t]);
            nrm2 = __dadd_rn(nrm2, __dmul_rn(x, x));
        }
        const double norm = __dsqrt_rn(nrm2);
        double eta = 1.0;
        if (T > 0.0 && norm > 0.0) {
            const double tn = __ddiv_rn(T, norm);
            const double tt = __dmul_rn(tn, tn);
            if (tt < 1.0) eta = __ddiv_rn(__dmul_rn(static_cast<double>(d - 1), tt), __dadd_rn(1.0, -tt));
        }
        const double e1 = __dadd_rn(eta, -1.0);
        double* su = su_all + static_cast<size_t>(half) * d;
        if (USE_U) {
            for (int t = j; t < d; t += 16) {
                const double x = static_cast<double>(xr[t]);
                su[t] = norm > 0.0 ? __ddiv_rn(x, norm) : 0.0;
            }
            __syncwarp(mask);
        }
        auto unit = [&](int t, double x) { return USE_U ? su[t] : (norm > 0.0 ? __ddiv_rn(x, norm) : 0.0); };
        // start: per block the nearest center
        for (int b = 0; b < B; ++b) {
            double e = 0.0;
            for (int s = 0; s < dpb; ++s) {
                const double df = __dadd_rn(static_cast<double>(xr[b * dpb + s]),
                                            -static_cast<double>(cb[(b * 16 + j) * dpb + s]));
                e = __dadd_rn(e, __dmul_rn(df, df));
            }
            int best = j;
            half_argmin(e, best, mask);
            if (j == 0) code[b] = static_cast<uint8_t>(best);
        }
        __syncwarp(mask);
        double rpar = 0.0, rn2 = 0.0;
        for (int b = 0; b < B; ++b) {
            const int c = code[b];
            for (int s = 0; s < dpb; ++s) {
                const double x = static_cast<double>(xr[b * dpb + s]);
                const double u = unit(b * dpb + s, x);
                const double r = __dadd_rn(x, -static_cast<double>(cb[(b * 16 + c) * dpb + s]));
                rpar = __dadd_rn(rpar, __dmul_rn(r, u));
                rn2 = __dadd_rn(rn2, __dmul_rn(r, r));
            }
        }
        int used = 0;
        for (int p = 0; p < passes; ++p) {
            int changed = 0;
            for (int b = 0; b < B; ++b) {
                const int cur = code[b];
                double sp = 0.0, sn = 0.0;
                for (int s = 0; s < dpb; ++s) {
                    const double x = static_cast<double>(xr[b * dpb + s]);
                    const double u = unit(b * dpb + s, x);
                    const double r = __dadd_rn(x, -static_cast<double>(cb[(b * 16 + j) * dpb + s]));
                    sp = __dadd_rn(sp, __dmul_rn(r, u));
                    sn = __dadd_rn(sn, __dmul_rn(r, r));
                }
                // the current center's sums are lane cur's own (same operations)
                const double cp = __shfl_sync(mask, sp, cur, 16), cn = __shfl_sync(mask, sn, cur, 16);
                const double wp = __dadd_rn(rpar, -cp), wn = __dadd_rn(rn2, -cn);
                const double pj = __dadd_rn(wp, sp), nj = __dadd_rn(wn, sn);
                const double l = __dadd_rn(__dmul_rn(e1, __dmul_rn(pj, pj)), nj);
                const double lcur = __shfl_sync(mask, l, cur, 16);
                double bl = l;
                int best = j;
                half_argmin(bl, best, mask);
                if (bl < lcur) {                     // the same decision on every lane
                    rpar = __shfl_sync(mask, pj, best, 16);
                    rn2 = __shfl_sync(mask, nj, best, 16);
                    if (j == 0) code[b] = static_cast<uint8_t>(best);
                    ++changed;
                }
                __syncwarp(mask);                    // code[b] visible to the half-warp
            }
            used = p + 1;
            if (changed == 0) break;
        }
        if (passes_used && j == 0) passes_used[i] = used;
        uint8_t* out = codes + i * static_cast<int64_t>(B / 2);
        for (int c = j; c < B / 2; c += 16) out[c] = static_cast<uint8_t>(code[2 * c] | (code[2 * c + 1] << 4));
        __syncwarp(mask);
    }
}

}  // namespace

// Dynamic shared memory: the codebook (when it fits), 16 half-warps' codes
// and, when it fits, 16 half-warps' unit vectors.
size_t encode_smem_bytes(int d, int dpb, bool* cb_in_smem, bool* use_u) {
    const size_t B = static_cast<size_t>(d / dpb);
    const size_t cb = B * 16 * dpb * sizeof(float);
    const size_t codes = 16 * B;
    const size_t u = 16 * static_cast<size_t>(d) * sizeof(double) + 16;
    *cb_in_smem = cb + codes <= 100 * 1024;
    const size_t base = (*cb_in_smem ? cb : 0) + codes;
    *use_u = base + u <= 200 * 1024;
    return base + (*use_u ? u : 0);
}

cudaError_t launch_encode(const float* X, int64_t n, int d, int dpb, const float* codebook, double T, int passes,
                          uint8_t* codes, int32_t* passes_used, int num_sms, cudaStream_t s) {
    if (n <= 0) return cudaSuccess;
    bool in_smem = false, use_u = false;
    const size_t smem = encode_smem_bytes(d, dpb, &in_smem, &use_u);
    void (*kern)(const float*, int64_t, int, int, const float*, double, int, int, uint8_t*, int32_t*);
    switch (dpb) {
        case 1: kern = use_u ? encode_kernel<true, 1> : encode_kernel<false, 1>; break;
        case 2: kern = use_u ? encode_kernel<true, 2> : encode_kernel<false, 2>; break;
        case 4: kern = use_u ? encode_kernel<true, 4> : encode_kernel<false, 4>; break;
        case 8: kern = use_u ? encode_kernel<true, 8> : encode_kernel<false, 8>; break;
        default: kern = use_u ? encode_kernel<true, 0> : encode_kernel<false, 0>; break;
    }
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 256, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const int64_t need = (n + 15) / 16;
    const int64_t grid = std::min<int64_t>(need, static_cast<int64_t>(num_sms) * per_sm);
    kern<<<static_cast<unsigned>(grid), 256, smem, s>>>(X, n, d, dpb, codebook, T, passes, in_smem ? 1 : 0, codes,
                                                        passes_used);
    return cudaGetLastError();
}

}  // namespace ah
