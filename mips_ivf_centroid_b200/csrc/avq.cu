// Closed-form anisotropic center update (index build), ScaNN blog post,
// "Training an anisotropic codebook yourself": after every point has been
// assigned to a center, each center moves to the minimiser of its members'
// summed anisotropic loss
//     sum_i (eta_i - 1) ((x_i - c) . u_i)^2 + ||x_i - c||^2,  u_i = x_i / ||x_i||,
// (the loss of "The loss in one paragraph" with h_perp = 1).  Setting its
// gradient to zero gives the linear system (Theorem 4.2 form)
//     (m I + sum_i (eta_i - 1) u_i u_i^T) c = sum_i eta_i x_i,
// which is the plain mean when every eta_i = 1.  eta_i comes from the
// threshold T and the point's norm as for the code assignment: eta =
// (d - 1) t / (1 - t), t = (T / ||x||)^2, and eta = 1 when T <= 0, ||x|| = 0 or
// t >= 1.
//
// The system matrix is never formed.  With eta_i > 0 it is symmetric positive
// definite with eigenvalues between m min(1, eta_min) and m max(1, eta_max),
// so conjugate gradients converge in a few tens of steps; each step applies it
// as m p + sum_i (eta_i - 1) (u_i . p) u_i, reading the members' rows.  One
// CTA per center, fp64, every reduction in a fixed order (the result does not
// depend on scheduling).
//
// Kernels: count members per center, exclusive offsets, an order-preserving
// member list (each center's members in ascending point order), and the solve.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "kernels.h"

namespace ah {

namespace {

constexpr int kVT = 256;          // threads per CTA
constexpr int kFillC = 8;         // centers per member-list CTA
constexpr int kFillChunk = 1024;  // assignments scanned per step

__global__ void avq_count_kernel(const int32_t* __restrict__ assign, int64_t n, int nl, int32_t* __restrict__ counts) {
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const int a = assign[i];
    if (a >= 0 && a < nl) atomicAdd(&counts[a], 1);
}

// Single CTA of 1024 threads: offs = exclusive prefix sums of counts (int64).
__global__ void __launch_bounds__(1024) avq_offsets_kernel(const int32_t* __restrict__ counts, int nl,
                                                           int64_t* __restrict__ offs) {
    __shared__ long long warp_sums[32];
    __shared__ long long s_total;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    long long carry = 0;
    for (int base = 0; base < nl; base += 1024) {
        const int c = base + threadIdx.x;
        const long long v = (c < nl) ? counts[c] : 0;
        long long x = v;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const long long y = __shfl_up_sync(0xFFFFFFFFu, x, off);
            if (lane >= off) x += y;
        }
        if (lane == 31) warp_sums[warp] = x;
        __syncthreads();
        if (warp == 0) {
            const long long w = warp_sums[lane];
            long long xs = w;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const long long y = __shfl_up_sync(0xFFFFFFFFu, xs, off);
                if (lane >= off) xs += y;
            }
            warp_sums[lane] = xs - w;
            if (lane == 31) s_total = xs;
        }
        __syncthreads();
        if (c < nl) offs[c] = carry + warp_sums[warp] + x - v;
        carry += s_total;
        __syncthreads();
    }
    if (threadIdx.x == 0) offs[nl] = carry;
}

// CTA owns centers c0 .. c0 + kFillC - 1: it walks the assignment in
// ascending point order, kFillChunk entries at a time, and appends each of its
// centers' members in that order.
__global__ void __launch_bounds__(kVT) avq_fill_kernel(const int32_t* __restrict__ assign, int64_t n, int nl,
                                                       const int64_t* __restrict__ offs,
                                                       int32_t* __restrict__ members) {
    __shared__ int warp_n[kVT / 32][kFillC];
    __shared__ long long cursor[kFillC];
    const int c0 = blockIdx.x * kFillC;
    const int cn = min(kFillC, nl - c0);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid < kFillC) cursor[tid] = (tid < cn) ? offs[c0 + tid] : 0;
    __syncthreads();
    for (int64_t base = 0; base < n; base += kFillChunk) {
        // thread-major within a warp's 128 entries, warps in order: entry order
        int lc[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int64_t i = base + warp * 128 + u * 32 + lane;
            const int a = (i < n) ? assign[i] : -1;
            lc[u] = (a >= c0 && a < c0 + cn) ? a - c0 : -1;
        }
        // members per (warp, center) in this chunk
        for (int c = 0; c < cn; ++c) {
            int cnt = 0;
#pragma unroll
            for (int u = 0; u < 4; ++u) cnt += __popc(__ballot_sync(0xFFFFFFFFu, lc[u] == c));
            if (lane == 0) warp_n[warp][c] = cnt;
        }
        __syncthreads();
        for (int c = 0; c < cn; ++c) {
            long long pos = cursor[c];
            for (int w = 0; w < warp; ++w) pos += warp_n[w][c];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const unsigned m = __ballot_sync(0xFFFFFFFFu, lc[u] == c);
                if (lc[u] == c) members[pos + __popc(m & ((1u << lane) - 1u))] = static_cast<int32_t>(base + warp * 128 + u * 32 + lane);
                pos += __popc(m);
            }
        }
        __syncthreads();
        if (tid < cn) {
            long long add = 0;
            for (int w = 0; w < kVT / 32; ++w) add += warp_n[w][tid];
            cursor[tid] += add;
        }
        __syncthreads();
    }
}

// Sum of v over the CTA in a fixed order: per-thread values, then a tree over
// threads in shared memory.  Returns the sum on every thread.
__device__ __forceinline__ double block_sum(double v, double* red) {
    red[threadIdx.x] = v;
    __syncthreads();
#pragma unroll
    for (int s = kVT / 2; s > 0; s >>= 1) {
        if (threadIdx.x < s) red[threadIdx.x] = __dadd_rn(red[threadIdx.x], red[threadIdx.x + s]);
        __syncthreads();
    }
    const double r = red[0];
    __syncthreads();
    return r;
}

// One CTA per center: eta and 1/||x|| of every member, b = sum_i eta_i x_i,
// then conjugate gradients on (m I + sum_i w_i u_i u_i^T) c = b, w_i = eta_i - 1,
// from c = 0, until ||r|| <= tol ||b|| or max_iters steps.
__global__ void __launch_bounds__(kVT) avq_solve_kernel(const float* __restrict__ X, int d,
                                                        const int32_t* __restrict__ members,
                                                        const int64_t* __restrict__ offs, double T,
                                                        double* __restrict__ mscal, double* __restrict__ coef,
                                                        const float* __restrict__ C_old, float* __restrict__ C_new,
                                                        int64_t* __restrict__ counts, int32_t* __restrict__ iters,
                                                        int max_iters, double tol) {
    extern __shared__ __align__(16) unsigned char smem[];
    double* x = reinterpret_cast<double*>(smem);    // [d] solution
    double* r = x + d;                              // [d] residual
    double* p = r + d;                              // [d] search direction
    double* q = p + d;                              // [d] A p
    __shared__ double red[kVT];
    const int c = blockIdx.x;
    const int64_t m0 = offs[c];
    const int64_t m = offs[c + 1] - m0;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) {
        if (counts) counts[c] = m;
    }
    if (m == 0) {
        for (int t = tid; t < d; t += kVT) C_new[static_cast<int64_t>(c) * d + t] = C_old[static_cast<int64_t>(c) * d + t];
        if (tid == 0 && iters) iters[c] = 0;
        return;
    }
    // per member: 1/||x|| and eta (warp per member; lanes stride the row, then
    // a fixed shuffle tree)
    for (int64_t k = warp; k < m; k += kVT / 32) {
        const float* xr = X + static_cast<int64_t>(members[m0 + k]) * d;
        double s = 0.0;
        for (int t = lane; t < d; t += 32) {
            const double v = static_cast<double>(xr[t]);
            s = fma(v, v, s);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) s = __dadd_rn(s, __shfl_xor_sync(0xFFFFFFFFu, s, off));
        if (lane == 0) {
            const double norm = sqrt(s);
            double eta = 1.0;
            if (T > 0.0 && norm > 0.0) {
                const double tn = T / norm;
                const double tt = tn * tn;
                if (tt < 1.0) eta = static_cast<double>(d - 1) * tt / (1.0 - tt);
            }
            mscal[2 * (m0 + k)] = norm > 0.0 ? 1.0 / norm : 0.0;
            mscal[2 * (m0 + k) + 1] = eta;
        }
    }
    __syncthreads();
    // b = sum_i eta_i x_i (each coordinate by one thread, members in order);
    // x = 0, r = p = b
    double bb_part = 0.0;
    for (int t = tid; t < d; t += kVT) {
        double acc = 0.0;
        for (int64_t k = 0; k < m; ++k)
            acc = fma(mscal[2 * (m0 + k) + 1], static_cast<double>(X[static_cast<int64_t>(members[m0 + k]) * d + t]), acc);
        x[t] = 0.0;
        r[t] = acc;
        p[t] = acc;
        bb_part = fma(acc, acc, bb_part);
    }
    const double bb = block_sum(bb_part, red);
    double rr = bb;
    const double md = static_cast<double>(m);
    int it = 0;
    while (it < max_iters && rr > tol * tol * bb) {
        // coef_i = w_i (u_i . p) / ||x_i|| = w_i inv_i^2 (x_i . p)
        for (int64_t k = warp; k < m; k += kVT / 32) {
            const float* xr = X + static_cast<int64_t>(members[m0 + k]) * d;
            double s = 0.0;
            for (int t = lane; t < d; t += 32) s = fma(static_cast<double>(xr[t]), p[t], s);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) s = __dadd_rn(s, __shfl_xor_sync(0xFFFFFFFFu, s, off));
            if (lane == 0) {
                const double inv = mscal[2 * (m0 + k)];
                const double w = mscal[2 * (m0 + k) + 1] - 1.0;
                coef[m0 + k] = w * inv * inv * s;
            }
        }
        __syncthreads();
        // q = m p + sum_i coef_i x_i
        double pq_part = 0.0;
        for (int t = tid; t < d; t += kVT) {
            double acc = 0.0;
            for (int64_t k = 0; k < m; ++k)
                acc = fma(coef[m0 + k], static_cast<double>(X[static_cast<int64_t>(members[m0 + k]) * d + t]), acc);
            const double qt = fma(md, p[t], acc);
            q[t] = qt;
            pq_part = fma(p[t], qt, pq_part);
        }
        const double pq = block_sum(pq_part, red);
        if (!(pq > 0.0)) break;              // not positive definite (or p = 0): stop where we are
        const double alpha = rr / pq;
        double rn_part = 0.0;
        for (int t = tid; t < d; t += kVT) {
            x[t] = fma(alpha, p[t], x[t]);
            const double rt = fma(-alpha, q[t], r[t]);
            r[t] = rt;
            rn_part = fma(rt, rt, rn_part);
        }
        const double rn = block_sum(rn_part, red);
        const double beta = rn / rr;
        for (int t = tid; t < d; t += kVT) p[t] = fma(beta, p[t], r[t]);
        rr = rn;
        ++it;
        __syncthreads();
    }
    for (int t = tid; t < d; t += kVT) C_new[static_cast<int64_t>(c) * d + t] = __double2float_rn(x[t]);
    if (tid == 0 && iters) iters[c] = it;
}

}  // namespace

size_t avq_solve_smem_bytes(int d) { return static_cast<size_t>(4) * d * sizeof(double); }

size_t avq_workspace_bytes(int64_t n, int nl) {
    auto al = [](size_t b) { return (b + 255) / 256 * 256; };
    return al(sizeof(int32_t) * static_cast<size_t>(nl)) + al(sizeof(int64_t) * (static_cast<size_t>(nl) + 1)) +
           al(sizeof(int32_t) * static_cast<size_t>(n)) + al(2 * sizeof(double) * static_cast<size_t>(n)) +
           al(sizeof(double) * static_cast<size_t>(n));
}

cudaError_t launch_avq_update(const float* X, int64_t n, int d, const int32_t* assign, int nl, const float* C_old,
                              double T, float* C_new, int64_t* counts, int32_t* iters, int max_iters, double tol,
                              void* workspace, cudaStream_t s) {
    auto al = [](size_t b) { return (b + 255) / 256 * 256; };
    char* w = static_cast<char*>(workspace);
    int32_t* cnt = reinterpret_cast<int32_t*>(w);
    w += al(sizeof(int32_t) * static_cast<size_t>(nl));
    int64_t* offs = reinterpret_cast<int64_t*>(w);
    w += al(sizeof(int64_t) * (static_cast<size_t>(nl) + 1));
    int32_t* members = reinterpret_cast<int32_t*>(w);
    w += al(sizeof(int32_t) * static_cast<size_t>(n));
    double* mscal = reinterpret_cast<double*>(w);
    w += al(2 * sizeof(double) * static_cast<size_t>(n));
    double* coef = reinterpret_cast<double*>(w);
    cudaError_t e = cudaMemsetAsync(cnt, 0, sizeof(int32_t) * static_cast<size_t>(nl), s);
    if (e != cudaSuccess) return e;
    if (n > 0) {
        avq_count_kernel<<<static_cast<unsigned>((n + kVT - 1) / kVT), kVT, 0, s>>>(assign, n, nl, cnt);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    avq_offsets_kernel<<<1, 1024, 0, s>>>(cnt, nl, offs);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (n > 0) {
        avq_fill_kernel<<<(nl + kFillC - 1) / kFillC, kVT, 0, s>>>(assign, n, nl, offs, members);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    const size_t smem = avq_solve_smem_bytes(d);
    if ((e = cudaFuncSetAttribute(avq_solve_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(smem))) != cudaSuccess)
        return e;
    avq_solve_kernel<<<nl, kVT, smem, s>>>(X, d, members, offs, T, mscal, coef, C_old, C_new, counts, iters,
                                            max_iters, tol);
    return cudaGetLastError();
}

}  // namespace ah
