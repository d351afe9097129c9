// Centroid scores on the 5th-generation tensor cores (ScaNN blog post, "Three
// stages of a search": a query scores every centroid, s[q][c] = q . c).
//
// S = Q C^T is a dense fp32 contraction.  The tensor cores take tf32 operands
// (10 explicit mantissa bits), so each operand x is split into x_hi = x with
// its 13 low mantissa bits cleared (exact in tf32) and x_lo = x - x_hi (exact
// in fp32, rounded to tf32 by the MMA), and
//     q . c  ~  q_hi . c_hi + q_hi . c_lo + q_lo . c_hi;
// the dropped q_lo . c_lo term and the rounding of the lo parts are below
// 2^-21 of sum |q_t c_t| <= |q| |c|.  Integer-valued data of at most 11
// significant bits (e.g. coordinates 0..255) splits with lo = 0 and its
// products and sums stay exact.
//
// The MMA's fp32 accumulation rounds toward zero, so its error grows with the
// number of accumulations into one accumulator rather than as a random walk.
// Tensor memory therefore holds four 128-column fp32 accumulators per tile:
// three take the hi . hi products of every third K slice in turn, the fourth
// the (2^-10 smaller) cross terms; the epilogue adds the four with IEEE
// round-to-nearest.  At d = 1536 each hi . hi accumulator sees 64 MMAs, so
// the accumulated error stays below about 64 ulps of sum |q_t c_t| (4e-6 on
// unit vectors); d is limited to 4096 (171 MMAs, 1e-5).
//
// One CTA computes a 128 x 128 tile of S: one thread (warp 0) issues the TMA
// loads of 16-wide K slices of Q_hi, Q_lo and C_hi, C_lo (128 rows each) into a
// six-stage ring (64-byte swizzle, mbarrier completion), another (warp 1)
// waits for each slice and issues tcgen05.mma kind::tf32 (M = N = 128, K = 8;
// three per half slice), committing the stage free, and the four warps then
// read the accumulators back with tcgen05.ld and store the sums.
// Every mbarrier wait is bounded: on expiry the kernel records an error,
// waits (bounded) for its own transfers, frees its tensor memory and returns.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <mutex>

#include "kernels.h"

namespace ah {

namespace {

constexpr int kTcM = 128;                  // queries per tile
constexpr int kTcN = 128;                  // centroids per tile
constexpr int kTcK = 16;                   // fp32 K elements per stage (64 bytes per row)
constexpr int kTcStages = 6;
constexpr int kTcThreads = 128;
constexpr uint32_t kATileBytes = kTcM * kTcK * 4;          // 8 KB
constexpr uint32_t kBTileBytes = kTcN * kTcK * 4;          // 8 KB
constexpr uint32_t kStageBytes = 2 * kATileBytes + 2 * kBTileBytes;   // 32 KB
constexpr uint32_t kTmemCols = 512;                        // 4 accumulators of kTcN columns
constexpr int kMaxTcD = 4096;
constexpr long long kWaitLimit = 1ll << 26;                // polls before a wait gives up

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

// Bounded wait for the barrier's phase with the given parity; false if the
// limit ran out.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
    const uint32_t a = smem_u32(bar);
    for (long long i = 0; i < kWaitLimit; ++i) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.b32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(a), "r"(parity)
            : "memory");
        if (done) return true;
    }
    return false;
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// Shared-memory matrix descriptor of a K-major tile with 64-byte swizzle:
// rows of 64 bytes, 8-row atoms of 512 bytes (stride byte offset), leading
// byte offset unused (1), descriptor version 1, layout type 4 (64B swizzle).
__device__ __forceinline__ uint64_t sw64_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFF);
    d |= static_cast<uint64_t>(1) << 16;                    // leading byte offset (16-byte units)
    d |= static_cast<uint64_t>(512 >> 4) << 32;             // stride byte offset (16-byte units)
    d |= static_cast<uint64_t>(1) << 46;                    // version
    d |= static_cast<uint64_t>(4) << 61;                    // 64-byte swizzle
    return d;
}

// Instruction descriptor: fp32 accumulator, tf32 A and B, both K-major,
// N = 128, M = 128.
constexpr uint32_t kIdesc = (1u << 4) | (2u << 7) | (2u << 10) | (static_cast<uint32_t>(kTcN >> 3) << 17) |
                            (static_cast<uint32_t>(kTcM >> 4) << 24);

__device__ __forceinline__ void mma_tf32(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t accumulate) {
    const uint32_t z = 0;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}"
        ::"r"(tmem_d), "l"(da), "l"(db), "r"(kIdesc), "r"(accumulate), "r"(z), "r"(z), "r"(z), "r"(z));
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__global__ void __launch_bounds__(kTcThreads, 1) centroid_scores_tc_kernel(
    const __grid_constant__ CUtensorMap qhi, const __grid_constant__ CUtensorMap qlo,
    const __grid_constant__ CUtensorMap chi, const __grid_constant__ CUtensorMap clo, float* __restrict__ S,
    int nq, int nl, int d, int* __restrict__ err) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    extern __shared__ unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t full[kTcStages];
    __shared__ __align__(8) uint64_t empty[kTcStages];
    __shared__ __align__(8) uint64_t done;
    __shared__ uint32_t s_tmem;
    __shared__ int s_fail, s_issued, s_consumed;
    // 1024-byte aligned stage buffers (the swizzle pattern repeats every 512 B)
    unsigned char* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int m0 = blockIdx.y * kTcM, n0 = blockIdx.x * kTcN;
    const int KT = (d + kTcK - 1) / kTcK;

    if (tid == 0) {
        for (int s = 0; s < kTcStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(&done, 1);
        s_fail = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s_tmem)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = s_tmem;

    auto stage_ptr = [&](int s) { return smem + static_cast<size_t>(s) * kStageBytes; };
    if (tid == 0) {
        // producer: a stage is refilled once the MMAs that read it are done
        int kt = 0;
        for (; kt < KT; ++kt) {
            const int s = kt % kTcStages;
            if (kt >= kTcStages && !mbar_wait(&empty[s], ((kt / kTcStages) + 1) & 1)) {
                s_fail = 1;
                break;
            }
            unsigned char* p = stage_ptr(s);
            mbar_expect_tx(&full[s], kStageBytes);
            const int k0 = kt * kTcK;
            tma_load_2d(p, &qhi, &full[s], k0, m0);
            tma_load_2d(p + kATileBytes, &qlo, &full[s], k0, m0);
            tma_load_2d(p + 2 * kATileBytes, &chi, &full[s], k0, n0);
            tma_load_2d(p + 2 * kATileBytes + kBTileBytes, &clo, &full[s], k0, n0);
        }
        s_issued = kt;
    } else if (tid == 32) {
        // MMA issuer: hi . hi into accumulator kt % 3 (slices kt < 3 start
        // it), the cross terms into accumulator 3 (slice 0 starts it)
        int kt = 0;
        for (; kt < KT; ++kt) {
            const int s = kt % kTcStages;
            if (!mbar_wait(&full[s], (kt / kTcStages) & 1)) {
                s_fail = 1;
                break;
            }
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            const uint32_t a_hi = smem_u32(stage_ptr(s));
            const uint32_t a_lo = a_hi + kATileBytes;
            const uint32_t b_hi = a_hi + 2 * kATileBytes;
            const uint32_t b_lo = b_hi + kBTileBytes;
            const uint32_t main = tmem + static_cast<uint32_t>((kt % 3) * kTcN);
            const uint32_t cross = tmem + static_cast<uint32_t>(3 * kTcN);
#pragma unroll
            for (int kk = 0; kk < kTcK / 8; ++kk) {
                const uint32_t off = kk * 32;     // 8 tf32 = 32 bytes along the swizzled row
                mma_tf32(main, sw64_desc(a_hi + off), sw64_desc(b_hi + off), (kt >= 3 || kk > 0) ? 1u : 0u);
                mma_tf32(cross, sw64_desc(a_hi + off), sw64_desc(b_lo + off), (kt > 0 || kk > 0) ? 1u : 0u);
                mma_tf32(cross, sw64_desc(a_lo + off), sw64_desc(b_hi + off), 1u);
            }
            mma_commit(&empty[s]);
        }
        mma_commit(&done);                    // arrives once every MMA issued above has completed
        s_consumed = kt;
    }
    // a failed wait can leave loads the MMA thread never consumed: let them
    // land (bounded) before this CTA's shared memory goes away
    __syncthreads();
    if (tid == 0 && s_fail) {
        atomicCAS(err, 0, kDevTimeout);
        for (int j = s_consumed; j < s_issued; ++j) mbar_wait(&full[j % kTcStages], (j / kTcStages) & 1);
    }
    __syncthreads();
    // epilogue: warp w reads accumulator lanes 32w .. 32w + 31 (its rows)
    const bool ready = __all_sync(0xFFFFFFFFu, mbar_wait(&done, 0)) && !s_fail;
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (ready) {
        const int row = m0 + warp * 32 + lane;
        float* out = S + static_cast<int64_t>(row) * nl;
        const bool vec = (nl % 4) == 0;
        const uint32_t lanes = static_cast<uint32_t>(warp * 32) << 16;
        for (int c0 = 0; c0 < kTcN; c0 += 32) {
            // ((acc0 + acc1) + acc2) + cross, IEEE fp32 adds; an accumulator
            // no slice reached (fewer than 3 slices) is left out
            uint32_t r[32], t[32];
            tmem_ld32(tmem + lanes + c0, r);
            for (int a = 1; a < 4; ++a) {
                if (a < 3 && a >= KT) continue;
                tmem_ld32(tmem + lanes + static_cast<uint32_t>(a * kTcN) + c0, t);
#pragma unroll
                for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(__fadd_rn(__uint_as_float(r[j]), __uint_as_float(t[j])));
            }
            if (row < nq) {
                const int col = n0 + c0;
                if (vec && col + 32 <= nl) {
#pragma unroll
                    for (int j = 0; j < 32; j += 4)
                        *reinterpret_cast<float4*>(out + col + j) =
                            make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]), __uint_as_float(r[j + 2]),
                                        __uint_as_float(r[j + 3]));
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (col + j < nl) out[col + j] = __uint_as_float(r[j]);
                }
            }
        }
    } else if (tid == 0) {
        atomicCAS(err, 0, kDevTimeout);
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
}

// x -> (x with its 13 low mantissa bits cleared, x minus that)
__global__ void split_tf32_kernel(const float* __restrict__ x, int64_t n, float* __restrict__ hi,
                                  float* __restrict__ lo) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const float v = x[i];
    const float h = __uint_as_float(__float_as_uint(v) & 0xFFFFE000u);
    hi[i] = h;
    lo[i] = __fsub_rn(v, h);
}

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

cudaError_t encode_rows(CUtensorMap* map, const float* base, int rows, int d, int box_rows) {
    std::call_once(g_encode_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    if (!g_encode) return cudaErrorNotSupported;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(d) * sizeof(float)};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(kTcK), static_cast<cuuint32_t>(box_rows)};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides, box,
                                estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace

size_t centroid_tc_smem_bytes() { return static_cast<size_t>(kTcStages) * kStageBytes + 1024; }

bool centroid_tc_usable(int nq, int nl, int d) {
    // row strides of whole 16-byte units for the tensor maps, extents of at
    // least one box, and enough tiles to be worth a 192 KB CTA (smaller
    // problems use the SIMT tiles)
    return d % 4 == 0 && d >= kTcK && d <= kMaxTcD && nq >= kTcM && nl >= kTcN &&
           static_cast<int64_t>(nq) * nl >= (int64_t(1) << 20);
}

cudaError_t launch_split_tf32(const float* x, int64_t n, float* hi, float* lo, cudaStream_t s) {
    if (n <= 0) return cudaSuccess;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>((n + 255) / 256));
    cfg.blockDim = dim3(256);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, split_tf32_kernel, x, n, hi, lo);
    return e == cudaSuccess ? cudaGetLastError() : e;
}

cudaError_t launch_centroid_scores_tc(const float* q_hi, const float* q_lo, const float* c_hi, const float* c_lo,
                                      float* S, int nq, int nl, int d, int* err, cudaStream_t s) {
    CUtensorMap m[4];
    cudaError_t e;
    if ((e = encode_rows(&m[0], q_hi, nq, d, kTcM)) != cudaSuccess) return e;
    if ((e = encode_rows(&m[1], q_lo, nq, d, kTcM)) != cudaSuccess) return e;
    if ((e = encode_rows(&m[2], c_hi, nl, d, kTcN)) != cudaSuccess) return e;
    if ((e = encode_rows(&m[3], c_lo, nl, d, kTcN)) != cudaSuccess) return e;
    const size_t smem = centroid_tc_smem_bytes();
    {
        // the shared-memory limit is raised once per device
        static std::mutex mu;
        static bool set[64] = {};
        int dev = 0;
        if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
        std::lock_guard<std::mutex> lock(mu);
        if (dev < 0 || dev >= 64 || !set[dev]) {
            e = cudaFuncSetAttribute(centroid_scores_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(smem));
            if (e != cudaSuccess) return e;
            if (dev >= 0 && dev < 64) set[dev] = true;
        }
    }
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((nl + kTcN - 1) / kTcN, (nq + kTcM - 1) / kTcM);
    cfg.blockDim = dim3(kTcThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, centroid_scores_tc_kernel, m[0], m[1], m[2], m[3], S, nq, nl, d, err);
    return e == cudaSuccess ? cudaGetLastError() : e;
}

}  // namespace ah
