// The 4-bit code scan with uint8 tables on the int8 tensor cores (ScaNN blog
// post, "Three stages of a search": a point's approximate score is the sum of
// its table entries, one per block).
//
// With uint8 tables the sum for query q and point p is an integer,
//     sum(q, p) = sum_b lut8[q][b][code_b(p)] = sum_{b, j} lut8[q][b][j] * [code_b(p) == j],
// the product of the query's table row (A, B x 16 bytes) with the point's
// one-hot code expansion (B, B x 16 bytes of 0/1).  tcgen05.mma kind::i8
// multiplies unsigned bytes and accumulates in int32, exactly, so the sums are
// the same integers the table lookups give, whatever the order: the result
// is bit-identical to the lookup scan, the threshold sample and the rescan.
//
// A work item is (leaf, up to 128 of its queries, 256 of its points).  Per
// slice of 8 blocks (128 bytes of K) the CTA stages the queries' table bytes
// (A: 128 rows x 128 B) and builds the points' one-hot rows from their code
// word (B: 256 rows x 128 B), both K-major with the 128-byte swizzle, while
// the tensor core multiplies the previous slice (two stages; an MMA commit on
// an mbarrier frees a stage).  The 128 x 256 int32 accumulator lives in
// tensor memory; four warps read it back (one query per lane) and keep the
// points whose sum reaches the query's bound, as the lookup scan does.  Every
// mbarrier wait is bounded; on expiry the kernel records an error in the
// index's error word, drains its own MMAs (bounded), frees its tensor memory
// and returns.
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.h"

namespace ah {

namespace {

constexpr int kQM = 128;                           // queries per item (MMA M)
constexpr int kPN = 256;                           // points per item (MMA N): 8 code tiles
constexpr int kSliceK = 128;                       // bytes of K per slice: 8 blocks x 16 centers
constexpr int kThreads = 256;
constexpr uint32_t kABytes = kQM * kSliceK;        // 16 KB
constexpr uint32_t kBBytes = kPN * kSliceK;        // 32 KB
constexpr uint32_t kStage = kABytes + kBBytes;     // 48 KB
constexpr uint32_t kTmemCols = kPN;                // int32 accumulator columns
constexpr long long kWaitLimit = 1ll << 26;
// int32 accumulator, unsigned 8-bit A and B, both K-major, N = 256, M = 128
constexpr uint32_t kIdesc = (2u << 4) | (0u << 7) | (0u << 10) | (static_cast<uint32_t>(kPN >> 3) << 17) |
                            (static_cast<uint32_t>(kQM >> 4) << 24);

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

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

// K-major tile with 128-byte rows and the 128-byte swizzle: 8-row atoms of
// 1 KB (stride byte offset), leading byte offset unused, version 1, layout 2.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFF);
    d |= static_cast<uint64_t>(1) << 16;
    d |= static_cast<uint64_t>(1024 >> 4) << 32;
    d |= static_cast<uint64_t>(1) << 46;
    d |= static_cast<uint64_t>(2) << 61;
    return d;
}

// Byte offset of 16-byte chunk c (0..7) of row r in a 128-byte-swizzled tile.
__device__ __forceinline__ uint32_t sw128_off(int r, int c) {
    return static_cast<uint32_t>(r * 128 + ((c ^ (r & 7)) << 4));
}

__device__ __forceinline__ void mma_i8(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t accumulate) {
    const uint32_t z = 0;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}"
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

// Word w of lane `lane` within a tile of the code copy ([W/V][32][V] words).
__device__ __forceinline__ int tc_code_word(int w, int lane, int V) {
    const int r = w & (V - 1);
    return (w - r) * 32 + lane * V + r;
}

__global__ void __launch_bounds__(kThreads, 2) scan_tc_kernel(DeviceIndex ix, SearchArgs a, SearchBuffers b) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    extern __shared__ unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t empty[2];
    __shared__ __align__(8) uint64_t done;
    __shared__ uint32_t s_tmem;
    __shared__ int s_item, s_leaf;
    __shared__ int s_q[kQM];
    __shared__ uint32_t s_th[kQM], s_tl[kQM];
    unsigned char* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int B = ix.B, row_bytes = B * 16, S = (B + 7) / 8;
    const int total_items = b.item_off[ix.nl];

    if (tid == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&empty[0])) : "memory");
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&empty[1])) : "memory");
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&done)) : "memory");
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

    uint32_t g = 0;              // slices issued by this CTA (stage = g & 1)
    uint32_t done_phase = 0;
    bool ok = true;
    for (;;) {
        __syncthreads();
        if (tid == 0) {
            const int item = atomicAdd(&b.counters[a.scan_counter], 1);
            s_item = item;
            if (item < total_items) {
                int lo = 0, hi = ix.nl;
                while (lo < hi) {
                    const int mid = (lo + hi + 1) >> 1;
                    if (b.item_off[mid] <= item) lo = mid; else hi = mid - 1;
                }
                s_leaf = lo;
            }
        }
        __syncthreads();
        const int item = s_item;
        if (item >= total_items) break;
        const int leaf = s_leaf;
        const int pt0 = ix.ptile[leaf], ntile = ix.ptile[leaf + 1] - pt0;
        const int npc = (ntile + (kPN / 32) - 1) / (kPN / 32);
        const int local = item - b.item_off[leaf];
        const int qt = local / npc, c = local - qt * npc;
        const int m = min(kQM, b.qcount[leaf] - qt * kQM);
        const int t0 = pt0 + c * (kPN / 32), t1 = min(pt0 + ntile, t0 + kPN / 32);
        const int slot_base = ix.offs[leaf] - 32 * pt0, send = ix.offs[leaf + 1];
        if (tid < kQM) {
            const int qq = (tid < m) ? b.qlist[b.qoff[leaf] + qt * kQM + tid] : -1;
            s_q[tid] = qq;
            const uint64_t t = (qq >= 0) ? b.tau[qq] : ~0ull;
            s_th[tid] = static_cast<uint32_t>(t >> 32);
            s_tl[tid] = static_cast<uint32_t>(t);
        }
        __syncthreads();
        // the point this thread expands into one-hot rows
        const int pn = tid;                                   // 0 .. 255
        const int ptile_i = t0 + (pn >> 5);
        const bool p_in = ptile_i < t1;
        const uint32_t* ptw = ix.codes_il + static_cast<int64_t>(p_in ? ptile_i : t0) * ix.W * 32;
        for (int s = 0; s < S; ++s, ++g) {
            const uint32_t stage = g & 1u;
            unsigned char* st = smem + stage * kStage;
            // the stage is free once the MMAs of slice g - 2 are done: thread
            // 0 waits, the barrier shares the outcome with every thread
            const int late = (tid == 0 && g >= 2) ? !mbar_wait(&empty[stage], ((g >> 1) + 1) & 1u) : 0;
            if (__syncthreads_or(late)) {
                ok = false;
                break;
            }
            // A: the queries' table bytes of blocks 8s .. 8s+7 (zero past the
            // table's end and for rows without a query)
#pragma unroll
            for (int i = 0; i < (kQM * 8) / kThreads; ++i) {
                const int idx = tid + kThreads * i;
                const int r = idx >> 3, ch = idx & 7;
                const int k0 = s * kSliceK + ch * 16;
                const int qq = s_q[r];
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if (qq >= 0 && k0 < row_bytes)
                    v = *reinterpret_cast<const uint4*>(b.lut_u8 + static_cast<int64_t>(qq) * row_bytes + k0);
                *reinterpret_cast<uint4*>(st + sw128_off(r, ch)) = v;
            }
            // B: one-hot rows of this thread's point for blocks 8s .. 8s+7
            const uint32_t code = p_in ? ptw[tc_code_word(s, pn & 31, ix.V)] : 0u;
            unsigned char* bt = st + kABytes;
#pragma unroll
            for (int blk = 0; blk < 8; ++blk) {
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if (8 * s + blk < B) {
                    const uint32_t nib = (code >> (4 * blk)) & 15u;
                    const uint32_t one = 1u << (8 * (nib & 3u));
                    const uint32_t w = nib >> 2;
                    v = make_uint4(w == 0 ? one : 0u, w == 1 ? one : 0u, w == 2 ? one : 0u, w == 3 ? one : 0u);
                }
                *reinterpret_cast<uint4*>(bt + sw128_off(pn, blk)) = v;
            }
            // the generic-proxy stores above must be visible to the tensor core
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncthreads();
            if (tid == 0) {
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                const uint32_t a_addr = smem_u32(st), b_addr = a_addr + kABytes;
#pragma unroll
                for (int kk = 0; kk < kSliceK / 32; ++kk)   // K = 32 bytes per MMA
                    mma_i8(tmem, sw128_desc(a_addr + 32 * kk), sw128_desc(b_addr + 32 * kk),
                           (s > 0 || kk > 0) ? 1u : 0u);
                mma_commit(&empty[stage]);
            }
        }
        // every MMA of the item done (thread 0 waits; the barrier shares it)
        int late = 0;
        if (tid == 0) {
            mma_commit(&done);
            late = !mbar_wait(&done, done_phase);
            if (!ok || late) atomicCAS(b.err, 0, kDevTimeout);
        }
        const bool ready = !__syncthreads_or(late);
        done_phase ^= 1u;
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        // epilogue: warp w < 4 reads accumulator lanes 32w .. 32w + 31, one
        // query per lane, and keeps the points whose sum reaches its bound
        if (warp < 4 && ok && ready) {
            const int qr = warp * 32 + lane;
            const int q = s_q[qr];
            const uint32_t th = s_th[qr], tl = s_tl[qr];
            for (int c0 = 0; c0 < kPN; c0 += 32) {
                uint32_t r[32];
                tmem_ld32(tmem + (static_cast<uint32_t>(warp * 32) << 16) + static_cast<uint32_t>(c0), r);
                if (q < 0) continue;
                const int tile = t0 + (c0 >> 5);
                if (tile >= t1) continue;
                const int sb = slot_base + 32 * tile;
                uint32_t passm = 0u;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int slot = sb + j;
                    bool pass = slot < send && r[j] >= th;
                    if (pass && r[j] == th) pass = (0xFFFFFFFFu - static_cast<uint32_t>(ix.slot_ids[slot])) >= tl;
                    if (pass) passm |= 1u << j;
                }
                if (passm) {
                    int pos = atomicAdd(&b.count[q], __popc(passm));
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        if (passm & (1u << j)) {
                            if (pos < b.cap) {
                                const int slot = sb + j;
                                const int64_t o = static_cast<int64_t>(q) * b.cap + pos;
                                b.ckey[o] = make_key(r[j], ix.slot_ids[slot]);
                                b.cslot[o] = slot;
                            }
                            ++pos;
                        }
                    }
                }
            }
        }
        asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
        if (!ok || !ready) break;
    }
    // leave no MMA in flight: the last commit covers every earlier one
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
}

}  // namespace

int scan_tc_group() { return kQM; }
int scan_tc_chunk_tiles() { return kPN / 32; }
size_t scan_tc_smem_bytes() { return 2 * static_cast<size_t>(kStage) + 1024; }

cudaError_t launch_scan_tc(const DeviceIndex& ix, const SearchArgs& a, const SearchBuffers& b, int num_sms,
                           cudaStream_t s) {
    const size_t smem = scan_tc_smem_bytes();
    cudaError_t e;
    {
        static bool set[64] = {};
        int dev = 0;
        if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
        if (dev < 0 || dev >= 64 || !set[dev]) {
            e = cudaFuncSetAttribute(scan_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
            if (e != cudaSuccess) return e;
            if (dev >= 0 && dev < 64) set[dev] = true;
        }
    }
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(num_sms * 2);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, scan_tc_kernel, ix, a, b);
    return e == cudaSuccess ? cudaGetLastError() : e;
}

}  // namespace ah
