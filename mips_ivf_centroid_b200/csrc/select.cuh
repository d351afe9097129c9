// CTA-wide selection of the K largest 64-bit keys (radix select, MSB first,
// 8 bits per pass) and a bitonic sort of the selected keys.  Used for every
// "keep the best N" step of the search: leaves, candidates, final neighbours.
// Keys are distinct by construction (the low 32 bits encode the id), so the
// K-th largest key is unique and exactly K keys are selected.
#pragma once

#include <cstdint>

#include "common.cuh"

namespace ah {

// Shared scratch for block_select_threshold: 256 histogram bins + bookkeeping.
struct SelectScratch {
    int hist[256];
    int bucket;
    int above;
    int count;
    unsigned long long kand;
    unsigned long long kor;
};

// Among the warp's 256 bins (lane l owns bins 8l..8l+7), find the bucket b where
// the count of keys in bins above b is < need <= count in bins >= b.  Lane 0
// writes the bucket and the count strictly above it.
__device__ __forceinline__ void find_bucket_warp(SelectScratch& s, int need) {
    const int lane = threadIdx.x & 31;
    int local = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) local += s.hist[lane * 8 + i];
    // suffix sum over lanes: sum of lanes >= lane
    int suf = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        int v = __shfl_down_sync(0xFFFFFFFFu, suf, off);
        if (lane + off < 32) suf += v;
    }
    const int above_lane = suf - local;   // keys in lanes above this one
    const bool here = (above_lane < need) && (suf >= need);
    if (here) {
        int acc = above_lane;
        for (int i = 7; i >= 0; --i) {
            int h = s.hist[lane * 8 + i];
            if (acc + h >= need) {
                s.bucket = lane * 8 + i;
                s.above = acc;
                break;
            }
            acc += h;
        }
    }
}

// Radix select over n keys given by get(i).  On return (*prefix, *mask) define
// the selection: key selected  <=>  (key & mask) >= prefix, which holds for
// exactly K keys when keys are distinct.  Requires 1 <= K <= n.  All threads
// of the block must call it; NT must be a multiple of 32.
template <int NT, class GetKey>
__device__ void block_select_threshold(GetKey get, int n, int K, SelectScratch& s,
                                       uint64_t* prefix_out, uint64_t* mask_out) {
    // Bytes every key shares carry no information: find the first byte (from
    // the top) where keys differ with a block AND/OR reduction and start there.
    uint64_t kand = ~0ull, kor = 0ull;
    for (int i = threadIdx.x; i < n; i += NT) {
        const uint64_t k = get(i);
        kand &= k;
        kor |= k;
    }
    const unsigned a_hi = __reduce_and_sync(0xFFFFFFFFu, static_cast<unsigned>(kand >> 32));
    const unsigned a_lo = __reduce_and_sync(0xFFFFFFFFu, static_cast<unsigned>(kand));
    const unsigned o_hi = __reduce_or_sync(0xFFFFFFFFu, static_cast<unsigned>(kor >> 32));
    const unsigned o_lo = __reduce_or_sync(0xFFFFFFFFu, static_cast<unsigned>(kor));
    if (threadIdx.x == 0) {
        s.kand = ~0ull;
        s.kor = 0ull;
    }
    __syncthreads();
    if ((threadIdx.x & 31) == 0) {
        atomicAnd(&s.kand, (static_cast<unsigned long long>(a_hi) << 32) | a_lo);
        atomicOr(&s.kor, (static_cast<unsigned long long>(o_hi) << 32) | o_lo);
    }
    __syncthreads();
    const uint64_t diff = s.kand ^ s.kor;
    int shift = 56;
    uint64_t prefix = 0, mask = 0;
    if (diff != 0ull) {
        const int top = 63 - __clzll(static_cast<long long>(diff));   // highest differing bit
        shift = (top / 8) * 8;
        mask = (shift >= 56) ? 0ull : (~0ull << (shift + 8));
        prefix = s.kand & mask;
    }
    int need = K;
    for (; shift >= 0; shift -= 8) {
        for (int i = threadIdx.x; i < 256; i += NT) s.hist[i] = 0;
        if (threadIdx.x == 0) {
            s.bucket = 0;
            s.above = 0;
        }
        __syncthreads();
        // histogram; lanes of a warp that hit the same bin add once (keys of
        // close scores share their top bits, so one bin is typically hot)
        const int lane = threadIdx.x & 31;
        for (int base = 0; base < n; base += NT) {
            const int i = base + threadIdx.x;
            bool take = false;
            int bin = 256 + lane;                       // unique dummy for idle lanes
            if (i < n) {
                uint64_t k = get(i);
                take = (k & mask) == prefix;
                if (take) bin = static_cast<int>((k >> shift) & 255);
            }
            const unsigned peers = __match_any_sync(0xFFFFFFFFu, bin);
            if (take && lane == __ffs(peers) - 1) atomicAdd(&s.hist[bin], __popc(peers));
        }
        __syncthreads();
        if (threadIdx.x < 32) find_bucket_warp(s, need);
        __syncthreads();
        const int b = s.bucket;
        const int cnt_b = s.hist[b];
        need -= s.above;
        prefix |= static_cast<uint64_t>(b) << shift;
        mask |= 0xFFull << shift;
        __syncthreads();   // everyone has read bucket/above/hist before the next pass clears them
        if (cnt_b == need) break;
    }
    *prefix_out = prefix;
    *mask_out = mask;
}

// Bitonic sort (descending) of keys[0..P2) with int payloads, P2 a power of two.
template <int NT>
__device__ void block_sort_desc(uint64_t* keys, int32_t* vals, int P2) {
    for (int size = 2; size <= P2; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            __syncthreads();
            for (int t = threadIdx.x; t < (P2 >> 1); t += NT) {
                int i = 2 * t - (t & (stride - 1));
                int j = i + stride;
                bool desc = ((i & size) == 0);
                uint64_t a = keys[i], b = keys[j];
                bool swap = desc ? (a < b) : (a > b);
                if (swap) {
                    keys[i] = b;
                    keys[j] = a;
                    if (vals) {
                        int32_t t2 = vals[i];
                        vals[i] = vals[j];
                        vals[j] = t2;
                    }
                }
            }
        }
    }
    __syncthreads();
}

__host__ __device__ __forceinline__ int next_pow2(int x) {
    int p = 1;
    while (p < x) p <<= 1;
    return p;
}

// Select the K = min(K, n) largest keys of get(i) (payload pay(i)) into
// out_keys/out_vals (shared, capacity >= next_pow2(K)), sorted descending
// (unless `sort` is false: then in no particular order).
// Returns K.  Slots K..next_pow2(K)-1 hold key 0.  err is raised if more than
// K keys qualify (duplicate keys).
template <int NT, class GetKey, class GetVal>
__device__ int block_topk(GetKey get, GetVal pay, int n, int K, SelectScratch& s,
                          uint64_t* out_keys, int32_t* out_vals, int* err, bool sort = true) {
    if (K > n) K = n;
    if (K <= 0) return 0;
    uint64_t prefix = 0, mask = 0;
    if (K < n) block_select_threshold<NT>(get, n, K, s, &prefix, &mask);
    const int P2 = next_pow2(K);
    for (int i = threadIdx.x; i < P2; i += NT) {
        out_keys[i] = 0ull;
        if (out_vals) out_vals[i] = -1;
    }
    if (threadIdx.x == 0) s.count = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += NT) {
        uint64_t k = get(i);
        if ((k & mask) >= prefix) {
            int pos = atomicAdd(&s.count, 1);
            if (pos < K) {
                out_keys[pos] = k;
                if (out_vals) out_vals[pos] = pay(i);
            }
        }
    }
    __syncthreads();
    if (threadIdx.x == 0 && s.count != K && err) raise_error(err, kDevSelectSize);
    if (sort) block_sort_desc<NT>(out_keys, out_vals, P2);
    return K;
}

}  // namespace ah

// ---------------------------------------------------------------------------
// Warp-cooperative versions: one warp selects for one query with no block
// barrier.  `hist` is this warp's 256-int shared histogram; outputs are this
// warp's shared arrays of capacity next_pow2(K).
// ---------------------------------------------------------------------------
namespace ah {

__device__ __forceinline__ uint64_t warp_and64(uint64_t v) {
    const unsigned hi = __reduce_and_sync(0xFFFFFFFFu, static_cast<unsigned>(v >> 32));
    const unsigned lo = __reduce_and_sync(0xFFFFFFFFu, static_cast<unsigned>(v));
    return (static_cast<uint64_t>(hi) << 32) | lo;
}
__device__ __forceinline__ uint64_t warp_or64(uint64_t v) {
    const unsigned hi = __reduce_or_sync(0xFFFFFFFFu, static_cast<unsigned>(v >> 32));
    const unsigned lo = __reduce_or_sync(0xFFFFFFFFu, static_cast<unsigned>(v));
    return (static_cast<uint64_t>(hi) << 32) | lo;
}

// Same selection rule as block_select_threshold: (key & mask) >= prefix holds
// for exactly K of n distinct keys.  Requires 1 <= K < n.
template <class GetKey>
__device__ void warp_select_threshold(GetKey get, int n, int K, int* hist, uint64_t* prefix_out, uint64_t* mask_out) {
    const int lane = threadIdx.x & 31;
    uint64_t kand = ~0ull, kor = 0ull;
    for (int i = lane; i < n; i += 32) {
        const uint64_t k = get(i);
        kand &= k;
        kor |= k;
    }
    kand = warp_and64(kand);
    kor = warp_or64(kor);
    const uint64_t diff = kand ^ kor;
    int shift = 56;
    uint64_t prefix = 0ull, mask = 0ull;
    if (diff != 0ull) {
        const int top = 63 - __clzll(static_cast<long long>(diff));
        shift = (top / 8) * 8;
        mask = (shift >= 56) ? 0ull : (~0ull << (shift + 8));
        prefix = kand & mask;
    }
    int need = K;
    for (; shift >= 0; shift -= 8) {
#pragma unroll
        for (int i = 0; i < 8; ++i) hist[lane * 8 + i] = 0;
        __syncwarp();
        for (int base = 0; base < n; base += 32) {
            const int i = base + lane;
            bool take = false;
            int bin = 256 + lane;
            if (i < n) {
                const uint64_t k = get(i);
                take = (k & mask) == prefix;
                if (take) bin = static_cast<int>((k >> shift) & 255);
            }
            const unsigned peers = __match_any_sync(0xFFFFFFFFu, bin);
            if (take && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
        }
        __syncwarp();
        int local = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) local += hist[lane * 8 + i];
        int suf = local;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int v = __shfl_down_sync(0xFFFFFFFFu, suf, off);
            if (lane + off < 32) suf += v;
        }
        const int above_lane = suf - local;
        const bool here = (above_lane < need) && (suf >= need);
        int my_bucket = 0, my_above = 0;
        if (here) {
            int acc = above_lane;
            for (int i = 7; i >= 0; --i) {
                const int h = hist[lane * 8 + i];
                if (acc + h >= need) {
                    my_bucket = lane * 8 + i;
                    my_above = acc;
                    break;
                }
                acc += h;
            }
        }
        const unsigned hb = __ballot_sync(0xFFFFFFFFu, here);
        const int src = hb ? (__ffs(hb) - 1) : 0;
        const int bucket = __shfl_sync(0xFFFFFFFFu, my_bucket, src);
        const int above = __shfl_sync(0xFFFFFFFFu, my_above, src);
        const int cnt_b = hist[bucket];
        __syncwarp();
        need -= above;
        prefix |= static_cast<uint64_t>(bucket) << shift;
        mask |= 0xFFull << shift;
        if (cnt_b == need) break;
    }
    *prefix_out = prefix;
    *mask_out = mask;
}

__device__ __forceinline__ void warp_sort_desc(uint64_t* keys, int32_t* vals, int P2) {
    const int lane = threadIdx.x & 31;
    for (int size = 2; size <= P2; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            __syncwarp();
            for (int t = lane; t < (P2 >> 1); t += 32) {
                const int i = 2 * t - (t & (stride - 1));
                const int j = i + stride;
                const bool desc = ((i & size) == 0);
                const uint64_t a = keys[i], b = keys[j];
                if (desc ? (a < b) : (a > b)) {
                    keys[i] = b;
                    keys[j] = a;
                    if (vals) {
                        const int32_t t2 = vals[i];
                        vals[i] = vals[j];
                        vals[j] = t2;
                    }
                }
            }
        }
    }
    __syncwarp();
}

// The K = min(K, n) largest keys of get(i) (payload pay(i)), sorted
// descending into out_keys/out_vals; slots K..next_pow2(K)-1 hold key 0.
// Compaction is by ballot, so the kept set is written in index order before
// the sort.  Returns K.
template <class GetKey, class GetVal>
__device__ int warp_topk(GetKey get, GetVal pay, int n, int K, int* hist, uint64_t* out_keys, int32_t* out_vals,
                         bool sort = true) {
    const int lane = threadIdx.x & 31;
    if (K > n) K = n;
    if (K <= 0) return 0;
    uint64_t prefix = 0ull, mask = 0ull;
    if (K < n) warp_select_threshold(get, n, K, hist, &prefix, &mask);
    const int P2 = next_pow2(K);
    for (int i = lane; i < P2; i += 32) {
        out_keys[i] = 0ull;
        if (out_vals) out_vals[i] = -1;
    }
    __syncwarp();
    int base = 0;
    for (int b0 = 0; b0 < n; b0 += 32) {
        const int i = b0 + lane;
        bool sel = false;
        uint64_t k = 0ull;
        if (i < n) {
            k = get(i);
            sel = (k & mask) >= prefix;
        }
        const unsigned m = __ballot_sync(0xFFFFFFFFu, sel);
        if (sel) {
            const int pos = base + __popc(m & ((1u << lane) - 1u));
            if (pos < K) {
                out_keys[pos] = k;
                if (out_vals) out_vals[pos] = pay(i);
            }
        }
        base += __popc(m);
    }
    if (sort) warp_sort_desc(out_keys, out_vals, P2);
    else __syncwarp();
    return K;
}

}  // namespace ah

namespace ah {

// The K-th largest of n distinct keys (1 <= K <= n) without sorting: the
// minimum of the selected set.  All threads of the block call it; all get it.
template <int NT, class GetKey>
__device__ uint64_t block_kth_largest(GetKey get, int n, int K, SelectScratch& s) {
    uint64_t prefix = 0ull, mask = 0ull;
    if (K < n) block_select_threshold<NT>(get, n, K, s, &prefix, &mask);
    uint64_t mn = ~0ull;
    for (int i = threadIdx.x; i < n; i += NT) {
        const uint64_t k = get(i);
        if ((k & mask) >= prefix && k < mn) mn = k;
    }
    // warp min, then across warps through the scratch word
    const unsigned hi = __reduce_min_sync(0xFFFFFFFFu, static_cast<unsigned>(mn >> 32));
    const unsigned lo = __reduce_min_sync(0xFFFFFFFFu, (static_cast<unsigned>(mn >> 32) == hi)
                                                           ? static_cast<unsigned>(mn) : 0xFFFFFFFFu);
    if (threadIdx.x == 0) s.kand = ~0ull;
    __syncthreads();
    if ((threadIdx.x & 31) == 0) atomicMin(&s.kand, (static_cast<unsigned long long>(hi) << 32) | lo);
    __syncthreads();
    const uint64_t r = s.kand;
    __syncthreads();
    return r;
}

}  // namespace ah

namespace ah {

}  // namespace ah

// ---------------------------------------------------------------------------
// Register-resident warp selection: each lane holds up to KPL keys in
// registers (unused entries hold 0, which no real key equals or undercuts:
// real keys have a nonzero score part).  Radix selection one bit at a time:
// per bit every lane counts its keys in the candidate bucket and the warp sums
// the counts, so there are no shared-memory passes and no block barriers.
// ---------------------------------------------------------------------------
namespace ah {

// The K-th largest of the warp's keys (n > 0 real keys in total, key 0 =
// empty, 1 <= K <= n); all lanes return it.  Bitwise radix from the highest
// bit where the keys differ: each step counts the current bucket's keys with
// the bit set (one warp reduction; the running bucket size gives the other
// half), and the walk stops once the bucket holding the K-th key is exactly
// the remainder.  While the bit is in the upper word only those words are
// compared.
template <int KPL>
__device__ uint64_t warp_kth_reg(const uint64_t (&k)[KPL], int n, int K) {
    uint64_t kand = ~0ull, kor = 0ull;
#pragma unroll
    for (int j = 0; j < KPL; ++j) {
        if (k[j] != 0ull) kand &= k[j];
        kor |= k[j];
    }
    kand = warp_and64(kand);
    kor = warp_or64(kor);
    const uint64_t diff = kand ^ kor;
    if (diff == 0ull) return kor;                       // one distinct real key
    int bit = 63 - __clzll(static_cast<long long>(diff));
    uint64_t prefix = (bit >= 63) ? 0ull : (kand & (~0ull << (bit + 1)));
    int need = K, in_bucket = n;
    bool done = false;
    if (bit >= 32) {                                    // prefix has no low bits yet
        unsigned phi = static_cast<unsigned>(prefix >> 32);
        for (; bit >= 32; --bit) {
            const unsigned hm = ~0u << (bit - 32);
            const unsigned cand = phi | (1u << (bit - 32));
            int c = 0;
#pragma unroll
            for (int j = 0; j < KPL; ++j) c += ((static_cast<unsigned>(k[j] >> 32) & hm) == cand) ? 1 : 0;
            c = __reduce_add_sync(0xFFFFFFFFu, c);
            if (c >= need) {
                phi = cand;
                in_bucket = c;
            } else {
                need -= c;
                in_bucket -= c;
            }
            if (in_bucket == need) {
                done = true;
                break;
            }
        }
        prefix = static_cast<uint64_t>(phi) << 32;
    }
    if (!done) {
        for (; bit >= 0; --bit) {
            const uint64_t hm = ~0ull << bit;
            const uint64_t cand = prefix | (1ull << bit);
            int c = 0;
#pragma unroll
            for (int j = 0; j < KPL; ++j) c += ((k[j] & hm) == cand) ? 1 : 0;
            c = __reduce_add_sync(0xFFFFFFFFu, c);
            if (c >= need) {
                prefix = cand;
                in_bucket = c;
            } else {
                need -= c;
                in_bucket -= c;
            }
            if (in_bucket == need) break;
        }
    }
    // the K-th largest is the smallest real key of the final bucket, which is
    // the smallest real key >= prefix
    uint64_t mn = ~0ull;
#pragma unroll
    for (int j = 0; j < KPL; ++j)
        if (k[j] >= prefix && k[j] != 0ull && k[j] < mn) mn = k[j];
    const unsigned hi = __reduce_min_sync(0xFFFFFFFFu, static_cast<unsigned>(mn >> 32));
    const unsigned lo = __reduce_min_sync(0xFFFFFFFFu, (static_cast<unsigned>(mn >> 32) == hi)
                                                           ? static_cast<unsigned>(mn) : 0xFFFFFFFFu);
    return (static_cast<uint64_t>(hi) << 32) | lo;
}

}  // namespace ah

namespace ah {

// Compact the warp's keys >= thr (and payloads) to out_k/out_v; returns the
// count.  Order: register slot j, then lane.
template <int KPL>
__device__ __forceinline__ int warp_gather_ge(const uint64_t (&k)[KPL], const int32_t (&v)[KPL], uint64_t thr,
                                              uint64_t* out_k, int32_t* out_v) {
    const int lane = threadIdx.x & 31;
    int base = 0;
#pragma unroll
    for (int j = 0; j < KPL; ++j) {
        const bool sel = k[j] != 0ull && k[j] >= thr;
        const unsigned m = __ballot_sync(0xFFFFFFFFu, sel);
        if (sel) {
            const int pos = base + __popc(m & ((1u << lane) - 1u));
            out_k[pos] = k[j];
            if (out_v) out_v[pos] = v[j];
        }
        base += __popc(m);
    }
    __syncwarp();
    return base;
}

// The K = min(K, n) largest of n <= 32*KPL keys read by get(i) (payload pay(i)),
// by one warp through registers; written to out_k/out_v (capacity
// next_pow2(K)), sorted descending if `sort` (padding key 0).  Returns K.
template <int KPL, class GetKey, class GetVal>
__device__ int warp_topk_reg(GetKey get, GetVal pay, int n, int K, uint64_t* out_k, int32_t* out_v, bool sort) {
    const int lane = threadIdx.x & 31;
    uint64_t k[KPL];
    int32_t v[KPL];
#pragma unroll
    for (int j = 0; j < KPL; ++j) {
        const int i = lane + 32 * j;
        k[j] = (i < n) ? get(i) : 0ull;
        v[j] = (i < n && out_v) ? pay(i) : -1;
    }
    if (K > n) K = n;
    if (K <= 0) return 0;
    const uint64_t thr = (K < n) ? warp_kth_reg<KPL>(k, n, K) : 1ull;
    const int P2 = next_pow2(K);
    for (int i = K + lane; i < P2; i += 32) {
        out_k[i] = 0ull;
        if (out_v) out_v[i] = -1;
    }
    warp_gather_ge<KPL>(k, v, thr, out_k, out_v);
    if (sort) warp_sort_desc(out_k, out_v, P2);
    return K;
}


// The K = min(K, n) largest of keys[0..n) (n <= 32*KPL; any address space)
// by one warp, with payload vals[i] (may be null) fetched only for the keys
// kept.  Output as warp_topk_reg.  Returns K.
template <int KPL>
__device__ int warp_topk_src(const uint64_t* keys, const int32_t* vals, int n, int K, uint64_t* out_k,
                             int32_t* out_v, bool sort) {
    const int lane = threadIdx.x & 31;
    uint64_t k[KPL];
#pragma unroll
    for (int j = 0; j < KPL; ++j) {
        const int i = lane + 32 * j;
        k[j] = (i < n) ? keys[i] : 0ull;
    }
    if (K > n) K = n;
    if (K <= 0) return 0;
    const uint64_t thr = (K < n) ? warp_kth_reg<KPL>(k, n, K) : 1ull;
    const int P2 = next_pow2(K);
    for (int i = K + lane; i < P2; i += 32) {
        out_k[i] = 0ull;
        if (out_v) out_v[i] = -1;
    }
    int base = 0;
#pragma unroll
    for (int j = 0; j < KPL; ++j) {
        const bool sel = k[j] != 0ull && k[j] >= thr;
        const unsigned m = __ballot_sync(0xFFFFFFFFu, sel);
        if (sel) {
            const int pos = base + __popc(m & ((1u << lane) - 1u));
            out_k[pos] = k[j];
            if (out_v) out_v[pos] = vals[lane + 32 * j];
        }
        base += __popc(m);
    }
    __syncwarp();
    if (sort) warp_sort_desc(out_k, out_v, P2);
    return K;
}

}  // namespace ah

namespace ah {

// Scratch for block_kth_reg: per-warp partial counts, double-buffered by bit
// parity so one barrier per bit suffices, plus the and/or/min exchange.
template <int NT>
struct RegSelectScratch {
    int part[2][NT / 32];
    unsigned long long w64[NT / 32];
    unsigned long long w64b[NT / 32];
};

template <int NT>
__device__ __forceinline__ int block_sum_parity(int v, RegSelectScratch<NT>& s, int parity) {
    v = __reduce_add_sync(0xFFFFFFFFu, v);
    if ((threadIdx.x & 31) == 0) s.part[parity][threadIdx.x >> 5] = v;
    __syncthreads();
    int t = 0;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) t += s.part[parity][w];
    return t;
}

// K-th largest of the block's register-held keys (KPL per thread, key 0 =
// empty, n > 0 real keys in total, 1 <= K <= n).  Bitwise radix from the
// highest bit where the keys differ; a bit's step counts the keys of the
// current bucket that have the bit set (one warp reduction and one barrier).
// The running bucket size makes the count of the other half free, and the
// walk stops as soon as the bucket holding the K-th key is exactly the
// remainder, whose minimum is then the answer.  Every thread returns it.
template <int KPL, int NT>
__device__ uint64_t block_kth_reg(const uint64_t (&k)[KPL], int n, int K, RegSelectScratch<NT>& s) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint64_t kand = ~0ull, kor = 0ull;
#pragma unroll
    for (int j = 0; j < KPL; ++j) {
        if (k[j] != 0ull) kand &= k[j];
        kor |= k[j];
    }
    kand = warp_and64(kand);
    kor = warp_or64(kor);
    if (lane == 0) {
        s.w64[warp] = kand;
        s.w64b[warp] = kor;
    }
    __syncthreads();
    kand = ~0ull;
    kor = 0ull;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) {
        kand &= s.w64[w];
        kor |= s.w64b[w];
    }
    __syncthreads();  // s.w64 is reused for the minimum below
    const uint64_t diff = kand ^ kor;
    if (diff == 0ull) return kor;  // all keys equal
    const int top = 63 - __clzll(diff);
    uint64_t prefix = (top >= 63) ? 0ull : (kand & (~0ull << (top + 1)));
    int need = K, in_bucket = n, parity = 0;
    for (int bit = top; bit >= 0; --bit) {
        const uint64_t hm = ~0ull << bit;
        const uint64_t cand = prefix | (1ull << bit);
        int c = 0;
#pragma unroll
        for (int j = 0; j < KPL; ++j) c += ((k[j] & hm) == cand) ? 1 : 0;
        c = block_sum_parity<NT>(c, s, parity);
        parity ^= 1;
        if (c >= need) {
            prefix = cand;
            in_bucket = c;
        } else {
            need -= c;
            in_bucket -= c;
        }
        if (in_bucket == need) break;
    }
    uint64_t mn = ~0ull;
#pragma unroll
    for (int j = 0; j < KPL; ++j)
        if (k[j] != 0ull && k[j] >= prefix && k[j] < mn) mn = k[j];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const uint64_t o = __shfl_xor_sync(0xFFFFFFFFu, mn, off);
        mn = o < mn ? o : mn;
    }
    if (lane == 0) s.w64[warp] = mn;
    __syncthreads();
    mn = ~0ull;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) mn = s.w64[w] < mn ? s.w64[w] : mn;
    __syncthreads();
    return mn;
}

}  // namespace ah
