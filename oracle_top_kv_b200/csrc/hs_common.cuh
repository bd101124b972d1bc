// hs_common.cuh -- device helpers shared by the sm_100a kernels of the
// HySparse / HySparse2 hot path: element I/O, warp reductions, the sticky
// device status word, mma.sync / ldmatrix / cp.async wrappers, and the exact
// streaming top-k candidate buffer used by every selection step.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/hs.h"

namespace hs {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Sticky per-device status word (first error wins).  Set by kernels that find
// an out-of-range index or length; read and cleared by hs_device_status.
__device__ int g_status = 0;

__device__ __forceinline__ void set_status(int code) { atomicCAS(&g_status, 0, code); }

// SM clock cycles a bounded wait may take before it gives up (per device; the
// host sets it through hs_set_wait_limit, a failure-detection diagnostic).
__device__ long long g_wait_limit = 2000000000ll;

// Sampled start threshold of the token selectors (per device; set by the
// host through hs_set_select_sampling): -1 = rank chosen from the sample
// density, 0 = off, r > 0 = always the r-th best sampled score.
__device__ int g_sel_sample = -1;

// Rank, among `n_samples` keys drawn evenly from `range_keys` keys, of the
// sampled score a selector may start from as its admission threshold when it
// ranks the best `kc` keys of at least those `range_keys`.  The number of
// samples that fall among the true best kc is about Poisson(lambda), lambda =
// kc * n_samples / range_keys; the threshold is too high only if at least r of
// them do, so r = lambda + 4.3 sqrt(lambda) + 3 keeps that below 1e-5 (the
// selector then detects it and rescans without a threshold).  0 = do not
// sample (off, or samples too dense to save admissions).
__device__ __forceinline__ int sample_rank(int kc, int n_samples, long long range_keys) {
    const int mode = g_sel_sample;
    if (mode >= 0) return mode < n_samples ? mode : 0;
    const float lam = (float)kc * (float)n_samples / (float)range_keys;
    if (!(lam <= 200.f)) return 0;
    return (int)ceilf(lam + 4.3f * sqrtf(lam) + 3.f);
}

// ---------------------------------------------------------------- element I/O
__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// ---------------------------------------------------------------- warp helpers
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Sortable image of a float: larger float <-> larger unsigned.
__device__ __forceinline__ uint32_t float_order(float f) {
    uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float order_float(uint32_t u) {
    return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}
// Composite selection key: larger = better.  High word: the score; low word:
// the complement of the id, so that equal scores prefer the LOWER id.
__device__ __forceinline__ uint64_t sel_key(float score, uint32_t id) {
    return ((uint64_t)float_order(score) << 32) | (uint64_t)(0xffffffffu - id);
}
__device__ __forceinline__ uint32_t sel_key_id(uint64_t key) {
    return 0xffffffffu - (uint32_t)(key & 0xffffffffu);
}
__device__ __forceinline__ float sel_key_score(uint64_t key) {
    return order_float((uint32_t)(key >> 32));
}

// ---------------------------------------------------------------- PTX wrappers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
    // valid == false zero-fills the 16 destination bytes without reading src.
    const int n = valid ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(n));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n"); }
template <int N> __device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
// D = A(16x16 bf16, row) * B(16x8 bf16, col) + D (fp32)
__device__ __forceinline__ void mma_bf16(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// Byte offset of 16-byte chunk `chunk` of row `row` in a tile whose rows are
// `row_bytes` long, with the chunk index XOR-swizzled by the row so that
// ldmatrix over 8 consecutive rows touches 8 distinct bank groups.
__device__ __forceinline__ uint32_t swz(int row, int chunk, int row_bytes) {
    return (uint32_t)(row * row_bytes + ((chunk ^ (row & 7)) << 4));
}

// ------------------------------------------------- exact streaming top-k buffer
//
// One selection = the K best (score, id) pairs under "higher score first,
// lower id on ties".  Candidates are appended to a shared-memory buffer of
// capacity `cap` (>= 2K) as 64-bit composite keys (sel_key).  When the buffer
// runs full, the buffer is cut to its K best, and `thresh` becomes the K-th
// best key: a later candidate can only enter the final K if its key is above
// it, so nothing that could still be selected is ever dropped.

__device__ __forceinline__ uint64_t shfl_xor_u64(uint64_t v, int o) {
    const uint32_t lo = __shfl_xor_sync(0xffffffffu, (uint32_t)v, o);
    const uint32_t hi = __shfl_xor_sync(0xffffffffu, (uint32_t)(v >> 32), o);
    return ((uint64_t)hi << 32) | lo;
}

// K-th largest of n unique keys (1 <= K <= n), computed by one warp with a
// range bucket select: each pass spreads the keys of the live range [lo, hi]
// over 256 equal-width buckets (bucket = (key - lo) >> shift, with shift set
// by the width of the range, so nearby scores still land in different
// buckets), keeps the bucket holding the K-th key, and stops as soon as that
// bucket holds a single key.  hist: 256 words of shared scratch for this warp.
__device__ __forceinline__ uint64_t warp_kth_largest(const uint64_t* buf, int n, int K,
                                                     uint32_t* hist) {
    const int lane = threadIdx.x & 31;
    uint64_t lo = ~0ull, hi = 0ull;
    for (int base = 0; base < n; base += 8 * 32) {  // 8 loads in flight per lane
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = base + u * 32 + lane;
            if (i < n) {
                const uint64_t key = buf[i];
                lo = key < lo ? key : lo;
                hi = key > hi ? key : hi;
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const uint64_t a = shfl_xor_u64(lo, o), b = shfl_xor_u64(hi, o);
        lo = a < lo ? a : lo;
        hi = b > hi ? b : hi;
    }
    int need = K;  // rank of the wanted key, counted from the top of [lo, hi]
    for (int pass = 0; pass < 16; ++pass) {
        if (lo == hi) return lo;
        const uint64_t range = hi - lo;
        const int top = 63 - __clzll((long long)range);
        const int shift = top > 7 ? top - 7 : 0;  // (range >> shift) <= 255
#pragma unroll
        for (int x = 0; x < 8; ++x) hist[lane * 8 + x] = 0;
        __syncwarp();
        for (int base = 0; base < n; base += 8 * 32) {
            uint64_t key[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {  // all loads first, then the atomics
                const int i = base + u * 32 + lane;
                key[u] = i < n ? buf[i] : 0ull;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (base + u * 32 + lane < n && key[u] >= lo && key[u] <= hi)
                    atomicAdd(&hist[(uint32_t)((key[u] - lo) >> shift)], 1u);
        }
        __syncwarp();
        // lane L owns buckets 255-8L .. 248-8L (descending).  Count above each.
        uint32_t own[8];
        uint32_t s = 0;
#pragma unroll
        for (int x = 0; x < 8; ++x) { own[x] = hist[255 - (lane * 8 + x)]; s += own[x]; }
        uint32_t incl = s;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        uint32_t above = incl - s;
        int bucket = -1;
        uint32_t above_b = 0, in_b = 0;
#pragma unroll
        for (int x = 0; x < 8; ++x) {
            if (bucket < 0 && above < (uint32_t)need && above + own[x] >= (uint32_t)need) {
                bucket = 255 - (lane * 8 + x);
                above_b = above;
                in_b = own[x];
            }
            above += own[x];
        }
        const uint32_t found = __ballot_sync(0xffffffffu, bucket >= 0);
        const int src = __ffs(found) - 1;
        bucket = __shfl_sync(0xffffffffu, bucket, src);
        above_b = __shfl_sync(0xffffffffu, above_b, src);
        in_b = __shfl_sync(0xffffffffu, in_b, src);
        need -= (int)above_b;
        const uint64_t nlo = lo + ((uint64_t)bucket << shift);
        const uint64_t nhi = nlo + (((uint64_t)1 << shift) - 1);
        lo = nlo;
        hi = nhi < hi ? nhi : hi;
        __syncwarp();
        if (in_b == 1) {
            // the K-th key is the only one left in [lo, hi]: fetch it
            uint64_t hit = 0;
            for (int base = 0; base < n; base += 8 * 32) {
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int i = base + u * 32 + lane;
                    if (i < n) {
                        const uint64_t key = buf[i];
                        if (key >= lo && key <= hi) hit = key;
                    }
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const uint64_t y = shfl_xor_u64(hit, o);
                hit = y > hit ? y : hit;
            }
            return hit;
        }
    }
    return lo;  // not reached for unique keys: each pass shrinks the range 256-fold
}

// Keep only keys >= kth, compacted in place in their original order; returns
// the new count.  Chunks of 8 x 32 keys: the whole chunk is read into
// registers before any of it is written back (so the loads overlap instead of
// each waiting for the previous store), which is safe in place because a kept
// key's new position is never past its old one.
__device__ __forceinline__ int warp_keep_at_least(uint64_t* buf, int n, uint64_t kth) {
    const int lane = threadIdx.x & 31;
    int out = 0;
    for (int base = 0; base < n; base += 8 * 32) {
        uint64_t key[8];
        bool keep[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = base + u * 32 + lane;
            key[u] = i < n ? buf[i] : 0ull;
            keep[u] = i < n && key[u] >= kth;
        }
        __syncwarp();
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const uint32_t bal = __ballot_sync(0xffffffffu, keep[u]);
            if (keep[u]) buf[out + __popc(bal & ((1u << lane) - 1))] = key[u];
            out += __popc(bal);
        }
        __syncwarp();
    }
    return out;
}

// Number of keys >= thr among buf[0 .. n) (warp-wide; 8 loads in flight per lane).
__device__ __forceinline__ int warp_count_at_least(const uint64_t* buf, int n, uint64_t thr) {
    const int lane = threadIdx.x & 31;
    int c = 0;
    for (int base = 0; base < n; base += 8 * 32) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = base + u * 32 + lane;
            c += (i < n && buf[i] >= thr) ? 1 : 0;
        }
    }
    return __reduce_add_sync(0xffffffffu, c);
}

// Cut the buffer to its K best keys; returns the K-th best key (the new
// admission threshold).  Requires n > K.
__device__ __forceinline__ uint64_t warp_cut_to_k(uint64_t* buf, int n, int K, uint32_t* hist) {
    const uint64_t kth = warp_kth_largest(buf, n, K, hist);
    warp_keep_at_least(buf, n, kth);
    return kth;
}

// Ascending bitonic sort of 64 values held two per lane (a = element lane,
// b = element lane + 32), in registers.
__device__ __forceinline__ void warp_sort64(uint64_t& a, uint64_t& b) {
    const int lane = threadIdx.x & 31;
    for (int size = 2; size <= 64; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            if (stride == 32) {  // a <-> b of the same lane
                const bool up = true;  // size == 64
                if ((a > b) == up) { const uint64_t t = a; a = b; b = t; }
                continue;
            }
            // element e = lane (+32 for b); partner e ^ stride is in the same half
            const uint64_t pa = shfl_xor_u64(a, stride), pb = shfl_xor_u64(b, stride);
            const bool lower = (lane & stride) == 0;
            const bool up_a = (lane & size) == 0, up_b = ((lane + 32) & size) == 0;
            // the lower element keeps min when ascending, max when descending
            a = (lower == up_a) ? (a < pa ? a : pa) : (a > pa ? a : pa);
            b = (lower == up_b) ? (b < pb ? b : pb) : (b > pb ? b : pb);
        }
    }
}

// Cut a streaming buffer by a sampled quantile: sort 64 evenly spaced keys,
// take the one a little below the K-th best's expected sample rank as the
// threshold, count the keys at or above it and, if that keeps at least K
// (so the K best are all kept) and frees at least `min_free` slots, compact;
// otherwise move the threshold down the sample and count again, and fall
// back to the exact cut when the sample runs out.  No shared atomics, and
// outlying scores do not bunch the rest up.  Returns the surviving count;
// *thresh gets an admission threshold (a key must exceed it) that is at most
// the K-th best key.  Requires n > K.
__device__ __forceinline__ int warp_cut_sampled(uint64_t* buf, int n, int K, int min_free,
                                                uint32_t* hist, uint64_t* thresh) {
    const int lane = threadIdx.x & 31;
    uint64_t a = buf[(int)(((long long)(2 * lane) * n) >> 6)];
    uint64_t b = buf[(int)(((long long)(2 * lane + 1) * n) >> 6)];
    warp_sort64(a, b);  // ascending: element e = a of lane e, b of lane e - 32
    // expected descending sample rank of the K-th best, plus 3 samples of slack
    int q = (int)(((long long)K * 64 + n - 1) / n) + 3;
    for (; q < 64; q += 4) {
        const int e = 63 - q;  // ascending index
        const uint64_t thr = __shfl_sync(0xffffffffu, (uint32_t)(e < 32 ? a : b), e & 31) |
                             ((uint64_t)__shfl_sync(0xffffffffu, (uint32_t)((e < 32 ? a : b) >> 32),
                                                    e & 31) << 32);
        const int c = warp_count_at_least(buf, n, thr);
        if (c < K) continue;            // too high: a top-K key would go
        if (n - c < min_free) break;    // keeps too much: exact cut instead
        const int m = warp_keep_at_least(buf, n, thr);
        *thresh = thr ? thr - 1ull : 0ull;
        return m;
    }
    const uint64_t kth = warp_cut_to_k(buf, n, K, hist);
    *thresh = kth;
    return K;
}

// In-place ascending bitonic sort of n_pow2 values by one warp.
template <typename U>
__device__ __forceinline__ void warp_bitonic_sort(U* a, int n_pow2) {
    const int lane = threadIdx.x & 31;
    for (int size = 2; size <= n_pow2; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int t = lane; t < (n_pow2 >> 1); t += 32) {
                const int i = 2 * t - (t & (stride - 1));
                const int j = i + stride;
                const bool up = (i & size) == 0;
                const U x = a[i], y = a[j];
                if ((x > y) == up) { a[i] = y; a[j] = x; }
            }
            __syncwarp();
        }
    }
}

__host__ __device__ constexpr int next_pow2(int x) {
    int p = 1;
    while (p < x) p <<= 1;
    return p;
}

}  // namespace hs
