// cta_select.cuh -- exact selection by a whole CTA over keys held in shared
// memory: the k-th largest of n distinct 64-bit keys (sel_key composites, so
// "largest" is higher score first, lower id on equal scores), and a bitonic
// sort.  Every thread of the CTA calls these; they synchronise internally.
#pragma once

#include "hs_common.cuh"

namespace hs {

// Shared scratch of cta_kth_largest.
struct CtaSelectSmem {
    uint32_t hist[256];
    unsigned long long lo, hi, found;
    int need;
};

__device__ __forceinline__ int top_bit64(uint64_t x) { return 63 - __clzll((long long)x); }

// The k-th largest (1 <= k <= n) of the distinct keys get(0) .. get(n-1).
// Range bucket select: the live range [lo, hi] is cut into 256 equal buckets
// per pass, the bucket holding the k-th largest becomes the new range.  The
// range shrinks 256-fold per pass, so at most 8 passes; a pass whose bucket
// holds a single key ends with one scan that picks that key.
template <typename Get>
__device__ uint64_t cta_kth_largest(Get get, int n, int k, CtaSelectSmem& sh) {
    const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31;
    uint64_t mn = ~0ull, mx = 0ull;
    for (int i = tid; i < n; i += nt) {
        const uint64_t v = get(i);
        mn = v < mn ? v : mn;
        mx = v > mx ? v : mx;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const uint64_t a = shfl_xor_u64(mn, o), b = shfl_xor_u64(mx, o);
        mn = a < mn ? a : mn;
        mx = b > mx ? b : mx;
    }
    if (tid == 0) { sh.lo = ~0ull; sh.hi = 0ull; sh.need = k; sh.found = 0ull; }
    __syncthreads();
    if (lane == 0) { atomicMin(&sh.lo, (unsigned long long)mn); atomicMax(&sh.hi, (unsigned long long)mx); }
    __syncthreads();
    uint64_t lo = sh.lo, hi = sh.hi;
    for (int pass = 0; pass < 9 && lo != hi; ++pass) {
        const int shift = max(0, top_bit64(hi - lo) - 7);
        for (int x = tid; x < 256; x += nt) sh.hist[x] = 0u;
        __syncthreads();
        for (int i = tid; i < n; i += nt) {
            const uint64_t v = get(i);
            if (v >= lo && v <= hi) atomicAdd(&sh.hist[(uint32_t)((v - lo) >> shift)], 1u);
        }
        __syncthreads();
        bool single = false;
        if (tid < 32) {
            // lane l owns buckets 255 - 8l .. 248 - 8l (from the top)
            uint32_t c[8], s = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) { c[j] = sh.hist[255 - 8 * lane - j]; s += c[j]; }
            uint32_t incl = s;  // inclusive prefix over lanes (top first)
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            const int need = sh.need;
            const uint32_t excl = incl - s;
            const bool mine = excl < (uint32_t)need && incl >= (uint32_t)need;
            if (mine) {
                uint32_t above = excl;
                int j = 0;
                while (above + c[j] < (uint32_t)need) { above += c[j]; ++j; }
                const uint32_t b = 255u - 8u * lane - j;
                const uint64_t nlo = lo + ((uint64_t)b << shift);
                const uint64_t span = shift >= 64 ? ~0ull : ((1ull << shift) - 1ull);
                const uint64_t nhi = (hi - nlo) < span ? hi : nlo + span;
                sh.lo = nlo;
                sh.hi = nhi;
                sh.need = need - (int)above;
                sh.found = c[j] == 1u ? 1ull : 0ull;
            }
        }
        __syncthreads();
        lo = sh.lo;
        hi = sh.hi;
        single = sh.found != 0ull;
        __syncthreads();
        if (single && lo != hi) {  // the bucket holds one key: fetch it
            for (int i = tid; i < n; i += nt) {
                const uint64_t v = get(i);
                if (v >= lo && v <= hi) sh.lo = v;
            }
            __syncthreads();
            lo = hi = sh.lo;
            __syncthreads();
        }
    }
    return lo;
}

// Exclusive prefix sum of one int per thread over the CTA (thread order);
// `scratch` is one shared int per warp plus one.  All threads call.
__device__ __forceinline__ int cta_exclusive_sum(int v, int* scratch) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    __syncthreads();
    if (lane == 31) scratch[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = lane < nw ? scratch[lane] : 0;
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += y;
        }
        if (lane < nw) scratch[lane] = wi - w;  // exclusive warp offsets
    }
    __syncthreads();
    return scratch[warp] + incl - v;
}

// Ascending bitonic sort of a[0 .. n) in shared memory, n a power of two.
template <typename U>
__device__ void cta_bitonic_sort(U* a, int n) {
    for (int k = 2; k <= n; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = threadIdx.x; i < n; i += blockDim.x) {
                const int p = i ^ j;
                if (p > i) {
                    const U x = a[i], y = a[p];
                    const bool up = (i & k) == 0;
                    if ((x > y) == up) { a[i] = y; a[p] = x; }
                }
            }
            __syncthreads();
        }
    }
}

}  // namespace hs
