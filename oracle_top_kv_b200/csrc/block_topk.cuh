// block_topk.cuh -- exact top-K selection by one CTA over a stream of
// (score, id) candidates, for one query row and KV group.
//
// Order: higher score first, equal scores to the lower id.  Threads offer
// candidates in rounds (at most `round` offers per round); between rounds
// every thread calls end_round(), which cuts the buffer back to its K best
// once it could overflow.  finish() (warp 0) writes the winners in ascending
// id order, optionally followed by a forced contiguous range (the HySparse2
// window), and -1 / 0 padding.
#pragma once

#include "hs_common.cuh"

namespace hs {

struct BlockTopK {
    uint64_t* buf;     // [cap]
    uint64_t* sortb;   // [sort_n]
    uint32_t* hist;    // [256]
    int* count;        // shared
    unsigned long long* thresh;  // shared
    int cap, K, sort_n, round;

    // Shared-memory bytes for K winners and `round` offers per round.
    __host__ __device__ static size_t smem_bytes(int K, int round) {
        const int kk = K > 0 ? K : 1;
        return sizeof(uint64_t) * (2 * kk + round + next_pow2(kk)) + sizeof(uint32_t) * 256;
    }
    __device__ void setup(unsigned char* smem, int K_, int round_, int* cnt_sh,
                          unsigned long long* th_sh) {
        K = K_;
        round = round_;
        const int kk = K > 0 ? K : 1;
        cap = 2 * kk + round;
        sort_n = next_pow2(kk);
        buf = reinterpret_cast<uint64_t*>(smem);
        sortb = buf + cap;
        hist = reinterpret_cast<uint32_t*>(sortb + sort_n);
        count = cnt_sh;
        thresh = th_sh;
        if (threadIdx.x == 0) { *count = 0; *thresh = 0ull; }
    }
    __device__ __forceinline__ void offer(float score, uint32_t id) {
        const uint64_t key = sel_key(score, id);
        if (key > *thresh) buf[atomicAdd(count, 1)] = key;
    }
    // Called by every thread of the CTA after each round of offers.
    __device__ void end_round() {
        __syncthreads();
        const int cur = *count;
        __syncthreads();  // all reads of the count happen before the next offers
        if (cur > cap - round) {
            if (threadIdx.x < 32) {
                const uint64_t th = warp_cut_to_k(buf, cur, K, hist);
                if (threadIdx.x == 0) { *thresh = th; *count = K; }
            }
            __syncthreads();
        }
    }
    // Warp 0 only.  Writes min(count, K) winners sorted by id into irow (and
    // their scores exp2(score) into srow if non-null), then ids
    // forced_lo..forced_hi, then padding up to ksel.  Returns the count written.
    __device__ int finish(int32_t* irow, float* srow, int ksel, int forced_lo, int forced_hi) {
        const int lane = threadIdx.x & 31;
        int n = K > 0 ? *count : 0;
        if (n > K) { warp_cut_to_k(buf, n, K, hist); n = K; }
        __syncwarp();
        for (int x = lane; x < sort_n; x += 32)
            sortb[x] = x < n ? (((uint64_t)sel_key_id(buf[x]) << 32) | (buf[x] >> 32)) : ~0ull;
        __syncwarp();
        warp_bitonic_sort(sortb, sort_n);
        for (int x = lane; x < n; x += 32) {
            irow[x] = (int32_t)(sortb[x] >> 32);
            if (srow) srow[x] = exp2f(order_float((uint32_t)(sortb[x] & 0xffffffffu)));
        }
        int n_out = n;
        if (forced_hi >= forced_lo) {
            for (int x = lane; x <= forced_hi - forced_lo; x += 32) irow[n + x] = forced_lo + x;
            n_out += forced_hi - forced_lo + 1;
        }
        for (int x = n_out + lane; x < ksel; x += 32) {
            irow[x] = -1;
            if (srow) srow[x] = 0.f;
        }
        return n_out;
    }
};

}  // namespace hs
