// attend_mma.cuh -- one warp attends the (up to 16) query heads of a GQA group
// over a list of key rows of that group's K/V, with mma.sync tensor-core
// fragments (bf16 in, fp32 accumulate) and an online softmax.
//
// The 16 MMA rows are the heads of the group, so every gathered K/V row is
// loaded once and used by all of them ("HySparse 混合稀疏注意力（一）", GQA:
// the group shares one index set so each selected row is read once).  Rows are
// fetched 32 at a time into a 2-stage shared-memory ring owned by the warp:
// runs of consecutive keys (selected blocks, windows, cache splits) by TMA
// (one lane, 2-D boxes, 128-byte swizzle), gathered keys (token selection) by
// 16-byte cp.async into the same swizzled layout.  Masked rows get a -inf
// logit.
#pragma once

#include "hs_common.cuh"
#include "tc_ptx.cuh"

namespace hs {

constexpr int kChunk = 32;  // key rows per pipeline stage
constexpr int kStages = 2;

template <int D>
struct WarpSmem {
    static constexpr int kRowBytes = D * 2;
    static constexpr int kTileBytes = kChunk * kRowBytes;
    static constexpr int kStageBytes = 2 * kTileBytes;  // K tile + V tile
    static constexpr int kBytes = kStages * kStageBytes;
};

// Byte offset of 16-byte chunk c (elements 8c..8c+7) of row `row` in a tile of
// kChunk rows: the tile is stored as d-halves of [kChunk][64] elements with
// 128-byte rows, each XOR-swizzled by the row -- exactly the layout a TMA box
// {64, kChunk} with 128-byte swizzle writes at a 1 KB-aligned address.
__device__ __forceinline__ uint32_t tile_off(int row, int c) {
    return (uint32_t)(((c >> 3) * (kChunk * 128)) + row * 128 + (((c & 7) ^ (row & 7)) << 4));
}

// Online-softmax state of one warp: rows gid and gid+8 of the 16-row tile.
template <int D>
struct AttnState {
    float m[2], l[2];          // running max (log2 domain) and partial row sum
    float o[D / 8][4];         // O accumulator fragments (16 x D)
    __device__ __forceinline__ void init() {
        m[0] = m[1] = -INFINITY;
        l[0] = l[1] = 0.f;
#pragma unroll
        for (int n = 0; n < D / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    }
};

// A fragments of the 16 x D query tile: rows = heads h0 .. h0+15 (rows >= g
// are zero), columns = d.  q points at head h0's row; head stride in elements.
template <int D>
__device__ __forceinline__ void load_q_frags(uint32_t (&qf)[D / 16][4],
                                             const __nv_bfloat16* q, size_t head_stride, int g) {
    const int lane = threadIdx.x & 31, gid = lane >> 2, tig = lane & 3;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        const int c0 = kk * 16 + tig * 2;
        qf[kk][0] = gid < g ? *reinterpret_cast<const uint32_t*>(q + gid * head_stride + c0) : 0u;
        qf[kk][1] = gid + 8 < g
                        ? *reinterpret_cast<const uint32_t*>(q + (gid + 8) * head_stride + c0)
                        : 0u;
        qf[kk][2] = gid < g ? *reinterpret_cast<const uint32_t*>(q + gid * head_stride + c0 + 8)
                            : 0u;
        qf[kk][3] = gid + 8 < g
                        ? *reinterpret_cast<const uint32_t*>(q + (gid + 8) * head_stride + c0 + 8)
                        : 0u;
    }
}

// Issue the cp.async loads of one chunk: row r of the chunk reads key
// `key_of_lane_r` (held by lane r; < 0 = masked, zero-filled).
template <int D>
__device__ __forceinline__ void load_chunk(uint32_t stage_base, const __nv_bfloat16* kbase,
                                           const __nv_bfloat16* vbase, int my_key) {
    const int lane = threadIdx.x & 31;
    constexpr int CPR = D / 8;  // 16-byte chunks per row
#pragma unroll
    for (int it = 0; it < CPR; ++it) {
        const int x = it * 32 + lane;
        const int r = x / CPR, c = x % CPR;
        const int key = __shfl_sync(0xffffffffu, my_key, r);
        const bool ok = key >= 0;
        const size_t off = (size_t)(ok ? key : 0) * D + c * 8;
        const uint32_t so = tile_off(r, c);
        cp_async16(stage_base + so, kbase + off, ok);
        cp_async16(stage_base + WarpSmem<D>::kTileBytes + so, vbase + off, ok);
    }
}

// Issue the cp.async loads of a chunk of 32 consecutive keys key0..key0+31;
// rows whose bit is clear in `valid` are zero-filled without being read.
template <int D>
__device__ __forceinline__ void load_chunk_contig(uint32_t stage_base, const __nv_bfloat16* kbase,
                                                  const __nv_bfloat16* vbase, int key0,
                                                  uint32_t valid) {
    const int lane = threadIdx.x & 31;
    constexpr int CPR = D / 8;  // 16-byte chunks per row
#pragma unroll
    for (int it = 0; it < CPR; ++it) {
        const int x = it * 32 + lane;
        const int r = x / CPR, c = x % CPR;
        const bool ok = (valid >> r) & 1u;
        const size_t off = (size_t)(ok ? key0 + r : 0) * D + c * 8;
        const uint32_t so = tile_off(r, c);
        cp_async16(stage_base + so, kbase + off, ok);
        cp_async16(stage_base + WarpSmem<D>::kTileBytes + so, vbase + off, ok);
    }
}

// S = Q K^T for one chunk (16 x 32), raw logits, masked rows at -inf.
template <int D>
__device__ __forceinline__ void chunk_scores(float (&s)[4][4], const uint32_t (&qf)[D / 16][4],
                                             uint32_t kst, uint32_t valid_mask) {
    const int lane = threadIdx.x & 31, tig = lane & 3;
#pragma unroll
    for (int n = 0; n < 4; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
        for (int np = 0; np < 2; ++np) {  // pairs of 8-key n-tiles
            const int key = np * 16 + (lane & 7) + ((lane >> 4) << 3);
            const int chunk = kk * 2 + ((lane >> 3) & 1);
            uint32_t b0, b1, b2, b3;
            ldsm_x4(kst + tile_off(key, chunk), b0, b1, b2, b3);
            mma_bf16(s[np * 2], qf[kk], b0, b1);
            mma_bf16(s[np * 2 + 1], qf[kk], b2, b3);
        }
    }
#pragma unroll
    for (int n = 0; n < 4; ++n) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int col = n * 8 + tig * 2 + (e & 1);
            s[n][e] = ((valid_mask >> col) & 1u) ? s[n][e] : -INFINITY;
        }
    }
}

__device__ __forceinline__ float ex2f_fast(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Online-softmax update with one chunk of raw logits, then O += P V.  The
// reference max m (log2 domain) only moves when a chunk exceeds it by more
// than 2^8, so O is rescaled rarely; p = 2^(s * scale_log2 - m) <= 2^8.
template <int D>
__device__ __forceinline__ void chunk_update(AttnState<D>& st, float (&s)[4][4], uint32_t vst,
                                             float scale_log2) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {  // row gid (hr=0) and gid+8 (hr=1)
        float mx = fmaxf(fmaxf(fmaxf(s[0][2 * hr], s[0][2 * hr + 1]),
                               fmaxf(s[1][2 * hr], s[1][2 * hr + 1])),
                         fmaxf(fmaxf(s[2][2 * hr], s[2][2 * hr + 1]),
                               fmaxf(s[3][2 * hr], s[3][2 * hr + 1])));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        mx *= scale_log2;  // -inf stays -inf
        if (mx > st.m[hr] + 8.f) {
            const float corr = ex2f_fast(st.m[hr] - mx);  // 0 while nothing was seen
            st.l[hr] *= corr;
#pragma unroll
            for (int n = 0; n < D / 8; ++n) {
                st.o[n][2 * hr] *= corr;
                st.o[n][2 * hr + 1] *= corr;
            }
            st.m[hr] = mx;
        }
        const float nm = st.m[hr] == -INFINITY ? 0.f : -st.m[hr];
        float sum = 0.f;
#pragma unroll
        for (int n = 0; n < 4; ++n) {
            s[n][2 * hr] = ex2f_fast(fmaf(s[n][2 * hr], scale_log2, nm));
            s[n][2 * hr + 1] = ex2f_fast(fmaf(s[n][2 * hr + 1], scale_log2, nm));
            sum += s[n][2 * hr] + s[n][2 * hr + 1];
        }
        st.l[hr] += sum;
    }
    // P (16 x 32) as two k-steps of A fragments.
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
        uint32_t a[4];
        a[0] = pack_bf16(s[2 * ks][0], s[2 * ks][1]);
        a[1] = pack_bf16(s[2 * ks][2], s[2 * ks][3]);
        a[2] = pack_bf16(s[2 * ks + 1][0], s[2 * ks + 1][1]);
        a[3] = pack_bf16(s[2 * ks + 1][2], s[2 * ks + 1][3]);
#pragma unroll
        for (int dp = 0; dp < D / 16; ++dp) {  // pairs of 8-wide d tiles
            const int key = ks * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
            const int chunk = dp * 2 + (lane >> 4);
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(vst + tile_off(key, chunk), b0, b1, b2, b3);
            mma_bf16(st.o[dp * 2], a, b0, b1);
            mma_bf16(st.o[dp * 2 + 1], a, b2, b3);
        }
    }
}

// Finish the row sums across the quad (each lane summed its own columns).
template <int D>
__device__ __forceinline__ void finish_rows(AttnState<D>& st) {
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
        st.l[hr] += __shfl_xor_sync(0xffffffffu, st.l[hr], 1);
        st.l[hr] += __shfl_xor_sync(0xffffffffu, st.l[hr], 2);
    }
}

// Run the pipeline over n_chunks chunks of 32 gathered rows; src.key(r) gives
// the key of list row r (< 0: masked).  cp.async, 2 stages.
template <int D, typename Src, typename Hook>
__device__ __forceinline__ void attend_rows(AttnState<D>& st, const uint32_t (&qf)[D / 16][4],
                                            const __nv_bfloat16* kbase,
                                            const __nv_bfloat16* vbase, int n_chunks,
                                            const Src& src, uint32_t smem_base, float scale_log2,
                                            Hook hook) {
    static_assert(!Src::kContig, "gathered rows");
    const int lane = threadIdx.x & 31;
    uint32_t mask_a = 0, mask_b = 0;  // valid-row masks of the two stages
    auto issue = [&](int c, uint32_t& mask) {
        const uint32_t sb = smem_base + (c & 1) * WarpSmem<D>::kStageBytes;
        const int key = src.key(c * kChunk + lane);
        mask = __ballot_sync(0xffffffffu, key >= 0);
        load_chunk<D>(sb, kbase, vbase, key);
    };
    static_assert(kStages == 2, "two-stage ring");
    if (n_chunks > 0) issue(0, mask_a);
    cp_async_commit();
    for (int c = 0; c < n_chunks; ++c) {
        if (c + 1 < n_chunks) {
            if ((c + 1) & 1) issue(c + 1, mask_b);
            else issue(c + 1, mask_a);
        }
        cp_async_commit();
        cp_async_wait<1>();
        __syncwarp();
        const uint32_t sb = smem_base + (c & 1) * WarpSmem<D>::kStageBytes;
        const uint32_t mask = (c & 1) ? mask_b : mask_a;
        float s[4][4];
        chunk_scores<D>(s, qf, sb, mask);
        hook(c, s, 0);
        chunk_update<D>(st, s, sb + WarpSmem<D>::kTileBytes, scale_log2);
        __syncwarp();  // the stage is refilled by the next iteration
    }
    cp_async_wait<0>();
    finish_rows<D>(st);
}

// Per-warp TMA pipeline state: two mbarriers (one per stage) and how many
// times each has been used, so that the phases stay right across calls.
struct TmaRing {
    uint32_t bar;      // shared address of 2 consecutive mbarriers
    uint32_t uses[2];
};

// Run the pipeline over n_chunks chunks of 32 consecutive keys each;
// src.chunk(c, &key0) gives chunk c's first key and its valid-row mask.  One
// lane issues the TMA boxes {64, 32} of K and V (coordinates d, key, unit);
// rows past the cache end are zero-filled by the TMA.  The optional per-chunk
// hook sees the masked raw logits and the chunk's first key.  Returns false if
// a wait timed out (HS_ERR_TIMEOUT is then set).
template <int D, typename Src, typename Hook>
__device__ __forceinline__ bool attend_rows_tma(AttnState<D>& st, const uint32_t (&qf)[D / 16][4],
                                                const CUtensorMap* tk, const CUtensorMap* tv,
                                                int unit, int n_chunks, const Src& src,
                                                uint32_t smem_base, TmaRing& ring,
                                                float scale_log2, Hook hook) {
    static_assert(Src::kContig, "consecutive keys");
    constexpr uint32_t kHalf = kChunk * 128;          // one d-half box
    constexpr uint32_t kTx = 2 * (D / 64) * kHalf;    // K and V, all halves
    const int lane = threadIdx.x & 31;
    uint32_t mask_a = 0, mask_b = 0;
    int key0_a = 0, key0_b = 0;
    int dummy = 0;
    volatile int* no_abort = &dummy;
    auto issue = [&](int c, uint32_t& mask, int& key0) {
        const uint32_t sb = smem_base + (c & 1) * WarpSmem<D>::kStageBytes;
        mask = src.chunk(c, &key0);
        if (lane == 0) {
            const uint32_t b = ring.bar + 8u * (c & 1);
            tc::mbar_arrive_expect_tx(b, kTx);
#pragma unroll
            for (int h = 0; h < D / 64; ++h) {
                tc::tma_load_3d(sb + h * kHalf, tk, b, 64 * h, key0, unit);
                tc::tma_load_3d(sb + WarpSmem<D>::kTileBytes + h * kHalf, tv, b, 64 * h, key0,
                                unit);
            }
        }
    };
    int issued = 0, failed = -1;
    if (n_chunks > 0) { issue(0, mask_a, key0_a); issued = 1; }
    for (int c = 0; c < n_chunks; ++c) {
        if (c + 1 < n_chunks) {
            if ((c + 1) & 1) issue(c + 1, mask_b, key0_b);
            else issue(c + 1, mask_a, key0_a);
            issued = c + 2;
        }
        const int sidx = c & 1;
        const bool got = tc::mbar_wait(ring.bar + 8u * sidx, ring.uses[sidx] & 1, no_abort);
        if (!__all_sync(0xffffffffu, got)) { failed = c; break; }
        ring.uses[sidx]++;
        const uint32_t sb = smem_base + sidx * WarpSmem<D>::kStageBytes;
        const uint32_t mask = sidx ? mask_b : mask_a;
        const int key0 = sidx ? key0_b : key0_a;
        float s[4][4];
        chunk_scores<D>(s, qf, sb, mask);
        hook(c, s, key0);
        chunk_update<D>(st, s, sb + WarpSmem<D>::kTileBytes, scale_log2);
        __syncwarp();  // the stage is refilled by the next iteration
    }
    if (failed >= 0) {
        // wait (bounded) for every load issued but not consumed before the
        // buffers can be reused, keeping the phase counts consistent
        for (int c = failed; c < issued; ++c) {
            const int sidx = c & 1;
            const long long t0 = clock64();
            while (!tc::mbar_try_wait(ring.bar + 8u * sidx, ring.uses[sidx] & 1))
                if (clock64() - t0 > tc::kWaitCycles) break;
            ring.uses[sidx]++;
        }
        return false;
    }
    finish_rows<D>(st);
    return true;
}

// Keys first..last (inclusive) as contiguous chunks.
struct ContiguousKeys {
    static constexpr bool kContig = true;
    int first, last;
    __device__ __forceinline__ int n_chunks() const { return (last - first + kChunk) / kChunk; }
    __device__ __forceinline__ uint32_t chunk(int c, int* key0) const {
        *key0 = first + c * kChunk;
        const int n = last - *key0 + 1;  // valid rows in this chunk
        return n >= 32 ? 0xffffffffu : (n <= 0 ? 0u : ((1u << n) - 1u));
    }
};

// Partial result of one split: per head (m2, l, O[D]) fp32, unnormalised.
// Layout [16][D + 2]: m2, l, o[0..D).
template <int D>
__device__ __forceinline__ void store_partial(const AttnState<D>& st, float* part, int g) {
    const int lane = threadIdx.x & 31, gid = lane >> 2, tig = lane & 3;
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
        const int h = gid + 8 * hr;
        if (h >= g) continue;
        float* ph = part + h * (D + 2);
        if (tig == 0) { ph[0] = st.m[hr]; ph[1] = st.l[hr]; }
#pragma unroll
        for (int n = 0; n < D / 8; ++n) {
            const int col = n * 8 + tig * 2;
            ph[2 + col] = st.o[n][2 * hr];
            ph[2 + col + 1] = st.o[n][2 * hr + 1];
        }
    }
}

struct NoHook {
    __device__ __forceinline__ void operator()(int, float (&)[4][4], int) const {}
};

}  // namespace hs
