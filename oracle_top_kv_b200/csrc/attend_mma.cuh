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
#include "hs_kernels.cuh"
#include "tc_ptx.cuh"

namespace hs {

constexpr int kChunk = 32;  // key rows per pipeline stage
constexpr int kStages = 2;

template <int D, int S = kStages>
struct WarpSmem {
    static constexpr int kRowBytes = D * 2;
    static constexpr int kTileBytes = kChunk * kRowBytes;
    static constexpr int kStageBytes = 2 * kTileBytes;  // K tile + V tile
    static constexpr int kBytes = S * kStageBytes;
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

// Per-lane ldmatrix offsets into a swizzled chunk tile, computed once per
// call.  tile_off(row, c) of the row and 16-byte column a lane addresses in
// an x4 load splits into a part fixed for the lane (its row within a 16-row
// group and the XOR of its column with the row) and a constant: the column's
// d-half (c >> 3) and the 16-row group.  The XOR takes four values, one per
// (c >> 1) & 3.
struct LaneOffs {
    uint32_t k[4];  // Q K^T: K tile rows = keys, non-transposed x4 loads
    uint32_t v[4];  // P V:   V tile rows = keys, transposed x4 loads
    __device__ __forceinline__ void init() {
        const int lane = threadIdx.x & 31, r7 = lane & 7;
        const uint32_t rk = (uint32_t)((lane & 7) + ((lane >> 4) << 3)) * 128u;
        const uint32_t rv = (uint32_t)((lane & 7) + (((lane >> 3) & 1) << 3)) * 128u;
        const int bk = (lane >> 3) & 1, bv = lane >> 4;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            k[j] = rk + ((uint32_t)((2 * j + bk) ^ r7) << 4);
            v[j] = rv + ((uint32_t)((2 * j + bv) ^ r7) << 4);
        }
    }
};

// S = Q K^T for one chunk (16 x 32), raw logits, masked rows at -inf.
template <int D>
__device__ __forceinline__ void chunk_scores(float (&s)[4][4], const uint32_t (&qf)[D / 16][4],
                                             uint32_t kst, uint32_t valid_mask,
                                             const LaneOffs& lo) {
    const int lane = threadIdx.x & 31, tig = lane & 3;
#pragma unroll
    for (int n = 0; n < 4; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
        for (int np = 0; np < 2; ++np) {  // pairs of 8-key n-tiles
            // == tile_off(np*16 + (lane&7) + ((lane>>4)<<3), kk*2 + ((lane>>3)&1))
            const uint32_t off = (uint32_t)((kk >> 2) * (kChunk * 128) + np * 16 * 128);
            uint32_t b0, b1, b2, b3;
            ldsm_x4(kst + lo.k[kk & 3] + off, b0, b1, b2, b3);
            mma_bf16(s[np * 2], qf[kk], b0, b1);
            mma_bf16(s[np * 2 + 1], qf[kk], b2, b3);
        }
    }
    if (valid_mask != 0xffffffffu) {
#pragma unroll
        for (int n = 0; n < 4; ++n) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int col = n * 8 + tig * 2 + (e & 1);
                s[n][e] = ((valid_mask >> col) & 1u) ? s[n][e] : -INFINITY;
            }
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
                                             float scale_log2, const LaneOffs& lo) {
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
            // == tile_off(ks*16 + (lane&7) + (((lane>>3)&1)<<3), dp*2 + (lane>>4))
            const uint32_t off = (uint32_t)((dp >> 2) * (kChunk * 128) + ks * 16 * 128);
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(vst + lo.v[dp & 3] + off, b0, b1, b2, b3);
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

// Gathered-row pipeline: n_chunks chunks of 32 list rows, src.key(r) the key
// of list row r (< 0: masked), loaded by cp.async into an S-stage ring (S - 1
// chunks of lookahead); consume(c, stage, valid_mask, 0) runs the math of
// chunk c.  The valid-row masks of the chunks in flight rotate through
// registers.
template <int D, int S = kStages, typename Src, typename Consume>
__device__ __forceinline__ void gather_pipeline(const __nv_bfloat16* kbase,
                                                const __nv_bfloat16* vbase, int n_chunks,
                                                const Src& src, uint32_t smem_base,
                                                Consume&& consume) {
    static_assert(!Src::kContig, "gathered rows");
    static_assert(S >= 1 && S <= 4, "ring depth");
    const int lane = threadIdx.x & 31;
    if constexpr (S == 1) {  // no lookahead: load, wait, compute
        for (int c = 0; c < n_chunks; ++c) {
            const int key = src.key(c * kChunk + lane);
            const uint32_t mask = __ballot_sync(0xffffffffu, key >= 0);
            load_chunk<D>(smem_base, kbase, vbase, key);
            cp_async_commit();
            cp_async_wait<0>();
            __syncwarp();
            consume(c, smem_base, mask, 0);
            __syncwarp();
        }
        return;
    }
    uint32_t mq[S > 1 ? S - 1 : 1];  // masks of chunks c .. c+S-2
    auto issue = [&](int c) -> uint32_t {
        const uint32_t sb = smem_base + (uint32_t)(c % S) * WarpSmem<D, S>::kStageBytes;
        const int key = src.key(c * kChunk + lane);
        const uint32_t mask = __ballot_sync(0xffffffffu, key >= 0);
        load_chunk<D>(sb, kbase, vbase, key);
        return mask;
    };
#pragma unroll
    for (int i = 0; i < S - 1; ++i) {
        mq[i] = i < n_chunks ? issue(i) : 0u;
        cp_async_commit();
    }
    for (int c = 0; c < n_chunks; ++c) {
        const uint32_t mnext = c + S - 1 < n_chunks ? issue(c + S - 1) : 0u;
        cp_async_commit();
        cp_async_wait<S - 1>();
        __syncwarp();
        consume(c, smem_base + (uint32_t)(c % S) * WarpSmem<D, S>::kStageBytes, mq[0], 0);
#pragma unroll
        for (int i = 0; i < S - 2; ++i) mq[i] = mq[i + 1];
        mq[S - 2] = mnext;
        __syncwarp();  // the stage is refilled by the next iteration
    }
    cp_async_wait<0>();
}

// Per-warp TMA ring: S consecutive mbarriers (one per stage) and the number
// of chunks that went through the ring so far; chunk k overall uses stage
// k % S with phase parity (k / S) & 1, across calls.
struct TmaRing {
    uint32_t bar;   // shared address of the stage mbarriers
    uint32_t next;  // chunks consumed (or drained) so far
};

// Contiguous-key pipeline: n_chunks chunks of 32 consecutive keys each;
// src.chunk(c, &key0) gives chunk c's first key and its valid-row mask.  One
// lane issues the TMA boxes {64, 32} of K and V (coordinates d, key, unit);
// rows past the cache end are zero-filled by the TMA.  S - 1 chunks of
// lookahead.  consume(c, stage, valid_mask, key0) runs the math of chunk c.
// Returns false if a wait timed out (HS_ERR_TIMEOUT is then set) after
// draining the loads in flight.
template <int D, int S = kStages, typename Src, typename Consume>
__device__ __forceinline__ bool tma_pipeline(const CUtensorMap* tk, const CUtensorMap* tv,
                                             int unit, int n_chunks, const Src& src,
                                             uint32_t smem_base, TmaRing& ring,
                                             Consume&& consume) {
    static_assert(Src::kContig, "consecutive keys");
    static_assert(S >= 1 && S <= 4, "ring depth");
    constexpr uint32_t kHalf = kChunk * 128;          // one d-half box
    constexpr uint32_t kTx = 2 * (D / 64) * kHalf;    // K and V, all halves
    const int lane = threadIdx.x & 31;
    const uint32_t k0 = ring.next;
    uint32_t mq[S > 1 ? S - 1 : 1];  // masks and first keys of chunks c .. c+S-2
    int kq[S > 1 ? S - 1 : 1];
    int dummy = 0;
    volatile int* no_abort = &dummy;
    auto issue = [&](int c, int& key0) -> uint32_t {
        const uint32_t st = (k0 + (uint32_t)c) % S;
        const uint32_t sb = smem_base + st * WarpSmem<D, S>::kStageBytes;
        const uint32_t mask = src.chunk(c, &key0);
        if (lane == 0) {
            const uint32_t b = ring.bar + 8u * st;
            tc::mbar_arrive_expect_tx(b, kTx);
#pragma unroll
            for (int h = 0; h < D / 64; ++h) {
                tc::tma_load_3d(sb + h * kHalf, tk, b, 64 * h, key0, unit);
                tc::tma_load_3d(sb + WarpSmem<D, S>::kTileBytes + h * kHalf, tv, b, 64 * h,
                                key0, unit);
            }
        }
        return mask;
    };
#pragma unroll
    for (int i = 0; i < S - 1; ++i) {
        kq[i] = 0;
        mq[i] = i < n_chunks ? issue(i, kq[i]) : 0u;
    }
    if constexpr (S == 1) { mq[0] = 0u; kq[0] = 0; }
    int issued = min(n_chunks, S - 1), failed = -1;
    for (int c = 0; c < n_chunks; ++c) {
        int knext = 0;
        uint32_t mnext = 0u;
        if (c + S - 1 < n_chunks) {
            mnext = issue(c + S - 1, knext);
            issued = c + S;
        }
        if constexpr (S == 1) { mq[0] = mnext; kq[0] = knext; }
        const uint32_t k = k0 + (uint32_t)c, st = k % S;
        // poll: a suspended warp wakes up late on this short critical path
        const bool got = tc::mbar_wait(ring.bar + 8u * st, (k / S) & 1u, no_abort, false);
        if (!__all_sync(0xffffffffu, got)) { failed = c; break; }
        consume(c, smem_base + st * WarpSmem<D, S>::kStageBytes, mq[0], kq[0]);
        if constexpr (S > 1) {
#pragma unroll
            for (int i = 0; i < S - 2; ++i) { mq[i] = mq[i + 1]; kq[i] = kq[i + 1]; }
            mq[S - 2] = mnext;
            kq[S - 2] = knext;
        }
        __syncwarp();  // the stage is refilled by the next iteration
    }
    if (failed >= 0) {
        // wait (bounded) for every load issued but not consumed before the
        // buffers can be reused, keeping the phase counts consistent
        for (int c = failed; c < issued; ++c) {
            const uint32_t k = k0 + (uint32_t)c, st = k % S;
            const long long t0 = clock64();
            while (!tc::mbar_try_wait(ring.bar + 8u * st, (k / S) & 1u))
                if (clock64() - t0 > tc::kWaitCycles) break;
        }
        ring.next = k0 + (uint32_t)issued;
        return false;
    }
    ring.next = k0 + (uint32_t)n_chunks;
    return true;
}

// Heads-as-rows attention over gathered rows (cp.async).
template <int D, int S = kStages, typename Src, typename Hook>
__device__ __forceinline__ void attend_rows(AttnState<D>& st, const uint32_t (&qf)[D / 16][4],
                                            const __nv_bfloat16* kbase,
                                            const __nv_bfloat16* vbase, int n_chunks,
                                            const Src& src, uint32_t smem_base, float scale_log2,
                                            Hook hook) {
    LaneOffs lo;
    lo.init();
    gather_pipeline<D, S>(kbase, vbase, n_chunks, src, smem_base,
                       [&](int c, uint32_t sb, uint32_t mask, int key0) {
                           float s[4][4];
                           chunk_scores<D>(s, qf, sb, mask, lo);
                           hook(c, s, key0);
                           chunk_update<D>(st, s, sb + WarpSmem<D>::kTileBytes, scale_log2, lo);
                       });
    finish_rows<D>(st);
}

// Heads-as-rows attention over runs of consecutive keys (TMA).  The optional
// per-chunk hook sees the masked raw logits and the chunk's first key.
template <int D, int S = kStages, typename Src, typename Hook>
__device__ __forceinline__ bool attend_rows_tma(AttnState<D>& st, const uint32_t (&qf)[D / 16][4],
                                                const CUtensorMap* tk, const CUtensorMap* tv,
                                                int unit, int n_chunks, const Src& src,
                                                uint32_t smem_base, TmaRing& ring,
                                                float scale_log2, Hook hook) {
    LaneOffs lo;
    lo.init();
    const bool ok = tma_pipeline<D, S>(tk, tv, unit, n_chunks, src, smem_base, ring,
                                    [&](int c, uint32_t sb, uint32_t mask, int key0) {
                                        float s[4][4];
                                        chunk_scores<D>(s, qf, sb, mask, lo);
                                        hook(c, s, key0);
                                        chunk_update<D>(st, s, sb + WarpSmem<D>::kTileBytes,
                                                        scale_log2, lo);
                                    });
    if (ok) finish_rows<D>(st);
    return ok;
}

// ---------------------------------------------------------- keys as rows
// For a group of at most 8 heads the heads-as-rows tile leaves at least half
// of the 16 MMA rows empty.  This form computes S^T = K Q^T instead: the 32
// keys of a chunk are the MMA rows (two 16-row tiles) and the heads the 8
// columns; then O^T += V^T P^T, with V^T tiles as the A operand (transposed
// ldmatrix of the V tile) and P^T as the B operand, taken from the S^T
// accumulators by an in-register 8x8 transpose (movmatrix).  It issues half
// the MMAs of the heads-as-rows form.  Lane l holds the columns (heads)
// 2(l&3) and 2(l&3)+1.

template <int D>
struct AttnStateT {
    float m[2], l[2];     // per head column j: running max (log2 domain), partial sum
    float o[D / 16][4];   // O^T fragments: rows d, columns heads
    __device__ __forceinline__ void init() {
        m[0] = m[1] = -INFINITY;
        l[0] = l[1] = 0.f;
#pragma unroll
        for (int n = 0; n < D / 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    }
};

// B fragments of Q^T (d x 8 heads): column = head lane/4 (zero if >= g).
template <int D>
__device__ __forceinline__ void load_qt_frags(uint32_t (&qb)[D / 16][2],
                                              const __nv_bfloat16* q, size_t head_stride,
                                              int g) {
    const int lane = threadIdx.x & 31, h = lane >> 2, tig = lane & 3;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        const int c0 = kk * 16 + tig * 2;
        qb[kk][0] = h < g ? *reinterpret_cast<const uint32_t*>(q + h * head_stride + c0) : 0u;
        qb[kk][1] = h < g ? *reinterpret_cast<const uint32_t*>(q + h * head_stride + c0 + 8) : 0u;
    }
}

__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

// One chunk: S^T = K Q^T, masking, online softmax per head column (lazy
// rescale as in chunk_update), O^T += V^T P^T.
template <int D>
__device__ __forceinline__ void chunk_t(AttnStateT<D>& st, const uint32_t (&qb)[D / 16][2],
                                        uint32_t sb, uint32_t valid_mask, float scale_log2,
                                        const LaneOffs& lo) {
    const int lane = threadIdx.x & 31;
    float s[2][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) s[mt][0] = s[mt][1] = s[mt][2] = s[mt][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
            // A = K rows mt*16.. (keys) x d kk*16..: matrices (keys 0-7 | 8-15) x (d 0-7 | 8-15)
            // == tile_off(mt*16 + (lane&7) + (((lane>>3)&1)<<3), kk*2 + (lane>>4))
            uint32_t a[4];
            ldsm_x4(sb + lo.v[kk & 3] + (uint32_t)((kk >> 2) * (kChunk * 128) + mt * 16 * 128),
                    a[0], a[1], a[2], a[3]);
            mma_bf16(s[mt], a, qb[kk][0], qb[kk][1]);
        }
    }
    if (valid_mask != 0xffffffffu) {
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int key = mt * 16 + (lane >> 2) + 8 * (e >> 1);
                s[mt][e] = ((valid_mask >> key) & 1u) ? s[mt][e] : -INFINITY;
            }
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {  // head column 2(lane&3) + j
        float mx = fmaxf(fmaxf(s[0][j], s[0][j + 2]), fmaxf(s[1][j], s[1][j + 2]));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        mx *= scale_log2;  // -inf stays -inf
        if (mx > st.m[j] + 8.f) {
            const float corr = ex2f_fast(st.m[j] - mx);  // 0 while nothing was seen
            st.l[j] *= corr;
#pragma unroll
            for (int n = 0; n < D / 16; ++n) {
                st.o[n][j] *= corr;
                st.o[n][j + 2] *= corr;
            }
            st.m[j] = mx;
        }
        const float nm = st.m[j] == -INFINITY ? 0.f : -st.m[j];
        float sum = 0.f;
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
            s[mt][j] = ex2f_fast(fmaf(s[mt][j], scale_log2, nm));
            s[mt][j + 2] = ex2f_fast(fmaf(s[mt][j + 2], scale_log2, nm));
            sum += s[mt][j] + s[mt][j + 2];
        }
        st.l[j] += sum;
    }
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {  // keys ks*16 .. ks*16+15
        // P^T B fragments: transpose the [key][head] 8x8 blocks to [head][key]
        const uint32_t b0 = movmatrix_t(pack_bf16(s[ks][0], s[ks][1]));
        const uint32_t b1 = movmatrix_t(pack_bf16(s[ks][2], s[ks][3]));
#pragma unroll
        for (int dt = 0; dt < D / 16; ++dt) {
            // A = V^T: d dt*16.. x keys; matrices (d 0-7 | 8-15) x (keys 0-7 | 8-15)
            // == tile_off(ks*16 + (lane&7) + ((lane>>4)<<3), dt*2 + ((lane>>3)&1))
            uint32_t a[4];
            ldsm_x4_t(sb + WarpSmem<D>::kTileBytes + lo.k[dt & 3] +
                          (uint32_t)((dt >> 2) * (kChunk * 128) + ks * 16 * 128),
                      a[0], a[1], a[2], a[3]);
            mma_bf16(st.o[dt], a, b0, b1);
        }
    }
}

// Finish the per-head sums across the 8 lanes sharing a head column.
template <int D>
__device__ __forceinline__ void finish_rows_t(AttnStateT<D>& st) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        st.l[j] += __shfl_xor_sync(0xffffffffu, st.l[j], 4);
        st.l[j] += __shfl_xor_sync(0xffffffffu, st.l[j], 8);
        st.l[j] += __shfl_xor_sync(0xffffffffu, st.l[j], 16);
    }
}

template <int D, int S, typename Src>
__device__ __forceinline__ void attend_rows_t(AttnStateT<D>& st,
                                              const uint32_t (&qb)[D / 16][2],
                                              const __nv_bfloat16* kbase,
                                              const __nv_bfloat16* vbase, int n_chunks,
                                              const Src& src, uint32_t smem_base,
                                              float scale_log2) {
    LaneOffs lo;
    lo.init();
    gather_pipeline<D, S>(kbase, vbase, n_chunks, src, smem_base,
                       [&](int, uint32_t sb, uint32_t mask, int) {
                           chunk_t<D>(st, qb, sb, mask, scale_log2, lo);
                       });
    finish_rows_t<D>(st);
}

template <int D, int S, typename Src>
__device__ __forceinline__ bool attend_rows_tma_t(AttnStateT<D>& st,
                                                  const uint32_t (&qb)[D / 16][2],
                                                  const CUtensorMap* tk, const CUtensorMap* tv,
                                                  int unit, int n_chunks, const Src& src,
                                                  uint32_t smem_base, TmaRing& ring,
                                                  float scale_log2) {
    LaneOffs lo;
    lo.init();
    const bool ok = tma_pipeline<D, S>(tk, tv, unit, n_chunks, src, smem_base, ring,
                                    [&](int, uint32_t sb, uint32_t mask, int) {
                                        chunk_t<D>(st, qb, sb, mask, scale_log2, lo);
                                    });
    if (ok) finish_rows_t<D>(st);
    return ok;
}

// Normalise and store heads < g: o[h * head_stride + d] (bf16), lse natural
// log.  Lanes l and l^4 hold neighbouring d of the same two heads; one
// exchange lets each store a bf16 pair of one head.
template <int D>
__device__ __forceinline__ void store_rows_t(const AttnStateT<D>& st, __nv_bfloat16* o,
                                             size_t head_stride, float* lse, size_t lse_stride,
                                             int g) {
    const int lane = threadIdx.x & 31, h0 = 2 * (lane & 3), r = lane >> 2;
    const float inv0 = st.l[0] > 0.f ? 1.f / st.l[0] : 0.f;
    const float inv1 = st.l[1] > 0.f ? 1.f / st.l[1] : 0.f;
    const bool odd = r & 1;
#pragma unroll
    for (int dt = 0; dt < D / 16; ++dt) {
#pragma unroll
        for (int e2 = 0; e2 < 2; ++e2) {
            const int d = dt * 16 + r + 8 * e2;
            const float va = st.o[dt][2 * e2] * inv0, vb = st.o[dt][2 * e2 + 1] * inv1;
            const float recv = __shfl_xor_sync(0xffffffffu, odd ? va : vb, 4);
            if (!odd) {  // head h0 at d, d+1
                if (h0 < g)
                    *reinterpret_cast<uint32_t*>(o + h0 * head_stride + d) = pack_bf16(va, recv);
            } else {     // head h0+1 at d-1, d
                if (h0 + 1 < g)
                    *reinterpret_cast<uint32_t*>(o + (h0 + 1) * head_stride + d - 1) =
                        pack_bf16(recv, vb);
            }
        }
    }
    if (r == 0) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            if (h0 + j >= g) continue;
            const float l = st.l[j];
            lse[(h0 + j) * lse_stride] = l > 0.f ? (st.m[j] + log2f(l)) * kLn2 : -INFINITY;
        }
    }
}

// Keys first..last (inclusive) as contiguous chunks.
// Logical key -> row of a paged pool for one (sequence, kv group): the
// index sets keep logical token ids and the block table turns each into its
// page and row as the gather loads it ("HySparse 混合稀疏注意力（一）",
// 工程实现中的关键约束 item 2: the sparse index keeps logical token ranges,
// a block table translates them into physical page pieces, the kernel reads
// them directly).  A page id outside the pool marks the row masked and sets
// HS_ERR_BOUNDS.
struct PageMap {
    const int32_t* bt;  // this sequence's row of the block table
    int page_size, max_pages, n_pages, hkv, u;
    __device__ __forceinline__ int row(int key) const {
        const int lp = key / page_size;
        const int pg = lp < max_pages ? bt[lp] : -1;
        if (pg < 0 || pg >= n_pages) { set_status(HS_ERR_BOUNDS); return -1; }
        return (pg * hkv + u) * page_size + (key - lp * page_size);
    }
};

// A gathered-row source whose keys are translated through a PageMap; the
// gather then reads from the pool's base.
template <class Src>
struct PagedSrc {
    static constexpr bool kContig = false;
    Src src;
    PageMap pm;
    __device__ __forceinline__ int key(int r) const {
        const int k = src.key(r);
        return k < 0 ? -1 : pm.row(k);
    }
};

// Consecutive keys first..last as a gathered-row source (for pools, whose
// rows are not consecutive across pages).
struct KeyRange {
    static constexpr bool kContig = false;
    int first, last;
    __device__ __forceinline__ int n_chunks() const { return (last - first + kChunk) / kChunk; }
    __device__ __forceinline__ int key(int r) const { return first + r <= last ? first + r : -1; }
};

__device__ __forceinline__ PageMap page_map(const KParams& p, int b, int u) {
    return PageMap{p.bt + (size_t)b * p.max_pages, p.page_size, p.max_pages, p.n_pages, p.hkv, u};
}

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
