// attend_mma.cuh -- one warp attends the (up to 16) query heads of a GQA group
// over a list of key rows of that group's K/V, with mma.sync tensor-core
// fragments (bf16 in, fp32 accumulate) and an online softmax.
//
// The 16 MMA rows are the heads of the group, so every gathered K/V row is
// loaded once and used by all of them ("HySparse 混合稀疏注意力（一）", GQA:
// the group shares one index set so each selected row is read once).  Rows are
// fetched 32 at a time with 16-byte cp.async into a 2-stage, XOR-swizzled
// shared-memory ring owned by the warp; masked rows are zero-filled and get a
// -inf logit.
#pragma once

#include "hs_common.cuh"

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
        const uint32_t so = swz(r, c, WarpSmem<D>::kRowBytes);
        cp_async16(stage_base + so, kbase + off, ok);
        cp_async16(stage_base + WarpSmem<D>::kTileBytes + so, vbase + off, ok);
    }
}

// S = Q K^T for one chunk (16 x 32), scaled to log2 domain and masked.
template <int D>
__device__ __forceinline__ void chunk_scores(float (&s)[4][4], const uint32_t (&qf)[D / 16][4],
                                             uint32_t kst, uint32_t valid_mask,
                                             float scale_log2) {
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
            ldsm_x4(kst + swz(key, chunk, WarpSmem<D>::kRowBytes), b0, b1, b2, b3);
            mma_bf16(s[np * 2], qf[kk], b0, b1);
            mma_bf16(s[np * 2 + 1], qf[kk], b2, b3);
        }
    }
#pragma unroll
    for (int n = 0; n < 4; ++n) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int col = n * 8 + tig * 2 + (e & 1);
            s[n][e] = ((valid_mask >> col) & 1u) ? s[n][e] * scale_log2 : -INFINITY;
        }
    }
}

// Online-softmax update with one chunk of scores, then O += P V.
template <int D>
__device__ __forceinline__ void chunk_update(AttnState<D>& st, float (&s)[4][4], uint32_t vst) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {  // row gid (hr=0) and gid+8 (hr=1)
        float mx = -INFINITY;
#pragma unroll
        for (int n = 0; n < 4; ++n) mx = fmaxf(mx, fmaxf(s[n][2 * hr], s[n][2 * hr + 1]));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        const float m_new = fmaxf(st.m[hr], mx);
        // all -inf so far: keep exp2 arguments finite
        const float m_use = m_new == -INFINITY ? 0.f : m_new;
        const float corr = exp2f(st.m[hr] - m_use);
        float sum = 0.f;
#pragma unroll
        for (int n = 0; n < 4; ++n) {
            s[n][2 * hr] = exp2f(s[n][2 * hr] - m_use);
            s[n][2 * hr + 1] = exp2f(s[n][2 * hr + 1] - m_use);
            sum += s[n][2 * hr] + s[n][2 * hr + 1];
        }
        st.l[hr] = st.l[hr] * corr + sum;
        st.m[hr] = m_new;
#pragma unroll
        for (int n = 0; n < D / 8; ++n) {
            st.o[n][2 * hr] *= corr;
            st.o[n][2 * hr + 1] *= corr;
        }
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
            ldsm_x4_t(vst + swz(key, chunk, WarpSmem<D>::kRowBytes), b0, b1, b2, b3);
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

// Run the pipeline over n_rows rows; key_of(r) gives the key of list row r
// (< 0: masked).  Optional per-chunk hook sees the scaled logits before the
// softmax (used by the decode indexer to export logits).
template <int D, typename KeyOf, typename Hook>
__device__ __forceinline__ void attend_rows(AttnState<D>& st, const uint32_t (&qf)[D / 16][4],
                                            const __nv_bfloat16* kbase,
                                            const __nv_bfloat16* vbase, int n_rows,
                                            KeyOf key_of, uint32_t smem_base, float scale_log2,
                                            Hook hook) {
    const int lane = threadIdx.x & 31;
    const int n_chunks = (n_rows + kChunk - 1) / kChunk;
    int keys[kStages];
    uint32_t masks[kStages];
    // prologue
#pragma unroll
    for (int sgi = 0; sgi < kStages - 1; ++sgi) {
        if (sgi < n_chunks) {
            const int r = sgi * kChunk + lane;
            const int key = r < n_rows ? key_of(r) : -1;
            keys[sgi] = key;
            masks[sgi] = __ballot_sync(0xffffffffu, key >= 0);
            load_chunk<D>(smem_base + sgi * WarpSmem<D>::kStageBytes, kbase, vbase, key);
        }
        cp_async_commit();
    }
    for (int c = 0; c < n_chunks; ++c) {
        const int nxt = c + kStages - 1;
        if (nxt < n_chunks) {
            const int r = nxt * kChunk + lane;
            const int key = r < n_rows ? key_of(r) : -1;
            keys[nxt % kStages] = key;
            masks[nxt % kStages] = __ballot_sync(0xffffffffu, key >= 0);
            load_chunk<D>(smem_base + (nxt % kStages) * WarpSmem<D>::kStageBytes, kbase, vbase,
                          key);
        }
        cp_async_commit();
        cp_async_wait<kStages - 1>();
        __syncwarp();
        const uint32_t sb = smem_base + (c % kStages) * WarpSmem<D>::kStageBytes;
        float s[4][4];
        chunk_scores<D>(s, qf, sb, masks[c % kStages], scale_log2);
        hook(c, s, keys[c % kStages]);
        chunk_update<D>(st, s, sb + WarpSmem<D>::kTileBytes);
        __syncwarp();  // the stage is refilled by the next iteration
    }
    cp_async_wait<0>();
    finish_rows<D>(st);
}

struct ContiguousKeys {
    int first, last;  // inclusive range
    __device__ __forceinline__ int operator()(int r) const {
        const int key = first + r;
        return key <= last ? key : -1;
    }
};

// Partial result of one split: per head (m2, l, O[D]) fp32, unnormalised.
// Layout [16][D + 2]: m2, l, o[0..D).
template <int D>
__device__ __forceinline__ void store_partial(const AttnState<D>& st, float* part, int g) {
    // part layout: [16][D + 2]: m2, l, o[0..D)
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
