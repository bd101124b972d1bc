// sparse.cu -- the sparse layers that reuse the full layer's K^F / V^F and
// index set ("HySparse 混合稀疏注意力（一）", "跨层 KV Cache 复用怎样成立" and
// "同一个 Query，查询两种记忆"; "HySparse: ..." 3.3; "HySparse2 ..." 4.2).
//
// For query row t of KV group u, with the layer's own query q'_h:
//   R_t  = selected tokens (token mode), or the keys of the selected blocks
//          clipped to i <= t (block mode, in-block causal mask: "工程实现中的
//          关键约束" item 4);
//   o_h  = sum_{i in R_t} softmax_{R_t}(tau q'_h . k_i) v_i.
// HySparse sparse layers also run a window branch over their own K'/V' for
// keys max(0, t-w+1)..t, returned as a second output.
//
// Kernels
//   sparse_simt_kernel  fp32 / any shape: one CTA per row, one warp per head.
//   sparse_mma_kernel   bf16: one warp per (row, group), so each gathered row
//                       is read once for all the group's heads; the heads are
//                       the 16 MMA rows (groups of 9-16 heads), or the keys
//                       are (S^T = K Q^T, groups of at most 8 heads).
//   decode_sparse_*     bf16 decode: the selected rows of one (sequence, group)
//                       split across warps, then an exact log-sum-exp merge.
#include <atomic>

#include "attend_mma.cuh"
#include "hs_common.cuh"
#include "hs_kernels.cuh"

namespace hs {

// Key of row r of the gathered list, -1 if masked; flags out-of-range ids.
// Token mode: the selected keys themselves.  Block mode: block r / B, offset
// r % B, clipped to keys <= t (a selected block may cross the query).
struct GatherKeys {
    static constexpr bool kContig = false;
    const int32_t* ids;
    int n_rows, B, t, mode;
    __device__ __forceinline__ int key(int r) const {
        if (r >= n_rows) return -1;
        if (mode == 0) {
            const int jb = r / B;
            const int id = ids[jb];
            if (id < 0 || id > t / B) { set_status(HS_ERR_BOUNDS); return -1; }
            const int key = id * B + (r - jb * B);
            return key <= t ? key : -1;
        }
        const int key = ids[r];
        if (key < 0 || key > t) { set_status(HS_ERR_BOUNDS); return -1; }
        return key;
    }
    __device__ __forceinline__ int operator()(int r) const { return key(r); }
};

// Block mode with B a multiple of 32: every 32-row chunk is 32 consecutive
// keys of one selected block, so it is loaded as one contiguous range.
struct BlockChunks {
    static constexpr bool kContig = true;
    const int32_t* ids;
    int B, t;
    __device__ __forceinline__ uint32_t chunk(int c, int* key0) const {
        const int per = B / kChunk;
        const int jb = c / per;
        const int id = ids[jb];
        if (id < 0 || id > t / B) {
            set_status(HS_ERR_BOUNDS);
            *key0 = 0;
            return 0u;
        }
        *key0 = id * B + (c - jb * per) * kChunk;
        const int n = t - *key0 + 1;
        return n >= 32 ? 0xffffffffu : (n <= 0 ? 0u : ((1u << n) - 1u));
    }
};

__device__ __forceinline__ int clamp_count(int c, int ksel) {
    if (c < 0 || c > ksel) { set_status(HS_ERR_BOUNDS); return c < 0 ? 0 : ksel; }
    return c;
}

// ------------------------------------------------------------------ SIMT path
template <typename T, int D, typename KeyOf>
__device__ void simt_attend(const float* qh, const T* kbase, const T* vbase, int n_rows,
                            KeyOf key_of, T* orow, float* lse_out) {
    const int lane = threadIdx.x & 31;
    constexpr int E = D / 32;
    float m = -INFINITY, l = 0.f, acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.f;
    for (int c0 = 0; c0 < n_rows; c0 += 32) {
        const int r = c0 + lane;
        const int key = r < n_rows ? key_of(r) : -1;
        float a = -INFINITY;
        if (key >= 0) {
            const T* kr = kbase + (size_t)key * D;
            float s = 0.f;
#pragma unroll 8
            for (int x = 0; x < D; ++x) s += qh[x] * to_f(kr[x]);
            a = s;
        }
        const float mx = warp_max(a);
        const float m_new = fmaxf(m, mx);
        const float m_use = m_new == -INFINITY ? 0.f : m_new;
        const float pr = key >= 0 ? exp2f(a - m_use) : 0.f;
        const float corr = exp2f(m - m_use);
        l = l * corr + warp_sum(pr);
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] *= corr;
        const int nk = min(32, n_rows - c0);
        for (int jj = 0; jj < nk; ++jj) {
            const float pj = __shfl_sync(0xffffffffu, pr, jj);
            const int kj = __shfl_sync(0xffffffffu, key, jj);
            if (kj >= 0) {
                const T* vr = vbase + (size_t)kj * D + lane * E;
#pragma unroll
                for (int e = 0; e < E; ++e) acc[e] += pj * to_f(vr[e]);
            }
        }
        m = m_new;
    }
    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) orow[lane * E + e] = from_f<T>(acc[e] * inv);
    if (lane == 0 && lse_out) *lse_out = l > 0.f ? (m + log2f(l)) * kLn2 : -INFINITY;
}

// One CTA per (batch, kv group, query row) -- in decode per (sequence, kv
// group) at the newest position -- whose warps take the group's heads in
// turn (groups of up to 64 heads, head_dim up to 256).
template <typename T, int D>
__global__ void sparse_simt_kernel(KParams p, const T* __restrict__ q, const T* __restrict__ kf,
                                   const T* __restrict__ vf, const int32_t* __restrict__ idx,
                                   const int32_t* __restrict__ cnt, const T* __restrict__ kl,
                                   const T* __restrict__ vl, T* __restrict__ og,
                                   float* __restrict__ lseg, T* __restrict__ ol,
                                   float* __restrict__ lsel, const int32_t* __restrict__ seq_len) {
    extern __shared__ float qs[];  // [g][D]
    const int j = blockIdx.x, u = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int g = p.group;
    const int t = seq_len ? seq_len[b] - 1 : p.q_offset + j;
    const bool valid = t >= 0 && t < p.t_kv;
    if (!valid && threadIdx.x == 0) set_status(HS_ERR_BOUNDS);
    for (int x = threadIdx.x; x < g * D; x += blockDim.x) {
        const int h = u * g + x / D;
        qs[x] = to_f(q[(((size_t)b * p.hq + h) * p.t_q + j) * D + x % D]) * p.scale_log2;
    }
    __syncthreads();
    const size_t row = ((size_t)b * p.hkv + u) * p.t_q + j;
    const size_t kvoff = ((size_t)b * p.hkv + u) * p.t_kv * D;
    const int c = valid ? clamp_count(cnt[row], p.ksel) : 0;
    const int n_rows = p.mode == 0 ? c * p.block_size : c;
    const GatherKeys keys{idx + row * p.ksel, n_rows, p.block_size, t, p.mode};
    for (int hw = warp; hw < g; hw += nw) {
        const size_t orow = ((size_t)b * p.hq + u * g + hw) * p.t_q + j;
        simt_attend<T, D>(qs + hw * D, kf + kvoff, vf + kvoff, n_rows, keys, og + orow * D,
                          lseg ? lseg + orow : nullptr);
        if (kl) {
            const int first = max(0, t - p.window + 1);
            simt_attend<T, D>(qs + hw * D, kl + kvoff, vl + kvoff, valid ? t - first + 1 : 0,
                              [=](int r) { return first + r <= t ? first + r : -1; },
                              ol + orow * D, lsel + orow);
        }
    }
}

template <typename T, int D>
static cudaError_t launch_sparse_simt_t(const KParams& p, const void* q, const void* kf,
                                        const void* vf, const int32_t* idx, const int32_t* cnt,
                                        const void* kl, const void* vl, void* og, float* lseg,
                                        void* ol, float* lsel, const int32_t* seq_len,
                                        cudaStream_t st) {
    dim3 grid(p.t_q, p.hkv, p.batch);
    const int threads = 32 * (p.group < 16 ? p.group : 16);
    const size_t smem = sizeof(float) * p.group * D;
    auto kern = sparse_simt_kernel<T, D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, threads, smem, st>>>(p, (const T*)q, (const T*)kf, (const T*)vf, idx, cnt,
                                       (const T*)kl, (const T*)vl, (T*)og, lseg, (T*)ol, lsel,
                                       seq_len);
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_sparse_simt_d(const KParams& p, const void* q, const void* kf,
                                        const void* vf, const int32_t* idx, const int32_t* cnt,
                                        const void* kl, const void* vl, void* og, float* lseg,
                                        void* ol, float* lsel, const int32_t* seq_len,
                                        cudaStream_t st) {
    if (p.head_dim == 64)
        return launch_sparse_simt_t<T, 64>(p, q, kf, vf, idx, cnt, kl, vl, og, lseg, ol, lsel,
                                           seq_len, st);
    if (p.head_dim == 128)
        return launch_sparse_simt_t<T, 128>(p, q, kf, vf, idx, cnt, kl, vl, og, lseg, ol, lsel,
                                            seq_len, st);
    return launch_sparse_simt_t<T, 256>(p, q, kf, vf, idx, cnt, kl, vl, og, lseg, ol, lsel,
                                        seq_len, st);
}

cudaError_t launch_sparse_simt(const KParams& p, int dtype, const void* q, const void* kf,
                               const void* vf, const int32_t* idx, const int32_t* cnt,
                               const void* kl, const void* vl, void* og, float* lseg, void* ol,
                               float* lsel, cudaStream_t st, const int32_t* seq_len) {
    if (dtype == HS_FP32)
        return launch_sparse_simt_d<float>(p, q, kf, vf, idx, cnt, kl, vl, og, lseg, ol, lsel,
                                           seq_len, st);
    return launch_sparse_simt_d<__nv_bfloat16>(p, q, kf, vf, idx, cnt, kl, vl, og, lseg, ol, lsel,
                                               seq_len, st);
}

// ------------------------------------------------------------ tensor-core path
constexpr int kSparseWarps = 6;  // decode kernels: warps per CTA, 2-stage rings

// Normalise and store rows < g of a finished warp state.
template <int D>
__device__ __forceinline__ void store_rows(const AttnState<D>& st, __nv_bfloat16* o,
                                           size_t head_stride, float* lse, size_t lse_stride,
                                           int g) {
    const int lane = threadIdx.x & 31, gid = lane >> 2, tig = lane & 3;
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
        const int h = gid + 8 * hr;
        if (h >= g) continue;
        const float l = st.l[hr];
        const float inv = l > 0.f ? 1.f / l : 0.f;
        __nv_bfloat16* orow = o + h * head_stride;
#pragma unroll
        for (int n = 0; n < D / 8; ++n) {
            const int col = n * 8 + tig * 2;
            *reinterpret_cast<uint32_t*>(orow + col) =
                pack_bf16(st.o[n][2 * hr] * inv, st.o[n][2 * hr + 1] * inv);
        }
        if (tig == 0) lse[h * lse_stride] = l > 0.f ? (st.m[hr] + log2f(l)) * kLn2 : -INFINITY;
    }
}

// Dynamic shared memory: per warp an S-stage K/V ring, then per warp S mbarriers.
template <int D, int W, int S>
constexpr size_t sparse_smem_bytes() {
    return (size_t)W * WarpSmem<D, S>::kBytes + (size_t)W * 8 * S + 1024;
}

// W warps per CTA, each attending one (row, group) task through an S-stage
// ring.  kT: keys-as-rows form (groups of at most 8 heads); else heads as rows.
template <int D, bool kT, int W, int S>
__global__ void __launch_bounds__(W * 32)
    sparse_mma_kernel(const __grid_constant__ CUtensorMap tm_kf,
                      const __grid_constant__ CUtensorMap tm_vf,
                      const __grid_constant__ CUtensorMap tm_kl,
                      const __grid_constant__ CUtensorMap tm_vl, KParams p,
                      const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ kf,
                      const __nv_bfloat16* __restrict__ vf, const int32_t* __restrict__ idx,
                      const int32_t* __restrict__ cnt, int has_local,
                      __nv_bfloat16* __restrict__ og, float* __restrict__ lseg,
                      __nv_bfloat16* __restrict__ ol, float* __restrict__ lsel) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long task = (long long)blockIdx.x * W + warp;
    const long long n_tasks = (long long)p.batch * p.hkv * p.t_q;
    if (task >= n_tasks) return;
    const int j = (int)(task % p.t_q);
    const int u = (int)((task / p.t_q) % p.hkv);
    const int b = (int)(task / ((long long)p.t_q * p.hkv));
    const int g = p.group;
    const int t = p.q_offset + j;
    const uint32_t sbase = base + warp * WarpSmem<D, S>::kBytes;
    TmaRing ring{base + W * WarpSmem<D, S>::kBytes + 8u * S * warp, 0u};
    if (lane == 0) {
#pragma unroll
        for (int i = 0; i < S; ++i) tc::mbar_init(ring.bar + 8u * i, 1);
        tc::fence_mbar_init();
    }
    __syncwarp();

    const size_t head_stride = (size_t)p.t_q * D;
    const size_t q0 = (((size_t)b * p.hq + u * g) * p.t_q + j);  // row of head u*g
    const int unit = b * p.hkv + u;
    const size_t row = (size_t)unit * p.t_q + j;
    const size_t kvoff = (size_t)unit * p.t_kv * D;
    // has_local: bit 0 = run the window branch, bit 1 = skip the global branch
    // (computed by another kernel)
    const bool do_global = !(has_local & 2);
    const int c = do_global ? clamp_count(cnt[row], p.ksel) : 0;
    const int n_rows = p.mode == 0 ? c * p.block_size : c;
    if constexpr (kT) {
        uint32_t qb[D / 16][2];
        load_qt_frags<D>(qb, q + q0 * D, head_stride, g);
        AttnStateT<D> st;
        st.init();
        if (!do_global) {
        } else if (p.bt) {  // paged K^F/V^F: every row through the block table
            const PagedSrc<GatherKeys> keys{
                GatherKeys{idx + row * p.ksel, n_rows, p.block_size, t, p.mode}, page_map(p, b, u)};
            attend_rows_t<D, S>(st, qb, kf, vf, (n_rows + kChunk - 1) / kChunk, keys, sbase,
                                p.scale_log2);
        } else if (p.mode == 0 && p.block_size % kChunk == 0) {
            BlockChunks src{idx + row * p.ksel, p.block_size, t};
            attend_rows_tma_t<D, S>(st, qb, &tm_kf, &tm_vf, unit, c * (p.block_size / kChunk),
                                    src, sbase, ring, p.scale_log2);
        } else {
            GatherKeys keys{idx + row * p.ksel, n_rows, p.block_size, t, p.mode};
            attend_rows_t<D, S>(st, qb, kf + kvoff, vf + kvoff, (n_rows + kChunk - 1) / kChunk,
                                keys, sbase, p.scale_log2);
        }
        if (do_global) store_rows_t<D>(st, og + q0 * D, head_stride, lseg + q0, p.t_q, g);
        if (has_local & 1) {
            const int first = max(0, t - p.window + 1);
            AttnStateT<D> sl;
            sl.init();
            const ContiguousKeys win{first, t};
            attend_rows_tma_t<D, S>(sl, qb, &tm_kl, &tm_vl, unit, win.n_chunks(), win, sbase,
                                    ring, p.scale_log2);
            store_rows_t<D>(sl, ol + q0 * D, head_stride, lsel + q0, p.t_q, g);
        }
        return;
    }
    uint32_t qf[D / 16][4];
    load_q_frags<D>(qf, q + q0 * D, head_stride, g);

    AttnState<D> st;
    st.init();
    if (!do_global) {
    } else if (p.bt) {  // paged K^F/V^F: every row through the block table
        const PagedSrc<GatherKeys> keys{
            GatherKeys{idx + row * p.ksel, n_rows, p.block_size, t, p.mode}, page_map(p, b, u)};
        attend_rows<D, S>(st, qf, kf, vf, (n_rows + kChunk - 1) / kChunk, keys, sbase,
                          p.scale_log2, NoHook{});
    } else if (p.mode == 0 && p.block_size % kChunk == 0) {
        BlockChunks src{idx + row * p.ksel, p.block_size, t};
        attend_rows_tma<D, S>(st, qf, &tm_kf, &tm_vf, unit, c * (p.block_size / kChunk), src,
                              sbase, ring, p.scale_log2, NoHook{});
    } else {
        GatherKeys keys{idx + row * p.ksel, n_rows, p.block_size, t, p.mode};
        attend_rows<D, S>(st, qf, kf + kvoff, vf + kvoff, (n_rows + kChunk - 1) / kChunk, keys,
                          sbase, p.scale_log2, NoHook{});
    }
    if (do_global) store_rows<D>(st, og + q0 * D, head_stride, lseg + q0, p.t_q, g);
    if (has_local & 1) {
        const int first = max(0, t - p.window + 1);
        AttnState<D> sl;
        sl.init();
        const ContiguousKeys win{first, t};
        attend_rows_tma<D, S>(sl, qf, &tm_kl, &tm_vl, unit, win.n_chunks(), win, sbase, ring,
                              p.scale_log2, NoHook{});
        store_rows<D>(sl, ol + q0 * D, head_stride, lsel + q0, p.t_q, g);
    }
}

template <int D, bool kT, int W, int S>
static cudaError_t launch_sparse_cfg(const KParams& p, const CUtensorMap& mk,
                                     const CUtensorMap& mv, const CUtensorMap& mkl,
                                     const CUtensorMap& mvl, const void* q, const void* kf,
                                     const void* vf, const int32_t* idx, const int32_t* cnt,
                                     int has_local, void* og, float* lseg, void* ol, float* lsel,
                                     cudaStream_t st) {
    constexpr size_t smem = sparse_smem_bytes<D, W, S>();
    auto kern = sparse_mma_kernel<D, kT, W, S>;
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long n_tasks = (long long)p.batch * p.hkv * p.t_q;
    const unsigned grid = (unsigned)((n_tasks + W - 1) / W);
    kern<<<grid, W * 32, smem, st>>>(mk, mv, mkl, mvl, p, (const __nv_bfloat16*)q,
                                     (const __nv_bfloat16*)kf, (const __nv_bfloat16*)vf, idx, cnt,
                                     has_local, (__nv_bfloat16*)og, lseg,
                                     (__nv_bfloat16*)ol, lsel);
    return cudaGetLastError();
}

template <int D>
static cudaError_t launch_sparse_mma_t(const KParams& p, const void* q, const void* kf,
                                       const void* vf, const int32_t* idx, const int32_t* cnt,
                                       const void* kl, const void* vl, void* og, float* lseg,
                                       void* ol, float* lsel, bool global, cudaStream_t st) {
    const int flags = (kl ? 1 : 0) | (global ? 0 : 2);
    CUtensorMap mk, mv, mkl, mvl;
    const long long units = (long long)p.batch * p.hkv;
    // a paged pool is read by gathers only: its maps (unused) span the pool
    const long long rows = p.bt ? (long long)p.n_pages * p.hkv * p.page_size : p.t_kv;
    const long long mu = p.bt ? 1 : units;
    if (!tc::encode_rows(&mk, kf, D, rows, mu, kChunk) ||
        !tc::encode_rows(&mv, vf, D, rows, mu, kChunk))
        return cudaErrorInvalidValue;
    if (kl) {
        if (!tc::encode_rows(&mkl, kl, D, p.t_kv, units, kChunk) ||
            !tc::encode_rows(&mvl, vl, D, p.t_kv, units, kChunk))
            return cudaErrorInvalidValue;
    } else {
        mkl = mk;
        mvl = mv;
    }
    // The rate follows the number of resident warps: each warp's own chain of
    // dependent MMA, shuffle and exp2 steps is long, and other warps hide it
    // better than a deeper per-warp load lookahead does.  So one stage per
    // warp and as many warps as shared memory (16 KB each at d = 128) and
    // registers allow: 14 for the keys-as-rows form (126 registers), 12 for
    // the heads-as-rows form (168).  At d = 128 these beat 6 warps x 2 stages
    // by 1.6x and 1.4x; 4 x 3 and 3 x 4 were slower still.
    if (p.group <= 8)
        return launch_sparse_cfg<D, true, 14, 1>(p, mk, mv, mkl, mvl, q, kf, vf, idx, cnt, flags,
                                                 og, lseg, ol, lsel, st);
    return launch_sparse_cfg<D, false, 12, 1>(p, mk, mv, mkl, mvl, q, kf, vf, idx, cnt, flags, og,
                                              lseg, ol, lsel, st);
}

cudaError_t launch_sparse_mma(const KParams& p, const void* q, const void* kf, const void* vf,
                              const int32_t* idx, const int32_t* cnt, const void* kl,
                              const void* vl, void* og, float* lseg, void* ol, float* lsel,
                              cudaStream_t st, bool global) {
    if (p.head_dim == 64)
        return launch_sparse_mma_t<64>(p, q, kf, vf, idx, cnt, kl, vl, og, lseg, ol, lsel, global,
                                       st);
    return launch_sparse_mma_t<128>(p, q, kf, vf, idx, cnt, kl, vl, og, lseg, ol, lsel, global,
                                    st);
}

// ------------------------------------------------------------------- decode
// Partial result of one split: per head (m2, l, O[D]) in fp32, unnormalised.
constexpr int kDecodeSparseRows = 64;  // selected rows per split


template <int D>
__global__ void __launch_bounds__(kSparseWarps * 32)
    decode_sparse_split_kernel(KParams p, const __nv_bfloat16* __restrict__ q,
                               const __nv_bfloat16* __restrict__ kc,
                               const __nv_bfloat16* __restrict__ vc,
                               const int32_t* __restrict__ seq_len,
                               const int32_t* __restrict__ idx, const int32_t* __restrict__ cnt,
                               float* __restrict__ part, int n_split) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
    const int warp = threadIdx.x >> 5;
    const int task = blockIdx.x * kSparseWarps + warp;
    if (task >= p.batch * p.hkv * n_split) return;
    const int sp = task % n_split;
    const int unit = task / n_split;  // b * hkv + u
    const int u = unit % p.hkv, b = unit / p.hkv;
    const int g = p.group;
    float* mypart = part + (size_t)task * 16 * (D + 2);
    const int L = seq_len[b];
    AttnState<D> st;
    st.init();
    if (L >= 1 && L <= p.t_kv) {
        const int t = L - 1;
        const int c = clamp_count(cnt[unit], p.ksel);
        const int r0 = sp * kDecodeSparseRows;
        const int n_rows = max(0, min(kDecodeSparseRows, c - r0));
        const uint32_t sbase = base + warp * WarpSmem<D>::kBytes;
        uint32_t qf[D / 16][4];
        load_q_frags<D>(qf, q + ((size_t)b * p.hq + u * g) * D, D, g);
        GatherKeys keys{idx + (size_t)unit * p.ksel + r0, n_rows, 1, t, 1};
        const size_t kvoff = (size_t)unit * p.t_kv * D;
        attend_rows<D>(st, qf, kc + kvoff, vc + kvoff, (n_rows + kChunk - 1) / kChunk, keys,
                       sbase, p.scale_log2, NoHook{});
    } else if (sp == 0 && (threadIdx.x & 31) == 0) {
        set_status(HS_ERR_BOUNDS);
    }
    store_partial<D>(st, mypart, g);
}

// Exact merge of split partials: M = max m_s, l = sum l_s 2^(m_s - M),
// o = sum O_s 2^(m_s - M) / l.  One CTA of parts x D threads per (sequence,
// head): thread (part, d) accumulates element d over the splits s = part
// mod parts, and the parts are added in shared memory (parts = 4 when there
// are many splits -- long caches -- else 1).
constexpr int kCombineParts = 4;
static int combine_parts(int n_split) { return n_split >= 256 ? kCombineParts : 1; }

template <int D>
__global__ void __launch_bounds__(kCombineParts * D)
    decode_combine_kernel(KParams p, const float* __restrict__ part, int n_split,
                          const int32_t* __restrict__ seq_len, __nv_bfloat16* __restrict__ o,
                          float* __restrict__ lse, float* __restrict__ lse2_out) {
    constexpr int NWMAX = kCombineParts * D / 32;
    __shared__ float red_m[NWMAX], red_l[NWMAX];
    const int NW = blockDim.x >> 5, parts = blockDim.x / D;
    __shared__ float s_acc[kCombineParts][D];
    const int row = blockIdx.x;  // b * hq + h
    const int h = row % p.hq, b = row / p.hq;
    const int g = p.group, u = h / g, hh = h % g;
    const int unit = b * p.hkv + u;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int d = tid % D, prt = tid / D;
    const int L = seq_len[b];
    constexpr size_t S = 16 * (D + 2);  // floats between consecutive splits
    const float* base = part + (size_t)unit * n_split * S + (size_t)hh * (D + 2);
    float M = -INFINITY;
    for (int s = tid; s < n_split; s += blockDim.x) M = fmaxf(M, base[s * S]);
    M = warp_max(M);
    if (lane == 0) red_m[warp] = M;
    __syncthreads();
    for (int w = 0; w < NW; ++w) M = fmaxf(M, red_m[w]);
    const float Mu = M == -INFINITY ? 0.f : M;
    float l = 0.f;
    for (int s = tid; s < n_split; s += blockDim.x) l += base[s * S + 1] * exp2f(base[s * S] - Mu);
    l = warp_sum(l);
    if (lane == 0) red_l[warp] = l;
    float acc = 0.f;
#pragma unroll 4
    for (int s = prt; s < n_split; s += parts)
        acc += base[s * S + 2 + d] * exp2f(base[s * S] - Mu);
    s_acc[prt][d] = acc;
    __syncthreads();
    if (prt != 0) return;
    l = 0.f;
    for (int w = 0; w < NW; ++w) l += red_l[w];
    for (int x = 1; x < parts; ++x) acc += s_acc[x][d];
    const bool ok = L >= 1 && L <= p.t_kv && l > 0.f;
    o[(size_t)row * D + d] = __float2bfloat16_rn(ok ? acc / l : 0.f);
    if (d == 0) {
        const float l2 = ok ? M + log2f(l) : -INFINITY;
        if (lse) lse[row] = l2 * kLn2;
        if (lse2_out) lse2_out[row] = l2;
    }
}

size_t decode_sparse_split_workspace(const KParams& p) {
    const int n_split = (p.ksel + kDecodeSparseRows - 1) / kDecodeSparseRows;
    return (size_t)p.batch * p.hkv * n_split * 16 * (p.head_dim + 2) * sizeof(float);
}

// The split-k pair above with its partials in caller-provided scratch (used by
// the allocation-free entry point, whose scratch is a library array).
template <int D>
static cudaError_t launch_decode_sparse_split_t(const KParams& p, const void* q, const void* kc,
                                                const void* vc, const int32_t* seq_len,
                                                const int32_t* idx, const int32_t* cnt, void* o,
                                                float* lse, void* ws, cudaStream_t st) {
    const int n_split = (p.ksel + kDecodeSparseRows - 1) / kDecodeSparseRows;
    const size_t smem = (size_t)kSparseWarps * WarpSmem<D>::kBytes + 1024;
    auto kern = decode_sparse_split_kernel<D>;
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int n_tasks = p.batch * p.hkv * n_split;
    kern<<<(n_tasks + kSparseWarps - 1) / kSparseWarps, kSparseWarps * 32, smem, st>>>(
        p, (const __nv_bfloat16*)q, (const __nv_bfloat16*)kc, (const __nv_bfloat16*)vc, seq_len,
        idx, cnt, (float*)ws, n_split);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    decode_combine_kernel<D><<<p.batch * p.hq, combine_parts(n_split) * D, 0, st>>>(
        p, (const float*)ws, n_split, seq_len, (__nv_bfloat16*)o, lse, nullptr);
    return cudaGetLastError();
}

cudaError_t launch_decode_sparse_split(const KParams& p, const void* q, const void* kc,
                                       const void* vc, const int32_t* seq_len, const int32_t* idx,
                                       const int32_t* cnt, void* o, float* lse, void* ws,
                                       cudaStream_t st) {
    if (p.head_dim == 64)
        return launch_decode_sparse_split_t<64>(p, q, kc, vc, seq_len, idx, cnt, o, lse, ws, st);
    return launch_decode_sparse_split_t<128>(p, q, kc, vc, seq_len, idx, cnt, o, lse, ws, st);
}

// ---------------------------------------------- decode, one kernel per step
// One (sequence, group) unit per thread-block cluster of `csize` CTAs of
// kSparseWarps warps.  The unit's selected rows are dealt out to the
// 6 * csize warps in 32-row chunks (warp w takes chunks w, w + W, ...); each
// warp attends its chunks with the same cp.async gather ring as the prefill
// kernel, the CTA merges its warps' partials in shared memory, and CTA 0 of
// the cluster merges the CTAs' partials read through distributed shared
// memory and writes o and lse.  Every merge is the exact one of split-k
// attention: M = max m_s, l = sum l_s 2^(m_s - M), o = sum O_s 2^(m_s - M) / l.
// Nothing goes through global memory, so the step needs no workspace.

// Rows of the unit's index list owned by one warp: its chunk cc is the
// list's chunk first + cc * stride.
struct StridedGather {
    static constexpr bool kContig = false;
    const int32_t* ids;
    int n_rows, t, first, stride;
    __device__ __forceinline__ int key(int r) const {
        const int row = (first + (r >> 5) * stride) * kChunk + (r & 31);
        if (row >= n_rows) return -1;
        const int key = ids[row];
        if (key < 0 || key > t) { set_status(HS_ERR_BOUNDS); return -1; }
        return key;
    }
};

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
                 ::: "memory");
}

// fp32 at shared address `a` of cluster CTA `rank`.
__device__ __forceinline__ float ld_cluster_f32(uint32_t a, uint32_t rank) {
    uint32_t ra;
    float v;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(a), "r"(rank));
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(ra) : "memory");
    return v;
}

template <int D>
struct DecodeSmem {
    static constexpr int kPart = 16 * (D + 2);  // floats of one partial [16][D + 2]
    static constexpr size_t kRing = (size_t)kSparseWarps * WarpSmem<D>::kBytes;
    static constexpr size_t kBytes = kRing + kPart * sizeof(float) + 32 * sizeof(float) + 1024;
};

template <int D>
__global__ void __launch_bounds__(kSparseWarps * 32)
    decode_sparse_cluster_kernel(KParams p, const __nv_bfloat16* __restrict__ q,
                                 const __nv_bfloat16* __restrict__ kc,
                                 const __nv_bfloat16* __restrict__ vc,
                                 const int32_t* __restrict__ seq_len,
                                 const int32_t* __restrict__ idx,
                                 const int32_t* __restrict__ cnt, int csize,
                                 __nv_bfloat16* __restrict__ o, float* __restrict__ lse) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    using S = DecodeSmem<D>;
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char* gbase = smem_raw + (base - raw);
    float* cta_part = reinterpret_cast<float*>(gbase + S::kRing);  // [16][D + 2]
    float* s_ml = cta_part + S::kPart;                              // M[16], l[16]
    const int warp = threadIdx.x >> 5;
    const int crank = csize > 1 ? (int)cluster_rank() : 0;
    const int unit = blockIdx.x / csize;  // b * hkv + u
    const int u = unit % p.hkv, b = unit / p.hkv;
    const int g = p.group;
    const int L = seq_len[b];
    const bool valid = L >= 1 && L <= p.t_kv;
    float* wpart = reinterpret_cast<float*>(gbase + (size_t)warp * WarpSmem<D>::kBytes);

    AttnState<D> st;
    st.init();
    if (valid) {
        const int t = L - 1;
        const int c = clamp_count(cnt[unit], p.ksel);
        const int n_chunks = (c + kChunk - 1) / kChunk;
        const int W = kSparseWarps * csize;
        const int wg = crank * kSparseWarps + warp;
        const int mine = wg < n_chunks ? (n_chunks - 1 - wg) / W + 1 : 0;
        uint32_t qf[D / 16][4];
        load_q_frags<D>(qf, q + ((size_t)b * p.hq + u * g) * D, D, g);
        const StridedGather keys{idx + (size_t)unit * p.ksel, c, t, wg, W};
        if (p.bt) {  // paged cache: every row through the block table
            const PagedSrc<StridedGather> pkeys{keys, page_map(p, b, u)};
            attend_rows<D>(st, qf, kc, vc, mine, pkeys, base + warp * WarpSmem<D>::kBytes,
                           p.scale_log2, NoHook{});
        } else {
            const size_t kvoff = (size_t)unit * p.t_kv * D;
            attend_rows<D>(st, qf, kc + kvoff, vc + kvoff, mine, keys,
                           base + warp * WarpSmem<D>::kBytes, p.scale_log2, NoHook{});
        }
    } else if (crank == 0 && threadIdx.x == 0) {
        set_status(HS_ERR_BOUNDS);
    }
    __syncwarp();
    store_partial<D>(st, wpart, g);  // the warp's ring is drained: reuse it
    __syncthreads();

    // CTA merge of the warps' partials.
    constexpr int P = D + 2;
    if (threadIdx.x < g) {
        const int h = threadIdx.x;
        float M = -INFINITY;
        for (int w = 0; w < kSparseWarps; ++w)
            M = fmaxf(M, reinterpret_cast<const float*>(gbase + (size_t)w * WarpSmem<D>::kBytes)[h * P]);
        const float Mu = M == -INFINITY ? 0.f : M;
        float l = 0.f;
        for (int w = 0; w < kSparseWarps; ++w) {
            const float* ph = reinterpret_cast<const float*>(gbase + (size_t)w * WarpSmem<D>::kBytes) + h * P;
            l += ph[1] * exp2f(ph[0] - Mu);
        }
        s_ml[h] = M;
        s_ml[16 + h] = l;
        cta_part[h * P] = M;
        cta_part[h * P + 1] = l;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < g * D; e += blockDim.x) {
        const int h = e / D, d = e % D;
        const float M = s_ml[h];
        const float Mu = M == -INFINITY ? 0.f : M;
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < kSparseWarps; ++w) {
            const float* ph = reinterpret_cast<const float*>(gbase + (size_t)w * WarpSmem<D>::kBytes) + h * P;
            acc += ph[2 + d] * exp2f(ph[0] - Mu);
        }
        cta_part[h * P + 2 + d] = acc;
    }
    if (csize > 1) cluster_sync_all();  // the CTAs' partials are visible cluster-wide
    else __syncthreads();

    if (crank == 0) {
        const uint32_t part_addr = base + (uint32_t)S::kRing;
        auto rd = [&](int r, int off) -> float {
            return csize > 1 ? ld_cluster_f32(part_addr + 4u * off, (uint32_t)r) : cta_part[off];
        };
        for (int e = threadIdx.x; e < g * D; e += blockDim.x) {
            const int h = e / D, d = e % D;
            float M = -INFINITY;
            for (int r = 0; r < csize; ++r) M = fmaxf(M, rd(r, h * P));
            const float Mu = M == -INFINITY ? 0.f : M;
            float l = 0.f, acc = 0.f;
            for (int r = 0; r < csize; ++r) {
                const float w = exp2f(rd(r, h * P) - Mu);
                l += rd(r, h * P + 1) * w;
                acc += rd(r, h * P + 2 + d) * w;
            }
            const bool ok = valid && l > 0.f;
            const size_t orow = (size_t)b * p.hq + u * g + h;
            o[orow * D + d] = __float2bfloat16_rn(ok ? acc / l : 0.f);
            if (d == 0 && lse) lse[orow] = ok ? (M + log2f(l)) * kLn2 : -INFINITY;
        }
    }
    if (csize > 1) cluster_sync_all();  // peers keep their shared memory until CTA 0 is done
}

size_t decode_sparse_workspace(const KParams&) { return 0; }

template <int D>
static cudaError_t launch_decode_sparse_t(const KParams& p, const void* q, const void* kc,
                                          const void* vc, const int32_t* seq_len,
                                          const int32_t* idx, const int32_t* cnt, void* o,
                                          float* lse, cudaStream_t st) {
    auto kern = decode_sparse_cluster_kernel<D>;
    const size_t smem = DecodeSmem<D>::kBytes;
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return e;
    // Widest cluster (<= 8 CTAs, one per SM) that still fits the units in one wave.
    const int units = p.batch * p.hkv;
    const int chunks = (p.ksel + kChunk - 1) / kChunk;
    int csize = 1;
    while (csize < 8 && units * csize * 2 <= sms && kSparseWarps * csize < chunks) csize *= 2;
    for (;; csize /= 2) {
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        cfg.gridDim = dim3((unsigned)(units * csize));
        cfg.blockDim = dim3(kSparseWarps * 32);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = st;
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)csize;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = csize > 1 ? 1 : 0;
        if (csize > 1) {  // can the device co-schedule a cluster this wide? (cached)
            static std::atomic<int> fits[64][4];  // 0 unknown, 1 yes, -1 no
            const int lvl = csize == 2 ? 1 : csize == 4 ? 2 : 3;
            int f = dev < 64 ? fits[dev][lvl].load(std::memory_order_relaxed) : 0;
            if (f == 0) {
                int n = 0;
                f = cudaOccupancyMaxActiveClusters(&n, kern, &cfg) == cudaSuccess && n >= 1 ? 1
                                                                                             : -1;
                (void)cudaGetLastError();
                if (dev < 64) fits[dev][lvl].store(f, std::memory_order_relaxed);
            }
            if (f < 0) continue;
        }
        return cudaLaunchKernelEx(&cfg, kern, p, (const __nv_bfloat16*)q,
                                  (const __nv_bfloat16*)kc, (const __nv_bfloat16*)vc, seq_len,
                                  idx, cnt, csize, (__nv_bfloat16*)o, lse);
    }
}

cudaError_t launch_decode_sparse(const KParams& p, const void* q, const void* kc, const void* vc,
                                 const int32_t* seq_len, const int32_t* idx, const int32_t* cnt,
                                 void* o, float* lse, void*, cudaStream_t st) {
    if (p.head_dim == 64)
        return launch_decode_sparse_t<64>(p, q, kc, vc, seq_len, idx, cnt, o, lse, st);
    return launch_decode_sparse_t<128>(p, q, kc, vc, seq_len, idx, cnt, o, lse, st);
}

// Shared with decode_full.cu.
cudaError_t launch_decode_combine(const KParams& p, const float* part, int n_split,
                                  const int32_t* seq_len, void* o, float* lse, float* lse2,
                                  cudaStream_t st) {
    const int rows = p.batch * p.hq;
    if (p.head_dim == 64)
        decode_combine_kernel<64><<<rows, combine_parts(n_split) * 64, 0, st>>>(
            p, part, n_split, seq_len, (__nv_bfloat16*)o, lse, lse2);
    else
        decode_combine_kernel<128><<<rows, combine_parts(n_split) * 128, 0, st>>>(
            p, part, n_split, seq_len, (__nv_bfloat16*)o, lse, lse2);
    return cudaGetLastError();
}

}  // namespace hs
