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
//   sparse_mma_kernel   bf16: one warp per (row, group); the group's heads are
//                       the 16 MMA rows, so each gathered row is read once.
//   decode_sparse_*     bf16 decode: the selected rows of one (sequence, group)
//                       split across warps, then an exact log-sum-exp merge.
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
    if (lane == 0) *lse_out = l > 0.f ? (m + log2f(l)) * kLn2 : -INFINITY;
}

template <typename T, int D>
__global__ void sparse_simt_kernel(KParams p, const T* __restrict__ q, const T* __restrict__ kf,
                                   const T* __restrict__ vf, const int32_t* __restrict__ idx,
                                   const int32_t* __restrict__ cnt, const T* __restrict__ kl,
                                   const T* __restrict__ vl, T* __restrict__ og,
                                   float* __restrict__ lseg, T* __restrict__ ol,
                                   float* __restrict__ lsel) {
    __shared__ float qs[16 * D];
    const int j = blockIdx.x, u = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5;
    const int g = p.group;
    const int t = p.q_offset + j;
    for (int x = threadIdx.x; x < g * D; x += blockDim.x) {
        const int h = u * g + x / D;
        qs[x] = to_f(q[(((size_t)b * p.hq + h) * p.t_q + j) * D + x % D]) * p.scale_log2;
    }
    __syncthreads();
    if (warp >= g) return;
    const int h = u * g + warp;
    const size_t row = ((size_t)b * p.hkv + u) * p.t_q + j;
    const size_t orow = ((size_t)b * p.hq + h) * p.t_q + j;
    const size_t kvoff = ((size_t)b * p.hkv + u) * p.t_kv * D;
    const int c = clamp_count(cnt[row], p.ksel);
    const int n_rows = p.mode == 0 ? c * p.block_size : c;
    GatherKeys keys{idx + row * p.ksel, n_rows, p.block_size, t, p.mode};
    simt_attend<T, D>(qs + warp * D, kf + kvoff, vf + kvoff, n_rows, keys, og + orow * D,
                      lseg + orow);
    if (kl) {
        const int first = max(0, t - p.window + 1);
        simt_attend<T, D>(qs + warp * D, kl + kvoff, vl + kvoff, t - first + 1,
                          [=](int r) { return first + r <= t ? first + r : -1; }, ol + orow * D,
                          lsel + orow);
    }
}

template <typename T, int D>
static cudaError_t launch_sparse_simt_t(const KParams& p, const void* q, const void* kf,
                                        const void* vf, const int32_t* idx, const int32_t* cnt,
                                        const void* kl, const void* vl, void* og, float* lseg,
                                        void* ol, float* lsel, cudaStream_t st) {
    dim3 grid(p.t_q, p.hkv, p.batch);
    sparse_simt_kernel<T, D><<<grid, 32 * p.group, 0, st>>>(
        p, (const T*)q, (const T*)kf, (const T*)vf, idx, cnt, (const T*)kl, (const T*)vl, (T*)og,
        lseg, (T*)ol, lsel);
    return cudaGetLastError();
}

cudaError_t launch_sparse_simt(const KParams& p, int dtype, const void* q, const void* kf,
                               const void* vf, const int32_t* idx, const int32_t* cnt,
                               const void* kl, const void* vl, void* og, float* lseg, void* ol,
                               float* lsel, cudaStream_t st) {
    if (dtype == HS_FP32) {
        if (p.head_dim == 64)
            return launch_sparse_simt_t<float, 64>(p, q, kf, vf, idx, cnt, kl, vl, og, lseg, ol,
                                                   lsel, st);
        return launch_sparse_simt_t<float, 128>(p, q, kf, vf, idx, cnt, kl, vl, og, lseg, ol,
                                                lsel, st);
    }
    if (p.head_dim == 64)
        return launch_sparse_simt_t<__nv_bfloat16, 64>(p, q, kf, vf, idx, cnt, kl, vl, og, lseg,
                                                       ol, lsel, st);
    return launch_sparse_simt_t<__nv_bfloat16, 128>(p, q, kf, vf, idx, cnt, kl, vl, og, lseg, ol,
                                                    lsel, st);
}

// ------------------------------------------------------------ tensor-core path
constexpr int kSparseWarps = 6;

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

// Dynamic shared memory: per warp a 2-stage K/V ring, then per warp 2 mbarriers.
template <int D>
constexpr size_t sparse_smem_bytes() {
    return (size_t)kSparseWarps * WarpSmem<D>::kBytes + kSparseWarps * 16 + 1024;
}

template <int D>
__global__ void __launch_bounds__(kSparseWarps * 32)
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
    const long long task = (long long)blockIdx.x * kSparseWarps + warp;
    const long long n_tasks = (long long)p.batch * p.hkv * p.t_q;
    if (task >= n_tasks) return;
    const int j = (int)(task % p.t_q);
    const int u = (int)((task / p.t_q) % p.hkv);
    const int b = (int)(task / ((long long)p.t_q * p.hkv));
    const int g = p.group;
    const int t = p.q_offset + j;
    const uint32_t sbase = base + warp * WarpSmem<D>::kBytes;
    TmaRing ring{base + kSparseWarps * WarpSmem<D>::kBytes + 16u * warp, {0u, 0u}};
    if (lane == 0) {
        tc::mbar_init(ring.bar, 1);
        tc::mbar_init(ring.bar + 8, 1);
        tc::fence_mbar_init();
    }
    __syncwarp();

    const size_t head_stride = (size_t)p.t_q * D;
    const size_t q0 = (((size_t)b * p.hq + u * g) * p.t_q + j);  // row of head u*g
    uint32_t qf[D / 16][4];
    load_q_frags<D>(qf, q + q0 * D, head_stride, g);

    const int unit = b * p.hkv + u;
    const size_t row = (size_t)unit * p.t_q + j;
    const size_t kvoff = (size_t)unit * p.t_kv * D;
    const int c = clamp_count(cnt[row], p.ksel);
    const int n_rows = p.mode == 0 ? c * p.block_size : c;

    AttnState<D> st;
    st.init();
    if (p.mode == 0 && p.block_size % kChunk == 0) {
        BlockChunks src{idx + row * p.ksel, p.block_size, t};
        attend_rows_tma<D>(st, qf, &tm_kf, &tm_vf, unit, c * (p.block_size / kChunk), src, sbase,
                           ring, p.scale_log2, NoHook{});
    } else {
        GatherKeys keys{idx + row * p.ksel, n_rows, p.block_size, t, p.mode};
        attend_rows<D>(st, qf, kf + kvoff, vf + kvoff, (n_rows + kChunk - 1) / kChunk, keys,
                       sbase, p.scale_log2, NoHook{});
    }
    store_rows<D>(st, og + q0 * D, head_stride, lseg + q0, p.t_q, g);
    if (has_local) {
        const int first = max(0, t - p.window + 1);
        AttnState<D> sl;
        sl.init();
        const ContiguousKeys win{first, t};
        attend_rows_tma<D>(sl, qf, &tm_kl, &tm_vl, unit, win.n_chunks(), win, sbase, ring,
                           p.scale_log2, NoHook{});
        store_rows<D>(sl, ol + q0 * D, head_stride, lsel + q0, p.t_q, g);
    }
}

template <int D>
static cudaError_t launch_sparse_mma_t(const KParams& p, const void* q, const void* kf,
                                       const void* vf, const int32_t* idx, const int32_t* cnt,
                                       const void* kl, const void* vl, void* og, float* lseg,
                                       void* ol, float* lsel, cudaStream_t st) {
    const size_t smem = sparse_smem_bytes<D>();
    CUtensorMap mk, mv, mkl, mvl;
    const long long units = (long long)p.batch * p.hkv;
    if (!tc::encode_rows(&mk, kf, D, p.t_kv, units, kChunk) ||
        !tc::encode_rows(&mv, vf, D, p.t_kv, units, kChunk))
        return cudaErrorInvalidValue;
    if (kl) {
        if (!tc::encode_rows(&mkl, kl, D, p.t_kv, units, kChunk) ||
            !tc::encode_rows(&mvl, vl, D, p.t_kv, units, kChunk))
            return cudaErrorInvalidValue;
    } else {
        mkl = mk;
        mvl = mv;
    }
    auto kern = sparse_mma_kernel<D>;
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long n_tasks = (long long)p.batch * p.hkv * p.t_q;
    const unsigned grid = (unsigned)((n_tasks + kSparseWarps - 1) / kSparseWarps);
    kern<<<grid, kSparseWarps * 32, smem, st>>>(
        mk, mv, mkl, mvl, p, (const __nv_bfloat16*)q, (const __nv_bfloat16*)kf,
        (const __nv_bfloat16*)vf, idx, cnt, kl ? 1 : 0, (__nv_bfloat16*)og, lseg,
        (__nv_bfloat16*)ol, lsel);
    return cudaGetLastError();
}

cudaError_t launch_sparse_mma(const KParams& p, const void* q, const void* kf, const void* vf,
                              const int32_t* idx, const int32_t* cnt, const void* kl,
                              const void* vl, void* og, float* lseg, void* ol, float* lsel,
                              cudaStream_t st) {
    if (p.head_dim == 64)
        return launch_sparse_mma_t<64>(p, q, kf, vf, idx, cnt, kl, vl, og, lseg, ol, lsel, st);
    return launch_sparse_mma_t<128>(p, q, kf, vf, idx, cnt, kl, vl, og, lseg, ol, lsel, st);
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
// o = sum O_s 2^(m_s - M) / l.  One warp per (sequence, head).
template <int D>
__global__ void decode_combine_kernel(KParams p, const float* __restrict__ part, int n_split,
                                      const int32_t* __restrict__ seq_len,
                                      __nv_bfloat16* __restrict__ o, float* __restrict__ lse,
                                      float* __restrict__ lse2_out) {
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (warp >= p.batch * p.hq) return;
    const int h = warp % p.hq, b = warp / p.hq;
    const int g = p.group, u = h / g, hh = h % g;
    const int unit = b * p.hkv + u;
    const int L = seq_len[b];
    constexpr int E = D / 32;
    float M = -INFINITY;
    for (int s = 0; s < n_split; ++s)
        M = fmaxf(M, part[((size_t)unit * n_split + s) * 16 * (D + 2) + hh * (D + 2)]);
    const float Mu = M == -INFINITY ? 0.f : M;
    float l = 0.f, acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.f;
    for (int s = 0; s < n_split; ++s) {
        const float* ph = part + ((size_t)unit * n_split + s) * 16 * (D + 2) + hh * (D + 2);
        const float w = exp2f(ph[0] - Mu);
        l += ph[1] * w;
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] += ph[2 + lane * E + e] * w;
    }
    const bool ok = L >= 1 && L <= p.t_kv && l > 0.f;
    const float inv = ok ? 1.f / l : 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) o[(size_t)warp * D + lane * E + e] = __float2bfloat16_rn(acc[e] * inv);
    if (lane == 0) {
        const float l2 = ok ? M + log2f(l) : -INFINITY;
        if (lse) lse[warp] = l2 * kLn2;
        if (lse2_out) lse2_out[warp] = l2;
    }
}

size_t decode_sparse_workspace(const KParams& p) {
    const int n_split = (p.ksel + kDecodeSparseRows - 1) / kDecodeSparseRows;
    return (size_t)p.batch * p.hkv * n_split * 16 * (p.head_dim + 2) * sizeof(float);
}

template <int D>
static cudaError_t launch_decode_sparse_t(const KParams& p, const void* q, const void* kc,
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
    const int warps = p.batch * p.hq;
    decode_combine_kernel<D><<<(warps + 7) / 8, 256, 0, st>>>(p, (const float*)ws, n_split,
                                                              seq_len, (__nv_bfloat16*)o, lse,
                                                              nullptr);
    return cudaGetLastError();
}

cudaError_t launch_decode_sparse(const KParams& p, const void* q, const void* kc, const void* vc,
                                 const int32_t* seq_len, const int32_t* idx, const int32_t* cnt,
                                 void* o, float* lse, void* ws, cudaStream_t st) {
    if (p.head_dim == 64)
        return launch_decode_sparse_t<64>(p, q, kc, vc, seq_len, idx, cnt, o, lse, ws, st);
    return launch_decode_sparse_t<128>(p, q, kc, vc, seq_len, idx, cnt, o, lse, ws, st);
}

// Shared with decode_full.cu.
cudaError_t launch_decode_combine(const KParams& p, const float* part, int n_split,
                                  const int32_t* seq_len, void* o, float* lse, float* lse2,
                                  cudaStream_t st) {
    const int warps = p.batch * p.hq;
    if (p.head_dim == 64)
        decode_combine_kernel<64><<<(warps + 7) / 8, 256, 0, st>>>(
            p, part, n_split, seq_len, (__nv_bfloat16*)o, lse, lse2);
    else
        decode_combine_kernel<128><<<(warps + 7) / 8, 256, 0, st>>>(
            p, part, n_split, seq_len, (__nv_bfloat16*)o, lse, lse2);
    return cudaGetLastError();
}

}  // namespace hs
