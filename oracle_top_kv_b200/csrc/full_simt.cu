// full_simt.cu -- full-attention layer + oracle indexer, CUDA-core (SIMT)
// version.  Exact fp32 arithmetic for any supported shape; this is the path
// of the fp32 configurations and the general fallback of the bf16 ones.
//
// One CTA per (batch, kv group u, query row j) -- or, in decode, per (sequence,
// kv group) at the sequence's newest position -- with up to 16 warps that
// take the group's heads in turn for the attention (groups of up to 64
// heads, head_dim 64, 128 or 256: the MQA 64/1 d = 256 shape of "HySparse2
// ...", 6.4), then all warps for the selection:
//
//  phase A (per head h):  online softmax over keys 0..t in chunks of 32
//      ("HySparse 混合稀疏注意力（一）", exact attention and the online-softmax
//      statistics m_i, l_i of "为什么不需要重新物化注意力矩阵"): writes o_h and
//      lse_h, and keeps lse_h (log2 domain) in shared memory;
//  phase B (selection):  every candidate (a block r of B keys, or a key i) gets
//      the group score in log2 domain
//          s = max_{h in u} max_{i in candidate} (a2_{h,i} - lse2_h)
//      i.e. log2 of S_bar = max_h max_i p_{h,t,i} (block max probability, then
//      GQA group max: "GQA 下为什么要组内共享索引"; token mode: the same with
//      B = 1), and enters the exact streaming top-k buffer.  Token mode keeps
//      the last w keys out of the ranking and selects them unconditionally
//      ("HySparse2 ..." 4.2, forced local window).
#include "block_topk.cuh"
#include "hs_common.cuh"
#include "hs_kernels.cuh"

namespace hs {

template <typename T, int D>
__device__ __forceinline__ float dot_row(const float* __restrict__ qs, const T* __restrict__ kr) {
    float s = 0.f;
#pragma unroll 8
    for (int x = 0; x < D; ++x) s += qs[x] * to_f(kr[x]);
    return s;
}

constexpr int kSimtMaxGroup = 64;

template <typename T, int D>
__global__ void __launch_bounds__(512) full_simt_kernel(KParams p, const T* __restrict__ q,
                                                        const T* __restrict__ k,
                                                        const T* __restrict__ v, T* __restrict__ o,
                                                        float* __restrict__ lse,
                                                        int32_t* __restrict__ idx,
                                                        int32_t* __restrict__ cnt,
                                                        float* __restrict__ sel, int do_attn,
                                                        const int32_t* __restrict__ seq_len) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const int j = blockIdx.x, u = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nw = blockDim.x >> 5;
    const int g = p.group;
    // decode (seq_len given): the one query is the sequence's newest token
    const int t = seq_len ? seq_len[b] - 1 : p.q_offset + j;
    if (t < 0 || t >= p.t_kv) {  // uniform over the CTA
        if (threadIdx.x == 0) {
            set_status(HS_ERR_BOUNDS);
            cnt[((size_t)b * p.hkv + u) * p.t_q + j] = 0;
        }
        return;
    }

    const int Kc = p.mode == 0 ? p.ksel : p.k - p.window;  // ranked slots

    float* qs = reinterpret_cast<float*>(smem_raw);   // [g][D]
    float* lse2 = qs + g * D;                          // [kSimtMaxGroup]
    __shared__ int s_count;
    __shared__ unsigned long long s_thresh;
    BlockTopK topk;
    topk.setup(reinterpret_cast<unsigned char*>(lse2 + kSimtMaxGroup), Kc, blockDim.x, &s_count,
               &s_thresh);

    const T* kbase = k + ((size_t)b * p.hkv + u) * p.t_kv * D;
    const T* vbase = v + ((size_t)b * p.hkv + u) * p.t_kv * D;

    for (int x = threadIdx.x; x < g * D; x += blockDim.x) {
        const int hh = x / D, c = x % D;
        const int h = u * g + hh;
        qs[x] = to_f(q[(((size_t)b * p.hq + h) * p.t_q + j) * D + c]) * p.scale_log2;
    }
    __syncthreads();

    // ---------------- phase A: exact attention, the warps take the heads in turn
    constexpr int E = D / 32;
    if (!do_attn) {
        // selection only: the attention (and lse) came from another kernel
        for (int hh = threadIdx.x; hh < g; hh += blockDim.x)
            lse2[hh] = lse[((size_t)b * p.hq + u * g + hh) * p.t_q + j] * kLog2e;
    } else for (int hw = warp; hw < g; hw += nw) {
        const int h = u * g + hw;
        const float* qh = qs + hw * D;
        float m = -INFINITY, l = 0.f, acc[E];
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] = 0.f;
        for (int c0 = 0; c0 <= t; c0 += 32) {
            const int i = c0 + lane;
            const bool valid = i <= t;
            const float a = valid ? dot_row<T, D>(qh, kbase + (size_t)i * D) : -INFINITY;
            const float m_new = fmaxf(m, warp_max(a));
            const float pr = valid ? exp2f(a - m_new) : 0.f;
            const float corr = exp2f(m - m_new);
            l = l * corr + warp_sum(pr);
#pragma unroll
            for (int e = 0; e < E; ++e) acc[e] *= corr;
            const int nk = min(32, t + 1 - c0);
            for (int jj = 0; jj < nk; ++jj) {
                const float pj = __shfl_sync(0xffffffffu, pr, jj);
                const T* vr = vbase + (size_t)(c0 + jj) * D + lane * E;
#pragma unroll
                for (int e = 0; e < E; ++e) acc[e] += pj * to_f(vr[e]);
            }
            m = m_new;
        }
        const float inv = 1.f / l;
        T* orow = o + (((size_t)b * p.hq + h) * p.t_q + j) * D + lane * E;
#pragma unroll
        for (int e = 0; e < E; ++e) orow[e] = from_f<T>(acc[e] * inv);
        const float l2 = m + log2f(l);
        if (lane == 0) {
            lse2[hw] = l2;
            lse[((size_t)b * p.hq + h) * p.t_q + j] = l2 * kLn2;
        }
    }
    __syncthreads();

    // ---------------- phase B: group scores and exact top-k
    const size_t row = ((size_t)b * p.hkv + u) * p.t_q + j;
    int32_t* irow = idx + row * p.ksel;
    float* srow = sel ? sel + row * p.ksel : nullptr;
    const int B = p.block_size;
    const int n_cand = (t + 1 + B - 1) / B;           // blocks, or tokens (B = 1)
    const bool select_all = p.mode == 0 ? (n_cand <= p.ksel) : (t + 1 <= p.k);
    const int lo = p.mode == 1 ? t - p.window + 1 : n_cand;  // first forced id (token mode)
    // Scores are needed for ranked candidates always, for the others only if
    // the caller wants sel_scores.
    const bool ranked = !select_all && Kc > 0;
    int n_scored;
    if (select_all) n_scored = srow ? n_cand : 0;
    else if (p.mode == 1) n_scored = srow ? n_cand : lo;
    else n_scored = n_cand;

    for (int c0 = 0; c0 < n_scored; c0 += blockDim.x) {
        const int id = c0 + threadIdx.x;
        if (id < n_scored) {
            float s = -INFINITY;
            const int i0 = id * B, i1 = min(id * B + B - 1, t);
            for (int i = i0; i <= i1; ++i) {
                const T* kr = kbase + (size_t)i * D;
                for (int hh = 0; hh < g; ++hh)
                    s = fmaxf(s, dot_row<T, D>(qs + hh * D, kr) - lse2[hh]);
            }
            if (select_all) {
                srow[id] = exp2f(s);
            } else if (p.mode == 1 && id >= lo) {
                if (srow) srow[Kc + (id - lo)] = exp2f(s);
            } else if (ranked) {
                topk.offer(s, (uint32_t)id);
            }
        }
        if (ranked) topk.end_round();
    }
    __syncthreads();

    if (warp != 0) return;
    int n_out;
    if (select_all) {
        n_out = n_cand;
        for (int x = lane; x < n_out; x += 32) irow[x] = x;
        for (int x = n_out + lane; x < p.ksel; x += 32) {
            irow[x] = -1;
            if (srow) srow[x] = 0.f;
        }
    } else if (p.mode == 1) {
        n_out = topk.finish(irow, srow, p.ksel, lo, t);
    } else {
        n_out = topk.finish(irow, srow, p.ksel, 0, -1);
    }
    if (lane == 0) cnt[row] = n_out;
}

template <typename T, int D>
static cudaError_t launch_full_simt_t(const KParams& p, const void* q, const void* k,
                                      const void* v, void* o, float* lse, int32_t* idx,
                                      int32_t* cnt, float* sel, int do_attn,
                                      const int32_t* seq_len, cudaStream_t st) {
    const int nwarps = p.group < 4 ? 4 : (p.group > 16 ? 16 : p.group);
    const int Kc = p.mode == 0 ? p.ksel : p.k - p.window;
    const size_t smem = sizeof(float) * (p.group * D + kSimtMaxGroup) +
                        BlockTopK::smem_bytes(Kc, nwarps * 32);
    auto kern = full_simt_kernel<T, D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(p.t_q, p.hkv, p.batch);
    kern<<<grid, nwarps * 32, smem, st>>>(p, (const T*)q, (const T*)k, (const T*)v, (T*)o, lse,
                                           idx, cnt, sel, do_attn, seq_len);
    return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_full_simt_d(const KParams& p, const void* q, const void* k,
                                      const void* v, void* o, float* lse, int32_t* idx,
                                      int32_t* cnt, float* sel, int do_attn,
                                      const int32_t* seq_len, cudaStream_t st) {
    if (p.head_dim == 64)
        return launch_full_simt_t<T, 64>(p, q, k, v, o, lse, idx, cnt, sel, do_attn, seq_len, st);
    if (p.head_dim == 128)
        return launch_full_simt_t<T, 128>(p, q, k, v, o, lse, idx, cnt, sel, do_attn, seq_len, st);
    return launch_full_simt_t<T, 256>(p, q, k, v, o, lse, idx, cnt, sel, do_attn, seq_len, st);
}

cudaError_t launch_full_simt(const KParams& p, int dtype, const void* q, const void* k,
                             const void* v, void* o, float* lse, int32_t* idx, int32_t* cnt,
                             float* sel, int do_attn, cudaStream_t st, const int32_t* seq_len) {
    if (dtype == HS_FP32)
        return launch_full_simt_d<float>(p, q, k, v, o, lse, idx, cnt, sel, do_attn, seq_len, st);
    return launch_full_simt_d<__nv_bfloat16>(p, q, k, v, o, lse, idx, cnt, sel, do_attn, seq_len,
                                             st);
}

}  // namespace hs
