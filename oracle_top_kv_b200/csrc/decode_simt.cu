// decode_simt.cu -- split-k decode steps on the CUDA cores for the shapes the
// tensor-core decode kernels do not take: groups of more than 16 query heads
// per KV head (HySparse2's MQA 64/1) and head dim 256 ("HySparse2 ...", 6.4).
//
// The same three-stage decode as decode_full.cu, with CUDA-core arithmetic:
//  1. dsm_split_kernel: CTA (split, sequence-group) takes a slice of the keys
//     -- a range of the cache (full step) or a range of the index list
//     (sparse step) -- 32 keys at a time staged in shared memory; warp w owns
//     the group's heads w, w + 8, ... and keeps an online-softmax partial (m,
//     l, O) per head ("HySparse 混合稀疏注意力（一）": exact attention with the
//     online-softmax statistics).  The full step also exports every scaled
//     logit a2_{h,i} (log2 domain): the group score max_h (a2_{h,i} - lse2_h)
//     needs every head's final lse, known only after all splits;
//  2. dsm_combine_kernel: the exact log-sum-exp merge of the splits -> o,
//     lse (and lse2 for the selector);
//  3. (full step) dsm_score_kernel turns every key's logits into its group
//     score max_h (a2_{h,i} - lse2_h) on many CTAs, and dsm_select_kernel (one
//     CTA per sequence-group) ranks keys 0..t-w by it with the exact streaming
//     top-k and appends the forced window t-w+1..t ("HySparse2 ..." 4.2).
// The one-CTA SIMT kernels (full_simt.cu, sparse.cu) remain for callers that
// give no workspace.
#include "block_topk.cuh"
#include "hs_common.cuh"
#include "hs_kernels.cuh"

namespace hs {
namespace dsm {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kTile = 32;            // keys staged per step
constexpr int kFullKeys = 512;       // cache keys per split (full step)
constexpr int kSparseKeys = 32;      // index entries per split (sparse step): one tile
constexpr int kMaxGroup = 64;
constexpr int kHeadsPerWarp = kMaxGroup / kWarps;  // 8
constexpr int kSelThreads = 512;

template <int D>
struct Smem {
    static constexpr int kKRow = D * 2 + 16;  // padded K rows: lane = key reads are conflict-free
    static constexpr size_t kQ = 0;                                   // fp32 [g][D]
    static constexpr size_t kK = sizeof(float) * kMaxGroup * D;       // bf16 [kTile][kKRow]
    static constexpr size_t kV = kK + (size_t)kTile * kKRow;          // bf16 [kTile][D]
    static constexpr size_t kIds = kV + (size_t)kTile * D * 2;        // int [kTile]
    static constexpr size_t kBytes = kIds + sizeof(int) * kTile;
};

struct Ws {
    float* logits;  // full step: [units][t_kv][g]
    float* part;    // [units][n_split][g][D + 2]
    float* lse2;    // full step: [batch * hq]
    float* score;   // full step: [units][t_kv] group scores (log2 domain)
    int n_split;
};
constexpr int kScoreKeys = 1024;  // keys per CTA of the score kernel

__host__ __device__ inline int full_splits(const KParams& p) {
    return (p.t_kv + kFullKeys - 1) / kFullKeys;
}
__host__ __device__ inline int sparse_splits(const KParams& p) {
    return (p.ksel + kSparseKeys - 1) / kSparseKeys;
}

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

static Ws ws_layout(const KParams& p, void* base, bool full) {
    Ws w;
    const size_t units = (size_t)p.batch * p.hkv;
    w.n_split = full ? full_splits(p) : sparse_splits(p);
    char* c = static_cast<char*>(base);
    const size_t logits_b = full ? align256(units * p.t_kv * p.group * sizeof(float)) : 0;
    const size_t part_b = align256(units * w.n_split * p.group * (p.head_dim + 2) * sizeof(float));
    const size_t lse_b = full ? align256((size_t)p.batch * p.hq * sizeof(float)) : 0;
    w.logits = full ? reinterpret_cast<float*>(c) : nullptr;
    w.part = reinterpret_cast<float*>(c + logits_b);
    w.lse2 = full ? reinterpret_cast<float*>(c + logits_b + part_b) : nullptr;
    w.score = full ? reinterpret_cast<float*>(c + logits_b + part_b + lse_b) : nullptr;
    return w;
}

static size_t ws_bytes(const KParams& p, bool full) {
    const size_t units = (size_t)p.batch * p.hkv;
    const int n_split = full ? full_splits(p) : sparse_splits(p);
    size_t b = align256(units * n_split * p.group * (p.head_dim + 2) * sizeof(float));
    if (full)
        b += align256(units * p.t_kv * p.group * sizeof(float)) +
             align256((size_t)p.batch * p.hq * sizeof(float)) +
             align256(units * p.t_kv * sizeof(float));
    return b;
}

// kMode 0: keys sp*kFullKeys .. of the cache (decode full step, keys <= t);
// 1: entries sp*kSparseKeys .. of the sequence-group's index row (decode
// sparse step); 2: a sparse layer in prefill -- CTA (query row) takes all
// of the row's index entries and writes o and lse itself (no split, no
// workspace).  Paged caches are not taken here.
template <int D, int kMode>
__global__ void __launch_bounds__(kThreads)
    dsm_split_kernel(KParams p, const __nv_bfloat16* __restrict__ q,
                     const __nv_bfloat16* __restrict__ kc, const __nv_bfloat16* __restrict__ vc,
                     const int32_t* __restrict__ seq_len, const int32_t* __restrict__ idx,
                     const int32_t* __restrict__ cnt, Ws ws, __nv_bfloat16* __restrict__ o_out,
                     float* __restrict__ lse_out) {
    constexpr bool kGather = kMode != 0, kPrefill = kMode == 2;
    using S = Smem<D>;
    constexpr int E = D / 32;  // d elements per lane in the PV accumulation
    extern __shared__ __align__(16) unsigned char smem[];
    float* qs = reinterpret_cast<float*>(smem + S::kQ);
    unsigned char* ks = smem + S::kK;
    __nv_bfloat16* vs = reinterpret_cast<__nv_bfloat16*>(smem + S::kV);
    int* ids = reinterpret_cast<int*>(smem + S::kIds);
    // row: the index row / query row (prefill), else the sequence-group
    const int sp = kPrefill ? 0 : (int)blockIdx.x;
    const int row = kPrefill ? (int)blockIdx.x : (int)blockIdx.y;
    const int j = kPrefill ? row % p.t_q : 0;
    const int unit = kPrefill ? row / p.t_q : row;
    const int u = unit % p.hkv, b = unit / p.hkv;
    const int g = p.group;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int L = kPrefill ? p.q_offset + j + 1 : seq_len[b];
    const bool valid = L >= 1 && L <= p.t_kv;
    const int t = L - 1;
    int n_keys = 0, first = 0;
    if (valid) {
        if (kGather) {
            const int c = clamp_count(cnt[row], p.ksel);
            first = kPrefill ? 0 : sp * kSparseKeys;
            n_keys = kPrefill ? c : max(0, min(c, first + kSparseKeys) - first);
        } else {
            first = sp * kFullKeys;
            n_keys = max(0, min(L, first + kFullKeys) - first);
        }
    }
    for (int x = threadIdx.x; x < g * D; x += kThreads) {
        const int h = u * g + x / D;
        qs[x] = __bfloat162float(q[(((size_t)b * p.hq + h) * p.t_q + j) * D + x % D]) *
                p.scale_log2;
    }
    const size_t kvoff = (size_t)unit * p.t_kv * D;
    const int32_t* irow = idx + (size_t)row * p.ksel;
    const int my_n = g > warp ? (g - 1 - warp) / kWarps + 1 : 0;  // heads of this warp
    float m[kHeadsPerWarp], l[kHeadsPerWarp], o[kHeadsPerWarp][E];
#pragma unroll
    for (int hh = 0; hh < kHeadsPerWarp; ++hh) {
        m[hh] = -INFINITY;
        l[hh] = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) o[hh][e] = 0.f;
    }
    float* lg = kGather ? nullptr : ws.logits + (size_t)unit * p.t_kv * g;
    for (int k0 = 0; k0 < n_keys; k0 += kTile) {
        __syncthreads();  // the previous tile is consumed (and q is in place)
        if (threadIdx.x < kTile) {
            const int r = k0 + threadIdx.x;
            int key = -1;
            if (r < n_keys) {
                key = kGather ? irow[first + r] : first + r;
                if (key < 0 || key > t) {
                    key = -1;
                    if (kGather) set_status(HS_ERR_BOUNDS);
                }
            }
            ids[threadIdx.x] = key;
        }
        __syncthreads();
        constexpr int kChunks = D / 8;  // 16-byte chunks per row
        for (int x = threadIdx.x; x < kTile * kChunks; x += kThreads) {
            const int r = x / kChunks, c = x % kChunks;
            const int key = ids[r];
            uint4 kv = make_uint4(0u, 0u, 0u, 0u), vv = kv;
            if (key >= 0) {
                kv = *reinterpret_cast<const uint4*>(kc + kvoff + (size_t)key * D + c * 8);
                vv = *reinterpret_cast<const uint4*>(vc + kvoff + (size_t)key * D + c * 8);
            }
            *reinterpret_cast<uint4*>(ks + (size_t)r * S::kKRow + c * 16) = kv;
            *reinterpret_cast<uint4*>(vs + (size_t)r * D + c * 8) = vv;
        }
        __syncthreads();
        const int key = ids[lane];
        // logits: lane = key of the tile, the warp's heads in registers
        float s[kHeadsPerWarp];
#pragma unroll
        for (int hh = 0; hh < kHeadsPerWarp; ++hh) s[hh] = 0.f;
        const unsigned char* krow = ks + (size_t)lane * S::kKRow;
#pragma unroll 4
        for (int c = 0; c < D / 8; ++c) {
            const uint4 kw = *reinterpret_cast<const uint4*>(krow + c * 16);
            const uint32_t w4[4] = {kw.x, kw.y, kw.z, kw.w};
            float kf[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w4[i]));
                kf[2 * i] = f.x;
                kf[2 * i + 1] = f.y;
            }
#pragma unroll
            for (int hh = 0; hh < kHeadsPerWarp; ++hh) {
                if (hh >= my_n) break;
                const float4* qv =
                    reinterpret_cast<const float4*>(qs + (warp + hh * kWarps) * D + c * 8);
                const float4 q0 = qv[0], q1 = qv[1];
                s[hh] += q0.x * kf[0] + q0.y * kf[1] + q0.z * kf[2] + q0.w * kf[3] +
                         q1.x * kf[4] + q1.y * kf[5] + q1.z * kf[6] + q1.w * kf[7];
            }
        }
        if (!kGather && key >= 0) {
#pragma unroll
            for (int hh = 0; hh < kHeadsPerWarp; ++hh)
                if (hh < my_n) lg[(size_t)key * g + warp + hh * kWarps] = s[hh];
        }
        // online softmax per head, then O += P V with lane = d slice
        float pr[kHeadsPerWarp];
#pragma unroll
        for (int hh = 0; hh < kHeadsPerWarp; ++hh) {
            if (hh >= my_n) break;
            const float a = key >= 0 ? s[hh] : -INFINITY;
            const float mt = warp_max(a);
            const float mn = fmaxf(m[hh], mt);
            const float mu = mn == -INFINITY ? 0.f : mn;
            pr[hh] = key >= 0 ? exp2f(a - mu) : 0.f;
            const float corr = exp2f(m[hh] - mu);
            l[hh] = l[hh] * corr + warp_sum(pr[hh]);
#pragma unroll
            for (int e = 0; e < E; ++e) o[hh][e] *= corr;
            m[hh] = mn;
        }
        const int nk = min(kTile, n_keys - k0);
        for (int r = 0; r < nk; ++r) {
            float vf[E];
            const __nv_bfloat16* vrow = vs + (size_t)r * D + lane * E;
#pragma unroll
            for (int e = 0; e < E; e += 2) {
                const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(vrow + e));
                vf[e] = f.x;
                vf[e + 1] = f.y;
            }
#pragma unroll
            for (int hh = 0; hh < kHeadsPerWarp; ++hh) {
                if (hh >= my_n) break;
                const float pj = __shfl_sync(0xffffffffu, pr[hh], r);
#pragma unroll
                for (int e = 0; e < E; ++e) o[hh][e] += pj * vf[e];
            }
        }
    }
    if (kPrefill) {  // the row's whole index set: final outputs
        if (!valid) return;
#pragma unroll
        for (int hh = 0; hh < kHeadsPerWarp; ++hh) {
            if (hh >= my_n) break;
            const size_t orow = ((size_t)b * p.hq + u * g + warp + hh * kWarps) * p.t_q + j;
            const float inv = l[hh] > 0.f ? 1.f / l[hh] : 0.f;
#pragma unroll
            for (int e = 0; e < E; e += 2)
                *reinterpret_cast<uint32_t*>(o_out + orow * D + lane * E + e) =
                    pack_bf16(o[hh][e] * inv, o[hh][e + 1] * inv);
            if (lane == 0) lse_out[orow] = l[hh] > 0.f ? (m[hh] + log2f(l[hh])) * kLn2 : -INFINITY;
        }
        return;
    }
    // partial of each of the warp's heads: m, l (log2 domain), O
    float* part = ws.part + ((size_t)unit * ws.n_split + sp) * g * (D + 2);
#pragma unroll
    for (int hh = 0; hh < kHeadsPerWarp; ++hh) {
        if (hh >= my_n) break;
        float* ph = part + (size_t)(warp + hh * kWarps) * (D + 2);
        if (lane == 0) { ph[0] = m[hh]; ph[1] = l[hh]; }
#pragma unroll
        for (int e = 0; e < E; ++e) ph[2 + lane * E + e] = o[hh][e];
    }
}

// One CTA per (sequence, query head), D threads: the exact merge of the
// splits' partials.
template <int D>
__global__ void __launch_bounds__(D)
    dsm_combine_kernel(KParams p, Ws ws, const int32_t* __restrict__ seq_len,
                       __nv_bfloat16* __restrict__ o, float* __restrict__ lse) {
    __shared__ float red[D / 32];
    const int row = blockIdx.x;  // b * hq + h
    const int h = row % p.hq, b = row / p.hq;
    const int g = p.group, u = h / g, hh = h % g;
    const int unit = b * p.hkv + u;
    const int d = threadIdx.x, lane = d & 31, warp = d >> 5;
    const size_t S = (size_t)g * (D + 2);  // floats between consecutive splits
    const float* base = ws.part + (size_t)unit * ws.n_split * S + (size_t)hh * (D + 2);
    float M = -INFINITY;
    for (int s = d; s < ws.n_split; s += D) M = fmaxf(M, base[s * S]);
    M = warp_max(M);
    if (lane == 0) red[warp] = M;
    __syncthreads();
    M = -INFINITY;
    for (int w = 0; w < D / 32; ++w) M = fmaxf(M, red[w]);
    __syncthreads();
    const float Mu = M == -INFINITY ? 0.f : M;
    float l = 0.f;
    for (int s = d; s < ws.n_split; s += D) l += base[s * S + 1] * exp2f(base[s * S] - Mu);
    l = warp_sum(l);
    if (lane == 0) red[warp] = l;
    float acc = 0.f;
    for (int s = 0; s < ws.n_split; ++s) acc += base[s * S + 2 + d] * exp2f(base[s * S] - Mu);
    __syncthreads();
    l = 0.f;
    for (int w = 0; w < D / 32; ++w) l += red[w];
    const int L = seq_len[b];
    const bool ok = L >= 1 && L <= p.t_kv && l > 0.f;
    o[(size_t)row * D + d] = __float2bfloat16_rn(ok ? acc / l : 0.f);
    if (d == 0) {
        const float l2 = ok ? M + log2f(l) : -INFINITY;
        if (lse) lse[row] = l2 * kLn2;
        if (ws.lse2) ws.lse2[row] = l2;
    }
}

// CTA (key block, sequence-group): group score max_h (a2_{h,i} - lse2_h) of
// keys kScoreKeys * blockIdx.x .. (every key <= t; a thread per key).
__global__ void __launch_bounds__(256)
    dsm_score_kernel(KParams p, const int32_t* __restrict__ seq_len, Ws ws) {
    __shared__ float s_lse2[kMaxGroup];
    const int unit = blockIdx.y;
    const int u = unit % p.hkv, b = unit / p.hkv;
    const int g = p.group;
    const int L = seq_len[b];
    if (L < 1 || L > p.t_kv) return;
    for (int x = threadIdx.x; x < g; x += blockDim.x) s_lse2[x] = ws.lse2[b * p.hq + u * g + x];
    __syncthreads();
    const float* lg = ws.logits + (size_t)unit * p.t_kv * g;
    float* sc = ws.score + (size_t)unit * p.t_kv;
    const int i_end = min(L, (int)(blockIdx.x + 1) * kScoreKeys);
    for (int i = blockIdx.x * kScoreKeys + threadIdx.x; i < i_end; i += blockDim.x) {
        const float* r = lg + (size_t)i * g;
        float s = -INFINITY;
        if ((g & 3) == 0) {  // rows are 16-byte aligned
            const float4* r4 = reinterpret_cast<const float4*>(r);
            for (int h4 = 0; h4 < g / 4; ++h4) {
                const float4 a = r4[h4];
                s = fmaxf(s, fmaxf(fmaxf(a.x - s_lse2[4 * h4], a.y - s_lse2[4 * h4 + 1]),
                                   fmaxf(a.z - s_lse2[4 * h4 + 2], a.w - s_lse2[4 * h4 + 3])));
            }
        } else {
            for (int h = 0; h < g; ++h) s = fmaxf(s, r[h] - s_lse2[h]);
        }
        sc[i] = s;
    }
}

// One CTA per sequence-group: exact streaming top-(k-w) of the ranked keys'
// group scores, then the window.
__global__ void __launch_bounds__(kSelThreads)
    dsm_select_kernel(KParams p, const int32_t* __restrict__ seq_len, Ws ws,
                      int32_t* __restrict__ idx, int32_t* __restrict__ cnt,
                      float* __restrict__ sel) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    __shared__ int s_count;
    __shared__ unsigned long long s_thresh;
    const int unit = blockIdx.x;
    const int b = unit / p.hkv;
    const int L = seq_len[b];
    int32_t* irow = idx + (size_t)unit * p.ksel;
    float* srow = sel ? sel + (size_t)unit * p.ksel : nullptr;
    if (L < 1 || L > p.t_kv) {
        for (int x = threadIdx.x; x < p.ksel; x += blockDim.x) {
            irow[x] = -1;
            if (srow) srow[x] = 0.f;
        }
        if (threadIdx.x == 0) { cnt[unit] = 0; set_status(HS_ERR_BOUNDS); }
        return;
    }
    const int t = L - 1;
    const int Kc = p.k - p.window;
    BlockTopK topk;
    topk.setup(smem_raw, Kc, blockDim.x, &s_count, &s_thresh);
    __syncthreads();
    const bool select_all = t + 1 <= p.k;
    const int lo = t - p.window + 1;
    const bool ranked = !select_all && Kc > 0;
    int n_scored;
    if (select_all) n_scored = srow ? t + 1 : 0;
    else n_scored = srow ? t + 1 : lo;
    const float* sc = ws.score + (size_t)unit * p.t_kv;
    for (int c0 = 0; c0 < n_scored; c0 += blockDim.x) {
        const int i = c0 + threadIdx.x;
        if (i < n_scored) {
            const float s = sc[i];
            if (select_all) srow[i] = exp2f(s);
            else if (i >= lo) { if (srow) srow[Kc + (i - lo)] = exp2f(s); }
            else if (ranked) topk.offer(s, (uint32_t)i);
        }
        if (ranked) topk.end_round();
    }
    __syncthreads();
    if (threadIdx.x >= 32) return;
    int n_out;
    if (select_all) {
        n_out = t + 1;
        for (int x = threadIdx.x; x < n_out; x += 32) irow[x] = x;
        for (int x = n_out + threadIdx.x; x < p.ksel; x += 32) {
            irow[x] = -1;
            if (srow) srow[x] = 0.f;
        }
    } else {
        n_out = topk.finish(irow, srow, p.ksel, lo, t);
    }
    if (threadIdx.x == 0) cnt[unit] = n_out;
}

template <int D>
static cudaError_t launch_t(const KParams& p, bool full, const void* q, const void* kc,
                            const void* vc, const int32_t* seq_len, int32_t* idx, int32_t* cnt,
                            void* o, float* lse, float* sel, void* ws_base, cudaStream_t st) {
    Ws w = ws_layout(p, ws_base, full);
    const dim3 grid((unsigned)w.n_split, (unsigned)(p.batch * p.hkv));
    auto kern = full ? dsm_split_kernel<D, 0> : dsm_split_kernel<D, 1>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Smem<D>::kBytes);
    if (e != cudaSuccess) return e;
    kern<<<grid, kThreads, Smem<D>::kBytes, st>>>(p, (const __nv_bfloat16*)q,
                                                   (const __nv_bfloat16*)kc,
                                                   (const __nv_bfloat16*)vc, seq_len, idx, cnt, w,
                                                   nullptr, nullptr);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    dsm_combine_kernel<D><<<p.batch * p.hq, D, 0, st>>>(p, w, seq_len, (__nv_bfloat16*)o, lse);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (!full) return cudaSuccess;
    const dim3 sgrid((unsigned)((p.t_kv + kScoreKeys - 1) / kScoreKeys), (unsigned)(p.batch * p.hkv));
    dsm_score_kernel<<<sgrid, 256, 0, st>>>(p, seq_len, w);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const size_t s3 = BlockTopK::smem_bytes(p.k - p.window, kSelThreads);
    e = cudaFuncSetAttribute(dsm_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)s3);
    if (e != cudaSuccess) return e;
    dsm_select_kernel<<<p.batch * p.hkv, kSelThreads, s3, st>>>(p, seq_len, w, idx, cnt, sel);
    return cudaGetLastError();
}

template <int D>
static cudaError_t launch_prefill_t(const KParams& p, const void* q, const void* kc,
                                   const void* vc, const int32_t* idx, const int32_t* cnt,
                                   void* o, float* lse, cudaStream_t st) {
    Ws w{};
    auto kern = dsm_split_kernel<D, 2>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Smem<D>::kBytes);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)((long long)p.batch * p.hkv * p.t_q);
    kern<<<grid, kThreads, Smem<D>::kBytes, st>>>(p, (const __nv_bfloat16*)q,
                                                   (const __nv_bfloat16*)kc,
                                                   (const __nv_bfloat16*)vc, nullptr, idx, cnt, w,
                                                   (__nv_bfloat16*)o, lse);
    return cudaGetLastError();
}

}  // namespace dsm

// Token-mode sparse layer in prefill on the CUDA cores for wide groups and
// head_dim 256 (bf16, contiguous K^F/V^F, no window branch): one CTA per
// (query row, group), no workspace.
bool sparse_simt_rows_supported(const KParams& p, int dtype) {
    return dtype == HS_BF16 && p.mode == 1 && !p.bt && p.group <= dsm::kMaxGroup &&
           (p.head_dim == 64 || p.head_dim == 128 || p.head_dim == 256) &&
           (long long)p.batch * p.hkv * p.t_q < (1ll << 31);
}

cudaError_t launch_sparse_simt_rows(const KParams& p, const void* q, const void* kf,
                                    const void* vf, const int32_t* idx, const int32_t* cnt,
                                    void* o, float* lse, cudaStream_t st) {
    if (p.head_dim == 64) return dsm::launch_prefill_t<64>(p, q, kf, vf, idx, cnt, o, lse, st);
    if (p.head_dim == 128) return dsm::launch_prefill_t<128>(p, q, kf, vf, idx, cnt, o, lse, st);
    return dsm::launch_prefill_t<256>(p, q, kf, vf, idx, cnt, o, lse, st);
}

// Shapes this path takes: bf16, contiguous cache, groups of up to 64 heads,
// head_dim 64, 128 or 256.
bool decode_simt_split_supported(const KParams& p) {
    return !p.bt && p.group <= dsm::kMaxGroup &&
           (p.head_dim == 64 || p.head_dim == 128 || p.head_dim == 256);
}

size_t decode_simt_workspace(const KParams& p, bool full) { return dsm::ws_bytes(p, full); }

// Kernels one call launches (for the launch count).
int decode_simt_kernel_count(bool full) { return full ? 4 : 2; }

cudaError_t launch_decode_simt(const KParams& p, bool full, const void* q, const void* kc,
                               const void* vc, const int32_t* seq_len, int32_t* idx,
                               int32_t* cnt, void* o, float* lse, float* sel, void* ws,
                               cudaStream_t st) {
    if (p.head_dim == 64)
        return dsm::launch_t<64>(p, full, q, kc, vc, seq_len, idx, cnt, o, lse, sel, ws, st);
    if (p.head_dim == 128)
        return dsm::launch_t<128>(p, full, q, kc, vc, seq_len, idx, cnt, o, lse, sel, ws, st);
    return dsm::launch_t<256>(p, full, q, kc, vc, seq_len, idx, cnt, o, lse, sel, ws, st);
}

}  // namespace hs
