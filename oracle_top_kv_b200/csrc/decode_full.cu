// decode_full.cu -- decode step of the full-attention layer acting as the
// oracle indexer ("HySparse 混合稀疏注意力（一）": at decode step t the new token
// first passes the full layer, which selects for position t; cost model
// "Decode：关键收益来自少读 KV": the full layer streams the whole cache).
//
// Three launches per step:
//  1. decode_full_split_kernel: one warp per (sequence, kv group, 2048-key
//     split) streams its slice of the cache once; the group's heads are the
//     16 MMA rows.  It keeps an online-softmax partial (m, l, O) per head and
//     exports every scaled logit a2_{h,i} (log2 domain) to the workspace,
//     because the group score max_h (a2_{h,i} - lse2_h) needs every head's
//     final lse, known only after all splits;
//  2. the exact log-sum-exp merge of the splits (shared with the sparse
//     decode) -> o, lse, and lse2 for the selector;
//  3. the selector ranks keys 0..t-w by max_h (a2_{h,i} - lse2_h) (= log2 of
//     max_h p_{h,t,i}) with the exact streaming top-k and appends the forced
//     window t-w+1..t ("HySparse2 ..." 4.2): 8 CTAs per (sequence, group)
//     each keep the top-(k-w) of a slice of the keys, and a merge kernel
//     takes the top-(k-w) of their union (decode_select_kernel, one CTA per
//     unit, serves budgets above 1024).
#include "attend_mma.cuh"
#include "block_topk.cuh"
#include "cta_select.cuh"
#include "hs_common.cuh"
#include "hs_kernels.cuh"

namespace hs {

cudaError_t launch_decode_combine(const KParams& p, const float* part, int n_split,
                                  const int32_t* seq_len, void* o, float* lse, float* lse2,
                                  cudaStream_t st);

constexpr int kDecodeKeys = 2048;  // cache keys per split
constexpr int kDecodeWarps = 4;
constexpr int kSelectThreads = 512;

constexpr int kSelSlice = 16384;       // most ranked keys one selector CTA stages
constexpr int kSelMaxRanked = 1024;    // k - w handled by the split selector
constexpr int kMergeCap = 8192;        // candidate keys the merge holds at once
// The merge writes ids through a bitmap over 0..t below this (in its buffer).
constexpr int kBitmapKeys = (kMergeCap - kSelMaxRanked) * 64;

// CTAs per (sequence, group) in the split selector: slices of at most
// kSelSlice keys, and enough CTAs for about two per SM of a 148-SM part
// (slices not shorter than 2048 keys).
static int sel_splits(const KParams& p) {
    const int units = p.batch * p.hkv;
    const int by_len = (p.t_kv + kSelSlice - 1) / kSelSlice;
    const int by_fill = min((296 + units - 1) / units, (p.t_kv + 2047) / 2048);
    return max(1, max(by_len, by_fill));
}

constexpr int kSelGroup = 8;  // slices a first-level merge CTA folds (many slices)

struct DecodeWs {
    float* logits;    // [batch*hkv][t_kv][16]
    float* part;      // [batch*hkv][n_split][16][D+2]
    float* lse2;      // [batch*hq]
    uint64_t* cand;   // [batch*hkv][n_sel][kSelMaxRanked] selection keys
    int* cand_n;      // [batch*hkv][n_sel]
    uint64_t* cand2;  // [batch*hkv][n_grp][kSelMaxRanked] first-level merge output
    int* cand2_n;     // [batch*hkv][n_grp]
    int n_split, n_sel, n_grp;
};

// Many slices (few sequences, long caches) are merged in two levels.
static int sel_groups(int n_sel) { return n_sel > 2 * kSelGroup ? (n_sel + kSelGroup - 1) / kSelGroup : 0; }

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

static DecodeWs decode_ws_layout(const KParams& p, void* base) {
    DecodeWs w;
    w.n_split = (p.t_kv + kDecodeKeys - 1) / kDecodeKeys;
    w.n_sel = sel_splits(p);
    w.n_grp = sel_groups(w.n_sel);
    const size_t units = (size_t)p.batch * p.hkv;
    const size_t logits_b = align256(units * p.t_kv * 16 * sizeof(float));
    const size_t part_b = align256(units * w.n_split * 16 * (p.head_dim + 2) * sizeof(float));
    const size_t lse_b = align256((size_t)p.batch * p.hq * sizeof(float));
    const size_t cand_b = align256(units * w.n_sel * kSelMaxRanked * sizeof(uint64_t));
    char* c = static_cast<char*>(base);
    w.logits = reinterpret_cast<float*>(c);
    w.part = reinterpret_cast<float*>(c + logits_b);
    w.lse2 = reinterpret_cast<float*>(c + logits_b + part_b);
    w.cand = reinterpret_cast<uint64_t*>(c + logits_b + part_b + lse_b);
    w.cand_n = reinterpret_cast<int*>(c + logits_b + part_b + lse_b + cand_b);
    const size_t candn_b = align256(units * w.n_sel * sizeof(int));
    const size_t cand2_b = align256(units * w.n_grp * kSelMaxRanked * sizeof(uint64_t));
    w.cand2 = reinterpret_cast<uint64_t*>(c + logits_b + part_b + lse_b + cand_b + candn_b);
    w.cand2_n = reinterpret_cast<int*>(c + logits_b + part_b + lse_b + cand_b + candn_b + cand2_b);
    return w;
}

size_t decode_full_workspace(const KParams& p) {
    const int n_split = (p.t_kv + kDecodeKeys - 1) / kDecodeKeys;
    const size_t units = (size_t)p.batch * p.hkv;
    return align256(units * p.t_kv * 16 * sizeof(float)) +
           align256(units * n_split * 16 * (p.head_dim + 2) * sizeof(float)) +
           align256((size_t)p.batch * p.hq * sizeof(float)) +
           align256(units * sel_splits(p) * kSelMaxRanked * sizeof(uint64_t)) +
           align256(units * sel_splits(p) * sizeof(int)) +
           align256(units * sel_groups(sel_splits(p)) * kSelMaxRanked * sizeof(uint64_t)) +
           align256(units * sel_groups(sel_splits(p)) * sizeof(int));
}

// Writes every head's scaled logit a2 = scale_log2 * q.k of the chunk's keys.
template <int D>
struct LogitExport {
    float* logits;  // this unit's [t_kv][16]
    int last, g;
    float scale_log2;
    __device__ __forceinline__ void operator()(int, float (&s)[4][4], int key0) const {
        const int lane = threadIdx.x & 31, gid = lane >> 2, tig = lane & 3;
#pragma unroll
        for (int n = 0; n < 4; ++n) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int h = gid + 8 * (e >> 1);
                const int key = key0 + n * 8 + tig * 2 + (e & 1);
                if (h < g && key <= last) logits[(size_t)key * 16 + h] = s[n][e] * scale_log2;
            }
        }
    }
};

template <int D>
__global__ void __launch_bounds__(kDecodeWarps * 32)
    decode_full_split_kernel(const __grid_constant__ CUtensorMap tm_k,
                             const __grid_constant__ CUtensorMap tm_v, KParams p,
                             const __nv_bfloat16* __restrict__ q,
                             const __nv_bfloat16* __restrict__ kc,
                             const __nv_bfloat16* __restrict__ vc,
                             const int32_t* __restrict__ seq_len, DecodeWs ws) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int task = blockIdx.x * kDecodeWarps + warp;
    if (task >= p.batch * p.hkv * ws.n_split) return;
    const int sp = task % ws.n_split;
    const int unit = task / ws.n_split;
    const int u = unit % p.hkv, b = unit / p.hkv;
    const int g = p.group;
    const int L = seq_len[b];
    AttnState<D> st;
    st.init();
    const int first = sp * kDecodeKeys;
    if (L >= 1 && L <= p.t_kv && first < L) {
        const int last = min(L - 1, first + kDecodeKeys - 1);
        const uint32_t sbase = base + warp * WarpSmem<D>::kBytes;
        TmaRing ring{base + kDecodeWarps * WarpSmem<D>::kBytes + 16u * warp, 0u};
        if (lane == 0) {
            tc::mbar_init(ring.bar, 1);
            tc::mbar_init(ring.bar + 8, 1);
            tc::fence_mbar_init();
        }
        __syncwarp();
        uint32_t qf[D / 16][4];
        load_q_frags<D>(qf, q + ((size_t)b * p.hq + u * g) * D, D, g);
        LogitExport<D> hook{ws.logits + (size_t)unit * p.t_kv * 16, last, g, p.scale_log2};
        if (p.bt) {
            // paged cache: consecutive logical keys, gathered row by row through
            // the block table (a chunk may straddle pages); the hook gets each
            // chunk's first logical key
            const PagedSrc<KeyRange> src{KeyRange{first, last}, page_map(p, b, u)};
            attend_rows<D>(st, qf, kc, vc, src.src.n_chunks(), src, sbase, p.scale_log2,
                           [&](int c, float (&s)[4][4], int) { hook(c, s, first + c * kChunk); });
        } else {
            const ContiguousKeys src{first, last};
            attend_rows_tma<D>(st, qf, &tm_k, &tm_v, unit, src.n_chunks(), src, sbase, ring,
                               p.scale_log2, hook);
        }
    }
    store_partial<D>(st, ws.part + (size_t)task * 16 * (D + 2), g);
}

__global__ void __launch_bounds__(kSelectThreads)
    decode_select_kernel(KParams p, const int32_t* __restrict__ seq_len, DecodeWs ws,
                         int32_t* __restrict__ idx, int32_t* __restrict__ cnt,
                         float* __restrict__ sel) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    __shared__ int s_count;
    __shared__ unsigned long long s_thresh;
    __shared__ float s_lse2[16];
    const int unit = blockIdx.x;
    const int u = unit % p.hkv, b = unit / p.hkv;
    const int g = p.group;
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
    if (threadIdx.x < 16) s_lse2[threadIdx.x] = threadIdx.x < g ? ws.lse2[b * p.hq + u * g + threadIdx.x] : 0.f;
    __syncthreads();

    const bool select_all = t + 1 <= p.k;
    const int lo = t - p.window + 1;
    const bool ranked = !select_all && Kc > 0;
    int n_scored;
    if (select_all) n_scored = srow ? t + 1 : 0;
    else n_scored = srow ? t + 1 : lo;
    const float* lg = ws.logits + (size_t)unit * p.t_kv * 16;

    for (int c0 = 0; c0 < n_scored; c0 += blockDim.x) {
        const int i = c0 + threadIdx.x;
        if (i < n_scored) {
            const float4* r4 = reinterpret_cast<const float4*>(lg + (size_t)i * 16);
            float s = -INFINITY;
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                if (q4 * 4 >= g) break;
                const float4 a = r4[q4];
                const float av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    if (q4 * 4 + e < g) s = fmaxf(s, av[e] - s_lse2[q4 * 4 + e]);
            }
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

// Group log-score of key i: max over the group's heads of a2 - lse2 (log2 of
// max_h p_{h,t,i}).
__device__ __forceinline__ float group_score(const float* lg_row, const float* lse2, int g) {
    const float4* r4 = reinterpret_cast<const float4*>(lg_row);
    float s = -INFINITY;
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) {
        if (q4 * 4 >= g) break;
        const float4 a = r4[q4];
        const float av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
            if (q4 * 4 + e < g) s = fmaxf(s, av[e] - lse2[q4 * 4 + e]);
    }
    return s;
}

// Stage 1 of the split selector: CTA (unit, slice) stages the group scores of
// its slice of the ranked keys 0..t-w in shared memory (as order bits), finds
// the slice's (k-w)-th largest selection key with a CTA-wide bucket select,
// and writes the slice's top-(k-w) keys out unsorted.  The group's top-(k-w)
// is contained in the union of the slices' top-(k-w).
__global__ void __launch_bounds__(kSelectThreads, 2)
    decode_select_split_kernel(KParams p, const int32_t* __restrict__ seq_len, DecodeWs ws) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    __shared__ CtaSelectSmem cs;
    __shared__ float s_lse2[16];
    __shared__ int s_n;
    uint32_t* bits = reinterpret_cast<uint32_t*>(smem_raw);  // [kSelSlice]
    const int unit = blockIdx.x / ws.n_sel, sp = blockIdx.x % ws.n_sel;
    const int u = unit % p.hkv, b = unit / p.hkv;
    const int g = p.group;
    const int L = seq_len[b];
    const int Kc = p.k - p.window;
    int* out_n = ws.cand_n + (size_t)unit * ws.n_sel + sp;
    if (L < 1 || L > p.t_kv || L <= p.k || Kc <= 0) {  // nothing ranked here
        if (threadIdx.x == 0) *out_n = 0;
        return;
    }
    const int lo = L - p.window;  // ranked keys 0..lo-1
    const int per = (lo + ws.n_sel - 1) / ws.n_sel;  // <= kSelSlice
    const int i0 = sp * per;
    const int n = max(0, min(lo, i0 + per) - i0);
    if (threadIdx.x < 16) s_lse2[threadIdx.x] = threadIdx.x < g ? ws.lse2[b * p.hq + u * g + threadIdx.x] : 0.f;
    __syncthreads();
    const float* lg = ws.logits + (size_t)unit * p.t_kv * 16;
    if (g == 16) {
        // two keys per thread per round, all 8 loads issued before any use
        // (the logits are read once: streaming loads)
        float nl[16];
#pragma unroll
        for (int h = 0; h < 16; ++h) nl[h] = -s_lse2[h];
        const float4* l4 = reinterpret_cast<const float4*>(lg + (size_t)i0 * 16);
        constexpr int U = 2;
        for (int base = threadIdx.x; base < n; base += U * blockDim.x) {
            float4 r[U][4];
#pragma unroll
            for (int k = 0; k < U; ++k) {
                const int i = base + k * blockDim.x;
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4)
                    r[k][q4] = i < n ? __ldcs(l4 + (size_t)i * 4 + q4) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int k = 0; k < U; ++k) {
                const int i = base + k * blockDim.x;
                float v[16];
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    v[4 * q4] = r[k][q4].x + nl[4 * q4];
                    v[4 * q4 + 1] = r[k][q4].y + nl[4 * q4 + 1];
                    v[4 * q4 + 2] = r[k][q4].z + nl[4 * q4 + 2];
                    v[4 * q4 + 3] = r[k][q4].w + nl[4 * q4 + 3];
                }
                const float sc = fmaxf(
                    tc::max3f(tc::max3f(v[0], v[1], v[2]), tc::max3f(v[3], v[4], v[5]),
                              tc::max3f(v[6], v[7], v[8])),
                    tc::max3f(tc::max3f(v[9], v[10], v[11]), tc::max3f(v[12], v[13], v[14]), v[15]));
                if (i < n) bits[i] = float_order(sc);
            }
        }
    } else {
        for (int i = threadIdx.x; i < n; i += blockDim.x)
            bits[i] = float_order(group_score(lg + (size_t)(i0 + i) * 16, s_lse2, g));
    }
    __syncthreads();
    auto key = [&](int i) -> uint64_t {
        return ((uint64_t)bits[i] << 32) | (uint64_t)(0xffffffffu - (uint32_t)(i0 + i));
    };
    uint64_t* dst = ws.cand + ((size_t)unit * ws.n_sel + sp) * kSelMaxRanked;
    if (n <= Kc) {
        for (int i = threadIdx.x; i < n; i += blockDim.x) dst[i] = key(i);
        if (threadIdx.x == 0) *out_n = n;
        return;
    }
    const uint64_t kth = cta_kth_largest(key, n, Kc, cs);
    if (threadIdx.x == 0) s_n = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const uint64_t v = key(i);
        if (v >= kth) dst[atomicAdd(&s_n, 1)] = v;
    }
    __syncthreads();
    if (threadIdx.x == 0) *out_n = s_n;  // exactly Kc: the keys are distinct
}

// Keep the K largest of buf[0..n) (n > K), in buf[0..K); tmp holds K keys.
__device__ int cta_cut(uint64_t* buf, int n, int K, uint64_t* tmp, CtaSelectSmem& cs,
                       int* s_n) {
    const uint64_t kth = cta_kth_largest([&](int i) { return buf[i]; }, n, K, cs);
    if (threadIdx.x == 0) *s_n = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += blockDim.x)
        if (buf[i] >= kth) tmp[atomicAdd(s_n, 1)] = buf[i];
    __syncthreads();
    for (int i = threadIdx.x; i < K; i += blockDim.x) buf[i] = tmp[i];
    __syncthreads();
    return K;
}

// Stage 2: per unit, the final top-(k-w) of the slices' candidates (cut to
// k-w whenever the buffer would overflow), sorted by id, then the forced
// window; or every key when the budget covers them all.
// First level of a two-level merge: CTA (unit, group) folds kSelGroup slices'
// candidates into their top-(k-w), written out unsorted as one group list.
__global__ void __launch_bounds__(kSelectThreads)
    decode_select_group_kernel(KParams p, const int32_t* __restrict__ seq_len, DecodeWs ws) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    __shared__ CtaSelectSmem cs;
    __shared__ int s_n;
    const int unit = blockIdx.x / ws.n_grp, grp = blockIdx.x % ws.n_grp;
    const int b = unit / p.hkv;
    const int L = seq_len[b];
    const int Kc = p.k - p.window;
    int* out_n = ws.cand2_n + (size_t)unit * ws.n_grp + grp;
    if (L < 1 || L > p.t_kv || L <= p.k || Kc <= 0) {
        if (threadIdx.x == 0) *out_n = 0;
        return;
    }
    uint64_t* buf = reinterpret_cast<uint64_t*>(smem_raw);  // [kSelGroup * kSelMaxRanked]
    uint64_t* tmp = buf + kSelGroup * kSelMaxRanked;         // [kSelMaxRanked]
    int n = 0;
    const int s0 = grp * kSelGroup, s1 = min(ws.n_sel, s0 + kSelGroup);
    for (int sp = s0; sp < s1; ++sp) {
        const int c = ws.cand_n[(size_t)unit * ws.n_sel + sp];
        const uint64_t* src = ws.cand + ((size_t)unit * ws.n_sel + sp) * kSelMaxRanked;
        for (int x = threadIdx.x; x < c; x += blockDim.x) buf[n + x] = src[x];
        n += c;
    }
    __syncthreads();
    if (n > Kc) n = cta_cut(buf, n, Kc, tmp, cs, &s_n);
    uint64_t* dst = ws.cand2 + ((size_t)unit * ws.n_grp + grp) * kSelMaxRanked;
    for (int x = threadIdx.x; x < n; x += blockDim.x) dst[x] = buf[x];
    if (threadIdx.x == 0) *out_n = n;
}

__global__ void __launch_bounds__(kSelectThreads)
    decode_select_merge_kernel(KParams p, const int32_t* __restrict__ seq_len, DecodeWs ws,
                               const uint64_t* __restrict__ cand, const int* __restrict__ cand_n,
                               int n_src, int32_t* __restrict__ idx, int32_t* __restrict__ cnt,
                               float* __restrict__ sel) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    __shared__ CtaSelectSmem cs;
    __shared__ float s_lse2[16];
    __shared__ int s_n;
    __shared__ int s_scan[33];
    const int unit = blockIdx.x;
    const int u = unit % p.hkv, b = unit / p.hkv;
    const int g = p.group;
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
    if (threadIdx.x < 16) s_lse2[threadIdx.x] = threadIdx.x < g ? ws.lse2[b * p.hq + u * g + threadIdx.x] : 0.f;
    __syncthreads();
    const float* lg = ws.logits + (size_t)unit * p.t_kv * 16;
    if (t + 1 <= p.k) {  // the budget covers every key
        for (int x = threadIdx.x; x < p.ksel; x += blockDim.x) {
            irow[x] = x <= t ? x : -1;
            if (srow) srow[x] = x <= t ? exp2f(group_score(lg + (size_t)x * 16, s_lse2, g)) : 0.f;
        }
        if (threadIdx.x == 0) cnt[unit] = t + 1;
        return;
    }
    const int lo = t - p.window + 1;
    // window scores (only wanted with sel)
    if (srow)
        for (int x = threadIdx.x; x <= t - lo; x += blockDim.x)
            srow[Kc + x] = exp2f(group_score(lg + (size_t)(lo + x) * 16, s_lse2, g));
    uint64_t* buf = reinterpret_cast<uint64_t*>(smem_raw);  // [kMergeCap]
    uint64_t* tmp = buf + kMergeCap;                         // [kSelMaxRanked]
    int n = 0;
    if (Kc > 0) {
        for (int sp = 0; sp < n_src; ++sp) {
            const int c = cand_n[(size_t)unit * n_src + sp];
            if (n + c > kMergeCap) n = cta_cut(buf, n, Kc, tmp, cs, &s_n);
            const uint64_t* src = cand + ((size_t)unit * n_src + sp) * kSelMaxRanked;
            for (int x = threadIdx.x; x < c; x += blockDim.x) buf[n + x] = src[x];
            n += c;
            __syncthreads();
        }
        if (n > Kc) n = cta_cut(buf, n, Kc, tmp, cs, &s_n);
    }
    if (!srow && t < kBitmapKeys) {
        // ascending ids without sorting: mark the winners in a bitmap over
        // 0..t (in the free part of buf), then each thread reads out a run of
        // consecutive words at its prefix-sum offset
        uint32_t* bm = reinterpret_cast<uint32_t*>(buf + kSelMaxRanked);
        const int words = (t >> 5) + 1;
        const int per = (words + blockDim.x - 1) / blockDim.x;
        for (int x = threadIdx.x; x < per * (int)blockDim.x; x += blockDim.x) bm[x] = 0u;
        __syncthreads();
        for (int x = threadIdx.x; x < n; x += blockDim.x) {
            const uint32_t id = sel_key_id(buf[x]);
            atomicOr(&bm[id >> 5], 1u << (id & 31));
        }
        __syncthreads();
        const int w0 = threadIdx.x * per;
        int c = 0;
        for (int x = 0; x < per; ++x) c += __popc(bm[w0 + x]);
        const int at = cta_exclusive_sum(c, s_scan);
        int o = at;
        for (int x = 0; x < per; ++x) {
            uint32_t m = bm[w0 + x];
            while (m) {
                irow[o++] = (w0 + x) * 32 + (__ffs(m) - 1);
                m &= m - 1u;
            }
        }
    } else {
        const int sort_n = next_pow2(Kc > 0 ? Kc : 1);
        for (int x = threadIdx.x; x < sort_n; x += blockDim.x)
            tmp[x] = x < n ? (((uint64_t)sel_key_id(buf[x]) << 32) | (buf[x] >> 32)) : ~0ull;
        __syncthreads();
        cta_bitonic_sort(tmp, sort_n);
        for (int x = threadIdx.x; x < n; x += blockDim.x) {
            irow[x] = (int32_t)(tmp[x] >> 32);
            if (srow) srow[x] = exp2f(order_float((uint32_t)(tmp[x] & 0xffffffffu)));
        }
    }
    for (int x = threadIdx.x; x <= t - lo; x += blockDim.x) irow[n + x] = lo + x;
    const int n_out = n + (t - lo + 1);
    for (int x = n_out + threadIdx.x; x < p.ksel; x += blockDim.x) {
        irow[x] = -1;
        if (srow) srow[x] = 0.f;
    }
    if (threadIdx.x == 0) cnt[unit] = n_out;
}

template <int D>
static cudaError_t launch_decode_full_t(const KParams& p, const void* q, const void* kc,
                                        const void* vc, const int32_t* seq_len, int32_t* idx,
                                        int32_t* cnt, void* o, float* lse, float* sel, void* ws,
                                        cudaStream_t st) {
    DecodeWs w = decode_ws_layout(p, ws);
    const size_t smem = (size_t)kDecodeWarps * (WarpSmem<D>::kBytes + 16) + 1024;
    CUtensorMap mk, mv;
    const long long units = (long long)p.batch * p.hkv;
    // a paged pool is read by gathers only: its maps (unused) span the pool
    const long long rows = p.bt ? (long long)p.n_pages * p.hkv * p.page_size : p.t_kv;
    const long long mu = p.bt ? 1 : units;
    if (!tc::encode_rows(&mk, kc, D, rows, mu, kChunk) ||
        !tc::encode_rows(&mv, vc, D, rows, mu, kChunk))
        return cudaErrorInvalidValue;
    auto kern = decode_full_split_kernel<D>;
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int n_tasks = p.batch * p.hkv * w.n_split;
    kern<<<(n_tasks + kDecodeWarps - 1) / kDecodeWarps, kDecodeWarps * 32, smem, st>>>(
        mk, mv, p, (const __nv_bfloat16*)q, (const __nv_bfloat16*)kc, (const __nv_bfloat16*)vc,
        seq_len, w);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = launch_decode_combine(p, w.part, w.n_split, seq_len, o, lse, w.lse2, st)) !=
        cudaSuccess)
        return e;
    const int Kc = p.k - p.window;
    if (Kc <= kSelMaxRanked) {
        const size_t s1 = sizeof(uint32_t) * kSelSlice;
        e = cudaFuncSetAttribute(decode_select_split_kernel,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s1);
        if (e != cudaSuccess) return e;
        decode_select_split_kernel<<<p.batch * p.hkv * w.n_sel, kSelectThreads, s1, st>>>(
            p, seq_len, w);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        const uint64_t* cand = w.cand;
        const int* cand_n = w.cand_n;
        int n_src = w.n_sel;
        if (w.n_grp > 0) {  // many slices: fold groups of them on more CTAs first
            const size_t sg = sizeof(uint64_t) * (kSelGroup * kSelMaxRanked + kSelMaxRanked);
            e = cudaFuncSetAttribute(decode_select_group_kernel,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sg);
            if (e != cudaSuccess) return e;
            decode_select_group_kernel<<<p.batch * p.hkv * w.n_grp, kSelectThreads, sg, st>>>(
                p, seq_len, w);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
            cand = w.cand2;
            cand_n = w.cand2_n;
            n_src = w.n_grp;
        }
        const size_t s2 = sizeof(uint64_t) * (kMergeCap + kSelMaxRanked);
        e = cudaFuncSetAttribute(decode_select_merge_kernel,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s2);
        if (e != cudaSuccess) return e;
        decode_select_merge_kernel<<<p.batch * p.hkv, kSelectThreads, s2, st>>>(
            p, seq_len, w, cand, cand_n, n_src, idx, cnt, sel);
        return cudaGetLastError();
    }
    const size_t sel_smem = BlockTopK::smem_bytes(Kc, kSelectThreads);
    e = cudaFuncSetAttribute(decode_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)sel_smem);
    if (e != cudaSuccess) return e;
    decode_select_kernel<<<p.batch * p.hkv, kSelectThreads, sel_smem, st>>>(p, seq_len, w, idx,
                                                                           cnt, sel);
    return cudaGetLastError();
}

int decode_full_kernel_count(const KParams& p) {
    if (p.k - p.window > kSelMaxRanked) return 3;  // split, combine, one-CTA selector
    return sel_groups(sel_splits(p)) > 0 ? 5 : 4;  // + split selector, (group merge,) merge
}

cudaError_t launch_decode_full(const KParams& p, const void* q, const void* kc, const void* vc,
                               const int32_t* seq_len, int32_t* idx, int32_t* cnt, void* o,
                               float* lse, float* sel, void* ws, cudaStream_t st) {
    if (p.head_dim == 64)
        return launch_decode_full_t<64>(p, q, kc, vc, seq_len, idx, cnt, o, lse, sel, ws, st);
    return launch_decode_full_t<128>(p, q, kc, vc, seq_len, idx, cnt, o, lse, sel, ws, st);
}

}  // namespace hs
