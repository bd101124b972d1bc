// full_tc.cu -- full-attention layer + block-level oracle indexer on the
// sm_100a tensor cores (tcgen05 MMA with TMEM accumulators, TMA-fed).
//
// What it computes ("HySparse 混合稀疏注意力（一）", "为什么不需要重新物化注意力
// 矩阵"; "HySparse: ..." 3.2, Algorithm 1): flash attention over causal key
// tiles of B_C = 64 keys, which in block mode are exactly the sparse blocks
// (B = B_C).  The row max of each S tile, m~_ij, is the block's max logit;
// S_ij = exp(m~_ij - lse_i) is its block score after the scan (the page's
// corrected line 14).  Instead of writing the T x T/B score matrix, every row
// keeps its 16 best (m~, block) pairs in registers; ranking within a head by
// logit equals ranking by probability ("TopK 只需要排序，为什么还要归一化分数").
// After the scan the heads of a GQA group are merged exactly: every member of
// the group's top-K is in the list of the head that attains its max, so the
// union of the lists, re-scored as m~ - lse_h, contains the answer
// ("GQA 下为什么要组内共享索引": S_bar = max over the group's heads).
//
// Q tile: 128 query rows = g heads x (128/g) positions of one KV group (rows
// are head-major, exactly as one 4-D TMA box lands), so every K/V tile is
// loaded once for the whole group.  A CTA runs two consecutive Q tiles that
// share every K/V tile; their softmax warpgroups alternate on the tensor core.
// Warp roles:
//   warp 0       TMA producer (both Q tiles once; K and V tiles through
//                rings of 3 stages each)
//   warp 1       TMEM owner and MMA issuer of Q tile 0; warp 10 issues for
//                Q tile 1: S = Q K^T into one of two TMEM buffers, then
//                O += P V (P from TMEM, V MN-major).  One issuing
//                thread per tile: a single thread cannot issue the MMAs of
//                both tiles as fast as the tensor core runs them.
//   warps 2..9   two softmax warpgroups, one thread per row (TMEM lane):
//                online softmax with lazy rescaling of O (only when the max
//                grows by > 2^8), P back into TMEM, epilogue.  Block mode
//                takes every tile's maximum (the block score, captured into
//                the row's list) and runs a third of the exponentials on the
//                FMA pipe; token mode needs no maximum (lazy softmax).
// All waits are bounded (tc_ptx.cuh); a timeout aborts the CTA cleanly.
#include "flash_tc.cuh"
#include "hs_common.cuh"
#include "hs_kernels.cuh"
#include "tc_ptx.cuh"

namespace hs {
namespace tc {

using L = fl::Layout<3, 3, 0>;  // 3-stage K and V rings, nothing beyond the P buffers
constexpr int kBM = L::kBM, kNQ = L::kNQ, kBN = L::kBN, kD = L::kD;
constexpr int kList = 16;     // per-row candidate list (>= k/B)
constexpr int kThreads = L::kThreads;
constexpr uint32_t kSmemBytes = L::kMiscOff + 16 + 1024;  // + room to align the base to 1 KB

struct FullTcArgs {
    KParams p;
    __nv_bfloat16* o;
    float* lse;
    int32_t* idx;
    int32_t* cnt;
    float* sel;
    int n_ctas_q;  // CTAs along the query axis
    int P;         // positions per Q tile (128 / g)
    int capture;   // 1: block-mode selection
};

// Insert (v, id) into a list sorted by value descending; equal values keep the
// earlier (lower) id first.  Static indices only, so the list stays in registers.
__device__ __forceinline__ void list_insert(float (&lv)[kList], int (&li)[kList], float v, int id) {
    if (!(v > lv[kList - 1])) return;
#pragma unroll
    for (int i = kList - 1; i >= 1; --i) {
        if (lv[i - 1] < v) {
            lv[i] = lv[i - 1];
            li[i] = li[i - 1];
        } else if (lv[i] < v) {
            lv[i] = v;
            li[i] = id;
        }
    }
    if (lv[0] < v) { lv[0] = v; li[0] = id; }
}

// Number of K/V tiles a Q tile needs: keys up to its last valid row's position.
__device__ __forceinline__ int tiles_for(const KParams& p, int first_row, int P) {
    if (first_row >= p.t_q) return 0;
    const int last_row = min(p.t_q, first_row + P) - 1;
    return min((p.t_kv + kBN - 1) / kBN, (p.q_offset + last_row) / kBN + 1);
}

// kCapture: block-mode index (needs every tile's maximum); otherwise o and lse
// only, with the lazy softmax that skips the tile maximum and runs every
// exponential on the MUFU unit (measured: offloading a share to the FMA pipe,
// which the block path needs, no longer pays once the maximum is gone).
constexpr int kLazyPolyEvery = 0;
template <bool kCapture>
__global__ void __launch_bounds__(kThreads, 1)
    full_tc_kernel(const __grid_constant__ CUtensorMap tmap_q,
                   const __grid_constant__ CUtensorMap tmap_k,
                   const __grid_constant__ CUtensorMap tmap_v, FullTcArgs a) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char* gbase = smem_raw + (base - raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const KParams& p = a.p;
    const int g = p.group, P = a.P;

    // CTA -> (b, u, query tile pair), heaviest (latest) query tiles first
    const int bu_n = p.batch * p.hkv;
    const int qc = a.n_ctas_q - 1 - (int)(blockIdx.x / bu_n);
    const int bu = (int)(blockIdx.x % bu_n);
    const int b = bu / p.hkv, u = bu % p.hkv;
    const int row0 = qc * kNQ * P;  // first query row of the CTA
    int ntq[kNQ];
#pragma unroll
    for (int q = 0; q < kNQ; ++q) ntq[q] = tiles_for(p, row0 + q * P, P);
    int nt = 0;
#pragma unroll
    for (int q = 0; q < kNQ; ++q) nt = max(nt, ntq[q]);

    auto bar = [&](int i) { return base + L::kBarOff + 8u * i; };
    volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L::kMiscOff + 4);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + L::kMiscOff);

    if (threadIdx.x == 0) {
        fl::init_barriers<L>(base + L::kBarOff);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(base + L::kMiscOff, L::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0)
            fl::producer<L>(base, &tmap_q, &tmap_k, &tmap_v, row0, P, u * g, b, bu, nt,
                            [](int j) { return j * kBN; }, abort_flag);
    } else if (warp == 1 || warp == L::kIssuer1Warp) {
        if (lane == 0) {
            const int qi = warp == 1 ? 0 : 1;
            fl::mma_issuer<L>(base, tmem, qi, nt, qi == 0 ? ntq[0] : ntq[1], abort_flag);
        }
    } else {
        // ------------------------------------------------------ softmax
        const int q = (warp - 2) >> 2;   // warpgroup = Q tile
        const int quad = warp & 3;       // TMEM lane quadrant of this warp
        const int row = quad * 32 + lane;
        const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16) + q * 256;
        const int hh = row / P, pr = row % P;
        const int qrow0 = row0 + q * P;              // first query row of this Q tile
        const int pos = p.q_offset + qrow0 + pr;
        const int nt_me = ntq[q];
        const float sl2 = p.scale_log2;
        float m_ref = -INFINITY, l = 0.f;
        float lv[kList];
        int li[kList];
#pragma unroll
        for (int i = 0; i < kList; ++i) { lv[i] = -INFINITY; li[i] = -1; }
        bool ok = true;
        for (int j = 0; j < nt_me; ++j) {
            const int s = j & 1;
            if (!fl::warp_wait(bar(L::BSF + 2 * q + s), (j >> 1) & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            uint32_t r[64];
            tmem_ld32(trow + 64 * s, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
            tmem_ld32(trow + 64 * s + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
            tmem_wait_ld();

            // causal: keys <= pos (only the diagonal tile masks anything).  Key 0
            // is in every row's first tile, so every row keeps a key and a third
            // of the exponentials can run on the FMA pipe.
            float corr;
            uint32_t pk[32];
            bool resc;
            if (kCapture) {
                float mt;
                resc = fl::softmax_tile<3>(r, 0, pos - j * kBN, sl2, m_ref, l, mt, corr, pk);
                if (mt > -INFINITY) list_insert(lv, li, mt, j);
            } else {
                resc = fl::softmax_tile_lazy<kLazyPolyEvery>(r, pos - j * kBN, sl2, m_ref, l, corr, pk);
            }
            // P over the S buffer just read: its previous P (tile j-2) was consumed
            // by a PV that executed before this tile's S MMA
            fl::store_p_tmem(trow + 64 * s, pk);
            if (__any_sync(0xffffffffu, resc)) {
                // O may only be touched once the PV of tile j-1 has finished
                if (!fl::warp_wait(bar(L::BPVD + 2 * q + (s ^ 1)), ((j - 1) >> 1) & 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                fl::rescale_o(trow + 128, resc ? corr : 1.f);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(L::BPF + 2 * q + s));
        }
        if (ok && nt_me > 0) ok = fl::warp_wait(bar(L::BOF + q), 0, abort_flag);
        const bool row_ok = nt_me > 0 && qrow0 + pr < p.t_q;
        const int h = u * g + hh;
        const size_t orow = ((size_t)b * p.hq + h) * p.t_q + qrow0 + pr;
        const float lse2 = m_ref + log2f(l);
        if (ok && nt_me > 0) {
            tc_fence_after();
            fl::store_o(trow + 128, true, 1.f / l, row_ok, a.o + orow * kD);
            if (row_ok) a.lse[orow] = lse2 * kLn2;
        }
        if (kCapture) {
            // ---- group merge.  Rows hh*P + pr of the g heads share position
            // pr; each row's list is sorted by (score desc, id asc).  The g
            // lists of a position are k-way merged in that order, skipping ids
            // already taken: an id's first occurrence carries its largest
            // listed score, so this is the union rule's top-k.  The merge runs
            // on all 128 threads: a group of g consecutive lanes per position,
            // lane hh holding the front of head hh's list; each step the group
            // finds its best front with in-group shuffles and that lane moves on.
            unsigned char* reg = gbase + L::kPOff + q * 32768;    // this tile's P buffers
            float* cs = reinterpret_cast<float*>(reg);         // [128][kList]
            int* ci = reinterpret_cast<int*>(reg + 128 * kList * 4);
            // every PV has completed (BOF), so the P buffers are free to reuse
#pragma unroll
            for (int i = 0; i < kList; ++i) {
                cs[row * kList + i] = li[i] >= 0 ? lv[i] - lse2 : -INFINITY;
                ci[row * kList + i] = ok ? li[i] : -1;
            }
            asm volatile("bar.sync %0, 128;" ::"r"(1 + q) : "memory");
            const int wl = row >> 5;                  // warp within the warpgroup
            const int gh = lane % g;                  // head of this lane's list
            const int pp = wl * (32 / g) + lane / g;  // position of this lane's group
            const int* lid = ci + (gh * P + pp) * kList;
            const float* lsc = cs + (gh * P + pp) * kList;
            int ptr = 0;
            float fv = lsc[0];
            int fid = lid[0] >= 0 ? lid[0] : 0x7fffffff;
            if (lid[0] < 0) fv = -INFINITY;
            int sid[kList];
            float ssc[kList];
            int nsel = 0;
            const int ksel = p.ksel;
            // warp-uniform trip count: every group of the warp takes part in the shuffles
            for (int step = 0; step < g * kList; ++step) {
                float bv = fv;
                int bid = fid;
                for (int o = 1; o < g; o <<= 1) {
                    const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                    const int oid = __shfl_xor_sync(0xffffffffu, bid, o);
                    if (ov > bv || (ov == bv && oid < bid)) { bv = ov; bid = oid; }
                }
                const bool live = bv > -INFINITY && nsel < ksel;
                if (live && fv == bv && fid == bid) {  // this lane's front was taken
                    ++ptr;
                    if (ptr < kList && lid[ptr] >= 0) { fv = lsc[ptr]; fid = lid[ptr]; }
                    else { fv = -INFINITY; fid = 0x7fffffff; }
                }
                bool dup = false;
#pragma unroll
                for (int x = 0; x < kList; ++x)
                    if (x < nsel && sid[x] == bid) dup = true;
                if (live && !dup) {
#pragma unroll
                    for (int x = 0; x < kList; ++x)
                        if (x == nsel) { sid[x] = bid; ssc[x] = bv; }
                    ++nsel;
                }
                if (__all_sync(0xffffffffu, !live)) break;
            }
            if (ok && gh == 0 && pp < P && qrow0 + pp < p.t_q) {
                // write in ascending id order
                const size_t orow_i = ((size_t)b * p.hkv + u) * p.t_q + qrow0 + pp;
                int32_t* irow = a.idx + orow_i * p.ksel;
                float* srow = a.sel ? a.sel + orow_i * p.ksel : nullptr;
#pragma unroll
                for (int x = 0; x < kList; ++x) {
                    if (x >= nsel) continue;
                    int op = 0;
#pragma unroll
                    for (int y = 0; y < kList; ++y)
                        if (y < nsel && sid[y] < sid[x]) ++op;
                    irow[op] = sid[x];
                    if (srow) srow[op] = exp2f(ssc[x]);
                }
                for (int x = nsel; x < p.ksel; ++x) {
                    irow[x] = -1;
                    if (srow) srow[x] = 0.f;
                }
                a.cnt[orow_i] = nsel;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, L::kTmemCols);
    }
}

// ------------------------------------------------------------------- host
}  // namespace tc

bool full_tc_supported(const KParams& p, int dtype) {
    if (dtype != HS_BF16 || p.head_dim != 128) return false;
    if (128 % p.group != 0) return false;
    // block mode: the group merge runs on g consecutive lanes of a warp
    if (p.mode == 0) return p.block_size == tc::kBN && p.ksel <= tc::kList && p.group <= 16;
    return true;
}

// capture = 1: block-mode index into idx/cnt/sel.  capture = 0: o and lse only.
cudaError_t launch_full_tc(const KParams& p, const void* q, const void* k, const void* v,
                           void* o, float* lse, int32_t* idx, int32_t* cnt, float* sel,
                           int capture, cudaStream_t st) {
    using namespace tc;
    const int g = p.group, P = kBM / g;
    CUtensorMap mq, mk, mv;
    const cuuint64_t qd[4] = {(cuuint64_t)kD, (cuuint64_t)p.t_q, (cuuint64_t)p.hq,
                              (cuuint64_t)p.batch};
    const cuuint64_t qs[3] = {(cuuint64_t)kD * 2, (cuuint64_t)p.t_q * kD * 2,
                              (cuuint64_t)p.hq * p.t_q * kD * 2};
    const cuuint32_t qb[4] = {64, (cuuint32_t)P, (cuuint32_t)g, 1};
    const cuuint64_t kdims[3] = {(cuuint64_t)kD, (cuuint64_t)p.t_kv,
                                 (cuuint64_t)p.hkv * p.batch};
    const cuuint64_t ks[2] = {(cuuint64_t)kD * 2, (cuuint64_t)p.t_kv * kD * 2};
    const cuuint32_t kb[3] = {64, (cuuint32_t)kBN, 1};
    if (!encode(&mq, q, 4, qd, qs, qb) || !encode(&mk, k, 3, kdims, ks, kb) ||
        !encode(&mv, v, 3, kdims, ks, kb))
        return cudaErrorInvalidValue;
    FullTcArgs a;
    a.p = p;
    a.o = (__nv_bfloat16*)o;
    a.lse = lse;
    a.idx = idx;
    a.cnt = cnt;
    a.sel = sel;
    a.P = P;
    a.n_ctas_q = (p.t_q + kNQ * P - 1) / (kNQ * P);
    a.capture = capture;
    auto kern = capture ? full_tc_kernel<true> : full_tc_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kSmemBytes);
    if (e != cudaSuccess) return e;
    const long long grid = (long long)a.n_ctas_q * p.batch * p.hkv;
    kern<<<(unsigned)grid, kThreads, kSmemBytes, st>>>(mq, mk, mv, a);
    return cudaGetLastError();
}

}  // namespace hs
