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
//   warp 0       TMA producer (both Q tiles once; K and V tiles, 3-stage ring)
//   warp 1       TMEM owner and MMA issuer: per Q tile S = Q K^T into one of
//                two TMEM buffers, then O += P V (P from shared memory, V
//                MN-major)
//   warps 2..9   two softmax warpgroups, one thread per row (TMEM lane):
//                online softmax with lazy rescaling of O (only when the max
//                grows by > 2^8), P to shared memory, block-score capture,
//                epilogue.
// All waits are bounded (tc_ptx.cuh); a timeout aborts the CTA cleanly.
#include "hs_common.cuh"
#include "hs_kernels.cuh"
#include "tc_ptx.cuh"

namespace hs {
namespace tc {

constexpr int kBM = 128;      // rows per Q tile (one softmax warpgroup)
constexpr int kNQ = 2;        // Q tiles per CTA, sharing every K/V tile
constexpr int kBN = 64;       // keys per K/V tile (= block size B)
constexpr int kD = 128;
constexpr int kKV = 3;        // K/V ring stages
constexpr int kList = 16;     // per-row candidate list (>= k/B)
constexpr int kThreads = 64 + 128 * kNQ;
// The TMA producer and the MMA issuer are single threads on the critical
// path: they poll their barriers instead of sleeping.
constexpr bool kRoleSleep = false;

constexpr uint32_t kQOff = 0;                         // kNQ x 32 KB (two d halves each)
constexpr uint32_t kKOff = kNQ * 32768;               // kKV x 16 KB
constexpr uint32_t kVOff = kKOff + kKV * 16384;       // kKV x 16 KB
constexpr uint32_t kPOff = kVOff + kKV * 16384;       // kNQ x 2 x 16 KB
constexpr uint32_t kBarOff = kPOff + kNQ * 2 * 16384;
enum {
    BQ = 0,
    BKVF = 1,
    BKVE = BKVF + kKV,
    BSF = BKVE + kKV,      // [q][s]
    BSE = BSF + 2 * kNQ,
    BPF = BSE + 2 * kNQ,
    BPVD = BPF + 2 * kNQ,
    BOF = BPVD + 2 * kNQ,
    BDRAIN = BOF + 1,
    BCOUNT = BDRAIN + 1
};
constexpr uint32_t kMiscOff = kBarOff + BCOUNT * 8;
constexpr uint32_t kSmemBytes = kMiscOff + 16 + 1024;  // + room to align the base to 1 KB
constexpr uint32_t kTmemCols = 256 * kNQ;              // per Q tile: S0 | S1 | O

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

// Bounded wait that ignores the abort flag (used to drain in-flight work).
__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity) {
    const long long t0 = clock64();
    while (!mbar_try_wait_sleep(bar, parity)) {
        if (clock64() - t0 > kWaitCycles) { set_status(HS_ERR_TIMEOUT); return; }
    }
}

// Warp-uniform bounded wait: every lane polls, the warp proceeds only if all saw it.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort) {
    const bool ok = mbar_wait(bar, parity, abort);
    return __all_sync(0xffffffffu, ok);
}

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

    auto bar = [&](int i) { return base + kBarOff + 8u * i; };
    volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + kMiscOff + 4);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + kMiscOff);

    if (threadIdx.x == 0) {
        mbar_init(bar(BQ), 1);
        for (int i = 0; i < kKV; ++i) { mbar_init(bar(BKVF + i), 1); mbar_init(bar(BKVE + i), 1); }
        for (int i = 0; i < 2 * kNQ; ++i) {
            mbar_init(bar(BSF + i), 1);
            mbar_init(bar(BSE + i), 4);
            mbar_init(bar(BPF + i), 4);
            mbar_init(bar(BPVD + i), 1);
        }
        mbar_init(bar(BOF), 1);
        mbar_init(bar(BDRAIN), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(base + kMiscOff, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tmap(&tmap_q);
            prefetch_tmap(&tmap_k);
            prefetch_tmap(&tmap_v);
            mbar_arrive_expect_tx(bar(BQ), kNQ * 32768);
#pragma unroll
            for (int q = 0; q < kNQ; ++q) {
                tma_load_4d(base + kQOff + q * 32768, &tmap_q, bar(BQ), 0, row0 + q * P, u * g, b);
                tma_load_4d(base + kQOff + q * 32768 + 16384, &tmap_q, bar(BQ), 64, row0 + q * P,
                            u * g, b);
            }
            int issued = 0;
            for (int j = 0; j < nt; ++j) {
                const int st = j % kKV;
                if (j >= kKV &&
                    !mbar_wait(bar(BKVE + st), ((j / kKV) - 1) & 1, abort_flag, kRoleSleep))
                    break;
                const uint32_t f = bar(BKVF + st);
                mbar_arrive_expect_tx(f, 4 * 8192);
                const uint32_t kd = base + kKOff + st * 16384, vd = base + kVOff + st * 16384;
                const int key0 = j * kBN;
                tma_load_3d(kd, &tmap_k, f, 0, key0, bu);
                tma_load_3d(kd + 8192, &tmap_k, f, 64, key0, bu);
                tma_load_3d(vd, &tmap_v, f, 0, key0, bu);
                tma_load_3d(vd + 8192, &tmap_v, f, 64, key0, bu);
                issued = j + 1;
            }
            // every issued load must have landed before the CTA may exit
            mbar_drain(bar(BQ), 0);
            for (int j = max(0, issued - kKV); j < issued; ++j)
                mbar_drain(bar(BKVF + j % kKV), (j / kKV) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t id_s = idesc_bf16(kBM, kBN, false, false);
            const uint32_t id_o = idesc_bf16(kBM, kD, false, true);
            bool ok = mbar_wait(bar(BQ), 0, abort_flag, kRoleSleep);
            tc_fence_after();
            for (int j = 0; ok && j <= nt; ++j) {
                if (j < nt) {
                    const int st = j % kKV, s = j & 1;
                    if (!mbar_wait(bar(BKVF + st), (j / kKV) & 1, abort_flag, kRoleSleep)) break;
                    const uint32_t kb = base + kKOff + st * 16384;
#pragma unroll
                    for (int q = 0; q < kNQ; ++q) {
                        if (j >= ntq[q]) continue;
                        if (j >= 2 && !mbar_wait(bar(BSE + 2 * q + s), ((j >> 1) - 1) & 1,
                                                 abort_flag, kRoleSleep)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t qb = base + kQOff + q * 32768;
#pragma unroll
                        for (int kk = 0; kk < kD / 16; ++kk) {
                            const uint64_t ad = sw128_desc(qb + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
                            const uint64_t bd = sw128_desc(kb + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024);
                            umma_ss(tmem + q * 256 + 64 * s, ad, bd, id_s, kk > 0 ? 1u : 0u);
                        }
                        umma_commit(bar(BSF + 2 * q + s));
                    }
                    if (!ok) break;
                }
                if (j >= 1) {
                    const int jj = j - 1, sp = jj & 1, stp = jj % kKV;
                    const uint32_t vb = base + kVOff + stp * 16384;
#pragma unroll
                    for (int q = 0; q < kNQ; ++q) {
                        if (jj >= ntq[q]) continue;
                        if (!mbar_wait(bar(BPF + 2 * q + sp), (jj >> 1) & 1, abort_flag,
                                       kRoleSleep)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t pb = base + kPOff + (2 * q + sp) * 16384;
#pragma unroll
                        for (int kk = 0; kk < kBN / 16; ++kk) {
                            const uint64_t ad = sw128_desc(pb + kk * 32, 16, 1024);
                            const uint64_t bd = sw128_desc(vb + kk * 2048, 8192, 1024);
                            umma_ss(tmem + q * 256 + 128, ad, bd, id_o, (jj > 0 || kk > 0) ? 1u : 0u);
                        }
                        umma_commit(bar(BPVD + 2 * q + sp));
                    }
                    if (!ok) break;
                    umma_commit(bar(BKVE + stp));
                }
            }
            umma_commit(bar(BOF));
            umma_commit(bar(BDRAIN));
            mbar_drain(bar(BDRAIN), 0);
        }
    } else {
        // ------------------------------------------------------ softmax
        const int q = (warp - 2) >> 2;   // warpgroup = Q tile
        const int quad = warp & 3;       // TMEM lane quadrant of this warp
        const int row = quad * 32 + lane;
        const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16) + q * 256;
        const int hh = row / P, pr = row % P;
        const int qrow0 = row0 + q * P;              // first query row of this Q tile
        const int pos_first = p.q_offset + qrow0;    // its position
        const int pos = pos_first + pr;
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
            if (!warp_wait(bar(BSF + 2 * q + s), (j >> 1) & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            uint32_t r[64];
            tmem_ld32(trow + 64 * s, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
            tmem_ld32(trow + 64 * s + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(BSE + 2 * q + s));

            const int key0 = j * kBN;
            float x[64];
#pragma unroll
            for (int c = 0; c < 64; ++c) x[c] = __uint_as_float(r[c]);
            if (key0 + kBN - 1 > pos_first) {  // diagonal tile: causal mask per row
                const int lim = pos - key0;
#pragma unroll
                for (int c = 0; c < 64; ++c) x[c] = c <= lim ? x[c] : -INFINITY;
            }
            // tile max of the raw logits (tree), then to the log2 domain
            float mx[16];
#pragma unroll
            for (int c = 0; c < 16; ++c)
                mx[c] = fmaxf(fmaxf(x[c], x[c + 16]), fmaxf(x[c + 32], x[c + 48]));
#pragma unroll
            for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
                for (int c = 0; c < w; ++c) mx[c] = fmaxf(mx[c], mx[c + w]);
            const float mt = mx[0] * sl2;  // -inf stays -inf (sl2 > 0)
            if (a.capture && mt > -INFINITY) list_insert(lv, li, mt, j);
            // lazy rescale: keep the reference max unless the tile exceeds it by 2^8
            bool resc = false;
            float corr = 1.f;
            if (mt > m_ref + 8.f) {
                corr = ex2(m_ref - mt);  // 0 on the first tile
                resc = j > 0;
                m_ref = mt;
                l *= corr;
            }
            // p = 2^(x * scale_log2 - m): packed FFMA for the arguments and
            // packed adds for the row sum
            const float2 s2 = make_float2(sl2, sl2), n2 = make_float2(-m_ref, -m_ref);
            float e[64];
            float2 acc[8];
#pragma unroll
            for (int c2 = 0; c2 < 32; ++c2) {
                const float2 y = ffma2(make_float2(x[2 * c2], x[2 * c2 + 1]), s2, n2);
                e[2 * c2] = ex2(y.x);
                e[2 * c2 + 1] = ex2(y.y);
                const float2 ev = make_float2(e[2 * c2], e[2 * c2 + 1]);
                acc[c2 & 7] = c2 < 8 ? ev : fadd2(acc[c2 & 7], ev);
            }
#pragma unroll
            for (int w = 4; w >= 1; w >>= 1)
#pragma unroll
                for (int c = 0; c < w; ++c) acc[c] = fadd2(acc[c], acc[c + w]);
            l += acc[0].x + acc[0].y;
            uint32_t pk[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) pk[c] = pack_bf16(e[2 * c], e[2 * c + 1]);
            // P buffer s of this tile is free once the PV of tile j-2 is done
            if (j >= 2 && !warp_wait(bar(BPVD + 2 * q + s), ((j >> 1) - 1) & 1, abort_flag)) { ok = false; break; }
            unsigned char* prow = gbase + kPOff + (2 * q + s) * 16384 + row * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                uint4 v4 = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
                *reinterpret_cast<uint4*>(prow + ((c ^ (row & 7)) << 4)) = v4;
            }
            fence_proxy_async_smem();
            if (__any_sync(0xffffffffu, resc)) {
                // O may only be touched once the PV of tile j-1 has finished
                if (!warp_wait(bar(BPVD + 2 * q + (s ^ 1)), ((j - 1) >> 1) & 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const float cf = resc ? corr : 1.f;
#pragma unroll
                for (int c4 = 0; c4 < kD / 32; ++c4) {
                    uint32_t ro[32];
                    tmem_ld32(trow + 128 + 32 * c4, ro);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 32; ++c) ro[c] = __float_as_uint(__uint_as_float(ro[c]) * cf);
                    tmem_st32(trow + 128 + 32 * c4, ro);
                }
                tmem_wait_st();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(BPF + 2 * q + s));
        }
        if (ok && nt_me > 0) ok = warp_wait(bar(BOF), 0, abort_flag);
        const bool row_ok = nt_me > 0 && qrow0 + pr < p.t_q;
        const int h = u * g + hh;
        const size_t orow = ((size_t)b * p.hq + h) * p.t_q + qrow0 + pr;
        const float lse2 = m_ref + log2f(l);
        if (ok && nt_me > 0) {
            tc_fence_after();
            const float inv = 1.f / l;
            __nv_bfloat16* og = a.o + orow * kD;
#pragma unroll
            for (int c4 = 0; c4 < kD / 32; ++c4) {
                uint32_t ro[32];
                tmem_ld32(trow + 128 + 32 * c4, ro);
                tmem_wait_ld();
                if (row_ok) {
#pragma unroll
                    for (int c = 0; c < 32; c += 8) {
                        uint4 v4;
                        v4.x = pack_bf16(__uint_as_float(ro[c]) * inv, __uint_as_float(ro[c + 1]) * inv);
                        v4.y = pack_bf16(__uint_as_float(ro[c + 2]) * inv, __uint_as_float(ro[c + 3]) * inv);
                        v4.z = pack_bf16(__uint_as_float(ro[c + 4]) * inv, __uint_as_float(ro[c + 5]) * inv);
                        v4.w = pack_bf16(__uint_as_float(ro[c + 6]) * inv, __uint_as_float(ro[c + 7]) * inv);
                        *reinterpret_cast<uint4*>(og + c4 * 32 + c) = v4;
                    }
                }
            }
            if (row_ok) a.lse[orow] = lse2 * kLn2;
        }
        if (a.capture) {
            // ---- group merge.  Rows hh*P + pr of the g heads share position
            // pr; each row's list is sorted by (score desc, id asc).  The g
            // lists of a position are k-way merged in that order, skipping ids
            // already taken: an id's first occurrence carries its largest
            // listed score, so this is the union rule's top-k.  The merge runs
            // on all 128 threads: a group of g consecutive lanes per position,
            // lane hh holding the front of head hh's list; each step the group
            // finds its best front with in-group shuffles and that lane moves on.
            unsigned char* reg = gbase + kPOff + q * 32768;    // this tile's P buffers
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
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ------------------------------------------------------------------- host
}  // namespace tc

bool full_tc_supported(const KParams& p, int dtype) {
    if (dtype != HS_BF16 || p.head_dim != 128) return false;
    if (128 % p.group != 0) return false;
    if (p.mode == 0) return p.block_size == tc::kBN && p.ksel <= tc::kList;
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
    cudaError_t e = cudaFuncSetAttribute(full_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    const long long grid = (long long)a.n_ctas_q * p.batch * p.hkv;
    full_tc_kernel<<<(unsigned)grid, kThreads, kSmemBytes, st>>>(mq, mk, mv, a);
    return cudaGetLastError();
}

}  // namespace hs
