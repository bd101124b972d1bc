// token_select_tc.cu -- HySparse2 token-level selection on the tensor cores.
//
// For a query at position t and KV group u the token score of key i is
//     S_bar_{t,i} = max_{h in u} p_{h,t,i} = 2^( max_h (a2_{h,t,i} - lse2_{h,t}) )
// (block score of "HySparse 混合稀疏注意力（一）" with B = 1; group max from
// "GQA 下为什么要组内共享索引"), and the index set is the most recent w keys
// plus the k - w best keys of 0..t-w ("HySparse2 ..." 4.2, forced window).
// lse comes from the attention pass.  This pass recomputes the logits:
//
//     S^T = K_tile * Q^T      (M = 128 keys, N = 8 positions x 16 heads, K = d)
//
// with Q's rows position-major (one 4-D TMA box with the head and position
// strides swapped), so a thread owns one key and holds all 16 heads of each
// of its positions in registers: the group max is in-thread FFMA + FMNMX with
// the fp32 lse.  Each position keeps an exact streaming top-(k-w) buffer in
// shared memory (admission threshold = the k-w-th best key after each cut).
//
// Warps: 0 TMA (Q once, K tiles of 128 keys through a 2-stage ring), 1 TMEM +
// MMA issuer (S^T in 4 TMEM buffers), 2..17 scorers in four sets of four (each
// set covers the 128 TMEM lanes = keys, and 2 of the 8 positions).  The sets
// only meet at the TMEM buffers, so one set's buffer cut does not stall the
// others for up to 3 tiles.  The scorers' dependent chains (TMEM load, FMA,
// max, ballot, shared atomics) are latency-bound, so the work is spread over
// 16 warps with 2 positions per thread rather than 8 warps with 4.
#include "hs_common.cuh"
#include "hs_kernels.cuh"
#include "tc_ptx.cuh"

namespace hs {
namespace tsel {

using namespace tc;

constexpr int kG = 16;          // heads per group handled here
constexpr int kPos = 8;         // positions per CTA
constexpr int kKeys = 128;      // keys per K tile (= MMA M)
constexpr int kPP = 2;          // positions per scorer thread
constexpr int kSets = kPos / kPP;          // scorer sets of four warps
constexpr int kScorers = 4 * kSets;        // scorer warps
constexpr int kHd = 128;
constexpr int kStages = 2;       // K ring (the MMA is far ahead of the scorers)
constexpr int kSBufs = 4;        // S^T buffers in TMEM: the scorer sets may drift 3 tiles apart
constexpr int kThreads = 64 + 32 * kScorers;
constexpr int kMaxRanked = 1024;            // k - w handled here
// Per-position buffer entries: the k - w kept, two tiles of admissions
// between cut checks, and 5 tiles' worth of headroom (what shared memory holds).
constexpr int kCap = kMaxRanked + 7 * kKeys;
constexpr int kBitmapKeys = 65536;  // finalize by id bitmap (8 KB per position) below this
// a cut at n > kCap - 2 kKeys must leave room for two more tiles
static_assert((kCap - 2 * kKeys - kMaxRanked) / 2 >= 2 * kKeys, "cut headroom");

constexpr uint32_t kQOff = 0;                         // 2 x 16 KB
constexpr uint32_t kKOff = 32768;                     // kStages x 32 KB (sort scratch later)
constexpr uint32_t kBufOff = kKOff + kStages * 32768; // kPos x kCap x 8
constexpr uint32_t kHistOff = kBufOff + kPos * kCap * 8;   // kPos positions x 1 KB
constexpr uint32_t kBarOff = kHistOff + 8 * 1024;
enum { BQ = 0, BKF = 1, BKE = BKF + kStages, BSF = BKE + kStages, BSE = BSF + kSBufs,
       BDRAIN = BSE + kSBufs, BCOUNT = BDRAIN + 1 };
constexpr uint32_t kMiscOff = kBarOff + BCOUNT * 8;  // tmem(4) abort(4) cnt[8](32) thresh[8](64)
constexpr uint32_t kSmemBytes = kMiscOff + 8 + 32 + 64 + 1024;
constexpr uint32_t kTmemCols = 128 * kSBufs;
static_assert(kStages * 32768 >= 8 * kMaxRanked * 8, "sort scratch fits in the K ring");
static_assert(kStages * 32768 >= 8 * (kBitmapKeys / 8), "id bitmaps fit in the K ring");
static_assert(kSmemBytes <= 232448, "shared memory");

struct Args {
    KParams p;
    const float* lse;  // [b][hq][t_q] natural log, from the attention pass
    int32_t* idx;
    int32_t* cnt;
    float* sel;
    int n_ptiles;      // position tiles per (b, u)
};

__device__ __forceinline__ void drain(uint32_t bar, uint32_t parity) {
    const long long t0 = clock64();
    while (!mbar_try_wait_sleep(bar, parity)) {
        if (clock64() - t0 > kWaitCycles) { set_status(HS_ERR_TIMEOUT); return; }
    }
}

__global__ void __launch_bounds__(kThreads, 1)
    token_select_kernel(const __grid_constant__ CUtensorMap tmap_q,
                        const __grid_constant__ CUtensorMap tmap_k, Args a) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char* gb = smem_raw + (base - raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const KParams& p = a.p;

    const int bu_n = p.batch * p.hkv;
    const int pt = a.n_ptiles - 1 - (int)(blockIdx.x / bu_n);  // latest positions first
    const int bu = (int)(blockIdx.x % bu_n);
    const int b = bu / p.hkv, u = bu % p.hkv;
    const int row0 = pt * kPos;
    const int last_row = min(p.t_q, row0 + kPos) - 1;
    const int pos_max = p.q_offset + last_row;
    const int nt = min((p.t_kv + kKeys - 1) / kKeys, pos_max / kKeys + 1);
    const int Kc = p.k - p.window;

    auto bar = [&](int i) { return base + kBarOff + 8u * i; };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gb + kMiscOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(gb + kMiscOff + 4);
    int* s_cnt = reinterpret_cast<int*>(gb + kMiscOff + 8);
    unsigned long long* s_th = reinterpret_cast<unsigned long long*>(gb + kMiscOff + 40);

    if (threadIdx.x == 0) {
        mbar_init(bar(BQ), 1);
        for (int i = 0; i < kStages; ++i) { mbar_init(bar(BKF + i), 1); mbar_init(bar(BKE + i), 1); }
        for (int i = 0; i < kSBufs; ++i) { mbar_init(bar(BSF + i), 1); mbar_init(bar(BSE + i), kScorers); }
        mbar_init(bar(BDRAIN), 1);
        *abort_flag = 0;
        for (int i = 0; i < kPos; ++i) { s_cnt[i] = 0; s_th[i] = 0ull; }
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
        if (lane == 0) {
            prefetch_tmap(&tmap_q);
            prefetch_tmap(&tmap_k);
            mbar_arrive_expect_tx(bar(BQ), 32768);
            tma_load_4d(base + kQOff, &tmap_q, bar(BQ), 0, u * kG, row0, b);
            tma_load_4d(base + kQOff + 16384, &tmap_q, bar(BQ), 64, u * kG, row0, b);
            int issued = 0;
            for (int j = 0; j < nt; ++j) {
                const int st = j % kStages;
                if (j >= kStages && !mbar_wait(bar(BKE + st), ((j / kStages) - 1) & 1, abort_flag)) break;
                const uint32_t f = bar(BKF + st);
                mbar_arrive_expect_tx(f, 32768);
                const uint32_t kd = base + kKOff + st * 32768;
                tma_load_3d(kd, &tmap_k, f, 0, j * kKeys, bu);
                tma_load_3d(kd + 16384, &tmap_k, f, 64, j * kKeys, bu);
                issued = j + 1;
            }
            drain(bar(BQ), 0);
            for (int j = max(0, issued - kStages); j < issued; ++j)
                drain(bar(BKF + j % kStages), (j / kStages) & 1);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t id = idesc_bf16(kKeys, kPos * kG, false, false);
            bool ok = mbar_wait(bar(BQ), 0, abort_flag);
            tc_fence_after();
            for (int j = 0; ok && j < nt; ++j) {
                const int st = j % kStages, s = j % kSBufs;
                if (!mbar_wait(bar(BKF + st), (j / kStages) & 1, abort_flag)) break;
                if (j >= kSBufs && !mbar_wait(bar(BSE + s), ((j / kSBufs) - 1) & 1, abort_flag))
                    break;
                tc_fence_after();
                const uint32_t kb = base + kKOff + st * 32768;
#pragma unroll
                for (int kk = 0; kk < kHd / 16; ++kk) {
                    const uint64_t ad = sw128_desc(kb + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
                    const uint64_t bd = sw128_desc(base + kQOff + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
                    umma_ss(tmem + 128 * s, ad, bd, id, kk > 0 ? 1u : 0u);
                }
                umma_commit(bar(BSF + s));
                umma_commit(bar(BKE + st));
            }
            umma_commit(bar(BDRAIN));
            drain(bar(BDRAIN), 0);
        }
    } else {
        // ------------------------------------------------------------ scorers
        const int set = (warp - 2) >> 2;  // positions kPP*set ..
        const int quad = warp & 3;        // TMEM lane quadrant = keys 32*quad ..
        const int wid = warp - 2;         // 0 .. kScorers-1
        const uint32_t tq = tmem + ((uint32_t)(quad * 32) << 16) + set * (kPP * kG);
        const float sl2 = p.scale_log2;
        // this thread's kPP positions: lse (log2 domain) of their 16 heads
        float nlse2[kPP][kG];  // -lse2
        int tpos[kPP];
        bool live[kPP], all_sel[kPP];
#pragma unroll
        for (int i = 0; i < kPP; ++i) {
            const int r = row0 + set * kPP + i;
            live[i] = r < p.t_q;
            tpos[i] = p.q_offset + r;
            all_sel[i] = tpos[i] + 1 <= p.k;
#pragma unroll
            for (int hh = 0; hh < kG; ++hh)
                nlse2[i][hh] = live[i] ? -a.lse[((size_t)b * p.hq + u * kG + hh) * p.t_q + r] * kLog2e
                                       : 0.f;
        }
        uint64_t* bufs = reinterpret_cast<uint64_t*>(gb + kBufOff);
        // scratch of the position this warp cuts (quads 0..kPP-1 of a set cut)
        uint32_t* hist = reinterpret_cast<uint32_t*>(
            gb + kHistOff + (set * kPP + (quad < kPP ? quad : 0)) * 1024);
        const int bar_id = 1 + set;
        // Admission compares a key's float score with the float score of the
        // position's threshold key (thf, in registers): score >= thf admits
        // every key that beats the 64-bit threshold (and at most the few that
        // tie its score), and admitting more than necessary is always safe --
        // the cuts and the finalize select exactly.  Bulk tiles (the thread's
        // positions live, none selecting everything, no scores to write, the
        // tile entirely below the first position's window, hence below every
        // window of the set and visible to all) need nothing else.
        bool bulk_ok = Kc > 0 && a.sel == nullptr;
#pragma unroll
        for (int i = 0; i < kPP; ++i) bulk_ok = bulk_ok && live[i] && !all_sel[i];
        const int lo_first = tpos[0] - p.window + 1;
        float thf[kPP];
#pragma unroll
        for (int i = 0; i < kPP; ++i) thf[i] = -INFINITY;
        bool ok = true;
        // Every warp runs every iteration (the set meets at named barriers);
        // after an abort the waits fail at once and the work is skipped.
        for (int j = 0; j < nt; ++j) {
            const int s = j % kSBufs;
            bool got = ok && mbar_wait(bar(BSF + s), (j / kSBufs) & 1, abort_flag);
            got = __all_sync(0xffffffffu, got);
            if (!got) ok = false;
            if (got) {
            tc_fence_after();
            uint32_t r0[32];
            tmem_ld32(tq + 128 * s, r0);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(BSE + s));
            const int key = j * kKeys + quad * 32 + lane;
            const bool bulk = bulk_ok && (j + 1) * kKeys <= lo_first;  // warp-uniform
            float sc[kPP];
            uint32_t bal[kPP];
#pragma unroll
            for (int i = 0; i < kPP; ++i) {
                const uint32_t* rr = r0;
                const int c0 = i * kG;
                // a2 - lse2 of the 16 heads (packed FMA), then their max (3-input max)
                float v[kG];
#pragma unroll
                for (int hh = 0; hh < kG; hh += 2) {
                    const float2 r2 = ffma2(make_float2(__uint_as_float(rr[c0 + hh]),
                                                        __uint_as_float(rr[c0 + hh + 1])),
                                            make_float2(sl2, sl2),
                                            make_float2(nlse2[i][hh], nlse2[i][hh + 1]));
                    v[hh] = r2.x;
                    v[hh + 1] = r2.y;
                }
                sc[i] = fmaxf(max3f(max3f(v[0], v[1], v[2]), max3f(v[3], v[4], v[5]),
                                    max3f(v[6], v[7], v[8])),
                              max3f(max3f(v[9], v[10], v[11]), max3f(v[12], v[13], v[14]), v[15]));
                if (bulk) {
                    bal[i] = __ballot_sync(0xffffffffu, sc[i] >= thf[i]);
                    continue;
                }
                const int t = tpos[i];
                const bool visible = live[i] && key <= t;
                const int pos = set * kPP + i;
                const size_t orow = ((size_t)b * p.hkv + u) * p.t_q + row0 + pos;
                float* srow = a.sel ? a.sel + orow * p.ksel : nullptr;
                // Every lane reaches the ballot below: no per-lane early exit.
                const int lo = t - p.window + 1;
                bool cand = false;
                if (all_sel[i]) {
                    if (visible && srow) srow[key] = exp2f(sc[i]);
                } else if (visible && key >= lo) {
                    if (srow) srow[Kc + (key - lo)] = exp2f(sc[i]);
                } else {
                    cand = visible && Kc > 0 && key < lo && sc[i] >= thf[i];
                }
                bal[i] = __ballot_sync(0xffffffffu, cand);
            }
            // lanes 0..kPP-1 reserve the slots of the thread's positions at once
            uint32_t my_bal = bal[0];
#pragma unroll
            for (int i = 1; i < kPP; ++i) my_bal = lane == i ? bal[i] : my_bal;
            int my_base = 0;
            if (lane < kPP && my_bal != 0u) my_base = atomicAdd(&s_cnt[set * kPP + lane], __popc(my_bal));
#pragma unroll
            for (int i = 0; i < kPP; ++i) {
                if (!bal[i]) continue;  // warp-uniform
                const int bi = __shfl_sync(0xffffffffu, my_base, i);
                if ((bal[i] >> lane) & 1u)
                    bufs[(size_t)(set * kPP + i) * kCap + bi + __popc(bal[i] & ((1u << lane) - 1))] =
                        sel_key(sc[i], (uint32_t)key);
            }
            }  // got
            // Every second tile the set meets to cut the buffers that could
            // overflow within the next two tiles (a tile appends at most kKeys
            // keys per position; a cut frees at least kCutFree slots or leaves
            // Kc), then refreshes its thresholds.
            if (j & 1) {
                asm volatile("bar.sync %0, 128;" ::"r"(bar_id) : "memory");
                if (ok && quad < kPP) {
                    const int pos = set * kPP + quad;
                    const int n = s_cnt[pos];
                    if (n > kCap - 2 * kKeys) {
                        uint64_t th;
                        const int m = warp_cut_sampled(bufs + (size_t)pos * kCap, n, Kc,
                                                       (kCap - 2 * kKeys - Kc) / 2, hist, &th);
                        if (lane == 0) {
                            s_th[pos] = th > s_th[pos] ? th : s_th[pos];
                            s_cnt[pos] = m;
                        }
                    }
                }
                asm volatile("bar.sync %0, 128;" ::"r"(bar_id) : "memory");
                // a cut may have raised the thresholds: refresh their float scores
                // (-inf while nothing was cut, and never NaN)
#pragma unroll
                for (int i = 0; i < kPP; ++i) {
                    const uint64_t th = s_th[set * kPP + i];
                    const float x = order_float((uint32_t)(th >> 32));
                    thf[i] = (th == 0ull || x != x) ? -INFINITY : x;
                }
            }
        }
        // ---- finalize: one warp per position (K stages are free: all MMAs done)
        asm volatile("bar.sync %0, %1;" ::"r"(1 + kSets), "r"(32 * kScorers) : "memory");
        const int pos = wid;
        const int r = row0 + pos;
        if (ok && wid < kPos && r < p.t_q) {
            const int t = p.q_offset + r;
            const size_t orow = ((size_t)b * p.hkv + u) * p.t_q + r;
            int32_t* irow = a.idx + orow * p.ksel;
            float* srow = a.sel ? a.sel + orow * p.ksel : nullptr;
            int n_out;
            if (t + 1 <= p.k) {
                n_out = t + 1;
                for (int x = lane; x < n_out; x += 32) irow[x] = x;
            } else {
                uint64_t* buf = bufs + (size_t)pos * kCap;
                int n = Kc > 0 ? s_cnt[pos] : 0;
                uint32_t* fhist = reinterpret_cast<uint32_t*>(gb + kHistOff + pos * 1024);
                if (n > Kc) { warp_cut_to_k(buf, n, Kc, fhist); n = Kc; }
                __syncwarp();
                if (!srow && t < kBitmapKeys) {
                    // ascending ids without sorting: mark the winners in a bitmap
                    // over 0..t, then read the set bits out in word order
                    uint32_t* bm = reinterpret_cast<uint32_t*>(gb + kKOff) + (size_t)wid * (kBitmapKeys / 32);
                    const int words = (t >> 5) + 1;
                    const int per = (words + 31) >> 5;  // words per lane, consecutive
                    for (int x = lane; x < per * 32; x += 32) bm[x] = 0u;
                    __syncwarp();
                    for (int x = lane; x < n; x += 32) {
                        const uint32_t id = sel_key_id(buf[x]);
                        atomicOr(&bm[id >> 5], 1u << (id & 31));
                    }
                    __syncwarp();
                    int cnt_l = 0;
                    for (int x = 0; x < per; ++x) cnt_l += __popc(bm[lane * per + x]);
                    int incl = cnt_l;
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const int y = __shfl_up_sync(0xffffffffu, incl, o);
                        if (lane >= o) incl += y;
                    }
                    int at = incl - cnt_l;
                    for (int x = 0; x < per; ++x) {
                        const int wi = lane * per + x;
                        uint32_t m = bm[wi];
                        while (m) {
                            const int bit = __ffs(m) - 1;
                            irow[at++] = wi * 32 + bit;
                            m &= m - 1u;
                        }
                    }
                } else {
                    const int sort_n = next_pow2(Kc > 0 ? Kc : 1);
                    uint64_t* sb = reinterpret_cast<uint64_t*>(gb + kKOff) + (size_t)wid * kMaxRanked;
                    for (int x = lane; x < sort_n; x += 32)
                        sb[x] = x < n ? (((uint64_t)sel_key_id(buf[x]) << 32) | (buf[x] >> 32)) : ~0ull;
                    __syncwarp();
                    warp_bitonic_sort(sb, sort_n);
                    for (int x = lane; x < n; x += 32) {
                        irow[x] = (int32_t)(sb[x] >> 32);
                        if (srow) srow[x] = exp2f(order_float((uint32_t)(sb[x] & 0xffffffffu)));
                    }
                }
                const int lo = t - p.window + 1;
                for (int x = lane; x <= t - lo; x += 32) irow[n + x] = lo + x;
                n_out = n + (t - lo + 1);
            }
            for (int x = n_out + lane; x < p.ksel; x += 32) {
                irow[x] = -1;
                if (srow) srow[x] = 0.f;
            }
            if (lane == 0) a.cnt[orow] = n_out;
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

}  // namespace tsel

bool token_select_tc_supported(const KParams& p, int dtype) {
    return dtype == HS_BF16 && p.head_dim == 128 && p.mode == 1 && p.group == tsel::kG &&
           p.k - p.window <= tsel::kMaxRanked;
}

cudaError_t launch_token_select_tc(const KParams& p, const void* q, const void* k,
                                   const float* lse, int32_t* idx, int32_t* cnt, float* sel,
                                   cudaStream_t st) {
    using namespace tsel;
    CUtensorMap mq, mk;
    // Q viewed as [b][t_q][hq][d] through strides: position-major rows in smem
    const cuuint64_t qd[4] = {(cuuint64_t)kHd, (cuuint64_t)p.hq, (cuuint64_t)p.t_q,
                              (cuuint64_t)p.batch};
    const cuuint64_t qs[3] = {(cuuint64_t)p.t_q * kHd * 2, (cuuint64_t)kHd * 2,
                              (cuuint64_t)p.hq * p.t_q * kHd * 2};
    const cuuint32_t qb[4] = {64, (cuuint32_t)kG, (cuuint32_t)kPos, 1};
    const cuuint64_t kdims[3] = {(cuuint64_t)kHd, (cuuint64_t)p.t_kv, (cuuint64_t)p.hkv * p.batch};
    const cuuint64_t ks[2] = {(cuuint64_t)kHd * 2, (cuuint64_t)p.t_kv * kHd * 2};
    const cuuint32_t kb[3] = {64, (cuuint32_t)kKeys, 1};
    if (!tc::encode(&mq, q, 4, qd, qs, qb) || !tc::encode(&mk, k, 3, kdims, ks, kb))
        return cudaErrorInvalidValue;
    Args a;
    a.p = p;
    a.lse = lse;
    a.idx = idx;
    a.cnt = cnt;
    a.sel = sel;
    a.n_ptiles = (p.t_q + kPos - 1) / kPos;
    cudaError_t e = cudaFuncSetAttribute(
        token_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, tsel::kSmemBytes);
    if (e != cudaSuccess) return e;
    const long long grid = (long long)a.n_ptiles * p.batch * p.hkv;
    token_select_kernel<<<(unsigned)grid, tsel::kThreads, tsel::kSmemBytes, st>>>(mq, mk, a);
    return cudaGetLastError();
}

}  // namespace hs
