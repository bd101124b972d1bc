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
// of its positions in registers: the group max is in-thread packed FMA plus
// three-input max with the fp32 lse.  Each position keeps an exact streaming
// top-(k-w) buffer in shared memory (admission threshold = a key at or below
// the (k-w)-th best seen so far, raised by each cut of the buffer; a long scan
// starts from the rank-th best of a sample of its keys instead of from
// nothing, see token_select_kernel).
//
// What bounds it: per 128-key tile the tensor core reads its operands from
// shared memory (K 32 KB + Q^T 32 KB over the 8 MMAs) while TMA writes the
// next K tile (32 KB): 96 KB of shared-memory traffic per 512 MMA cycles,
// and the K tiles stream from L2 (every CTA of a group scans the same keys).
// So the K ring is as deep as shared memory allows next to the candidate
// buffers (two instantiations: a 3-stage ring for long scans, a 2-stage ring
// with larger buffers, hence fewer cuts, for shorter ones), and the scorers
// keep a short fast path: a tile in which no key of the thread's two
// positions reaches its threshold costs one TMEM load, the packed group max
// and one warp vote.
//
// Warps: 0 TMA (Q once, K tiles through the ring), 1 TMEM + MMA issuer (S^T
// into 4 TMEM buffers), 2..17 scorers in four sets of four (a set covers the
// 128 TMEM lanes = keys, and 2 of the 8 positions).  A set meets every second
// tile at a named barrier; its warps of quadrants 0 and 1 then cut their
// position's buffer if two more tiles could overflow it.  The sets only meet
// at the TMEM buffers, so one set's cut does not stall the others for up to 3
// tiles.  Producer and issuer waits may suspend the thread (measured ~4%
// faster than polling here).
#include "hs_common.cuh"
#include "hs_kernels.cuh"
#include "tc_ptx.cuh"

namespace hs {
namespace tsel {

using namespace tc;

constexpr int kG = 16;          // heads per group handled here
constexpr int kPos = 8;         // positions per CTA
constexpr int kKeys = 128;      // keys per K tile (= MMA M)
constexpr int kHd = 128;
constexpr int kSBufs = 4;        // S^T buffers in TMEM: the scorer sets may drift 3 tiles apart
constexpr int kCheck = 2;        // tiles between a set's cut checks
constexpr int kBitmapKeys = 65536;  // finalize by id bitmap (8 KB per position) below this
constexpr uint32_t kTmemCols = 128 * kSBufs;

// Shared-memory map of an instantiation with a kStages-deep K ring,
// candidate buffers of kCap entries per position and kPP positions per
// scorer thread (sets of four warps, one per TMEM lane quadrant).
template <int kStages, int kCap, int kPP_>
struct Cfg {
    static constexpr int kStagesN = kStages, kCapN = kCap, kPP = kPP_;
    static constexpr int kSets = kPos / kPP;      // scorer sets of four warps
    static constexpr int kScorers = 4 * kSets;    // scorer warps
    static constexpr int kThreads = 64 + 32 * kScorers;
    static_assert(kScorers >= kPos, "the finalize runs one scorer warp per position");
    // largest k - w handled: an exact cut leaves k - w entries, which must
    // leave room for the kCheck tiles of appends before the next check
    static constexpr int kMaxRanked = kCap - (kCheck + 1) * kKeys < 1024
                                          ? kCap - (kCheck + 1) * kKeys
                                          : 1024;
    static constexpr uint32_t kQOff = 0;                          // 2 x 16 KB
    static constexpr uint32_t kKOff = 32768;                      // kStages x 32 KB (finalize scratch later)
    static constexpr uint32_t kBufOff = kKOff + kStages * 32768;  // kPos x kCap x 8
    static constexpr uint32_t kHistOff = kBufOff + kPos * kCap * 8;  // kPos x 1 KB
    static constexpr uint32_t kBarOff = kHistOff + kPos * 1024;
    enum { BQ = 0, BKF = 1, BKE = BKF + kStages, BSF = BKE + kStages, BSE = BSF + kSBufs,
           BDRAIN = BSE + kSBufs, BCOUNT = BDRAIN + 1 };
    // tmem slot (4) | abort (4) | count[kPos] (32) | threshold key[kPos] (64) | rescan (4)
    static constexpr uint32_t kMiscOff = kBarOff + BCOUNT * 8;
    static constexpr uint32_t kFailOff = kMiscOff + 8 + 4 * kPos + 8 * kPos;
    static constexpr uint32_t kSmemBytes = kFailOff + 16 + 1024;
    // sampled tiles: an even count fills most of a buffer (the sampled
    // threshold is taken at a check, which falls on odd tiles)
    static constexpr int kSampleTiles = (kCap / kKeys) / kCheck * kCheck;
    static_assert(kSmemBytes <= 232448, "shared memory");
    static_assert(kStages * 32768 >= kPos * kMaxRanked * 8, "sort scratch fits in the K ring");
    static_assert(kStages * 32768 >= kPos * (kBitmapKeys / 8), "id bitmaps fit in the K ring");
    static_assert(kMaxRanked >= kKeys, "buffers hold at least one cut's worth");
};

// long scans: deeper ring; shorter scans: larger buffers (fewer cuts)
// Two positions per scorer thread (16 scorer warps): measured faster than
// four (8 warps) on both scan lengths -- the scorers' dependent chains (TMEM
// load, max tree, vote, appends) want more warps to hide their latency.
using CfgLong = Cfg<3, 1408, 2>;
using CfgShort = Cfg<2, 1920, 2>;

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

// max over 16 heads of a2 - lse2 for one key and position: raw logits r[0..16)
// (TMEM words), scale sl2, -lse2 of the heads in nl[0..16).
__device__ __forceinline__ float group_max16(const uint32_t* r, float sl2, const float* nl) {
    float v[kG];
#pragma unroll
    for (int hh = 0; hh < kG; hh += 2) {
        const float2 r2 = ffma2(make_float2(__uint_as_float(r[hh]), __uint_as_float(r[hh + 1])),
                                make_float2(sl2, sl2), make_float2(nl[hh], nl[hh + 1]));
        v[hh] = r2.x;
        v[hh + 1] = r2.y;
    }
    return fmaxf(max3f(max3f(v[0], v[1], v[2]), max3f(v[3], v[4], v[5]), max3f(v[6], v[7], v[8])),
                 max3f(max3f(v[9], v[10], v[11]), max3f(v[12], v[13], v[14]), v[15]));
}

// Key tile that pipeline step j of a sampled pass loads: the first
// kSampleTiles steps visit tiles spread evenly over 0 .. n_rt-1.
template <class C>
__device__ __forceinline__ int sample_tile(int j, int n_rt) {
    return ((2 * j + 1) * n_rt) / (2 * C::kSampleTiles);
}

// One scan of the CTA's key tiles and the finalize.  kSampled: the first
// kSampleTiles pipeline steps score sampled tiles straight into the buffers
// and set each position's threshold to the rank-th best sample; the
// finalize then flags (*s_fail) a position that saw fewer than k - w keys
// pass it.  reinit: the barriers of an earlier pass are invalidated first.
template <class C, bool kSampled>
__device__ __forceinline__ void select_pass(const CUtensorMap& tmap_q, const CUtensorMap& tmap_k,
                                            const Args& a, int rank, int n_rt, bool reinit) {
    constexpr int kStages = C::kStagesN, kCap = C::kCapN, kPP = C::kPP;
    constexpr int kSets = C::kSets, kScorers = C::kScorers;
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

    auto bar = [&](int i) { return base + C::kBarOff + 8u * i; };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gb + C::kMiscOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(gb + C::kMiscOff + 4);
    int* s_cnt = reinterpret_cast<int*>(gb + C::kMiscOff + 8);
    unsigned long long* s_th = reinterpret_cast<unsigned long long*>(gb + C::kMiscOff + 8 + 4 * kPos);
    volatile int* s_fail = reinterpret_cast<volatile int*>(gb + C::kFailOff);
    constexpr int ns = kSampled ? C::kSampleTiles : 0;  // sampled pipeline steps
    (void)s_fail;
    (void)rank;

    if (threadIdx.x == 0) {
        if (reinit)
            for (int i = 0; i < C::BCOUNT; ++i)
                asm volatile("mbarrier.inval.shared::cta.b64 [%0];" ::"r"(bar(i)) : "memory");
        mbar_init(bar(C::BQ), 1);
        for (int i = 0; i < kStages; ++i) { mbar_init(bar(C::BKF + i), 1); mbar_init(bar(C::BKE + i), 1); }
        for (int i = 0; i < kSBufs; ++i) { mbar_init(bar(C::BSF + i), 1); mbar_init(bar(C::BSE + i), kScorers); }
        mbar_init(bar(C::BDRAIN), 1);
        for (int i = 0; i < kPos; ++i) { s_cnt[i] = 0; s_th[i] = 0ull; }
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            if (!reinit) { prefetch_tmap(&tmap_q); prefetch_tmap(&tmap_k); }
            mbar_arrive_expect_tx(bar(C::BQ), 32768);
            tma_load_4d(base + C::kQOff, &tmap_q, bar(C::BQ), 0, u * kG, row0, b);
            tma_load_4d(base + C::kQOff + 16384, &tmap_q, bar(C::BQ), 64, u * kG, row0, b);
            int issued = 0;
            for (int j = 0; j < ns + nt; ++j) {
                const int st = j % kStages;
                if (j >= kStages &&
                    !mbar_wait(bar(C::BKE + st), ((j / kStages) - 1) & 1, abort_flag))
                    break;
                const uint32_t f = bar(C::BKF + st);
                mbar_arrive_expect_tx(f, 32768);
                const uint32_t kd = base + C::kKOff + st * 32768;
                const int key0 = (kSampled && j < ns ? sample_tile<C>(j, n_rt) : j - ns) * kKeys;
                tma_load_3d(kd, &tmap_k, f, 0, key0, bu);
                tma_load_3d(kd + 16384, &tmap_k, f, 64, key0, bu);
                issued = j + 1;
            }
            drain(bar(C::BQ), 0);
            for (int j = max(0, issued - kStages); j < issued; ++j)
                drain(bar(C::BKF + j % kStages), (j / kStages) & 1);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t id = idesc_bf16(kKeys, kPos * kG, false, false);
            // descriptors built once; an operand `off` bytes further is the
            // descriptor plus off >> 4 (every operand lies below 256 KB)
            const uint64_t dk0 = sw128_desc(base + C::kKOff, 16, 1024);
            const uint64_t dq = sw128_desc(base + C::kQOff, 16, 1024);
            bool ok = mbar_wait(bar(C::BQ), 0, abort_flag);
            tc_fence_after();
            for (int j = 0; ok && j < ns + nt; ++j) {
                const int st = j % kStages, s = j % kSBufs;
                if (!mbar_wait(bar(C::BKF + st), (j / kStages) & 1, abort_flag)) break;
                if (j >= kSBufs &&
                    !mbar_wait(bar(C::BSE + s), ((j / kSBufs) - 1) & 1, abort_flag))
                    break;
                tc_fence_after();
                const uint64_t dk = dk0 + (uint64_t)(st * (32768 >> 4));
                // K step kk: d columns 16kk.. = 32-byte column group kk&3 of d half kk>>2
#pragma unroll
                for (int kk = 0; kk < kHd / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                    umma_ss(tmem + 128 * s, dk + (uint64_t)(off >> 4), dq + (uint64_t)(off >> 4),
                            id, kk > 0 ? 1u : 0u);
                }
                umma_commit(bar(C::BSF + s));
                umma_commit(bar(C::BKE + st));
            }
            umma_commit(bar(C::BDRAIN));
            drain(bar(C::BDRAIN), 0);
        }
    } else {
        // ------------------------------------------------------------ scorers
        const int set = (warp - 2) >> 2;  // positions kPP*set ..
        const int quad = warp & 3;        // TMEM lane quadrant = keys 32*quad ..
        const int wid = warp - 2;         // 0 .. kScorers-1
        const uint32_t tq = tmem + ((uint32_t)(quad * 32) << 16) + set * (kPP * kG);
        const float sl2 = p.scale_log2;
        // this thread's kPP positions: -lse2 of their 16 heads, the last key
        // each may rank (t - w; -1 when it ranks nothing), and thresholds
        float nlse2[kPP][kG];
        int tpos[kPP], lim[kPP];
        bool live[kPP], all_sel[kPP];
#pragma unroll
        for (int i = 0; i < kPP; ++i) {
            const int r = row0 + set * kPP + i;
            live[i] = r < p.t_q;
            tpos[i] = p.q_offset + r;
            all_sel[i] = tpos[i] + 1 <= p.k;
            lim[i] = (live[i] && !all_sel[i] && Kc > 0) ? tpos[i] - p.window : -1;
#pragma unroll
            for (int hh = 0; hh < kG; ++hh)
                nlse2[i][hh] = live[i] ? -a.lse[((size_t)b * p.hq + u * kG + hh) * p.t_q + r] * kLog2e
                                       : 0.f;
        }
        uint64_t* bufs = reinterpret_cast<uint64_t*>(gb + C::kBufOff);
        // the position this warp cuts (quads 0..kPP-1 of a set cut)
        const bool cutter = quad < kPP;
        const int my_pos = set * kPP + (cutter ? quad : 0);
        uint32_t* hist = reinterpret_cast<uint32_t*>(gb + C::kHistOff + my_pos * 1024);
        const int bar_id = 1 + set;
        // Admission compares a key's float score with the float score of the
        // position's threshold key (thf): score >= thf admits every key that
        // beats the 64-bit threshold (and at most the few tying its score);
        // admitting more than necessary is always safe -- the cuts and the
        // finalize select exactly.
        float thf[kPP];
#pragma unroll
        for (int i = 0; i < kPP; ++i) thf[i] = -INFINITY;
        const uint32_t lt_mask = (1u << lane) - 1u;
        bool ok = true;
        // Pipeline step j scores key tile key0 (a sampled tile while sample).
        // Every warp runs every step (the set meets at named barriers); after
        // an abort the waits fail at once and the work is skipped.
        auto step = [&](const int j, const int key0, const bool sample) {
            const int s = j % kSBufs;
            bool got = ok && mbar_wait(bar(C::BSF + s), (j / kSBufs) & 1, abort_flag);
            got = __all_sync(0xffffffffu, got);
            if (!got) ok = false;
            if (got) {
                tc_fence_after();
                uint32_t r[kPP * kG];
#pragma unroll
                for (int c = 0; c < kPP * kG; c += 32)
                    tmem_ld32(tq + 128 * s + c, *reinterpret_cast<uint32_t(*)[32]>(&r[c]));
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(C::BSE + s));
                const int key = key0 + quad * 32 + lane;
                float sc[kPP];
                bool any = false;
#pragma unroll
                for (int i = 0; i < kPP; ++i) {
                    sc[i] = group_max16(&r[i * kG], sl2, nlse2[i]);
                    any |= (sc[i] >= thf[i]) & (key <= lim[i]);
                }
                if (__any_sync(0xffffffffu, any)) {
                    // appends: per position, one slot reservation for the warp
#pragma unroll
                    for (int i = 0; i < kPP; ++i) {
                        const bool cand = (sc[i] >= thf[i]) & (key <= lim[i]);
                        const uint32_t bal = __ballot_sync(0xffffffffu, cand);
                        if (bal == 0u) continue;  // warp-uniform
                        const int pos = set * kPP + i;
                        int at = 0;
                        if (lane == 0) at = atomicAdd(&s_cnt[pos], __popc(bal));
                        at = __shfl_sync(0xffffffffu, at, 0) + __popc(bal & lt_mask);
                        if (cand) {
                            if (at < kCap) bufs[(size_t)pos * kCap + at] = sel_key(sc[i], (uint32_t)key);
                            else set_status(HS_ERR_BOUNDS);  // not reached: the cuts keep room
                        }
                    }
                }
                if (!sample && a.sel) {
                    // scores of the keys selected without ranking (tests ask for them)
#pragma unroll
                    for (int i = 0; i < kPP; ++i) {
                        const int t = tpos[i];
                        if (!live[i] || key > t) continue;
                        float* srow = a.sel + (((size_t)b * p.hkv + u) * p.t_q + row0 + set * kPP + i) * p.ksel;
                        if (all_sel[i]) srow[key] = exp2f(sc[i]);
                        else if (key >= t - p.window + 1) srow[Kc + (key - (t - p.window + 1))] = exp2f(sc[i]);
                    }
                }
            }  // got
            // Every kCheck-th tile the set meets to cut the buffers that could
            // overflow within the next kCheck tiles (a tile appends at most
            // kKeys keys per position), then refreshes its thresholds.
            if (j % kCheck == kCheck - 1) {
                asm volatile("bar.sync %0, 128;" ::"r"(bar_id) : "memory");
                const int n = s_cnt[my_pos];
                if (sample) {
                    if (j == ns - 1 && cutter) {
                        // the samples are in: start from the rank-th best of
                        // them and empty the buffer (the scan proper sees
                        // them again)
                        const uint64_t th = (ok && n >= rank)
                            ? warp_kth_largest(bufs + (size_t)my_pos * kCap, n, rank, hist) : 0ull;
                        if (lane == 0) {
                            s_th[my_pos] = th ? th - 1ull : 0ull;
                            s_cnt[my_pos] = 0;
                        }
                    }
                } else if (ok && cutter && n > kCap - kCheck * kKeys) {
                    // keep at most halfway between k - w and the trigger
                    const int target = Kc + (kCap - kCheck * kKeys - Kc) / 2;
                    uint64_t th;
                    const int m = warp_cut_sampled(bufs + (size_t)my_pos * kCap, n, Kc, n - target,
                                                   hist, &th);
                    if (lane == 0) {
                        s_th[my_pos] = th > s_th[my_pos] ? th : s_th[my_pos];
                        s_cnt[my_pos] = m;
                    }
                }
                asm volatile("bar.sync %0, 128;" ::"r"(bar_id) : "memory");
                // a cut may have raised the thresholds: refresh their float
                // scores (-inf while nothing was cut, and never NaN)
#pragma unroll
                for (int i = 0; i < kPP; ++i) {
                    const uint64_t th = s_th[set * kPP + i];
                    const float x = order_float((uint32_t)(th >> 32));
                    thf[i] = (th == 0ull || x != x) ? -INFINITY : x;
                }
            }
        };
        if constexpr (kSampled)
            for (int j = 0; j < ns; ++j) step(j, sample_tile<C>(j, n_rt) * kKeys, true);
        for (int jj = 0; jj < nt; ++jj) step(jj + ns, jj * kKeys, false);
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
                int n = Kc > 0 ? min(s_cnt[pos], kCap) : 0;
                uint32_t* fhist = reinterpret_cast<uint32_t*>(gb + C::kHistOff + pos * 1024);
                // Every key above the threshold was admitted; with a sampled
                // start the k-w best are all among them only if at least k-w
                // of the buffer's keys reach it -- otherwise the CTA rescans.
                if (kSampled && warp_count_at_least(buf, n, s_th[pos]) < Kc && lane == 0)
                    *s_fail = 1;
                if (n > Kc) { warp_cut_to_k(buf, n, Kc, fhist); n = Kc; }
                __syncwarp();
                if (!srow && t < kBitmapKeys) {
                    // ascending ids without sorting: mark the winners in a bitmap
                    // over 0..t, then read the set bits out in word order
                    uint32_t* bm = reinterpret_cast<uint32_t*>(gb + C::kKOff) + (size_t)wid * (kBitmapKeys / 32);
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
                    uint64_t* sb = reinterpret_cast<uint64_t*>(gb + C::kKOff) + (size_t)wid * C::kMaxRanked;
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
    __syncthreads();  // the pass is done: every wait, load and MMA has drained
    tc_fence_after();
}

// One CTA = kPos positions of one (batch, KV group).  A scan whose ranked
// range is long enough starts from a sampled threshold: kSampleTiles key
// tiles spread evenly over the n_rt tiles that every position of the CTA
// ranks are scored first, and the rank-th best of each position's samples
// becomes its admission threshold (a few thousand admissions and a few cuts
// per position instead of ~2 (k-w) ln(T/(k-w))).  If the finalize finds a
// position for which fewer than k-w keys reach it, the CTA scans again
// without one.
template <class C>
__global__ void __launch_bounds__(C::kThreads, 1)
    token_select_kernel(const __grid_constant__ CUtensorMap tmap_q,
                        const __grid_constant__ CUtensorMap tmap_k, Args a) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char* gb = smem_raw + (base - raw);
    const int warp = threadIdx.x >> 5;
    const KParams& p = a.p;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gb + C::kMiscOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(gb + C::kMiscOff + 4);
    volatile int* s_fail = reinterpret_cast<volatile int*>(gb + C::kFailOff);
    if (threadIdx.x == 0) { *abort_flag = 0; *s_fail = 0; }
    if (warp == 1) {
        tmem_alloc(base + C::kMiscOff, kTmemCols);
        tmem_relinquish();
    }
    const int Kc = p.k - p.window;
    const int row0 = (a.n_ptiles - 1 - (int)(blockIdx.x / (p.batch * p.hkv))) * kPos;
    const int n_rt = (p.q_offset + row0 - p.window + 1) / kKeys;  // tiles every position ranks
    const int rank = (Kc > 0 && n_rt >= 8 * C::kSampleTiles)
                         ? sample_rank(Kc, C::kSampleTiles * kKeys, (long long)n_rt * kKeys)
                         : 0;
    bool plain = true;
    if (rank > 0) {
        select_pass<C, true>(tmap_q, tmap_k, a, rank, n_rt, false);
        plain = *s_fail != 0 && *abort_flag == 0;  // read after the pass's barrier
    }
    if (plain) select_pass<C, false>(tmap_q, tmap_k, a, 0, n_rt, rank > 0);

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(*tmem_slot, kTmemCols);
    }
}

// Key tiles one CTA scans for the latest of its positions, and the scan
// length from which the deeper K ring pays off over fewer buffer cuts.
constexpr int kLongScanTiles = 2048;  // 262144 keys

}  // namespace tsel

bool token_select_tc_supported(const KParams& p, int dtype) {
    return dtype == HS_BF16 && p.head_dim == 128 && p.mode == 1 && p.group == tsel::kG &&
           p.k - p.window <= tsel::CfgShort::kMaxRanked;
}

template <class C>
static cudaError_t launch_tsel(const CUtensorMap& mq, const CUtensorMap& mk, const tsel::Args& a,
                               long long grid, cudaStream_t st) {
    cudaError_t e = cudaFuncSetAttribute(tsel::token_select_kernel<C>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::kSmemBytes);
    if (e != cudaSuccess) return e;
    tsel::token_select_kernel<C><<<(unsigned)grid, C::kThreads, C::kSmemBytes, st>>>(mq, mk, a);
    return cudaGetLastError();
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
    const long long grid = (long long)a.n_ptiles * p.batch * p.hkv;
    const long long scan = ((long long)p.q_offset + p.t_q + kKeys - 1) / kKeys;
    // the deeper ring's smaller buffers need headroom above k - w for their cuts
    if (scan >= kLongScanTiles && p.k - p.window <= CfgLong::kCapN - 4 * kKeys)
        return launch_tsel<CfgLong>(mq, mk, a, grid, st);
    return launch_tsel<CfgShort>(mq, mk, a, grid, st);
}

}  // namespace hs
