// token_select_wide.cu -- HySparse2 token-level selection for long scans:
// 16 positions per work item, S^T with N = 256, candidate buffers in a
// caller workspace.
//
// Same scores and selection rule as token_select_tc.cu (the token score
// S_bar_{t,i} = 2^(max_h (a2_{h,t,i} - lse2_{h,t})) of "HySparse 混合稀疏注意力
// （一）" with B = 1 and the GQA group max; the last w keys forced in and the
// k - w best of 0..t-w ranked, "HySparse2 ..." 4.2).  What changes is the
// shape, for scans of 2^18 keys and more (a 1M-token prefix):
//
//   S^T = K_tile * Q^T   (M = 128 keys, N = 16 positions x 16 heads, K = d)
//
// At N = 128 the tensor core's shared-memory operand reads (K and Q^T) plus
// the TMA writes of the next K tile come to 96 KB per 512 MMA cycles, more
// than shared memory delivers; at N = 256 they are 128 KB per 1024 cycles,
// and every K tile fetched from L2 serves twice the positions.  Q^T then
// takes 64 KB and 16 positions' candidate buffers no longer fit beside a
// 3-stage K ring, so they live in the workspace (global memory, L2-resident):
// over a long scan admissions are rare -- each work item starts from a
// threshold taken from a sample of its keys (below), so a position admits a
// few thousand of its T keys and its 2048-entry buffer is cut a few times.
//
// The grid is persistent (one CTA per SM at most): CTA c handles work items
// c, c + gridDim.x, ... (an item = 16 positions of one (batch, kv group),
// latest positions first) and owns workspace slot c.  TMEM (2 S^T buffers of
// 256 columns) is allocated once; the mbarriers are re-initialised per item.
//
// The lse is folded into the contraction: a ninth K step multiplies a ones
// column of the keys with -lse2/scale of each (position, head) row, split
// into three bf16 terms (hi + mid + lo, 24 significant bits), so TMEM holds
// a2/scale - lse2/scale and a key's group score is scale * (a max over 16
// TMEM words): no per-value FMA, no lse in registers.  One more MMA per tile
// (+12.5%) buys a scorer fast path of two TMEM loads, 4 x 16-way max and
// four compares per thread and tile.
//
// Warps: 0 TMA (Q^T of the item once, K tiles through the ring), 1 TMEM +
// MMA issuer, 2..17 scorers in four sets of four (a set covers the 128 keys
// of a tile and 4 of the 16 positions; a thread owns one key and its 64
// values).  A set meets every second tile;
// each of its warps then cuts its own position's buffer if two more tiles
// could overflow it.  Finalize: the exact top-(k-w) of each buffer, sorted
// by id in shared memory (the Q and K regions are free by then), then the
// window.
#include <algorithm>

#include "hs_common.cuh"
#include "hs_kernels.cuh"
#include "tc_ptx.cuh"

namespace hs {
namespace tsw {

using namespace tc;

constexpr int kG = 16;           // heads per group
constexpr int kPos = 16;         // positions per item
constexpr int kN = kPos * kG;    // MMA N
constexpr int kKeys = 128;       // keys per K tile (= MMA M)
constexpr int kHd = 128;
constexpr int kPP = 4;           // positions per scorer thread
constexpr int kSets = kPos / kPP;
constexpr int kScorers = 4 * kSets;  // 16
constexpr int kThreads = 64 + 32 * kScorers;
constexpr int kStages = 3;
constexpr int kSBufs = 2;
constexpr int kCheck = 2;
constexpr int kCap = 2048;       // workspace entries per position
constexpr int kMaxRanked = 1024;
constexpr int kSampleTiles = kCap / kKeys;  // sampled tiles fill a buffer exactly
constexpr int kMinSampleTiles = 64;         // ranked range worth sampling
constexpr uint32_t kTmemCols = kN * kSBufs;  // 512

constexpr uint32_t kQOff = 0;                          // 2 d halves x 32 KB
constexpr uint32_t kKOff = 65536;                      // kStages x 32 KB
// the ninth K step's operands (128B-swizzled rows of 128 bytes): column group
// 0 of rows 0..255 = the split -lse2/scale of each (position, head) row of
// Q^T, column group 1 of rows 0..127 = ones for every key
constexpr uint32_t kXOff = kKOff + kStages * 32768;    // 32 KB
constexpr uint32_t kHistOff = kXOff + kN * 128;        // kPos x 1 KB
constexpr uint32_t kBarOff = kHistOff + kPos * 1024;
enum { BQ = 0, BKF = 1, BKE = BKF + kStages, BSF = BKE + kStages, BSE = BSF + kSBufs,
       BDRAIN = BSE + kSBufs, BCOUNT = BDRAIN + 1 };
// tmem slot (4) | abort (4) | count[kPos] (64) | threshold key[kPos] (128) |
// admission threshold / scale [kPos] (64, 16-byte aligned) | rescan (4)
constexpr uint32_t kMiscOff = kBarOff + BCOUNT * 8;
constexpr uint32_t kThrOff = (kMiscOff + 8 + 4 * kPos + 8 * kPos + 15) & ~15u;
constexpr uint32_t kFailOff = kThrOff + 4 * kPos;
constexpr uint32_t kSmemBytes = kFailOff + 16 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory");
static_assert(kKOff + kStages * 32768 >= (uint32_t)kPos * kMaxRanked * 8,
              "finalize sort scratch fits in the Q and K regions");
static_assert(kXOff % 1024 == 0, "swizzled operand alignment");
static_assert(kPP == 4, "thresholds are reloaded as one float4 per set");
static_assert(kCap - kCheck * kKeys > kMaxRanked + kKeys, "cut headroom");

constexpr size_t kSlotBytes = (size_t)kPos * kCap * 8;  // workspace per CTA

struct Args {
    KParams p;
    const float* lse;
    int32_t* idx;
    int32_t* cnt;
    float* sel;
    uint64_t* ws;      // gridDim.x slots of kPos x kCap keys
    int n_ptiles;
    int n_items;
};

__device__ __forceinline__ void drain(uint32_t bar, uint32_t parity) {
    const long long t0 = clock64();
    while (!mbar_try_wait_sleep(bar, parity)) {
        if (clock64() - t0 > kWaitCycles) { set_status(HS_ERR_TIMEOUT); return; }
    }
}

__device__ __forceinline__ void mbar_inval(uint32_t bar) {
    asm volatile("mbarrier.inval.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

// Key tile that pipeline step j of a sampled scan loads: the first
// kSampleTiles steps visit tiles spread evenly over 0 .. n_rt-1.
__device__ __forceinline__ int sample_tile(int j, int n_rt) {
    return ((2 * j + 1) * n_rt) / (2 * kSampleTiles);
}

// One scan of work item `it` and its finalize.  kSampled: the first
// kSampleTiles pipeline steps score sampled tiles straight into the buffers
// and set each position's threshold to the rank-th best sample; the
// finalize then flags (*s_fail = it + 1) a position that saw fewer than
// k - w keys reach it.  first: the CTA's first scan (no barriers to invalidate yet).
template <bool kSampled>
__device__ __forceinline__ void scan_item(const CUtensorMap& tmap_q, const CUtensorMap& tmap_k,
                                          const Args& a, int it, int rank, int n_rt, bool first) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char* gb = smem_raw + (base - raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const KParams& p = a.p;
    const int Kc = p.k - p.window;
    const int bu_n = p.batch * p.hkv;

    auto bar = [&](int i) { return base + kBarOff + 8u * i; };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gb + kMiscOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(gb + kMiscOff + 4);
    int* s_cnt = reinterpret_cast<int*>(gb + kMiscOff + 8);
    unsigned long long* s_th = reinterpret_cast<unsigned long long*>(gb + kMiscOff + 8 + 4 * kPos);
    float* s_thr = reinterpret_cast<float*>(gb + kThrOff);
    volatile int* s_fail = reinterpret_cast<volatile int*>(gb + kFailOff);
    uint64_t* slot = a.ws + (size_t)blockIdx.x * kPos * kCap;
    constexpr int ns = kSampled ? kSampleTiles : 0;  // sampled pipeline steps
    (void)s_fail;
    (void)rank;

    const int pt = a.n_ptiles - 1 - it / bu_n;  // latest positions first
    const int bu = it % bu_n;
    const int b = bu / p.hkv, u = bu % p.hkv;
    const int row0 = pt * kPos;
    const int last_row = min(p.t_q, row0 + kPos) - 1;
    const int nt = min((p.t_kv + kKeys - 1) / kKeys, (p.q_offset + last_row) / kKeys + 1);

    // ---- set-up of the item (the previous one has fully drained)
    if (threadIdx.x == 0) {
        if (!first)
            for (int i = 0; i < BCOUNT; ++i) mbar_inval(bar(i));
        mbar_init(bar(BQ), 1);
        for (int i = 0; i < kStages; ++i) { mbar_init(bar(BKF + i), 1); mbar_init(bar(BKE + i), 1); }
        for (int i = 0; i < kSBufs; ++i) { mbar_init(bar(BSF + i), 1); mbar_init(bar(BSE + i), kScorers); }
        mbar_init(bar(BDRAIN), 1);
        for (int i = 0; i < kPos; ++i) { s_cnt[i] = 0; s_th[i] = 0ull; s_thr[i] = -INFINITY; }
        fence_mbar_init();
    }
    for (int x = (int)threadIdx.x; x < kN; x += kThreads) {
        // row x of Q^T = (position x / 16, head x % 16): -lse2 / scale as
        // hi + mid + lo in bf16 (logical chunk 0: columns 0..2)
        const int pos = x / kG, hh = x % kG, r = row0 + pos;
        const float v = r < p.t_q
            ? -a.lse[((size_t)b * p.hq + u * kG + hh) * p.t_q + r] * kLog2e / p.scale_log2
            : 0.f;
        const __nv_bfloat16 hi = __float2bfloat16_rn(v);
        const float r1 = v - __bfloat162float(hi);
        const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
        const __nv_bfloat16 lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
        const uint32_t w0 = (uint32_t)__bfloat16_as_ushort(hi) |
                            ((uint32_t)__bfloat16_as_ushort(mid) << 16);
        const uint32_t w1 = (uint32_t)__bfloat16_as_ushort(lo);
        *reinterpret_cast<uint4*>(gb + kXOff + x * 128 + ((0 ^ (x & 7)) << 4)) =
            make_uint4(w0, w1, 0u, 0u);
    }
    fence_proxy_async_smem();  // visible to the tensor core's operand reads
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (*abort_flag) return;  // a wait of an earlier scan gave up

    if (warp == 0) {
        if (lane == 0) {
            if (first) { prefetch_tmap(&tmap_q); prefetch_tmap(&tmap_k); }
            mbar_arrive_expect_tx(bar(BQ), 65536);
            tma_load_4d(base + kQOff, &tmap_q, bar(BQ), 0, u * kG, row0, b);
            tma_load_4d(base + kQOff + 32768, &tmap_q, bar(BQ), 64, u * kG, row0, b);
            int issued = 0;
            for (int j = 0; j < ns + nt; ++j) {
                const int st = j % kStages;
                if (j >= kStages &&
                    !mbar_wait(bar(BKE + st), ((j / kStages) - 1) & 1, abort_flag, false))
                    break;
                const uint32_t f = bar(BKF + st);
                mbar_arrive_expect_tx(f, 32768);
                const uint32_t kd = base + kKOff + st * 32768;
                const int key0 = (kSampled && j < ns ? sample_tile(j, n_rt) : j - ns) * kKeys;
                tma_load_3d(kd, &tmap_k, f, 0, key0, bu);
                tma_load_3d(kd + 16384, &tmap_k, f, 64, key0, bu);
                issued = j + 1;
            }
            drain(bar(BQ), 0);
            for (int j = max(0, issued - kStages); j < issued; ++j)
                drain(bar(BKF + j % kStages), (j / kStages) & 1);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t id = idesc_bf16(kKeys, kN, false, false);
            const uint64_t dk0 = sw128_desc(base + kKOff, 16, 1024);
            const uint64_t dq = sw128_desc(base + kQOff, 16, 1024);
            const uint64_t dx = sw128_desc(base + kXOff, 16, 1024);
            bool ok = mbar_wait(bar(BQ), 0, abort_flag, false);
            tc_fence_after();
            for (int j = 0; ok && j < ns + nt; ++j) {
                const int st = j % kStages, s = j % kSBufs;
                if (!mbar_wait(bar(BKF + st), (j / kStages) & 1, abort_flag, false)) break;
                if (j >= kSBufs &&
                    !mbar_wait(bar(BSE + s), ((j / kSBufs) - 1) & 1, abort_flag, false))
                    break;
                tc_fence_after();
                const uint64_t dk = dk0 + (uint64_t)(st * (32768 >> 4));
                // K step kk: d columns 16kk.. = 32-byte column group kk&3 of d
                // half kk>>2 (K halves 16 KB apart, Q^T halves 32 KB apart)
#pragma unroll
                for (int kk = 0; kk < kHd / 16; ++kk)
                    umma_ss(tmem + kN * s,
                            dk + (uint64_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4),
                            dq + (uint64_t)(((kk >> 2) * 32768 + (kk & 3) * 32) >> 4), id,
                            kk > 0 ? 1u : 0u);
                // ninth step: ones (group 1) x -lse2/scale (group 0)
                umma_ss(tmem + kN * s, dx + (uint64_t)(32 >> 4), dx, id, 1u);
                umma_commit(bar(BSF + s));
                umma_commit(bar(BKE + st));
            }
            umma_commit(bar(BDRAIN));
            drain(bar(BDRAIN), 0);
        }
    } else {
        // -------------------------------------------------------- scorers
        const int set = (warp - 2) >> 2;  // positions kPP*set ..
        const int quad = warp & 3;        // TMEM lane quadrant = keys 32*quad ..
        const int wid = warp - 2;
        const uint32_t tq = tmem + ((uint32_t)(quad * 32) << 16) + set * (kPP * kG);
        const float sl2 = p.scale_log2;
        int tpos[kPP], lim[kPP];
        bool live[kPP], all_sel[kPP];
#pragma unroll
        for (int i = 0; i < kPP; ++i) {
            const int r = row0 + set * kPP + i;
            live[i] = r < p.t_q;
            tpos[i] = p.q_offset + r;
            all_sel[i] = tpos[i] + 1 <= p.k;
            lim[i] = (live[i] && !all_sel[i] && Kc > 0) ? tpos[i] - p.window : -1;
        }
        const int my_pos = set * kPP + quad;  // the position this warp cuts
        uint64_t* my_buf = slot + (size_t)my_pos * kCap;
        uint32_t* hist = reinterpret_cast<uint32_t*>(gb + kHistOff + my_pos * 1024);
        const int bar_id = 1 + set;
        // Admission compares a key's raw group maximum m = max_h (a2 - lse2)
        // / scale with thr, the threshold key's score / scale nudged down by
        // 2^-20 of its size: score = scale * m >= the threshold's score
        // implies m >= thr, so every key that beats the 64-bit threshold
        // (and at most a few near-ties) is admitted; admitting more than
        // necessary is always safe -- the cuts and the finalize are exact.
        float thr[kPP];
#pragma unroll
        for (int i = 0; i < kPP; ++i) thr[i] = -INFINITY;
        const uint32_t lt_mask = (1u << lane) - 1u;
        bool ok = true;
        // pipeline step j scores key tile key0 (a sampled tile while sample)
        auto step = [&](const int j, const int key0, const bool sample) {
            const int s = j % kSBufs;
            bool got = ok && mbar_wait(bar(BSF + s), (j / kSBufs) & 1, abort_flag);
            got = __all_sync(0xffffffffu, got);
            if (!got) ok = false;
            if (got) {
                tc_fence_after();
                uint32_t r[kPP * kG];
                tmem_ld32(tq + kN * s, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
                tmem_ld32(tq + kN * s + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(BSE + s));
                const int key = key0 + quad * 32 + lane;
                float m[kPP];
                uint32_t cmask = 0u;  // positions with this key as a candidate
#pragma unroll
                for (int i = 0; i < kPP; ++i) {
                    const float* v = reinterpret_cast<const float*>(&r[i * kG]);
                    m[i] = fmaxf(max3f(max3f(v[0], v[1], v[2]), max3f(v[3], v[4], v[5]),
                                       max3f(v[6], v[7], v[8])),
                                 max3f(max3f(v[9], v[10], v[11]), max3f(v[12], v[13], v[14]),
                                       v[15]));
                    cmask |= ((m[i] >= thr[i]) & (key <= lim[i])) ? (1u << i) : 0u;
                }
                uint32_t wmask = __reduce_or_sync(0xffffffffu, cmask);
                while (wmask) {  // warp-uniform: the positions with candidates
                    const int i = __ffs(wmask) - 1;
                    wmask &= wmask - 1u;
                    const bool cand = (cmask >> i) & 1u;
                    const uint32_t bal = __ballot_sync(0xffffffffu, cand);
                    const int pos = set * kPP + i;
                    int at = 0;
                    if (lane == 0) at = atomicAdd(&s_cnt[pos], __popc(bal));
                    at = __shfl_sync(0xffffffffu, at, 0) + __popc(bal & lt_mask);
                    if (cand) {
                        float mi = m[0];
#pragma unroll
                        for (int x = 1; x < kPP; ++x) mi = x == i ? m[x] : mi;
                        if (at < kCap) slot[(size_t)pos * kCap + at] = sel_key(mi * sl2, (uint32_t)key);
                        else set_status(HS_ERR_BOUNDS);  // not reached: the cuts keep room
                    }
                }
                if (!sample && a.sel) {
                    // scores of the keys selected without ranking (tests ask for them)
#pragma unroll
                    for (int i = 0; i < kPP; ++i) {
                        const int t = tpos[i];
                        if (!live[i] || key > t) continue;
                        float* srow = a.sel + (((size_t)b * p.hkv + u) * p.t_q + row0 + set * kPP + i) * p.ksel;
                        if (all_sel[i]) srow[key] = exp2f(m[i] * sl2);
                        else if (key >= t - p.window + 1)
                            srow[Kc + (key - (t - p.window + 1))] = exp2f(m[i] * sl2);
                    }
                }
            }  // got
            if (j % kCheck == kCheck - 1) {
                asm volatile("bar.sync %0, 128;" ::"r"(bar_id) : "memory");
                const int n = min(s_cnt[my_pos], kCap);
                if (sample) {
                    if (j == ns - 1) {
                        // the samples are in: start from the rank-th best
                        // of them and empty the buffer (the scan proper
                        // sees them again)
                        const uint64_t th =
                            (ok && n >= rank) ? warp_kth_largest(my_buf, n, rank, hist) : 0ull;
                        if (lane == 0) {
                            s_th[my_pos] = th ? th - 1ull : 0ull;
                            s_cnt[my_pos] = 0;
                            const float x = order_float((uint32_t)(th >> 32)) / sl2;
                            s_thr[my_pos] =
                                (th == 0ull || x != x) ? -INFINITY : x - fabsf(x) * 0x1p-20f;
                        }
                    }
                } else if (ok && n > kCap - kCheck * kKeys) {
                    const int target = Kc + (kCap - kCheck * kKeys - Kc) / 2;
                    uint64_t th;
                    const int mm = warp_cut_sampled(my_buf, n, Kc, n - target, hist, &th);
                    if (lane == 0) {
                        const uint64_t t2 = th > s_th[my_pos] ? th : s_th[my_pos];
                        s_th[my_pos] = t2;
                        s_cnt[my_pos] = mm;
                        const float x = order_float((uint32_t)(t2 >> 32)) / sl2;
                        s_thr[my_pos] = (t2 == 0ull || x != x) ? -INFINITY : x - fabsf(x) * 0x1p-20f;
                    }
                }
                asm volatile("bar.sync %0, 128;" ::"r"(bar_id) : "memory");
                const float4 t4 = *reinterpret_cast<const float4*>(s_thr + set * kPP);
                thr[0] = t4.x; thr[1] = t4.y; thr[2] = t4.z; thr[3] = t4.w;
            }
        };
        if constexpr (kSampled)
            for (int j = 0; j < ns; ++j) step(j, sample_tile(j, n_rt) * kKeys, true);
        for (int jj = 0; jj < nt; ++jj) step(jj + ns, jj * kKeys, false);
        // ---- finalize: one warp per position; the Q and K regions are free
        asm volatile("bar.sync %0, %1;" ::"r"(1 + kSets), "r"(32 * kScorers) : "memory");
        const int pos = wid;
        const int r = row0 + pos;
        if (ok && r < p.t_q) {
            const int t = p.q_offset + r;
            const size_t orow = ((size_t)b * p.hkv + u) * p.t_q + r;
            int32_t* irow = a.idx + orow * p.ksel;
            float* srow = a.sel ? a.sel + orow * p.ksel : nullptr;
            int n_out;
            if (t + 1 <= p.k) {
                n_out = t + 1;
                for (int x = lane; x < n_out; x += 32) irow[x] = x;
            } else {
                uint64_t* buf = slot + (size_t)pos * kCap;
                int n = Kc > 0 ? min(s_cnt[pos], kCap) : 0;
                uint32_t* fhist = reinterpret_cast<uint32_t*>(gb + kHistOff + pos * 1024);
                // Every key above the threshold was admitted; with a
                // sampled start the k-w best are all among them only if
                // at least k-w of the buffer's keys reach it -- otherwise
                // the item is scanned again.
                if (kSampled && warp_count_at_least(buf, n, s_th[pos]) < Kc && lane == 0)
                    *s_fail = it + 1;  // tagged with the item: never stale
                if (n > Kc) { warp_cut_to_k(buf, n, Kc, fhist); n = Kc; }
                __syncwarp();
                const int sort_n = next_pow2(Kc > 0 ? Kc : 1);
                uint64_t* sb = reinterpret_cast<uint64_t*>(gb + kQOff) + (size_t)wid * kMaxRanked;
                for (int x = lane; x < sort_n; x += 32)
                    sb[x] = x < n ? (((uint64_t)sel_key_id(buf[x]) << 32) | (buf[x] >> 32)) : ~0ull;
                __syncwarp();
                warp_bitonic_sort(sb, sort_n);
                for (int x = lane; x < n; x += 32) {
                    irow[x] = (int32_t)(sb[x] >> 32);
                    if (srow) srow[x] = exp2f(order_float((uint32_t)(sb[x] & 0xffffffffu)));
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
    __syncthreads();  // the scan is done: every wait, load and MMA has drained
    tc_fence_after();
}

// Persistent: CTA c scans work items c, c + gridDim.x, ...  An item whose
// ranked range is long enough starts from a sampled threshold: kSampleTiles
// key tiles spread evenly over the n_rt tiles that every position of the
// item ranks are scored first, and the rank-th best of each position's
// samples becomes its admission threshold, so the scan admits a few thousand
// keys per position instead of ~(k-w) ln(T/(k-w)) times two.  If the
// finalize finds a position for which fewer than k-w keys reach it, the item
// is scanned again without one.
__global__ void __launch_bounds__(kThreads, 1)
    token_select_wide_kernel(const __grid_constant__ CUtensorMap tmap_q,
                             const __grid_constant__ CUtensorMap tmap_k, Args a) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char* gb = smem_raw + (base - raw);
    const int warp = threadIdx.x >> 5;
    const KParams& p = a.p;
    const int Kc = p.k - p.window;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gb + kMiscOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(gb + kMiscOff + 4);
    volatile int* s_fail = reinterpret_cast<volatile int*>(gb + kFailOff);

    if (warp == 1) {
        tmem_alloc(base + kMiscOff, kTmemCols);
        tmem_relinquish();
    }
    if (threadIdx.x == 0) { *abort_flag = 0; *s_fail = 0; }
    // zero the extra operand buffer once, then the ones column of the keys
    // (logical 16-byte chunk 2 of rows 0..127: columns 16..18 = 1.0)
    for (int x = (int)threadIdx.x; x < kN * 8; x += kThreads)
        *reinterpret_cast<uint4*>(gb + kXOff + x * 16) = make_uint4(0u, 0u, 0u, 0u);
    __syncthreads();
    for (int r = (int)threadIdx.x; r < kKeys; r += kThreads) {
        const uint32_t one = 0x3f80u;  // bf16 1.0
        *reinterpret_cast<uint4*>(gb + kXOff + r * 128 + ((2 ^ (r & 7)) << 4)) =
            make_uint4(one | (one << 16), one, 0u, 0u);
    }

    bool first = true;
    for (int it = blockIdx.x; it < a.n_items && !*abort_flag; it += gridDim.x) {
        const int row0 = (a.n_ptiles - 1 - it / (p.batch * p.hkv)) * kPos;
        const int n_rt = (p.q_offset + row0 - p.window + 1) / kKeys;  // tiles every position ranks
        const int rank = (Kc > 0 && n_rt >= kMinSampleTiles)
                             ? sample_rank(Kc, kSampleTiles * kKeys, (long long)n_rt * kKeys)
                             : 0;
        bool plain = true;
        if (rank > 0) {
            scan_item<true>(tmap_q, tmap_k, a, it, rank, n_rt, first);
            first = false;
            plain = *s_fail == it + 1 && *abort_flag == 0;  // read after the scan's barrier
        }
        if (plain) {
            scan_item<false>(tmap_q, tmap_k, a, it, 0, n_rt, first);
            first = false;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(*tmem_slot, kTmemCols);
    }
}

// Scans of at least this many key tiles take the wide selector.
constexpr int kMinScanTiles = 2048;  // 262144 keys

}  // namespace tsw

static int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return n;
}

bool token_select_wide_applies(const KParams& p, int dtype) {
    const long long scan = ((long long)p.q_offset + p.t_q + tsw::kKeys - 1) / tsw::kKeys;
    return dtype == HS_BF16 && p.head_dim == 128 && p.mode == 1 && p.group == tsw::kG &&
           p.k - p.window <= tsw::kMaxRanked && scan >= tsw::kMinScanTiles;
}

size_t token_select_wide_workspace(const KParams& p) {
    const long long items = (long long)((p.t_q + tsw::kPos - 1) / tsw::kPos) * p.batch * p.hkv;
    const long long grid = std::min<long long>(items, sm_count());
    return (size_t)grid * tsw::kSlotBytes;
}

cudaError_t launch_token_select_wide(const KParams& p, const void* q, const void* k,
                                     const float* lse, int32_t* idx, int32_t* cnt, float* sel,
                                     void* ws, size_t ws_bytes, cudaStream_t st) {
    using namespace tsw;
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
    a.ws = static_cast<uint64_t*>(ws);
    a.n_ptiles = (p.t_q + kPos - 1) / kPos;
    a.n_items = a.n_ptiles * p.batch * p.hkv;
    // one CTA per workspace slot, at most one per SM
    const long long slots = (long long)(ws_bytes / kSlotBytes);
    const long long grid = std::min<long long>(std::min<long long>(a.n_items, slots),
                                               std::max(1, sm_count()));
    if (grid < 1) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(tsw::token_select_wide_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, tsw::kSmemBytes);
    if (e != cudaSuccess) return e;
    tsw::token_select_wide_kernel<<<(unsigned)grid, tsw::kThreads, tsw::kSmemBytes, st>>>(mq, mk, a);
    return cudaGetLastError();
}

}  // namespace hs
