// flash_tc.cuh -- the tcgen05 flash-attention pipeline shared by the full
// layer (full_tc.cu) and the row-grouped sparse layer (sparse_tc.cu).
//
// A CTA runs two 128-row Q tiles over a list of 64-key tiles that both share.
// Warp 0 is the TMA producer (K and V through rings of their own), warp 1
// owns TMEM, warps 2..9 are two softmax
// warpgroups with one thread per row, and one thread per Q tile (warp 1 for
// tile 0, warp 10 for tile 1) issues that tile's MMAs:
//   S = Q K^T  (M = 128, N = 64, K = 16 x 8) into one of two TMEM buffers,
//   O += P V   (N = 128, V as the MN-major operand; P from TMEM).
// The softmax writes P (bf16 pairs) back over the first 32 columns of the S
// buffer it read, and the PV MMA takes its A operand from there: P never
// touches shared memory, whose bandwidth the operand reads of the S MMAs
// (Q 4 KB + K 2 KB per 32-cycle MMA) and the TMA writes already saturate.
// An S buffer needs no release of its own: the MMAs of one issuer execute in
// issue order, so S of tile j + 2 (same buffer) follows PV of tile j, which
// waited for that tile's P.
// The kernels differ in which key tiles they visit, which keys a row keeps,
// and what they do besides attention (block-score capture, union building).
#pragma once

#include "hs_common.cuh"
#include "tc_ptx.cuh"

namespace hs {
namespace fl {

using namespace tc;

// Shared-memory map and mbarrier indices of a pipeline with a KS-stage K ring,
// a VS-stage V ring and `Extra` kernel-specific bytes after the P buffers.
// K and V have rings of their own: a K stage is free as soon as the S MMAs
// that read it are done, so K loads run ahead of V loads, which wait for PV.
template <int KS, int VS, uint32_t Extra>
struct Layout {
    static constexpr int kBM = 128, kNQ = 2, kBN = 64, kD = 128, kKS = KS, kVS = VS;
    static constexpr int kIssuer1Warp = 2 + 4 * kNQ;               // issuer of Q tile 1
    static constexpr int kThreads = 64 + 128 * kNQ + 32 * (kNQ - 1);
    static constexpr uint32_t kQOff = 0;                       // kNQ x 32 KB (two d halves)
    static constexpr uint32_t kKOff = kNQ * 32768;             // KS x 16 KB
    static constexpr uint32_t kVOff = kKOff + KS * 16384;      // VS x 16 KB
    static constexpr uint32_t kPOff = kVOff + VS * 16384;      // kNQ x 2 x 16 KB
    static constexpr uint32_t kExtraOff = kPOff + kNQ * 2 * 16384;
    static constexpr uint32_t kBarOff = kExtraOff + Extra;
    enum {
        BQ = 0,
        BKF = 1,          // K stage full / empty
        BKE = BKF + KS,
        BVF = BKE + KS,   // V stage full / empty
        BVE = BVF + VS,
        BSF = BVE + VS,   // [q][s]
        BSE = BSF + 2 * kNQ,
        BPF = BSE + 2 * kNQ,
        BPVD = BPF + 2 * kNQ,
        BOF = BPVD + 2 * kNQ,   // [q]: O of Q tile q is final
        BDRAIN = BOF + kNQ,     // [q]: issuer q's MMAs are done
        BCOUNT = BDRAIN + kNQ
    };
    static constexpr uint32_t kMiscOff = kBarOff + BCOUNT * 8;  // tmem slot, abort flag, ...
    static constexpr uint32_t kTmemCols = 256 * kNQ;            // per Q tile: S0 | S1 | O
    // every operand lies below 256 KB, so a descriptor's 14-bit addr >> 4 field never wraps
    static_assert(kMiscOff + 1024 <= 232448, "shared memory");
    static_assert(kNQ == 2, "one issuer warp per Q tile: warps 1 and 2 + 4 kNQ");
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

template <class L>
__device__ __forceinline__ void init_barriers(uint32_t bar0) {
    auto bar = [&](int i) { return bar0 + 8u * i; };
    mbar_init(bar(L::BQ), 1);
    // a K (V) stage is free once both issuers' S (PV) MMAs that read it are done
    for (int i = 0; i < L::kKS; ++i) { mbar_init(bar(L::BKF + i), 1); mbar_init(bar(L::BKE + i), L::kNQ); }
    for (int i = 0; i < L::kVS; ++i) { mbar_init(bar(L::BVF + i), 1); mbar_init(bar(L::BVE + i), L::kNQ); }
    for (int i = 0; i < 2 * L::kNQ; ++i) {
        mbar_init(bar(L::BSF + i), 1);
        mbar_init(bar(L::BSE + i), 4);
        mbar_init(bar(L::BPF + i), 4);
        mbar_init(bar(L::BPVD + i), 1);
    }
    for (int q = 0; q < L::kNQ; ++q) { mbar_init(bar(L::BOF + q), 1); mbar_init(bar(L::BDRAIN + q), 1); }
}

// TMA producer (one thread): both Q tiles once (4-D boxes: 64 d x P positions
// x g heads), then K and V of the key tiles key0_of(j), j < nt, in the order
// the MMAs need them: K(j) before V(j-1), since S of tile j is issued before
// PV of tile j-1.
template <class L, class KeyOf>
__device__ __forceinline__ void producer(uint32_t base, const CUtensorMap* tq, const CUtensorMap* tk,
                                         const CUtensorMap* tv, int row0, int P, int head0, int b,
                                         int bu, int nt, KeyOf key0_of, volatile int* abort) {
    auto bar = [&](int i) { return base + L::kBarOff + 8u * i; };
    prefetch_tmap(tq);
    prefetch_tmap(tk);
    prefetch_tmap(tv);
    mbar_arrive_expect_tx(bar(L::BQ), L::kNQ * 32768);
#pragma unroll
    for (int q = 0; q < L::kNQ; ++q) {
        tma_load_4d(base + L::kQOff + q * 32768, tq, bar(L::BQ), 0, row0 + q * P, head0, b);
        tma_load_4d(base + L::kQOff + q * 32768 + 16384, tq, bar(L::BQ), 64, row0 + q * P, head0, b);
    }
    int k_issued = 0, v_issued = 0, key_next = nt > 0 ? key0_of(0) : 0, key_prev = 0;
    for (int j = 0; j <= nt; ++j) {
        if (j < nt) {
            const int st = j % L::kKS;
            if (j >= L::kKS && !mbar_wait(bar(L::BKE + st), ((j / L::kKS) - 1) & 1, abort, false))
                break;
            const uint32_t f = bar(L::BKF + st), kd = base + L::kKOff + st * 16384;
            mbar_arrive_expect_tx(f, 16384);
            tma_load_3d(kd, tk, f, 0, key_next, bu);
            tma_load_3d(kd + 8192, tk, f, 64, key_next, bu);
            k_issued = j + 1;
        }
        if (j >= 1) {
            const int jj = j - 1, st = jj % L::kVS;
            if (jj >= L::kVS && !mbar_wait(bar(L::BVE + st), ((jj / L::kVS) - 1) & 1, abort, false))
                break;
            const uint32_t f = bar(L::BVF + st), vd = base + L::kVOff + st * 16384;
            mbar_arrive_expect_tx(f, 16384);
            tma_load_3d(vd, tv, f, 0, key_prev, bu);
            tma_load_3d(vd + 8192, tv, f, 64, key_prev, bu);
            v_issued = j;
        }
        key_prev = key_next;
        if (j + 1 < nt) key_next = key0_of(j + 1);
    }
    // every issued load must have landed before the CTA may exit
    mbar_drain(bar(L::BQ), 0);
    for (int j = max(0, k_issued - L::kKS); j < k_issued; ++j)
        mbar_drain(bar(L::BKF + j % L::kKS), (j / L::kKS) & 1);
    for (int j = max(0, v_issued - L::kVS); j < v_issued; ++j)
        mbar_drain(bar(L::BVF + j % L::kVS), (j / L::kVS) & 1);
}

// MMA issuer of Q tile q (one thread): iteration j issues S = Q K^T of tile j
// (after its S buffer is free) and releases tile j's K stage, then issues
// O += P V of tile j-1 (after its P is ready) and releases tile j-1's V stage.
// The Q tile uses ntq of the CTA's nt tiles; for the rest it still waits for
// each stage to fill before releasing it, so its release of a stage can never
// count towards a later use of that stage than the other issuer's.
// One thread's instruction stream bounds the MMA rate, hence one issuer per Q
// tile and shared-memory descriptors built once: a descriptor holds its start
// address as addr >> 4 in its low 14 bits, and every operand of the CTA lies
// below 256 KB, so moving an operand by `off` bytes adds off >> 4.
template <class L>
__device__ __forceinline__ void mma_issuer(uint32_t base, uint32_t tmem, int q, int nt, int ntq,
                                           volatile int* abort) {
    auto bar = [&](int i) { return base + L::kBarOff + 8u * i; };
    const uint32_t id_s = idesc_bf16(L::kBM, L::kBN, false, false);
    const uint32_t id_o = idesc_bf16(L::kBM, L::kD, false, true);
    const uint64_t dq = sw128_desc(base + L::kQOff + q * 32768, 16, 1024);
    const uint64_t dk0 = sw128_desc(base + L::kKOff, 16, 1024);
    const uint64_t dv0 = sw128_desc(base + L::kVOff, 8192, 1024);  // V: MN-major, d halves 8 KB apart
    const uint32_t ts = tmem + q * 256, to = tmem + q * 256 + 128;
    bool ok = mbar_wait(bar(L::BQ), 0, abort, false);
    tc_fence_after();
    for (int j = 0; ok && j <= nt; ++j) {
        if (j < nt) {
            const int st = j % L::kKS, s = j & 1;
            if (!mbar_wait(bar(L::BKF + st), (j / L::kKS) & 1, abort, false)) break;
            if (j < ntq) {
                tc_fence_after();
                const uint64_t dk = dk0 + (uint64_t)(st * (16384 >> 4));
                // K step kk: d columns 16kk.. = 32-byte column group kk&3 of d half kk>>2
#pragma unroll
                for (int kk = 0; kk < L::kD / 16; ++kk)
                    umma_ss(ts + 64 * s, dq + (uint64_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4),
                            dk + (uint64_t)(((kk >> 2) * 8192 + (kk & 3) * 32) >> 4), id_s,
                            kk > 0 ? 1u : 0u);
                umma_commit(bar(L::BSF + 2 * q + s));
            }
            umma_commit(bar(L::BKE + st));
        }
        if (j >= 1) {
            const int jj = j - 1, sp = jj & 1, stp = jj % L::kVS;
            if (!mbar_wait(bar(L::BVF + stp), (jj / L::kVS) & 1, abort, false)) break;
            if (jj < ntq) {
                if (!mbar_wait(bar(L::BPF + 2 * q + sp), (jj >> 1) & 1, abort, false)) break;
                tc_fence_after();
                const uint32_t tp = ts + 64 * sp;  // P: columns 0..31 of S buffer sp
                const uint64_t dv = dv0 + (uint64_t)(stp * (16384 >> 4));
                // K step kk: keys 16kk.. = P columns 8kk.. (two keys per column),
                // V rows 16kk..
#pragma unroll
                for (int kk = 0; kk < L::kBN / 16; ++kk)
                    umma_ts(to, tp + 8 * kk, dv + (uint64_t)((kk * 2048) >> 4), id_o,
                            (jj > 0 || kk > 0) ? 1u : 0u);
                umma_commit(bar(L::BPVD + 2 * q + sp));
            }
            umma_commit(bar(L::BVE + stp));
        }
    }
    umma_commit(bar(L::BOF + q));
    umma_commit(bar(L::BDRAIN + q));
    mbar_drain(bar(L::BDRAIN + q), 0);
}

// One 64-key tile of one row: raw logits r[] (TMEM), keep columns first..lim
// (the rest -> -inf), tile max mt (log2 domain, -inf if nothing kept), lazy
// rescale (the reference max m_ref moves only when the tile exceeds it by
// more than 2^8; *corr is then the factor for l and O, and the return value
// says whether O holds anything to rescale), p = 2^(x*scale_log2 - m_ref)
// with packed FMA, row sum into l, and P packed to bf16 pairs.
// kPolyEvery > 0: every kPolyEvery-th pair of exponentials runs on the FMA
// pipe (exp2_poly2) instead of the MUFU unit, whose throughput otherwise
// bounds the tile.  That path returns 2^-125 rather than 0 below 2^-125, e.g.
// for masked keys; kZero selects an exact 0 there, for callers whose rows may
// keep no key at all (whose l must then stay exactly 0).
template <int kPolyEvery = 0, bool kZero = false>
__device__ __forceinline__ bool softmax_tile(const uint32_t (&r)[64], int first, int lim, float sl2,
                                             float& m_ref, float& l, float& mt, float& corr,
                                             uint32_t (&pk)[32]) {
    float x[64];
#pragma unroll
    for (int c = 0; c < 64; ++c) x[c] = __uint_as_float(r[c]);
    if (lim < 63 || first > 0) {
#pragma unroll
        for (int c = 0; c < 64; ++c) x[c] = (c <= lim && c >= first) ? x[c] : -INFINITY;
    }
    float m3[22];
#pragma unroll
    for (int c = 0; c < 21; ++c) m3[c] = max3f(x[3 * c], x[3 * c + 1], x[3 * c + 2]);
    m3[21] = x[63];
#pragma unroll
    for (int c = 0; c < 7; ++c) m3[c] = max3f(m3[3 * c], m3[3 * c + 1], m3[3 * c + 2]);
    mt = max3f(max3f(m3[0], m3[1], m3[2]), max3f(m3[3], m3[4], m3[5]), fmaxf(m3[6], m3[21])) *
         sl2;  // -inf stays -inf (sl2 > 0)
    bool resc = false;
    corr = 1.f;
    if (mt > m_ref + 8.f) {
        corr = ex2(m_ref - mt);  // 0 while nothing was kept
        resc = m_ref > -INFINITY;
        m_ref = mt;
        l *= corr;
    }
    const float mu = m_ref == -INFINITY ? 0.f : m_ref;
    const float2 s2 = make_float2(sl2, sl2), n2 = make_float2(-mu, -mu);
    float e[64];
    float2 acc[8];
#pragma unroll
    for (int c2 = 0; c2 < 32; ++c2) {
        const float2 y = ffma2(make_float2(x[2 * c2], x[2 * c2 + 1]), s2, n2);
        if (kPolyEvery > 0 && c2 % (kPolyEvery > 0 ? kPolyEvery : 1) == kPolyEvery - 1) {
            const float2 ev = exp2_poly2(y);
            e[2 * c2] = (!kZero || y.x >= -125.f) ? ev.x : 0.f;
            e[2 * c2 + 1] = (!kZero || y.y >= -125.f) ? ev.y : 0.f;
        } else {
            e[2 * c2] = ex2(y.x);
            e[2 * c2 + 1] = ex2(y.y);
        }
        const float2 ev = make_float2(e[2 * c2], e[2 * c2 + 1]);
        acc[c2 & 7] = c2 < 8 ? ev : fadd2(acc[c2 & 7], ev);
    }
#pragma unroll
    for (int w = 4; w >= 1; w >>= 1)
#pragma unroll
        for (int c = 0; c < w; ++c) acc[c] = fadd2(acc[c], acc[c + w]);
    l += acc[0].x + acc[0].y;
#pragma unroll
    for (int c = 0; c < 32; ++c) pk[c] = pack_bf16(e[2 * c], e[2 * c + 1]);
    return resc;
}

// The same tile without the tile maximum, for callers that do not need it
// (no block-score capture): p = 2^(x*scale_log2 - m_ref) against the current
// reference directly.  The reference lags by design, so p may exceed 1; when
// the tile's sum stays below 2^8 every p of the tile is below 2^8 (the lazy
// rescale's own bound) and nothing else is needed.  Otherwise (a logit far
// above the reference, or inf/nan from one far enough above it) the tile
// takes its maximum, rescales l (and asks the caller to rescale O) and
// recomputes.  The first tile of a row (m_ref = -inf) starts from its
// maximum; it must keep at least one key (key 0 is in every row's first tile
// of the full layer).  Saves the 31 three-input max instructions of the
// maximum on all but the rare tiles that move the reference.
template <int kPolyEvery = 0>
__device__ __forceinline__ void exp_tile(const float (&x)[64], float sl2, float m_ref,
                                         float (&e)[64], float& sum) {
    const float2 s2 = make_float2(sl2, sl2), n2 = make_float2(-m_ref, -m_ref);
    float2 acc[8];
#pragma unroll
    for (int c2 = 0; c2 < 32; ++c2) {
        const float2 y = ffma2(make_float2(x[2 * c2], x[2 * c2 + 1]), s2, n2);
        if (kPolyEvery > 0 && c2 % (kPolyEvery > 0 ? kPolyEvery : 1) == kPolyEvery - 1) {
            const float2 ev = exp2_poly2(y);
            e[2 * c2] = ev.x;
            e[2 * c2 + 1] = ev.y;
        } else {
            e[2 * c2] = ex2(y.x);
            e[2 * c2 + 1] = ex2(y.y);
        }
        const float2 ev = make_float2(e[2 * c2], e[2 * c2 + 1]);
        acc[c2 & 7] = c2 < 8 ? ev : fadd2(acc[c2 & 7], ev);
    }
#pragma unroll
    for (int w = 4; w >= 1; w >>= 1)
#pragma unroll
        for (int c = 0; c < w; ++c) acc[c] = fadd2(acc[c], acc[c + w]);
    sum = acc[0].x + acc[0].y;
}

__device__ __forceinline__ float tile_max64(const float (&x)[64]) {
    float m3[22];
#pragma unroll
    for (int c = 0; c < 21; ++c) m3[c] = max3f(x[3 * c], x[3 * c + 1], x[3 * c + 2]);
    m3[21] = x[63];
#pragma unroll
    for (int c = 0; c < 7; ++c) m3[c] = max3f(m3[3 * c], m3[3 * c + 1], m3[3 * c + 2]);
    return max3f(max3f(m3[0], m3[1], m3[2]), max3f(m3[3], m3[4], m3[5]), fmaxf(m3[6], m3[21]));
}

template <int kPolyEvery = 0>
__device__ __forceinline__ bool softmax_tile_lazy(const uint32_t (&r)[64], int lim, float sl2,
                                                  float& m_ref, float& l, float& corr,
                                                  uint32_t (&pk)[32]) {
    float x[64];
#pragma unroll
    for (int c = 0; c < 64; ++c) x[c] = __uint_as_float(r[c]);
    if (lim < 63) {
#pragma unroll
        for (int c = 0; c < 64; ++c) x[c] = c <= lim ? x[c] : -INFINITY;
    }
    corr = 1.f;
    bool resc = false;
    if (m_ref == -INFINITY) m_ref = tile_max64(x) * sl2;  // first tile: O is still empty
    float e[64], lt;
    exp_tile<kPolyEvery>(x, sl2, m_ref, e, lt);
    if (!(lt < 256.f)) {
        const float mt = tile_max64(x) * sl2;  // > m_ref + 2: some p >= 4
        corr = ex2(m_ref - mt);
        resc = true;
        m_ref = mt;
        l *= corr;
        exp_tile<kPolyEvery>(x, sl2, m_ref, e, lt);
    }
    l += lt;
#pragma unroll
    for (int c = 0; c < 32; ++c) pk[c] = pack_bf16(e[2 * c], e[2 * c + 1]);
    return resc;
}

// P row (64 keys as 32 bf16 pairs) over the first 32 columns of the TMEM S
// buffer at trow_s (every lane of the warp calls this; the caller then
// fences and signals the MMA issuer).
__device__ __forceinline__ void store_p_tmem(uint32_t trow_s, const uint32_t (&pk)[32]) {
    tmem_st32(trow_s, pk);
    tmem_wait_st();
}

// P row (64 keys, bf16) into the 128B-swizzled P buffer, made visible to the
// tensor core's operand reads.
__device__ __forceinline__ void store_p(unsigned char* pbuf, int row, const uint32_t (&pk)[32]) {
    unsigned char* prow = pbuf + row * 128;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const uint4 v4 = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        *reinterpret_cast<uint4*>(prow + ((c ^ (row & 7)) << 4)) = v4;
    }
    fence_proxy_async_smem();
}

// O row *= cf in TMEM (every lane of the warp calls this).
__device__ __forceinline__ void rescale_o(uint32_t trow_o, float cf) {
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4) {
        uint32_t ro[32];
        tmem_ld32(trow_o + 32 * c4, ro);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c) ro[c] = __float_as_uint(__uint_as_float(ro[c]) * cf);
        tmem_st32(trow_o + 32 * c4, ro);
    }
    tmem_wait_st();
}

// O row * inv -> og[0..128) as bf16 (every lane of the warp calls this; only
// lanes with store = true write; have_o = false writes zeros).
__device__ __forceinline__ void store_o(uint32_t trow_o, bool have_o, float inv, bool store,
                                        __nv_bfloat16* og) {
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4) {
        uint32_t ro[32];
        if (have_o) {
            tmem_ld32(trow_o + 32 * c4, ro);
            tmem_wait_ld();
        } else {
#pragma unroll
            for (int c = 0; c < 32; ++c) ro[c] = 0u;
        }
        if (store) {
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
}

}  // namespace fl
}  // namespace hs
