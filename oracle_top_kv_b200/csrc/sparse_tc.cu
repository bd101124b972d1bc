// sparse_tc.cu -- the HySparse block-mode sparse layer on the tcgen05 tensor
// cores: row-grouped block-sparse attention.
//
// Query row t of a sparse layer attends over the keys of the blocks its index
// set selects, clipped to keys <= t ("HySparse: ..." 3.3; "跨层 KV Cache 复用
// 怎样成立"; the in-block causal mask of "工程实现中的关键约束" item 4):
//     o_h = sum_{i in R_t} softmax_{R_t}(tau q'_h . k_i) v_i.
// Nearby rows select overlapping block sets: on the HySparse-7B-shaped inputs
// the 64 positions of a CTA's two Q tiles select about 70 distinct 64-key
// blocks between them (16 each).  So a CTA forms the union of its rows'
// selected blocks and streams each union block once through the same tcgen05
// flash pipeline as the full layer: S = Q K^T for all 128 rows of a Q tile,
// each row keeping only the blocks it selected (and keys <= t), online
// softmax, O += P V.  A row pays tensor and exp work for union blocks it did
// not select (masked to -inf), but each K/V block is read once per CTA
// instead of once per row, and both contractions run on the tensor cores.
//
// Warp roles as in full_tc.cu: warp 0 TMA producer (Q once, the union blocks'
// K and V through 3- and 2-stage rings), warp 1 TMEM owner and MMA issuer of
// Q tile 0, warp 10 MMA issuer of Q tile 1, warps 2..9 two softmax warpgroups
// (one thread per row; a quarter of the exponentials on the FMA pipe, exact
// zeros for masked keys).  Supported: bf16, d = 128,
// block mode with B = 64 (= the key tile), 128 % g == 0, and a union of at
// most kMaxUnion blocks (2 * (128/g) positions x k/B ids).  The window branch
// over the layer's own K'/V' (keys t-w+1..t) is a second launch of the same
// kernel whose block list is the contiguous run the CTA's windows touch.
#include "cta_select.cuh"
#include "flash_tc.cuh"
#include "hs_common.cuh"
#include "hs_kernels.cuh"
#include "tc_ptx.cuh"

namespace hs {
namespace stc {

using namespace tc;

constexpr int kMaxSel = 16;    // selected blocks per row held in registers
constexpr int kMaxUnion = 1024;
using L = fl::Layout<3, 2, kMaxUnion * 4>;  // 3 K and 2 V stages; the union block list after P
constexpr int kBM = L::kBM, kNQ = L::kNQ, kBN = L::kBN, kD = L::kD;
constexpr int kThreads = L::kThreads;
constexpr uint32_t kUOff = L::kExtraOff;                  // union block ids, kMaxUnion ints
// misc: tmem(4) abort(4) U(4) pad(4) scan[16]
constexpr uint32_t kSmemBytes = L::kMiscOff + 16 + 64 + 1024;
constexpr uint32_t kBitmapWords = kNQ * 2 * 16384 / 4;  // blocks the union bitmap covers / 32
static_assert(kSmemBytes <= 232448, "shared memory");

struct Args {
    KParams p;
    const int32_t* idx;
    const int32_t* cnt;
    __nv_bfloat16* o;
    float* lse;
    int n_ctas_q;
    int P;  // positions per Q tile (128 / g)
};

// kWin: the window branch -- keys max(0, t-w+1)..t of the layer's own K'/V',
// so the block list is the contiguous run of blocks the CTA's windows touch.
template <bool kWin>
__global__ void __launch_bounds__(kThreads, 1)
    sparse_tc_kernel(const __grid_constant__ CUtensorMap tmap_q,
                     const __grid_constant__ CUtensorMap tmap_k,
                     const __grid_constant__ CUtensorMap tmap_v, Args a) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char* gbase = smem_raw + (base - raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const KParams& p = a.p;
    const int g = p.group, P = a.P;

    const int bu_n = p.batch * p.hkv;
    const int qc = a.n_ctas_q - 1 - (int)(blockIdx.x / bu_n);  // latest rows first
    const int bu = (int)(blockIdx.x % bu_n);
    const int b = bu / p.hkv, u = bu % p.hkv;
    const int row0 = qc * kNQ * P;  // first query row of the CTA
    const int last_row = min(p.t_q, row0 + kNQ * P) - 1;
    const int n_blocks = (p.q_offset + last_row) / kBN + 1;  // blocks any row may select
    const int win_b0 = max(0, p.q_offset + row0 - p.window + 1) / kBN;  // first window block

    auto bar = [&](int i) { return base + L::kBarOff + 8u * i; };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + L::kMiscOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L::kMiscOff + 4);
    int* s_union = reinterpret_cast<int*>(gbase + L::kMiscOff + 8);
    int* s_scan = reinterpret_cast<int*>(gbase + L::kMiscOff + 16);
    uint32_t* bitmap = reinterpret_cast<uint32_t*>(gbase + L::kPOff);  // prologue only
    int* ulist = reinterpret_cast<int*>(gbase + kUOff);
    const int words = kWin ? 0 : (n_blocks + 31) >> 5;

    if (threadIdx.x == 0) {
        fl::init_barriers<L>(base + L::kBarOff);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(base + L::kMiscOff, L::kTmemCols);
        tmem_relinquish();
    }
    for (int x = threadIdx.x; x < words; x += blockDim.x) bitmap[x] = 0u;

    // This thread's row (softmax warps): its position's selected block ids.
    const bool is_row = warp >= 2 && warp < L::kIssuer1Warp;
    const int q = is_row ? (warp - 2) >> 2 : 0;
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const int hh = row / P, pr = row % P;
    const int qrow0 = row0 + q * P;
    const int pos = p.q_offset + qrow0 + pr;
    const bool row_valid = is_row && qrow0 + pr < p.t_q;
    int sid[kMaxSel];
    int nsel = 0;
#pragma unroll
    for (int x = 0; x < kMaxSel; ++x) sid[x] = -1;
    __syncthreads();  // bitmap zeroed
    if (row_valid && !kWin) {
        const size_t irow = ((size_t)b * p.hkv + u) * p.t_q + qrow0 + pr;
        int c = a.cnt[irow];
        if (c < 0 || c > p.ksel) { if (hh == 0) set_status(HS_ERR_BOUNDS); c = c < 0 ? 0 : p.ksel; }
        const int32_t* ids = a.idx + irow * p.ksel;
#pragma unroll
        for (int x = 0; x < kMaxSel; ++x) {
            if (x < c) {
                const int id = ids[x];
                if (id < 0 || id > pos / kBN) {
                    if (hh == 0) set_status(HS_ERR_BOUNDS);
                } else {
                    sid[x] = id;
                    if (hh == 0) atomicOr(&bitmap[id >> 5], 1u << (id & 31));
                }
            }
        }
        nsel = c;
    }
    __syncthreads();  // bitmap complete
    {
        // union list, ascending: each thread reads out a run of words
        const int per = (words + blockDim.x - 1) / blockDim.x;
        const int w0 = threadIdx.x * per;
        int cbits = 0;
        for (int x = 0; x < per; ++x)
            if (w0 + x < words) cbits += __popc(bitmap[w0 + x]);
        int at = cta_exclusive_sum(cbits, s_scan);
        for (int x = 0; x < per; ++x) {
            if (w0 + x >= words) break;
            uint32_t m = bitmap[w0 + x];
            while (m) {
                if (at < kMaxUnion) ulist[at] = (w0 + x) * 32 + (__ffs(m) - 1);
                ++at;
                m &= m - 1u;
            }
        }
        if (threadIdx.x == blockDim.x - 1) *s_union = kWin ? n_blocks - win_b0 : min(at, kMaxUnion);
    }
    tc_fence_before();
    __syncthreads();  // union ready; the P region is free again
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int U = *s_union;
    int ntq[kNQ];
#pragma unroll
    for (int qq = 0; qq < kNQ; ++qq) ntq[qq] = row0 + qq * P < p.t_q ? U : 0;
    const int nt = U;

    if (warp == 0) {
        if (lane == 0)
            fl::producer<L>(base, &tmap_q, &tmap_k, &tmap_v, row0, P, u * g, b, bu, nt,
                            [&](int j) { return (kWin ? win_b0 + j : ulist[j]) * kBN; }, abort_flag);
    } else if (warp == 1 || warp == L::kIssuer1Warp) {
        if (lane == 0) {
            const int qi = warp == 1 ? 0 : 1;
            fl::mma_issuer<L>(base, tmem, qi, nt, qi == 0 ? ntq[0] : ntq[1], abort_flag);
        }
    } else {
        // ------------------------------------------------------ softmax
        const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16) + q * 256;
        const int nt_me = ntq[q];
        const float sl2 = p.scale_log2;
        float m_ref = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; j < nt_me; ++j) {
            const int s = j & 1;
            if (!fl::warp_wait(bar(L::BSF + 2 * q + s), (j >> 1) & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            uint32_t r[64];
            tmem_ld32(trow + 64 * s, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
            tmem_ld32(trow + 64 * s + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
            tmem_wait_ld();

            // global: this row keeps the block only if it selected it, and keys
            // <= t; window: keys t-w+1..t
            const int blk = kWin ? win_b0 + j : ulist[j];
            const int key0 = blk * kBN;
            bool sel = kWin;
            if (!kWin) {
#pragma unroll
                for (int x = 0; x < kMaxSel; ++x) sel |= (x < nsel) & (sid[x] == blk);
            }
            const int lim = (sel && row_valid) ? pos - key0 : -1;  // last kept column
            const int first = kWin ? pos - p.window + 1 - key0 : 0;  // first kept column
            // a row may see no kept key for a while (m_ref = -inf), or none at
            // all: masked keys must give exact zeros
            float mt, corr;
            uint32_t pk[32];
            const bool resc =
                fl::softmax_tile<4, true>(r, first, lim, sl2, m_ref, l, mt, corr, pk);
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
        const size_t orow = ((size_t)b * p.hq + u * g + hh) * p.t_q + qrow0 + pr;
        if (ok) {  // warp-uniform; the TMEM loads run on every lane of the warp
            if (nt_me > 0) tc_fence_after();
            const bool any = l > 0.f;
            const float inv = any ? 1.f / l : 0.f;
            fl::store_o(trow + 128, nt_me > 0, inv, row_valid, a.o + orow * kD);
            if (row_valid) a.lse[orow] = any ? (m_ref + log2f(l)) * kLn2 : -INFINITY;
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

}  // namespace stc

bool sparse_tc_supported(const KParams& p, int dtype) {
    if (dtype != HS_BF16 || p.head_dim != stc::kD || p.mode != 0 || p.group > 16) return false;
    if (p.block_size != stc::kBN || p.ksel > stc::kMaxSel || 128 % p.group != 0) return false;
    const int P = stc::kBM / p.group;
    if (stc::kNQ * P * p.ksel > stc::kMaxUnion) return false;  // the union always fits
    return (long long)(p.t_kv / stc::kBN + 1) <= (long long)stc::kBitmapWords * 32;
}

cudaError_t launch_sparse_tc(const KParams& p, const void* q, const void* kf, const void* vf,
                             const int32_t* idx, const int32_t* cnt, void* og, float* lseg,
                             bool window, cudaStream_t st) {
    const int g = p.group, P = stc::kBM / g;
    CUtensorMap mq, mk, mv;
    const cuuint64_t qd[4] = {(cuuint64_t)stc::kD, (cuuint64_t)p.t_q, (cuuint64_t)p.hq,
                              (cuuint64_t)p.batch};
    const cuuint64_t qs[3] = {(cuuint64_t)stc::kD * 2, (cuuint64_t)p.t_q * stc::kD * 2,
                              (cuuint64_t)p.hq * p.t_q * stc::kD * 2};
    const cuuint32_t qb[4] = {64, (cuuint32_t)P, (cuuint32_t)g, 1};
    const cuuint64_t kdims[3] = {(cuuint64_t)stc::kD, (cuuint64_t)p.t_kv, (cuuint64_t)p.hkv * p.batch};
    const cuuint64_t ks[2] = {(cuuint64_t)stc::kD * 2, (cuuint64_t)p.t_kv * stc::kD * 2};
    const cuuint32_t kb[3] = {64, (cuuint32_t)stc::kBN, 1};
    if (!tc::encode(&mq, q, 4, qd, qs, qb) || !tc::encode(&mk, kf, 3, kdims, ks, kb) ||
        !tc::encode(&mv, vf, 3, kdims, ks, kb))
        return cudaErrorInvalidValue;
    stc::Args a;
    a.p = p;
    a.idx = idx;
    a.cnt = cnt;
    a.o = (__nv_bfloat16*)og;
    a.lse = lseg;
    a.P = P;
    a.n_ctas_q = (p.t_q + stc::kNQ * P - 1) / (stc::kNQ * P);
    auto kern = window ? stc::sparse_tc_kernel<true> : stc::sparse_tc_kernel<false>;
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, stc::kSmemBytes);
    if (e != cudaSuccess) return e;
    const long long grid = (long long)a.n_ctas_q * p.batch * p.hkv;
    kern<<<(unsigned)grid, stc::kThreads, stc::kSmemBytes, st>>>(mq, mk, mv, a);
    return cudaGetLastError();
}

}  // namespace hs
