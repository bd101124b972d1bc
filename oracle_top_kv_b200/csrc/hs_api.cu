// hs_api.cu -- the C ABI declared in include/hs.h: argument validation,
// kernel selection and launch, workspace sizing and the device status word.
//
// The whole library is one translation unit (the kernel files are included
// below), so the sticky status word defined in hs_common.cuh is a single
// __device__ symbol without relocatable device code.
#include <math.h>
#include <stdint.h>

#include <atomic>

#include "../../include/hs.h"
#include "hs_common.cuh"
#include "hs_kernels.cuh"

#include "decode_full.cu"
#include "full_simt.cu"
#include "full_tc.cu"
#include "sparse_tc.cu"
#include "token_select_tc.cu"
#include "token_select_wide.cu"
#include "noalloc.cu"
#include "sparse.cu"
#include "decode_simt.cu"
#include "gate_sink.cu"

namespace hs {
static std::atomic<uint64_t> g_launches{0};
void count_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }
}  // namespace hs

namespace {

using hs::KParams;

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }
bool ok_ptr(const void* ptr) { return ptr != nullptr && aligned16(ptr); }
bool ok_opt(const void* ptr) { return ptr == nullptr || aligned16(ptr); }

// Common shape / knob checks.  Returns HS_OK and fills kp on success.
hs_status resolve(const hs_params* p, bool decode, KParams* kp) {
    if (!p) return HS_ERR_INVALID_ARG;
    if (p->batch < 1 || p->hq < 1 || p->hkv < 1 || p->t_q < 0 || p->t_kv < 1 || p->q_offset < 0)
        return HS_ERR_INVALID_ARG;
    if (p->hq % p->hkv != 0) return HS_ERR_INVALID_ARG;
    if (p->dtype != HS_BF16 && p->dtype != HS_FP32) return HS_ERR_INVALID_ARG;
    if (p->mode != HS_SEL_BLOCK && p->mode != HS_SEL_TOKEN) return HS_ERR_INVALID_ARG;
    if (!(p->scale >= 0.f) || !isfinite(p->scale)) return HS_ERR_INVALID_ARG;
    if (p->k < 1 || p->window < 0) return HS_ERR_INVALID_ARG;
    int ksel;
    if (p->mode == HS_SEL_BLOCK) {
        if (p->block_size < 1 || p->k % p->block_size != 0) return HS_ERR_INVALID_ARG;
        ksel = p->k / p->block_size;
    } else {
        if (p->window > p->k) return HS_ERR_INVALID_ARG;
        ksel = p->k;
    }
    if (decode) {
        if (p->t_q != 1) return HS_ERR_INVALID_ARG;
    } else if ((long long)p->q_offset + p->t_q > p->t_kv) {
        return HS_ERR_INVALID_ARG;
    }
    // element counts must stay far from overflow
    const double big = (double)p->batch * p->hq * (double)(p->t_kv > p->t_q ? p->t_kv : p->t_q) *
                       (p->head_dim > 0 ? p->head_dim : 1);
    if (big > 4.0e15) return HS_ERR_INVALID_ARG;
    // what this build implements
    const int g = p->hq / p->hkv;
    if (p->head_dim != 64 && p->head_dim != 128 && p->head_dim != 256) return HS_ERR_UNSUPPORTED;
    if (g > 64) return HS_ERR_UNSUPPORTED;
    if (p->mode == HS_SEL_BLOCK) {
        const int B = p->block_size;
        if (B != 16 && B != 32 && B != 64 && B != 128) return HS_ERR_UNSUPPORTED;
        if (ksel > 64) return HS_ERR_UNSUPPORTED;
    } else if (p->k > 4096) {
        return HS_ERR_UNSUPPORTED;
    }
    kp->batch = p->batch;
    kp->hq = p->hq;
    kp->hkv = p->hkv;
    kp->group = g;
    kp->head_dim = p->head_dim;
    kp->t_q = p->t_q;
    kp->t_kv = p->t_kv;
    kp->q_offset = decode ? 0 : p->q_offset;
    kp->mode = p->mode;
    kp->block_size = p->mode == HS_SEL_BLOCK ? p->block_size : 1;
    kp->k = p->k;
    kp->window = p->window;
    kp->ksel = ksel;
    const float scale = p->scale > 0.f ? p->scale : 1.0f / sqrtf((float)p->head_dim);
    kp->scale_log2 = scale * hs::kLog2e;
    return HS_OK;
}

hs_status from_cuda(cudaError_t e) { return e == cudaSuccess ? HS_OK : HS_ERR_CUDA; }

// The mma.sync gather and decode kernels: groups of up to 16 heads, d <= 128.
// Wider groups and d = 256 (the MQA 64/1, d = 256 shape) take the SIMT kernels.
bool mma_shape(const KParams& kp) { return kp.group <= 16 && kp.head_dim <= 128; }

// Launch a sequence through fn() and count its kernels when it succeeds.
template <typename Fn>
hs_status launched(int n_kernels, Fn fn) {
    const cudaError_t e = fn();
    if (e == cudaSuccess) hs::count_launches(n_kernels);
    return from_cuda(e);
}

}  // namespace

extern "C" {

hs_status hs_full_attn_index(const hs_params* p, const void* q, const void* k, const void* v,
                             void* o, float* lse, int32_t* idx, int32_t* idx_count,
                             float* sel_scores, void* workspace, size_t ws_bytes, void* stream) {
    KParams kp;
    hs_status s = resolve(p, false, &kp);
    if (s != HS_OK) return s;
    if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(o) || !ok_ptr(lse) || !ok_ptr(idx) ||
        !ok_ptr(idx_count) || !ok_opt(sel_scores))
        return HS_ERR_INVALID_ARG;
    if (kp.t_q == 0) return HS_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (hs::full_tc_supported(kp, p->dtype)) {
        if (kp.mode == HS_SEL_BLOCK)
            return launched(1, [&] {
                return hs::launch_full_tc(kp, q, k, v, o, lse, idx, idx_count, sel_scores, 1, st);
            });
        // token mode: tensor-core attention pass, then the selection pass
        return launched(2, [&] {
            cudaError_t e =
                hs::launch_full_tc(kp, q, k, v, o, lse, idx, idx_count, sel_scores, 0, st);
            if (e != cudaSuccess) return e;
            // long scans: the wide selector, when the caller gave its workspace
            if (hs::token_select_wide_applies(kp, p->dtype) && workspace != nullptr &&
                aligned16(workspace) && ws_bytes >= hs::token_select_wide_workspace(kp))
                return hs::launch_token_select_wide(kp, q, k, lse, idx, idx_count, sel_scores,
                                                    workspace, ws_bytes, st);
            if (hs::token_select_tc_supported(kp, p->dtype))
                return hs::launch_token_select_tc(kp, q, k, lse, idx, idx_count, sel_scores, st);
            return hs::launch_full_simt(kp, p->dtype, q, k, v, o, lse, idx, idx_count,
                                        sel_scores, 0, st);
        });
    }
    return launched(1, [&] {
        return hs::launch_full_simt(kp, p->dtype, q, k, v, o, lse, idx, idx_count, sel_scores,
                                    1, st);
    });
}

hs_status hs_sparse_attn_reuse(const hs_params* p, const void* q_sparse, const void* k_f,
                               const void* v_f, const int32_t* idx, const int32_t* idx_count,
                               const void* k_local, const void* v_local, void* o_global,
                               float* lse_global, void* o_local, float* lse_local,
                               void* workspace, size_t ws_bytes, void* stream) {
    (void)workspace;
    (void)ws_bytes;
    KParams kp;
    hs_status s = resolve(p, false, &kp);
    if (s != HS_OK) return s;
    if (!ok_ptr(q_sparse) || !ok_ptr(k_f) || !ok_ptr(v_f) || !ok_ptr(idx) || !ok_ptr(idx_count) ||
        !ok_ptr(o_global) || !ok_ptr(lse_global))
        return HS_ERR_INVALID_ARG;
    const bool local = k_local != nullptr || v_local != nullptr;
    if (local && (!ok_ptr(k_local) || !ok_ptr(v_local) || !ok_ptr(o_local) || !ok_ptr(lse_local)))
        return HS_ERR_INVALID_ARG;
    if (local && p->window < 1) return HS_ERR_INVALID_ARG;
    if (kp.t_q == 0) return HS_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (p->dtype == HS_FP32)
        return launched(1, [&] {
            return hs::launch_sparse_simt(kp, p->dtype, q_sparse, k_f, v_f, idx, idx_count,
                                          local ? k_local : nullptr, v_local, o_global,
                                          lse_global, o_local, lse_local, st);
        });
    if (!mma_shape(kp)) {
        // wide groups / d = 256: one CTA per query row and group with staged
        // K/V tiles (token mode, no window branch), else the per-head SIMT kernel
        if (!local && hs::sparse_simt_rows_supported(kp, p->dtype))
            return launched(1, [&] {
                return hs::launch_sparse_simt_rows(kp, q_sparse, k_f, v_f, idx, idx_count,
                                                   o_global, lse_global, st);
            });
        return launched(1, [&] {
            return hs::launch_sparse_simt(kp, p->dtype, q_sparse, k_f, v_f, idx, idx_count,
                                          local ? k_local : nullptr, v_local, o_global,
                                          lse_global, o_local, lse_local, st);
        });
    }
    if (hs::sparse_tc_supported(kp, p->dtype)) {
        // global branch, then the window branch, on the tensor cores
        return launched(local ? 2 : 1, [&] {
            cudaError_t e = hs::launch_sparse_tc(kp, q_sparse, k_f, v_f, idx, idx_count, o_global,
                                                 lse_global, false, st);
            if (e != cudaSuccess || !local) return e;
            return hs::launch_sparse_tc(kp, q_sparse, k_local, v_local, idx, idx_count, o_local,
                                        lse_local, true, st);
        });
    }
    return launched(1, [&] {
        return hs::launch_sparse_mma(kp, q_sparse, k_f, v_f, idx, idx_count,
                                     local ? k_local : nullptr, v_local, o_global, lse_global,
                                     o_local, lse_local, st);
    });
}

size_t hs_workspace_size(const hs_params* p, int32_t which) {
    KParams kp;
    const bool decode = which == HS_WS_DECODE_FULL || which == HS_WS_DECODE_SPARSE;
    if (which < HS_WS_FULL || which > HS_WS_DECODE_SPARSE) return (size_t)-1;
    if (resolve(p, decode, &kp) != HS_OK) return (size_t)-1;
    if (decode && !mma_shape(kp))  // wide groups / d = 256: the split-k CUDA-core steps
        return hs::decode_simt_split_supported(kp)
                   ? hs::decode_simt_workspace(kp, which == HS_WS_DECODE_FULL)
                   : 0;
    switch (which) {
        case HS_WS_FULL:
            return hs::full_tc_supported(kp, p->dtype) && hs::token_select_wide_applies(kp, p->dtype)
                       ? hs::token_select_wide_workspace(kp)
                       : 0;
        case HS_WS_DECODE_FULL: return hs::decode_full_workspace(kp);
        case HS_WS_DECODE_SPARSE: return hs::decode_sparse_workspace(kp);
        default: return 0;
    }
}

hs_status hs_decode_step(const hs_params* p, int32_t kind, const void* q, const void* k_cache,
                         const void* v_cache, const int32_t* seq_len, int32_t* idx,
                         int32_t* idx_count, void* o, float* lse, float* sel_scores,
                         void* workspace, size_t ws_bytes, void* stream) {
    KParams kp;
    hs_status s = resolve(p, true, &kp);
    if (s != HS_OK) return s;
    if (kind != HS_DECODE_FULL_INDEX && kind != HS_DECODE_SPARSE) return HS_ERR_INVALID_ARG;
    if (p->dtype != HS_BF16 || p->mode != HS_SEL_TOKEN) return HS_ERR_UNSUPPORTED;
    if (!ok_ptr(q) || !ok_ptr(k_cache) || !ok_ptr(v_cache) || !ok_ptr(seq_len) || !ok_ptr(idx) ||
        !ok_ptr(idx_count) || !ok_ptr(o) || !ok_opt(lse) || !ok_opt(sel_scores))
        return HS_ERR_INVALID_ARG;
    if (!mma_shape(kp)) {
        // wide groups / d = 256: split-k CUDA-core kernels with the workspace,
        // else one CTA per sequence and group (no workspace)
        cudaStream_t st = static_cast<cudaStream_t>(stream);
        const bool full = kind == HS_DECODE_FULL_INDEX;
        if (full && !lse) return HS_ERR_INVALID_ARG;
        if (hs::decode_simt_split_supported(kp) && workspace != nullptr && aligned16(workspace) &&
            ws_bytes >= hs::decode_simt_workspace(kp, full))
            return launched(hs::decode_simt_kernel_count(full), [&] {
                return hs::launch_decode_simt(kp, full, q, k_cache, v_cache, seq_len, idx,
                                              idx_count, o, lse, sel_scores, workspace, st);
            });
        if (kind == HS_DECODE_FULL_INDEX) {
            if (!lse) return HS_ERR_INVALID_ARG;
            return launched(1, [&] {
                return hs::launch_full_simt(kp, p->dtype, q, k_cache, v_cache, o, lse, idx,
                                            idx_count, sel_scores, 1, st, seq_len);
            });
        }
        return launched(1, [&] {
            return hs::launch_sparse_simt(kp, p->dtype, q, k_cache, v_cache, idx, idx_count,
                                          nullptr, nullptr, o, lse, nullptr, nullptr, st, seq_len);
        });
    }
    const size_t need = kind == HS_DECODE_FULL_INDEX ? hs::decode_full_workspace(kp)
                                                     : hs::decode_sparse_workspace(kp);
    if (need > 0 && (workspace == nullptr || ws_bytes < need || !aligned16(workspace)))
        return HS_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (kind == HS_DECODE_FULL_INDEX) {
        if (!lse) return HS_ERR_INVALID_ARG;
        const int n_kernels = hs::decode_full_kernel_count(kp);
        return launched(n_kernels, [&] {
            return hs::launch_decode_full(kp, q, k_cache, v_cache, seq_len, idx, idx_count, o,
                                          lse, sel_scores, workspace, st);
        });
    }
    return launched(1, [&] {
        return hs::launch_decode_sparse(kp, q, k_cache, v_cache, seq_len, idx, idx_count, o, lse,
                                        workspace, st);
    });
}

}  // extern "C"

namespace {
// Validates a block table description and records it in kp.
hs_status set_pages(const hs_params* p, const hs_pages* pages, KParams* kp) {
    if (!pages || !ok_ptr(pages->block_table)) return HS_ERR_INVALID_ARG;
    if (pages->page_size < 1 || pages->max_pages < 1 || pages->n_pages < 1)
        return HS_ERR_INVALID_ARG;
    if ((long long)pages->max_pages * pages->page_size != p->t_kv) return HS_ERR_INVALID_ARG;
    if ((long long)pages->n_pages * p->hkv * pages->page_size >= (1ll << 31))
        return HS_ERR_INVALID_ARG;
    kp->bt = pages->block_table;
    kp->page_size = pages->page_size;
    kp->max_pages = pages->max_pages;
    kp->n_pages = pages->n_pages;
    return HS_OK;
}
}  // namespace

extern "C" {

hs_status hs_sparse_attn_reuse_paged(const hs_params* p, const hs_pages* pages,
                                     const void* q_sparse, const void* k_pool,
                                     const void* v_pool, const int32_t* idx,
                                     const int32_t* idx_count, void* o_global,
                                     float* lse_global, void* stream) {
    KParams kp;
    hs_status s = resolve(p, false, &kp);
    if (s != HS_OK) return s;
    if ((s = set_pages(p, pages, &kp)) != HS_OK) return s;
    if (!ok_ptr(q_sparse) || !ok_ptr(k_pool) || !ok_ptr(v_pool) || !ok_ptr(idx) ||
        !ok_ptr(idx_count) || !ok_ptr(o_global) || !ok_ptr(lse_global))
        return HS_ERR_INVALID_ARG;
    if (p->dtype != HS_BF16 || !mma_shape(kp)) return HS_ERR_UNSUPPORTED;
    if (kp.t_q == 0) return HS_OK;
    return launched(1, [&] {
        return hs::launch_sparse_mma(kp, q_sparse, k_pool, v_pool, idx, idx_count, nullptr,
                                     nullptr, o_global, lse_global, nullptr, nullptr,
                                     static_cast<cudaStream_t>(stream));
    });
}

hs_status hs_decode_step_paged(const hs_params* p, const hs_pages* pages, int32_t kind,
                               const void* q, const void* k_pool, const void* v_pool,
                               const int32_t* seq_len, int32_t* idx, int32_t* idx_count,
                               void* o, float* lse, float* sel_scores, void* workspace,
                               size_t ws_bytes, void* stream) {
    KParams kp;
    hs_status s = resolve(p, true, &kp);
    if (s != HS_OK) return s;
    if ((s = set_pages(p, pages, &kp)) != HS_OK) return s;
    if (kind != HS_DECODE_FULL_INDEX && kind != HS_DECODE_SPARSE) return HS_ERR_INVALID_ARG;
    if (p->dtype != HS_BF16 || p->mode != HS_SEL_TOKEN || !mma_shape(kp)) return HS_ERR_UNSUPPORTED;
    if (!ok_ptr(q) || !ok_ptr(k_pool) || !ok_ptr(v_pool) || !ok_ptr(seq_len) || !ok_ptr(idx) ||
        !ok_ptr(idx_count) || !ok_ptr(o) || !ok_opt(lse) || !ok_opt(sel_scores))
        return HS_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (kind == HS_DECODE_FULL_INDEX) {
        const size_t need = hs::decode_full_workspace(kp);
        if (need > 0 && (workspace == nullptr || ws_bytes < need || !aligned16(workspace)))
            return HS_ERR_WORKSPACE;
        if (!lse) return HS_ERR_INVALID_ARG;
        return launched(hs::decode_full_kernel_count(kp), [&] {
            return hs::launch_decode_full(kp, q, k_pool, v_pool, seq_len, idx, idx_count, o, lse,
                                          sel_scores, workspace, st);
        });
    }
    return launched(1, [&] {
        return hs::launch_decode_sparse(kp, q, k_pool, v_pool, seq_len, idx, idx_count, o, lse,
                                        nullptr, st);
    });
}

hs_status hs_decode_sparse_noalloc(const hs_params* p, const void* q, const void* k_cache,
                                   const void* v_cache, const int32_t* seq_len,
                                   const int32_t* idx, const int32_t* idx_count, void* o,
                                   float* lse, void* stream) {
    KParams kp;
    hs_status s = resolve(p, true, &kp);
    if (s != HS_OK) return s;
    if (p->dtype != HS_BF16 || p->mode != HS_SEL_TOKEN || !mma_shape(kp)) return HS_ERR_UNSUPPORTED;
    if (!ok_ptr(q) || !ok_ptr(k_cache) || !ok_ptr(v_cache) || !ok_ptr(seq_len) || !ok_ptr(idx) ||
        !ok_ptr(idx_count) || !ok_ptr(o) || !ok_opt(lse))
        return HS_ERR_INVALID_ARG;
    if (hs::decode_sparse_split_workspace(kp) > hs::noalloc_scratch_bytes()) return HS_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return launched(2, [&] {
        return hs::launch_decode_sparse_noalloc(kp, q, k_cache, v_cache, seq_len, idx, idx_count,
                                                o, lse, st);
    });
}

hs_status hs_sparse_gate_sink(const hs_params* p, const void* o_global, float* lse_global,
                              const void* o_local, float* lse_local, const float* sink_global,
                              const float* sink_local, const float* gate_global,
                              const float* gate_local, void* o, void* stream) {
    KParams kp;
    hs_status s = resolve(p, false, &kp);
    if (s != HS_OK) return s;
    if (!ok_ptr(o_global) || !ok_ptr(lse_global) || !ok_ptr(o) || !ok_opt(o_local) ||
        !ok_opt(lse_local) || !ok_opt(sink_global) || !ok_opt(sink_local) ||
        !ok_opt(gate_global) || !ok_opt(gate_local))
        return HS_ERR_INVALID_ARG;
    // the local branch comes with its lse; its sink and gate only with it
    if ((o_local == nullptr) != (lse_local == nullptr)) return HS_ERR_INVALID_ARG;
    if (!o_local && (sink_local || gate_local)) return HS_ERR_INVALID_ARG;
    if (kp.t_q == 0) return HS_OK;
    return launched(1, [&] {
        return hs::launch_gate_sink(kp, p->dtype, o_global, lse_global, o_local, lse_local,
                                    sink_global, sink_local, gate_global, gate_local, o,
                                    static_cast<cudaStream_t>(stream));
    });
}

hs_status hs_device_status(void* stream, int32_t* out) {
    if (!out) return HS_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return HS_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, hs::g_status, sizeof(int)) != cudaSuccess) return HS_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpyToSymbol(hs::g_status, &zero, sizeof(int)) != cudaSuccess) return HS_ERR_CUDA;
    *out = v;
    return HS_OK;
}

uint64_t hs_launch_count(void) { return hs::g_launches.load(std::memory_order_relaxed); }

hs_status hs_set_wait_limit(int64_t cycles) {
    const long long v = cycles > 0 ? (long long)cycles : hs::tc::kWaitCycles;
    return cudaMemcpyToSymbol(hs::g_wait_limit, &v, sizeof(v)) == cudaSuccess ? HS_OK
                                                                               : HS_ERR_CUDA;
}

hs_status hs_set_select_sampling(int32_t rank) {
    const int v = rank < 0 ? -1 : (int)rank;
    return cudaMemcpyToSymbol(hs::g_sel_sample, &v, sizeof(v)) == cudaSuccess ? HS_OK
                                                                               : HS_ERR_CUDA;
}

const char* hs_status_string(int32_t status) {
    switch (status) {
        case HS_OK: return "HS_OK";
        case HS_ERR_INVALID_ARG: return "HS_ERR_INVALID_ARG";
        case HS_ERR_UNSUPPORTED: return "HS_ERR_UNSUPPORTED";
        case HS_ERR_CUDA: return "HS_ERR_CUDA";
        case HS_ERR_TIMEOUT: return "HS_ERR_TIMEOUT";
        case HS_ERR_BOUNDS: return "HS_ERR_BOUNDS";
        case HS_ERR_WORKSPACE: return "HS_ERR_WORKSPACE";
        default: return "HS_UNKNOWN_STATUS";
    }
}

}  // extern "C"
