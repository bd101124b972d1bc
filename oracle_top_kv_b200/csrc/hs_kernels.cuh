// hs_kernels.cuh -- launch parameters and host-side launchers shared between
// the C-ABI layer (hs_api.cu) and the kernel translation units.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace hs {

// Host-side count of kernel launches issued by this library (hs_launch_count).
void count_launches(int n);

// Resolved, validated parameters handed to every kernel (by value).
struct KParams {
    int batch, hq, hkv, group, head_dim;
    int t_q, t_kv, q_offset;
    int mode;        // 0 block, 1 token
    int block_size;  // B (1 in token mode)
    int k, window;
    int ksel;        // entries per index row
    float scale_log2;  // softmax scale * log2(e)
    // Paged K^F/V^F (bt != nullptr): the cache is a pool of pages of
    // page_size rows per kv head, [n_pages][hkv][page_size][d]; logical key i
    // of sequence b lives in page bt[b * max_pages + i / page_size], row
    // i % page_size.  t_kv is then max_pages * page_size.
    const int32_t* bt = nullptr;
    int page_size = 0, max_pages = 0, n_pages = 0;
};

// do_attn = 0: selection only, reading lse from a previous attention pass.
// seq_len (decode, t_q = 1): each sequence's query is its newest token.
// Groups of up to 64 heads, head_dim 64, 128 or 256.
cudaError_t launch_full_simt(const KParams& p, int dtype, const void* q, const void* k,
                             const void* v, void* o, float* lse, int32_t* idx, int32_t* cnt,
                             float* sel, int do_attn, cudaStream_t st,
                             const int32_t* seq_len = nullptr);

// tcgen05 flash attention (bf16, d = 128).  capture = 1: block-mode index.
bool full_tc_supported(const KParams& p, int dtype);
cudaError_t launch_full_tc(const KParams& p, const void* q, const void* k, const void* v,
                           void* o, float* lse, int32_t* idx, int32_t* cnt, float* sel,
                           int capture, cudaStream_t st);

// Split-k decode steps on the CUDA cores for groups of up to 64 heads and
// head_dim 64/128/256 (contiguous cache): full = full step with the index,
// else the sparse step.  Needs decode_simt_workspace(p, full) bytes.
bool decode_simt_split_supported(const KParams& p);
size_t decode_simt_workspace(const KParams& p, bool full);
int decode_simt_kernel_count(bool full);
cudaError_t launch_decode_simt(const KParams& p, bool full, const void* q, const void* kc,
                               const void* vc, const int32_t* seq_len, int32_t* idx,
                               int32_t* cnt, void* o, float* lse, float* sel, void* ws,
                               cudaStream_t st);

// Token-mode sparse layer in prefill on the CUDA cores (wide groups, head_dim
// 256; bf16, contiguous K^F/V^F, no window branch): one CTA per query row.
bool sparse_simt_rows_supported(const KParams& p, int dtype);
cudaError_t launch_sparse_simt_rows(const KParams& p, const void* q, const void* kf,
                                    const void* vf, const int32_t* idx, const int32_t* cnt,
                                    void* o, float* lse, cudaStream_t st);

// seq_len as for launch_full_simt.  Groups of up to 64 heads, head_dim 64,
// 128 or 256.
cudaError_t launch_sparse_simt(const KParams& p, int dtype, const void* q, const void* kf,
                               const void* vf, const int32_t* idx, const int32_t* cnt,
                               const void* kl, const void* vl, void* og, float* lseg, void* ol,
                               float* lsel, cudaStream_t st, const int32_t* seq_len = nullptr);

// bf16 tensor-core paths (mma.sync fragments; d = 64 or 128).  global = false:
// the window branch only (the global branch is computed by sparse_tc).
cudaError_t launch_sparse_mma(const KParams& p, const void* q, const void* kf, const void* vf,
                              const int32_t* idx, const int32_t* cnt, const void* kl,
                              const void* vl, void* og, float* lseg, void* ol, float* lsel,
                              cudaStream_t st, bool global = true);

// Block-mode global branch on tcgen05 (row-grouped block-sparse attention).
bool sparse_tc_supported(const KParams& p, int dtype);
// window = true: the window branch over the layer's own K'/V' (idx unused).
cudaError_t launch_sparse_tc(const KParams& p, const void* q, const void* kf, const void* vf,
                             const int32_t* idx, const int32_t* cnt, void* og, float* lseg,
                             bool window, cudaStream_t st);

// Decode (bf16, token mode).
size_t decode_full_workspace(const KParams& p);
int decode_full_kernel_count(const KParams& p);  // kernels one full decode step launches
size_t decode_sparse_workspace(const KParams& p);
cudaError_t launch_decode_full(const KParams& p, const void* q, const void* kc, const void* vc,
                               const int32_t* seq_len, int32_t* idx, int32_t* cnt, void* o,
                               float* lse, float* sel, void* ws, cudaStream_t st);
// One clustered kernel per sparse step; ws is unused (the workspace size is 0).
cudaError_t launch_decode_sparse(const KParams& p, const void* q, const void* kc, const void* vc,
                                 const int32_t* seq_len, const int32_t* idx, const int32_t* cnt,
                                 void* o, float* lse, void* ws, cudaStream_t st);
// Split-k sparse step (split kernel + combine) with partials in `ws`.
size_t decode_sparse_split_workspace(const KParams& p);
cudaError_t launch_decode_sparse_split(const KParams& p, const void* q, const void* kc,
                                       const void* vc, const int32_t* seq_len, const int32_t* idx,
                                       const int32_t* cnt, void* o, float* lse, void* ws,
                                       cudaStream_t st);

// Token-mode selection on the tensor cores (bf16, d = 128, 16 heads per group,
// k - w <= 1024); reads lse from the attention pass.
bool token_select_tc_supported(const KParams& p, int dtype);
// Sparse-layer output: per-head sinks and sigmoid-gate fusion of the branches
// (gate_sink.cu).  o_l / lse_l null: one branch; sink / gate null: none.
cudaError_t launch_gate_sink(const KParams& p, int dtype, const void* o_g, float* lse_g,
                             const void* o_l, float* lse_l, const float* sink_g,
                             const float* sink_l, const float* z_g, const float* z_l, void* o,
                             cudaStream_t st);
cudaError_t launch_token_select_tc(const KParams& p, const void* q, const void* k,
                                   const float* lse, int32_t* idx, int32_t* cnt, float* sel,
                                   cudaStream_t st);

// Token-mode selection for long scans (>= 2^18 keys): 16 positions per work
// item, N = 256, candidate buffers in the workspace (persistent grid).
bool token_select_wide_applies(const KParams& p, int dtype);
size_t token_select_wide_workspace(const KParams& p);
cudaError_t launch_token_select_wide(const KParams& p, const void* q, const void* k,
                                     const float* lse, int32_t* idx, int32_t* cnt, float* sel,
                                     void* ws, size_t ws_bytes, cudaStream_t st);

// Sparse decode step with its scratch in a file-scope device array.
size_t noalloc_scratch_bytes();
cudaError_t launch_decode_sparse_noalloc(const KParams& p, const void* q, const void* kc,
                                         const void* vc, const int32_t* seq_len,
                                         const int32_t* idx, const int32_t* cnt, void* o,
                                         float* lse, cudaStream_t st);

}  // namespace hs
