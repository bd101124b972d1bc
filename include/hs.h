/*
 * hs.h -- C ABI of the B200 (sm_100a) HySparse / HySparse2 hot path.
 *
 * Two halves of one hybrid block, as the pages describe them:
 *   1. a full-attention layer that is also the oracle indexer: exact causal
 *      GQA softmax attention that, besides O, emits per query and KV group the
 *      index set of the best keys ("HySparse 混合稀疏注意力（一）", sections
 *      "从精确注意力里提取块级分数" and "GQA 下为什么要组内共享索引";
 *      "HySparse: A Hybrid Sparse Attention Architecture ...", 3.2 and
 *      Algorithm 1; "HySparse2: Hybrid Sparse Attention with Two-Level KV
 *      Sharing", 4.2 "改造一"/"改造二");
 *   2. the sparse layers that follow it, which reuse that layer's K^F/V^F and
 *      index set and run attention over only the selected keys, with their own
 *      query ("HySparse 混合稀疏注意力（一）", "跨层 KV Cache 复用怎样成立" and
 *      "同一个 Query，查询两种记忆"; "HySparse ..." 3.3).
 *
 * Conventions shared by every entry point
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    never allocates or frees device memory.  Scratch is passed in through
 *    `workspace` (size from hs_workspace_size; NULL allowed when that is 0).
 *  - Every pointer must be 16-byte aligned.  Tensors are dense, row-major,
 *    with the innermost dimension = head_dim:
 *        q, o, q_sparse, o_global, o_local   [batch][hq ][t_q ][head_dim]
 *        k, v, k_f, v_f, k_local, v_local     [batch][hkv][t_kv][head_dim]
 *        lse, lse_global, lse_local          [batch][hq ][t_q ]            fp32 (natural log)
 *        idx                                 [batch][hkv][t_q ][ksel]      int32
 *        idx_count                           [batch][hkv][t_q ]            int32
 *    where ksel = k / block_size (block mode) or k (token mode).  Query head h
 *    belongs to KV group u = h / (hq / hkv).  Decode uses t_q = 1 and
 *    t_kv = cache capacity (the row stride of the cache).
 *  - Positions are 0-based and causal: query row j sits at position
 *    t = q_offset + j and sees keys 0..t (t < t_kv required).
 *  - Index sets are written in ascending order and padded with -1;
 *    idx_count holds the number of valid entries.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream).  Argument errors are detected on the host before any
 *    launch and returned synchronously; nothing is launched then.  A failed
 *    launch returns HS_ERR_CUDA.  Errors found on the device (an index or
 *    sequence length out of range) skip the offending row and set a sticky
 *    per-device status word that hs_device_status reads.  No kernel traps.
 *  - Supported: head_dim in {64, 128, 256}; hq % hkv == 0 with hq/hkv <= 64
 *    (HySparse2 is MQA 64/1 at head dim 256: "HySparse2 ...", 6.4, and its
 *    reading notes' KV-cache table).  Groups of up to 16 heads at head_dim
 *    <= 128 run on the tensor cores; wider groups and head_dim 256 run on
 *    CUDA-core kernels (same results, lower throughput).  The paged and the
 *    allocation-free entry points take groups of <= 16 heads, head_dim <= 128.
 *    block mode: block_size in {16, 32, 64, 128}, k % block_size == 0,
 *    k/block_size <= 64; token mode: 0 <= window <= k <= 4096;
 *    dtype fp32 or bf16 (decode: bf16 only).
 */
#ifndef HS_H_
#define HS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    HS_OK = 0,
    HS_ERR_INVALID_ARG = 1, /* a pointer, shape or knob is out of range        */
    HS_ERR_UNSUPPORTED = 2, /* valid, but not a shape this build implements   */
    HS_ERR_CUDA = 3,        /* a CUDA launch or runtime call failed           */
    HS_ERR_TIMEOUT = 4,     /* a bounded device wait gave up                  */
    HS_ERR_BOUNDS = 5,      /* a device-side index / length was out of range  */
    HS_ERR_WORKSPACE = 6    /* workspace missing or smaller than required     */
} hs_status;

typedef enum { HS_BF16 = 0, HS_FP32 = 1 } hs_dtype;

/* Selection granularity: HySparse blocks of B keys, or HySparse2 tokens with
 * the most recent `window` tokens always selected. */
typedef enum { HS_SEL_BLOCK = 0, HS_SEL_TOKEN = 1 } hs_sel_mode;

typedef struct {
    int32_t batch;      /* b                                                   */
    int32_t hq;         /* query heads                                         */
    int32_t hkv;        /* key/value heads (GQA groups)                        */
    int32_t head_dim;   /* d                                                   */
    int32_t t_q;        /* query rows per (batch, head)                        */
    int32_t t_kv;       /* key rows per (batch, kv head); decode: capacity     */
    int32_t q_offset;   /* position of query row 0 (chunked prefill)           */
    int32_t dtype;      /* hs_dtype of q, k, v and of the outputs o            */
    int32_t mode;       /* hs_sel_mode                                         */
    int32_t block_size; /* B (block mode)                                      */
    int32_t k;          /* token budget; token mode: total, window included    */
    int32_t window;     /* w (token mode: forced window; block mode: SWA width) */
    float scale;        /* softmax scale; 0 -> 1/sqrt(head_dim)                */
} hs_params;

/*
 * Full-attention layer + oracle indexer (prefill, or a prefill chunk).
 *
 * For every query row and head:  o = softmax(scale q K^T, causal) V and
 * lse = log sum exp(scale q K^T).  For every query row and KV group u it
 * writes the index set I_t:
 *   block mode: the k/B blocks with the largest group score
 *               S_bar_{t,r} = max_{h in u} max_{i in block r, i<=t} p_{h,t,i};
 *   token mode: {max(0,t-w+1)..t} plus the k-w keys of 0..t-w with the largest
 *               S_bar_{t,i} = max_{h in u} p_{h,t,i}.
 * When every candidate fits in the budget, all of them are selected.  Equal
 * scores go to the lower index.  No T x T (or T x T/B) matrix is written.
 *
 * q, k, v:    inputs (layouts above).  o, lse: outputs.
 * idx, idx_count: outputs (ascending, -1 padded).
 * sel_scores: optional output [batch][hkv][t_q][ksel] fp32, the S_bar of each
 *             selected entry (0 in the padding); NULL to skip.
 * workspace:  hs_workspace_size(p, HS_WS_FULL) bytes.  Non-zero only in token
 *             mode for long scans (q_offset + t_q >= 2^18 keys, bf16, d = 128,
 *             16 heads per group, k - w <= 1024): the candidate buffers of the
 *             wide selector (about 38 MB on a 148-SM GPU).  With a smaller
 *             workspace, or NULL, such a call takes the shared-memory selector
 *             instead: same result rule, slower on long scans.
 */
hs_status hs_full_attn_index(const hs_params* p, const void* q, const void* k,
                             const void* v, void* o, float* lse, int32_t* idx,
                             int32_t* idx_count, float* sel_scores, void* workspace,
                             size_t ws_bytes, void* stream);

/*
 * Sparse layer reusing the full layer's K^F, V^F and index set, with its own
 * query q_sparse:  o_global = softmax over R_t of (scale q' k_i) v_i, where R_t is
 * the selected tokens (token mode) or the keys of the selected blocks clipped
 * to i <= t (block mode).
 * When k_local / v_local are non-NULL (block mode), the local branch is also
 * computed: causal softmax attention of q' over the layer's OWN k_local,
 * v_local restricted to keys max(0,t-w+1)..t, into o_local / lse_local.
 * The two branches are returned unfused (the sigmoid gate needs trained
 * weights and is the caller's).  A row whose index set is empty gets o = 0 and
 * lse = -inf.  idx entries out of range set HS_ERR_BOUNDS on the device.
 */
hs_status hs_sparse_attn_reuse(const hs_params* p, const void* q_sparse, const void* k_f,
                               const void* v_f, const int32_t* idx,
                               const int32_t* idx_count, const void* k_local,
                               const void* v_local, void* o_global, float* lse_global,
                               void* o_local, float* lse_local, void* workspace,
                               size_t ws_bytes, void* stream);

/*
 * Output of a sparse layer: a per-head sink in each branch, then the sigmoid
 * gates that fuse the branches ("HySparse 混合稀疏注意力（一）", the section on
 * the two sigmoid gates; "HySparse: ..." 3.3, branch fusion, and the papers'
 * configuration notes on per-head sink biases in the sparse and window
 * branches).  For every row (b, h, t), in fp32:
 *     f_x = e^lse_x / (e^lse_x + e^sink_x[h])   (1 without a sink)
 *     o   = sigmoid(gate_global) f_g o_global + sigmoid(gate_local) f_l o_local
 * and lse_x is replaced IN PLACE by log(e^lse_x + e^sink_x[h]): the sink is
 * one more logit with a zero value vector in the branch's softmax.
 * o_global, o_local, o: [batch][hq][t_q][head_dim], p->dtype (bf16 or fp32);
 *           o may be o_global or o_local.
 * lse_global, lse_local: float [batch][hq][t_q] (as hs_sparse_attn_reuse writes them).
 * o_local / lse_local: both or neither (neither: one branch, e.g. HySparse2).
 * sink_global, sink_local: float [hq] or NULL (no sink); gate_global,
 *           gate_local: float [batch][hq][t_q] pre-activations or NULL (gate 1);
 *           the local ones only with a local branch.
 * p: batch, hq, hkv, head_dim (64 or 128), t_q and dtype as for the layer.
 * One elementwise kernel; asynchronous on `stream`; pointers 16-byte aligned.
 */
hs_status hs_sparse_gate_sink(const hs_params* p, const void* o_global, float* lse_global,
                              const void* o_local, float* lse_local, const float* sink_global,
                              const float* sink_local, const float* gate_global,
                              const float* gate_local, void* o, void* stream);

typedef enum { HS_DECODE_FULL_INDEX = 0, HS_DECODE_SPARSE = 1 } hs_decode_kind;

/*
 * One decode step for a batch of sequences, bf16, token mode
 * ("HySparse 混合稀疏注意力（一）": at step t the new token first passes the full
 * layer, which selects for position t, then the block's sparse layers).
 *
 * q:        [batch][hq][1][head_dim], the new token's query.
 * k_cache, v_cache: [batch][hkv][t_kv][head_dim]; the caller has already
 *           written the new token's k/v at row seq_len[b]-1.
 * seq_len:  DEVICE int32 [batch], 1 <= seq_len[b] <= t_kv (new token included).
 * HS_DECODE_FULL_INDEX: writes o, lse and idx/idx_count [batch][hkv][ksel]
 *           for position seq_len[b]-1 (same rule as hs_full_attn_index).
 * HS_DECODE_SPARSE: reads idx/idx_count and writes o (and lse) of the sparse
 *           layer with query q over K^F = k_cache, V^F = v_cache.
 * sel_scores: optional (FULL_INDEX only), as in hs_full_attn_index.
 * workspace: hs_workspace_size(p, HS_WS_DECODE_FULL) bytes for FULL_INDEX;
 *           HS_DECODE_SPARSE needs none (its size is 0; NULL allowed): one
 *           kernel per step, each (sequence, group) on a cluster of CTAs that
 *           merge their partial results in distributed shared memory.
 *           Groups of more than 16 heads and head_dim 256 (CUDA-core
 *           kernels): with hs_workspace_size(p, HS_WS_DECODE_FULL /
 *           HS_WS_DECODE_SPARSE) bytes both steps run split-k over many CTAs
 *           (the full step holds every key's head logits, 4 * group bytes per
 *           cache row, plus per-split partials); with a smaller workspace, or
 *           NULL, one CTA per (sequence, group) runs each step instead: same
 *           results, far slower on long caches.
 * The caller keeps k_cache, v_cache and idx alive until the last sparse layer
 * of the block has run.
 */
hs_status hs_decode_step(const hs_params* p, int32_t kind, const void* q,
                         const void* k_cache, const void* v_cache, const int32_t* seq_len,
                         int32_t* idx, int32_t* idx_count, void* o, float* lse,
                         float* sel_scores, void* workspace, size_t ws_bytes, void* stream);

/*
 * The sparse decode step of hs_decode_step(HS_DECODE_SPARSE), for callers that
 * cannot allocate device memory -- e.g. a plugin that only receives its input
 * and output buffers from an engine whose memory planner owns all device
 * memory, or a decode loop that must not call cudaMalloc (it can synchronise
 * the device).  It takes no workspace and allocates nothing: its scratch is a
 * fixed 32 MiB array inside the library, present on every GPU that loads the
 * library until the process exits.  (The pages have no counterpart of this
 * entry point.)  It runs the split-k form of the step -- a split kernel that
 * writes per-split partial results, then a combine kernel -- with those
 * partials in the library's array.
 *
 * Arguments, layouts and results are those of hs_decode_step with
 * kind = HS_DECODE_SPARSE.  Limits: batch * hkv * ceil(k / 64) split units of
 * 16 * (head_dim + 2) floats must fit in the 32 MiB (4032 units at
 * head_dim 128, e.g. 32 sequences x 4 kv groups x k = 1024); larger calls
 * return HS_ERR_WORKSPACE without launching anything.
 * The first call on a device looks up the array's device address (with that
 * device current); make that first call before any stream capture.  All calls
 * on a device share the one array: calls whose kernels could overlap on the
 * GPU (e.g. on unordered streams) race and must not be issued.  Nothing
 * persists from one call to the next.
 */
hs_status hs_decode_sparse_noalloc(const hs_params* p, const void* q, const void* k_cache,
                                   const void* v_cache, const int32_t* seq_len,
                                   const int32_t* idx, const int32_t* idx_count, void* o,
                                   float* lse, void* stream);

enum { HS_WS_FULL = 0, HS_WS_SPARSE = 1, HS_WS_DECODE_FULL = 2, HS_WS_DECODE_SPARSE = 3 };

/* Bytes of workspace the matching entry point needs for these parameters
 * (0 when none).  Returns (size_t)-1 for invalid parameters. */
size_t hs_workspace_size(const hs_params* p, int32_t which);

/* Waits for `stream`, then returns in *out the sticky device status word of
 * the current device (an hs_status value, HS_OK if nothing went wrong) and
 * clears it.  Returns HS_ERR_CUDA if the wait or the read failed. */
hs_status hs_device_status(void* stream, int32_t* out);

/* Static, human-readable name of a status code. */
const char* hs_status_string(int32_t status);

/* Number of kernels this library has launched in this process so far (all
 * devices, all streams).  A diagnostic for callers that account for launches;
 * it counts successful launch calls, not completed kernels. */
uint64_t hs_launch_count(void);

/*
 * Paged K^F/V^F ("HySparse 混合稀疏注意力（一）", 工程实现中的关键约束 items 2 and
 * 3: the sparse index keeps logical token ids, a block table translates them
 * into physical pages, and the kernel resolves the addresses while it loads
 * each K/V row instead of first copying the selected rows to a contiguous
 * buffer).  The cache is a pool of pages, k_pool and v_pool both
 * [n_pages][hkv][page_size][head_dim] bf16; logical key i of sequence b lives
 * in page block_table[b * max_pages + i / page_size] at row i % page_size.
 * Index sets (idx) hold logical ids, exactly as the contiguous entry points
 * write and read them.
 */
typedef struct {
    const int32_t* block_table; /* DEVICE int32 [batch][max_pages]               */
    int32_t page_size;          /* rows (tokens) per page, >= 1                  */
    int32_t max_pages;          /* logical pages per sequence (table row stride) */
    int32_t n_pages;            /* pages in the pool                             */
} hs_pages;

/*
 * hs_sparse_attn_reuse over a paged K^F/V^F: the global branch only (no
 * local window branch), bf16, token or block mode, any page size.
 * p->t_kv must equal pages->max_pages * pages->page_size (the logical
 * capacity), and n_pages * hkv * page_size must stay below 2^31.  A block
 * table entry outside [0, n_pages) for a row that is read masks that row and
 * sets HS_ERR_BOUNDS on the device.
 */
hs_status hs_sparse_attn_reuse_paged(const hs_params* p, const hs_pages* pages,
                                     const void* q_sparse, const void* k_pool,
                                     const void* v_pool, const int32_t* idx,
                                     const int32_t* idx_count, void* o_global,
                                     float* lse_global, void* stream);

/*
 * hs_decode_step over a paged cache: both kinds, same arguments and results
 * as hs_decode_step with k_cache/v_cache replaced by the pools; p->t_kv as
 * for hs_sparse_attn_reuse_paged; the workspace of HS_DECODE_FULL_INDEX is
 * hs_workspace_size(p, HS_WS_DECODE_FULL) bytes.
 */
hs_status hs_decode_step_paged(const hs_params* p, const hs_pages* pages, int32_t kind,
                               const void* q, const void* k_pool, const void* v_pool,
                               const int32_t* seq_len, int32_t* idx, int32_t* idx_count,
                               void* o, float* lse, float* sel_scores, void* workspace,
                               size_t ws_bytes, void* stream);

/* Failure-detection diagnostic (the pages have no counterpart).  Every wait
 * of a kernel on another role of its CTA (a TMA copy, an MMA, a stage of the
 * pipeline) is bounded: after `cycles` SM clock cycles it gives up, records
 * HS_ERR_TIMEOUT in the device status word (read with hs_device_status),
 * and the CTA drains the copies and MMAs it has in flight, frees its tensor
 * memory and returns, leaving its outputs unspecified and the context usable.
 * This sets that bound for kernels launched afterwards on the current device;
 * cycles <= 0 restores the default of 2e9 (about a second).  Synchronous:
 * call it while no kernel of this library runs on the device.  Tests use a
 * bound of a few hundred cycles to make waits run out on purpose. */
hs_status hs_set_wait_limit(int64_t cycles);

/* Token-selection tuning (HySparse2 token mode, hs_full_attn_index with a
 * workspace; the selection itself is unchanged).  Before a long scan the
 * selector scores 2048 keys spread evenly over the range every position of a
 * work item ranks and starts from the rank-th best of them as its admission
 * threshold, so far fewer keys enter its candidate buffers.  If fewer than
 * k - w keys of a position pass that threshold (the threshold was too high,
 * which the automatic rank makes a below-1e-5 event) the work item is scanned
 * again without one, so the result never depends on this setting.
 * rank < 0: automatic (the default; a rank from the sample density), 0: off,
 * rank > 0: always that rank (tests use 1 to force the rescan).  Applies to
 * kernels launched afterwards on the current device; synchronous. */
hs_status hs_set_select_sampling(int32_t rank);

#ifdef __cplusplus
}
#endif

#endif /* HS_H_ */
