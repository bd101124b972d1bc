// noalloc.cu -- the sparse decode step for callers that cannot allocate
// device memory.
//
// Some callers are handed only their input and output buffers: a plugin
// inside an inference engine whose memory planner owns every device byte, or
// a latency-critical decode loop where a cudaMalloc (which can synchronise
// the device) is not allowed.  This entry point runs the split-k form of the
// sparse decode step (a split kernel writing per-split partials, then a
// combine kernel) with its scratch in a fixed file-scope device array instead
// of a caller workspace; it allocates nothing.
//
// The array exists once per device context for as long as the library stays
// loaded (every GPU that loads the library holds it until exit).  Host code
// cannot pass the array's name to a kernel -- on the host it is only a
// stand-in, not a device address -- so the first call in each CUDA context
// looks up the real address with cudaGetSymbolAddress while that context is
// current, and caches it under the context's unique id (cuCtxGetId).  A new
// context (another driver context on the same device, or the primary context
// re-created after cudaDeviceReset) has its own copy of the array at another
// address and gets a lookup of its own.  Make the first call in a context
// before any stream capture.  All calls in a context share the array: two
// calls whose kernels overlap on the GPU (different streams, no ordering
// between them) race on it and must not be issued.  No state carries over
// between calls: every scratch entry a call reads was written earlier in the
// same call, so nothing needs clearing.
#include <cuda.h>

#include <mutex>

#include "hs_common.cuh"
#include "hs_kernels.cuh"

namespace hs {

// 32 MiB of float partials: (sequence, kv group, 64-row split) units of
// 16 x (head_dim + 2) floats each -- 4032 units at head_dim 128, enough for
// 32 sequences x 4 kv groups x 1024 selected tokens.
constexpr size_t kNoAllocScratchFloats = (size_t)8 << 20;
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchFloats];

// (context id, scratch address) pairs of the contexts seen so far.
constexpr int kMaxContexts = 64;
static unsigned long long g_noalloc_ctx[kMaxContexts];
static void* g_noalloc_ptr[kMaxContexts];
static int g_noalloc_n = 0, g_noalloc_evict = 0;
static std::mutex g_noalloc_mu;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Unique id of the current CUDA context (the device's primary context is
// made current first, as every runtime call would).
static cudaError_t current_context_id(unsigned long long* id) {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    if (!get_current || !get_id) {
        void* f1 = nullptr;
        void* f2 = nullptr;
        cudaDriverEntryPointQueryResult q1, q2;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) !=
                cudaSuccess || q1 != cudaDriverEntryPointSuccess ||
            cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) != cudaSuccess ||
            q2 != cudaDriverEntryPointSuccess)
            return cudaErrorNotSupported;
        get_current = reinterpret_cast<CtxGetCurrentFn>(f1);
        get_id = reinterpret_cast<CtxGetIdFn>(f2);
    }
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    e = cudaSetDevice(dev);  // binds (and if needed creates) the primary context
    if (e != cudaSuccess) return e;
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return cudaErrorDeviceUninitialized;
    if (get_id(ctx, id) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
    return cudaSuccess;
}

// Device address of the scratch array in the current context (looked up once
// per context).
static cudaError_t noalloc_scratch(void** out) {
    unsigned long long id = 0;
    cudaError_t e = current_context_id(&id);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    for (int i = 0; i < g_noalloc_n; ++i)
        if (g_noalloc_ctx[i] == id) {
            *out = g_noalloc_ptr[i];
            return cudaSuccess;
        }
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    // a full table keeps working: its entries are replaced in turn
    const int slot = g_noalloc_n < kMaxContexts ? g_noalloc_n++ : g_noalloc_evict++ % kMaxContexts;
    g_noalloc_ctx[slot] = id;
    g_noalloc_ptr[slot] = ptr;
    *out = ptr;
    return cudaSuccess;
}

size_t noalloc_scratch_bytes() { return kNoAllocScratchFloats * sizeof(float); }

cudaError_t launch_decode_sparse_noalloc(const KParams& p, const void* q, const void* kc,
                                         const void* vc, const int32_t* seq_len,
                                         const int32_t* idx, const int32_t* cnt, void* o,
                                         float* lse, cudaStream_t st) {
    void* scratch = nullptr;
    cudaError_t e = noalloc_scratch(&scratch);
    if (e != cudaSuccess) return e;
    return launch_decode_sparse_split(p, q, kc, vc, seq_len, idx, cnt, o, lse, scratch, st);
}

}  // namespace hs
