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
// The array exists once per device for as long as the library stays loaded
// (every GPU that loads the library holds it until exit).  Host code cannot
// pass the array's name to a kernel -- on the host it is only a stand-in, not
// a device address -- so the first call on each device looks up the real
// address with cudaGetSymbolAddress while that device is current, and
// caches it.  All calls on a device share the array: two calls whose kernels
// overlap on the GPU (different streams, no ordering between them) race on
// it and must not be issued.  No state carries over between calls: every
// scratch entry a call reads was written earlier in the same call, so nothing
// needs clearing.
#include <mutex>

#include "hs_common.cuh"
#include "hs_kernels.cuh"

namespace hs {

// 32 MiB of float partials: (sequence, kv group, 64-row split) units of
// 16 x (head_dim + 2) floats each -- 4032 units at head_dim 128, enough for
// 32 sequences x 4 kv groups x 1024 selected tokens.
constexpr size_t kNoAllocScratchFloats = (size_t)8 << 20;
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchFloats];

constexpr int kMaxDevices = 64;
static void* g_noalloc_ptr[kMaxDevices];
static std::mutex g_noalloc_mu;

// Device address of the scratch array on the current device (set up once).
static cudaError_t noalloc_scratch(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void* ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_noalloc_ptr[dev] = ptr;
    }
    *out = g_noalloc_ptr[dev];
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
