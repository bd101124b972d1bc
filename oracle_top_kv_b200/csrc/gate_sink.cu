// gate_sink.cu -- output of a sparse layer: per-head sinks and the sigmoid-gate
// fusion of its two branches, in one elementwise pass.
//
// "HySparse 混合稀疏注意力（一）" (the section on the two sigmoid gates) and
// "HySparse: ..." 3.3 (branch fusion): the global (block-sparse) and local
// (window) branch outputs each pass through an input-dependent sigmoid gate
// and are added,
//     o = sigmoid(z_G) * o_global' + sigmoid(z_L) * o_local',
// and, per the configuration notes of both papers, the sparse and window
// branches carry a learnable per-head sink bias (the gpt-oss construction):
// one more logit s_h in the branch's softmax with a zero value vector, so
//     o_x' = o_x * e^lse_x / (e^lse_x + e^s_x),  lse_x' = log(e^lse_x + e^s_x).
// Gates act per head (one pre-activation per row and head, supplied by the
// caller: the projection W_g x_t belongs to the model).
//
// One thread per 16 bytes of a row (8 bf16 or 4 fp32 channels); o may be
// o_global or o_local (each thread reads its 16 bytes before writing them).  A row's
// threads are consecutive and lie in one warp (32 is a multiple of d/8 and
// d/4 for d in {64, 128}), so the lse update is a warp-synchronous
// read-then-write.  Roofline: HBM -- the two branch outputs read once, the
// fused output written once.
#include "hs_common.cuh"
#include "hs_kernels.cuh"

namespace hs {
namespace gs {

template <typename T> struct Vec;
template <> struct Vec<__nv_bfloat16> {
    static constexpr int kN = 8;
    __device__ static void load(const __nv_bfloat16* p, float (&x)[8]) {
        const uint4 u = *reinterpret_cast<const uint4*>(p);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162*>(&w[i]);
            const float2 f = __bfloat1622float2(h);
            x[2 * i] = f.x;
            x[2 * i + 1] = f.y;
        }
    }
    __device__ static void store(__nv_bfloat16* p, const float (&x)[8]) {
        uint4 u;
        u.x = pack_bf16(x[0], x[1]);
        u.y = pack_bf16(x[2], x[3]);
        u.z = pack_bf16(x[4], x[5]);
        u.w = pack_bf16(x[6], x[7]);
        *reinterpret_cast<uint4*>(p) = u;
    }
};
template <> struct Vec<float> {
    static constexpr int kN = 4;
    __device__ static void load(const float* p, float (&x)[4]) {
        const float4 u = *reinterpret_cast<const float4*>(p);
        x[0] = u.x; x[1] = u.y; x[2] = u.z; x[3] = u.w;
    }
    __device__ static void store(float* p, const float (&x)[4]) {
        *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
    }
};

// log(e^a + e^b), -inf when both are -inf.
__device__ __forceinline__ float log_add_exp(float a, float b) {
    const float m = fmaxf(a, b);
    if (m == -INFINITY) return -INFINITY;
    return m + logf(expf(a - m) + expf(b - m));
}

// Share of the branch's softmax mass on its keys once the sink joins
// (e^lse / (e^lse + e^s)), and the updated lse.  No sink: 1 and lse.
__device__ __forceinline__ float sink_share(float lse, const float* sink, int h, float* lse_new) {
    if (!sink) { *lse_new = lse; return 1.f; }
    const float l2 = log_add_exp(lse, sink[h]);
    *lse_new = l2;
    return l2 == -INFINITY ? 0.f : expf(lse - l2);
}

__device__ __forceinline__ float sigmoid(float z) { return 1.f / (1.f + expf(-z)); }

struct Args {
    long long rows;  // batch * hq * t_q
    int hq, t_q, d;
    float* lse_g;
    float* lse_l;
    const float* sink_g;
    const float* sink_l;
    const float* z_g;
    const float* z_l;
};

template <typename T>
__global__ void __launch_bounds__(256) gate_sink_kernel(const T* o_g, const T* o_l, T* o, Args a) {
    constexpr int V = Vec<T>::kN;
    const int chunks = a.d / V;
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long row = idx / chunks;
    const int c = (int)(idx % chunks);
    const bool live = row < a.rows;
    const int h = live ? (int)((row / a.t_q) % a.hq) : 0;
    // every thread of the row reads the old lse before chunk 0 writes the new
    float fg = 0.f, fl = 0.f, lg_new = 0.f, ll_new = 0.f;
    if (live) {
        fg = sink_share(a.lse_g[row], a.sink_g, h, &lg_new);
        if (o_l) fl = sink_share(a.lse_l[row], a.sink_l, h, &ll_new);
        if (a.z_g) fg *= sigmoid(a.z_g[row]);
        if (o_l && a.z_l) fl *= sigmoid(a.z_l[row]);
    }
    __syncwarp();
    if (!live) return;
    if (c == 0) {
        a.lse_g[row] = lg_new;
        if (o_l) a.lse_l[row] = ll_new;
    }
    const size_t off = (size_t)row * a.d + (size_t)c * V;
    float x[V], y[V];
    Vec<T>::load(o_g + off, x);
#pragma unroll
    for (int i = 0; i < V; ++i) x[i] *= fg;
    if (o_l) {
        Vec<T>::load(o_l + off, y);
#pragma unroll
        for (int i = 0; i < V; ++i) x[i] += fl * y[i];
    }
    Vec<T>::store(o + off, x);
}

}  // namespace gs

cudaError_t launch_gate_sink(const KParams& p, int dtype, const void* o_g, float* lse_g,
                             const void* o_l, float* lse_l, const float* sink_g,
                             const float* sink_l, const float* z_g, const float* z_l, void* o,
                             cudaStream_t st) {
    gs::Args a;
    a.rows = (long long)p.batch * p.hq * p.t_q;
    a.hq = p.hq;
    a.t_q = p.t_q;
    a.d = p.head_dim;
    a.lse_g = lse_g;
    a.lse_l = lse_l;
    a.sink_g = sink_g;
    a.sink_l = sink_l;
    a.z_g = z_g;
    a.z_l = z_l;
    const int V = dtype == HS_BF16 ? 8 : 4;
    const long long threads = a.rows * (p.head_dim / V);
    const long long blocks = (threads + 255) / 256;
    if (dtype == HS_BF16)
        gs::gate_sink_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, st>>>(
            (const __nv_bfloat16*)o_g, (const __nv_bfloat16*)o_l, (__nv_bfloat16*)o, a);
    else
        gs::gate_sink_kernel<float><<<(unsigned)blocks, 256, 0, st>>>(
            (const float*)o_g, (const float*)o_l, (float*)o, a);
    return cudaGetLastError();
}

}  // namespace hs
