// Router for few tokens (decode): exact fp64 scores, warp top-k, softmax.
//
// "MoE稀疏架构是什么？从原理到落地的系统解读", section 三.1 (a small linear
// router scores every expert) and section 四 (top-k, softmax over the k).
//
// With few tokens the router is a matrix-vector product per token: the
// weights (E x H) stay in L2 and every SM can work on its own token.  One CTA
// per token: its 32 warps split the experts, the 32 lanes of a warp split H in
// 16-byte chunks (four in flight per lane), and each score is accumulated in
// fp64 (every product of two bf16 or float32 values is exact in fp64, so the
// scores are the exact sums up to fp64 rounding and the selection matches an
// fp64 reference except for ties closer than that).  Warp 0 then picks the k best by (score desc,
// index asc) with warp arg-max rounds and writes the softmax of those k.
#include "common.cuh"

namespace moe {
namespace {

constexpr int kWarps = 32;

template <typename TIn>
__device__ __forceinline__ void widen16(const uint4& q, double* out) {
    if constexpr (sizeof(TIn) == 2) {
        const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float2 f = __bfloat1622float2(p[i]);
            out[2 * i] = f.x;
            out[2 * i + 1] = f.y;
        }
    } else {
        const float* p = reinterpret_cast<const float*>(&q);
#pragma unroll
        for (int i = 0; i < 4; ++i) out[i] = p[i];
    }
}

template <typename TIn>
__global__ void __launch_bounds__(kWarps * 32) router_decode_kernel(
    int T, int H, int E, int k, const TIn* __restrict__ x, const TIn* __restrict__ wr,
    const float* __restrict__ b, int32_t* __restrict__ topk_idx, float* __restrict__ topk_w) {
    constexpr int V = 16 / sizeof(TIn);  // elements per 16-byte chunk
    __shared__ double sc[kMaxExperts];
    const int t = blockIdx.x;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int nch = H / V;
    const uint4* xr = reinterpret_cast<const uint4*>(x + (int64_t)t * H);

    for (int e = warp; e < E; e += kWarps) {
        const uint4* wrow = reinterpret_cast<const uint4*>(wr + (int64_t)e * H);
        // four 16-byte chunks per lane in flight, four accumulators
        double acc[4] = {0.0, 0.0, 0.0, 0.0};
        for (int c = lane; c < nch; c += 128) {
            uint4 xq[4], wq[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int cu = c + 32 * u;
                xq[u] = cu < nch ? xr[cu] : make_uint4(0, 0, 0, 0);
                wq[u] = cu < nch ? wrow[cu] : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                double fx[V], fw[V];
                widen16<TIn>(xq[u], fx);
                widen16<TIn>(wq[u], fw);
#pragma unroll
                for (int i = 0; i < V; ++i) acc[u] = fma(fx[i], fw[i], acc[u]);
            }
        }
        double s = (acc[0] + acc[1]) + (acc[2] + acc[3]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) sc[e] = s + (b ? (double)b[e] : 0.0);
    }
    __syncthreads();
    if (warp != 0) return;

    // k rounds of warp arg-max; round j takes the best ranking after pick j-1
    double pv = INFINITY;
    int pe = -1;
    double sel_v[kMaxTopK];
    int sel_e[kMaxTopK];
    for (int j = 0; j < k; ++j) {
        double bv = -INFINITY;
        int be = 0x7fffffff;
        for (int e = lane; e < E; e += 32) {
            const double v = sc[e];
            const bool after = (v < pv) || (v == pv && e > pe);
            if (after && (v > bv || (v == bv && e < be))) {
                bv = v;
                be = e;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const double ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oe = __shfl_xor_sync(0xffffffffu, be, o);
            if (ov > bv || (ov == bv && oe < be)) {
                bv = ov;
                be = oe;
            }
        }
        sel_v[j] = bv;
        sel_e[j] = be;
        pv = bv;
        pe = be;
    }
    if (lane == 0) {
        // softmax over the k selected, differences taken in fp64
        float z = 0.f;
        for (int j = 0; j < k; ++j) z += expf((float)(sel_v[j] - sel_v[0]));
        const float inv = 1.0f / z;
        for (int j = 0; j < k; ++j) {
            topk_idx[(int64_t)t * k + j] = sel_e[j];
            topk_w[(int64_t)t * k + j] = expf((float)(sel_v[j] - sel_v[0])) * inv;
        }
    }
}

}  // namespace

cudaError_t launch_router_decode(const Plan& p, const void* x, const void* router_w, const float* router_b,
                                 int32_t* topk_idx, float* topk_w, cudaStream_t st) {
    if (p.T == 0) return cudaSuccess;
    trace_before("router_decode", st);
    if (p.bf16)
        router_decode_kernel<bf16><<<(unsigned)p.T, kWarps * 32, 0, st>>>(
            (int)p.T, (int)p.H, (int)p.E, (int)p.k, (const bf16*)x, (const bf16*)router_w, router_b, topk_idx,
            topk_w);
    else
        router_decode_kernel<float><<<(unsigned)p.T, kWarps * 32, 0, st>>>(
            (int)p.T, (int)p.H, (int)p.E, (int)p.k, (const float*)x, (const float*)router_w, router_b,
            topk_idx, topk_w);
    trace_after(st);
    return cudaGetLastError();
}

}  // namespace moe
