// Router for few tokens (decode): exact scores, warp top-k, softmax.
//
// "MoE稀疏架构是什么？从原理到落地的系统解读", section 三.1 (a small linear
// router scores every expert) and section 四 (top-k, softmax over the k).
//
// With few tokens the router is a matrix-vector product per token.  Each
// token gets a thread-block cluster of C CTAs (C <= 8); CTA r scores experts
// [r*epc, (r+1)*epc) with one warp per expert at a time, the 32 lanes of a
// warp splitting H in 16-byte chunks (twelve in flight per lane).  Scores are
// exact up to fp64 rounding: for bf16 inputs each product of two bf16 values
// is exact in float32 (8-bit by 8-bit significands, for |product| in
// [2^-126, 2^128)) and is summed in fp64; float32 inputs are multiplied in
// fp64.  So the selection matches an fp64 reference except for ties closer
// than that.  After a cluster barrier, warp 0 of CTA 0 gathers all E scores
// through distributed shared memory, picks the k best by (score desc, index
// asc) with warp arg-max rounds and writes the softmax of those k; a second
// cluster barrier keeps the other CTAs' shared memory alive until then.
// When asked, the same warp adds the token's softmax over all E scores
// (fp64, from the exact scores) to the per-expert importance.
#include <algorithm>

#include "common.cuh"
#include "sm100.cuh"

namespace moe {
namespace {

using namespace sm100;

constexpr int kWarps = 8;
constexpr int kMaxCluster = 8;
constexpr int kExpertsPerWarpRound = kWarps;
constexpr int kRound = 12;  // 16-byte chunks per lane in flight

__device__ __forceinline__ double ld_dsmem_f64(uint32_t addr) {
    double v;
    asm volatile("ld.shared::cluster.f64 %0, [%1];" : "=d"(v) : "r"(addr) : "memory");
    return v;
}

// x . w over one 16-byte chunk, added to acc (fp64).
__device__ __forceinline__ void chunk_dot(const uint4& xq, const uint4& wq, double& acc, __nv_bfloat16) {
    const __nv_bfloat162* xp = reinterpret_cast<const __nv_bfloat162*>(&xq);
    const __nv_bfloat162* wp = reinterpret_cast<const __nv_bfloat162*>(&wq);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 xf = __bfloat1622float2(xp[i]);
        const float2 wf = __bfloat1622float2(wp[i]);
        // exact float32 products, summed in fp64
        acc += (double)__fmul_rn(xf.x, wf.x);
        acc += (double)__fmul_rn(xf.y, wf.y);
    }
}
__device__ __forceinline__ void chunk_dot(const uint4& xq, const uint4& wq, double& acc, float) {
    const float* xp = reinterpret_cast<const float*>(&xq);
    const float* wp = reinterpret_cast<const float*>(&wq);
#pragma unroll
    for (int i = 0; i < 4; ++i) acc = fma((double)xp[i], (double)wp[i], acc);
}

template <typename TIn>
__global__ void __launch_bounds__(kWarps * 32) router_decode_kernel(
    int T, int H, int E, int k, int C, int epc, const TIn* __restrict__ x, const TIn* __restrict__ wr,
    const float* __restrict__ b, int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
    float* __restrict__ importance) {
    constexpr int V = 16 / sizeof(TIn);  // elements per 16-byte chunk
    __shared__ double sc[kMaxExperts];   // this CTA's scores; CTA 0 gathers all E here
    const int t = blockIdx.x / C;  // clusters of C consecutive CTAs along x, one per token
    const uint32_t rank = cluster_ctarank();
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int nch = H / V;
    const uint4* xr = reinterpret_cast<const uint4*>(x + (int64_t)t * H);
    const int e0 = (int)rank * epc, e1 = min(E, e0 + epc);

    for (int e = e0 + warp; e < e1; e += kExpertsPerWarpRound) {
        const uint4* wrow = reinterpret_cast<const uint4*>(wr + (int64_t)e * H);
        // up to kRound chunks per lane loaded before any is used (one round
        // of memory latency for H up to 32 * kRound chunks)
        double acc[4] = {0.0, 0.0, 0.0, 0.0};
        for (int c = lane; c < nch; c += 32 * kRound) {
            uint4 xq[kRound], wq[kRound];
#pragma unroll
            for (int u = 0; u < kRound; ++u) {
                const int cu = c + 32 * u;
                xq[u] = cu < nch ? xr[cu] : make_uint4(0, 0, 0, 0);
                wq[u] = cu < nch ? wrow[cu] : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < kRound; ++u) chunk_dot(xq[u], wq[u], acc[u % 4], TIn());
        }
        double s = (acc[0] + acc[1]) + (acc[2] + acc[3]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) sc[e - e0] = s + (b ? (double)b[e] : 0.0);
    }
    cluster_sync();
    if (rank == 0 && warp == 0) {
        // gather the other CTAs' scores behind this CTA's own (same offsets)
        for (int e = epc + lane; e < E; e += 32) {
            const uint32_t r = (uint32_t)(e / epc);
            sc[e] = ld_dsmem_f64(mapa_shared(smem_u32(&sc[e - (int)r * epc]), r));
        }
        __syncwarp();
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
        if (importance) {
            // softmax over all E scores, shifted by the largest (sel_v[0])
            double z = 0.0;
            for (int e = lane; e < E; e += 32) z += exp(sc[e] - sel_v[0]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
            for (int e = lane; e < E; e += 32) atomicAdd(&importance[e], (float)(exp(sc[e] - sel_v[0]) / z));
        }
    }
    cluster_sync();  // CTA 0 has read every CTA's scores
}

template <typename TIn>
cudaError_t launch_typed(const Plan& p, const void* x, const void* router_w, const float* router_b,
                         int32_t* topk_idx, float* topk_w, cudaStream_t st) {
    // C CTAs per token, each scoring epc experts (at most 8 per warp round)
    const int E = (int)p.E;
    const int C = std::min(kMaxCluster, (E + kExpertsPerWarpRound - 1) / kExpertsPerWarpRound);
    const int epc = (E + C - 1) / C;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(C * p.T), 1, 1);
    cfg.blockDim = dim3(kWarps * 32, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, router_decode_kernel<TIn>, (int)p.T, (int)p.H, E, (int)p.k, C, epc,
                              (const TIn*)x, (const TIn*)router_w, router_b, topk_idx, topk_w, p.importance);
}

}  // namespace

cudaError_t launch_router_decode(const Plan& p, const void* x, const void* router_w, const float* router_b,
                                 int32_t* topk_idx, float* topk_w, cudaStream_t st) {
    if (p.T == 0) return cudaSuccess;
    trace_before("router_decode", st);
    cudaError_t e = p.bf16 ? launch_typed<bf16>(p, x, router_w, router_b, topk_idx, topk_w, st)
                           : launch_typed<float>(p, x, router_w, router_b, topk_idx, topk_w, st);
    trace_after(st);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace moe
