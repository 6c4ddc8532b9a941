// Router scores + top-k + softmax over the selected scores, CUDA-core version.
//
// "MoE稀疏架构是什么？从原理到落地的系统解读", section 三.1 (a small linear
// router gives one score per expert) and section 四 (keep the top-k scores,
// softmax over those k).  This kernel serves the float32 layer (tensor cores
// would round the inputs).  Scores are exact up to fp64 rounding: a product
// of two float32 values is exact in fp64 (24-bit by 24-bit significands), and
// the products are summed with fp64 FMAs, so the selection (ties to the lower
// index) matches an fp64 evaluation of the scores except for scores closer
// than that rounding.
//
// One block scores 16 tokens against all E experts: x and router-weight
// chunks of 32 columns are staged in shared memory as float; each thread owns
// up to 16 (token, expert) fp64 accumulators.  The scores then go to shared
// memory (fp64) and each warp selects the top-k of 2 tokens with warp
// arg-max rounds.
// When asked, each warp also forms its tokens' softmax over all E scores; the
// block sums them per expert in shared memory and adds the sums to the
// importance in global memory.
#include "common.cuh"

namespace moe {
namespace {

constexpr int kTB = 16;  // tokens per block
constexpr int kHC = 32;  // hidden columns per chunk
constexpr int kThreads = 256;

// Warp-wide arg-max of (v, e): larger v wins, equal v -> lower e wins.
__device__ __forceinline__ void warp_argmax(double& v, int& e) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        double ov = __shfl_xor_sync(0xffffffffu, v, o);
        int oe = __shfl_xor_sync(0xffffffffu, e, o);
        if (ov > v || (ov == v && oe < e)) {
            v = ov;
            e = oe;
        }
    }
}

template <typename TIn>
__global__ void __launch_bounds__(kThreads) router_simt_kernel(
    int T, int H, int E, int k, const TIn* __restrict__ x, const TIn* __restrict__ wr,
    const float* __restrict__ b, int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
    float* __restrict__ importance) {
    __shared__ float xs[kTB][kHC + 1];
    __shared__ float imp[kMaxExperts];  // this block's importance, when asked
    // weights chunk [E][kHC+1] (float) during the scores, then the scores
    // [kTB][E+1] (fp64); both fit in the same bytes
    static_assert(kTB * (kMaxExperts + 1) * sizeof(double) <= kMaxExperts * (kHC + 1) * sizeof(float) + 256,
                  "score buffer must fit in the staging buffer");
    __shared__ __align__(16) float buf[kMaxExperts * (kHC + 1) + 64];
    double* sc = reinterpret_cast<double*>(buf);

    const int tid = threadIdx.x;
    const int t0 = blockIdx.x * kTB;
    for (int e = tid; e < kMaxExperts; e += kThreads) imp[e] = 0.f;  // ordered by the loop's barriers
    const int P = kTB * E;  // (token, expert) pairs of this block

    double acc[kTB * kMaxExperts / kThreads];
#pragma unroll
    for (int i = 0; i < kTB * kMaxExperts / kThreads; ++i) acc[i] = 0.0;

    for (int h0 = 0; h0 < H; h0 += kHC) {
        for (int q = tid; q < kTB * kHC; q += kThreads) {
            int r = q / kHC, c = q % kHC;
            int t = t0 + r, h = h0 + c;
            xs[r][c] = (t < T && h < H) ? to_f32(x[(int64_t)t * H + h]) : 0.f;
        }
        for (int q = tid; q < E * kHC; q += kThreads) {
            int r = q / kHC, c = q % kHC;
            int h = h0 + c;
            buf[r * (kHC + 1) + c] = (h < H) ? to_f32(wr[(int64_t)r * H + h]) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int i = 0; i < kTB * kMaxExperts / kThreads; ++i) {
            int p = tid + i * kThreads;
            if (p < P) {
                int r = p / E, e = p % E;
                double s = acc[i];
#pragma unroll 8
                for (int c = 0; c < kHC; ++c) s = fma((double)xs[r][c], (double)buf[e * (kHC + 1) + c], s);
                acc[i] = s;
            }
        }
        __syncthreads();
    }

    // scores -> shared memory (bias added here, before selection)
#pragma unroll
    for (int i = 0; i < kTB * kMaxExperts / kThreads; ++i) {
        int p = tid + i * kThreads;
        if (p < P) {
            int r = p / E, e = p % E;
            sc[r * (E + 1) + e] = acc[i] + (b ? (double)b[e] : 0.0);
        }
    }
    __syncthreads();

    const int warp = tid / 32, lane = tid % 32;
    for (int r = warp; r < kTB; r += kThreads / 32) {
        int t = t0 + r;
        if (t >= T) break;
        const double* l = sc + r * (E + 1);
        // each lane holds experts lane, lane+32, ...; taken bits mark chosen ones
        uint32_t taken = 0;
        double sel_v[kMaxTopK];
        int sel_e[kMaxTopK];
        for (int j = 0; j < k; ++j) {
            double bv = -INFINITY;
            int be = 0x7fffffff;
            for (int q = 0; q * 32 + lane < E; ++q) {
                int e = q * 32 + lane;
                double v = l[e];
                if (!((taken >> q) & 1u) && (v > bv || (v == bv && e < be))) {
                    bv = v;
                    be = e;
                }
            }
            warp_argmax(bv, be);
            if ((be & 31) == lane) taken |= 1u << (be >> 5);
            sel_v[j] = bv;
            sel_e[j] = be;
        }
        if (lane == 0) {
            // softmax over the k selected, differences taken in fp64
            float z = 0.f;
            for (int j = 0; j < k; ++j) z += expf((float)(sel_v[j] - sel_v[0]));
            float inv = 1.0f / z;
            for (int j = 0; j < k; ++j) {
                topk_idx[(int64_t)t * k + j] = sel_e[j];
                topk_w[(int64_t)t * k + j] = expf((float)(sel_v[j] - sel_v[0])) * inv;
            }
        }
        if (importance) {
            // softmax over all E scores, shifted by the largest (sel_v[0])
            float z = 0.f;
            for (int e = lane; e < E; e += 32) z += expf((float)(l[e] - sel_v[0]));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
            const float inv = 1.0f / z;
            for (int e = lane; e < E; e += 32) atomicAdd(&imp[e], expf((float)(l[e] - sel_v[0])) * inv);
        }
    }
    if (importance) {
        __syncthreads();
        for (int e = tid; e < E; e += kThreads) atomicAdd(&importance[e], imp[e]);
    }
}

}  // namespace

cudaError_t launch_router_simt(const Plan& p, const void* x, const void* router_w,
                               const float* router_b, int32_t* topk_idx, float* topk_w,
                               cudaStream_t st) {
    if (p.T == 0) return cudaSuccess;
    dim3 grid((unsigned)((p.T + kTB - 1) / kTB));
    trace_before("router_simt", st);
    router_simt_kernel<float><<<grid, kThreads, 0, st>>>((int)p.T, (int)p.H, (int)p.E, (int)p.k,
                                                         (const float*)x, (const float*)router_w,
                                                         router_b, topk_idx, topk_w, p.importance);
    trace_after(st);
    return cudaGetLastError();
}

}  // namespace moe
