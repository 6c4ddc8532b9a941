// Expert parallelism: one shard of the experts per GPU.
//
// "Mixture of Experts (MoEs) in Transformers", section Expert Parallelism:
// the experts are split along their first dimension, each device holding E/N
// of them; the router's global expert indices are remapped to the device's
// local ones, the experts it does not hold are left out, and the devices'
// partial outputs are summed (an all-reduce).
//
// Two kernels here: the remap of the routing to shard-local expert ids (-1
// for another shard's expert, which the grouping then drops without counting
// it), and the sum of partial outputs in a fixed order with one rounding to
// the layer dtype (after the exchange, or over the shards of one device).
#include "common.cuh"

namespace moe {
namespace {

__global__ void remap_experts_kernel(const int32_t* __restrict__ idx, int64_t S, int begin, int count,
                                     int32_t* __restrict__ local) {
    for (int64_t s = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; s < S; s += (int64_t)gridDim.x * blockDim.x) {
        const int e = idx[s];
        local[s] = (e >= begin && e < begin + count) ? e - begin : -1;
    }
}

// Four consecutive elements per thread: partials [n][count] float32.
template <typename TOut>
__global__ void reduce_partials_kernel(const float* __restrict__ partials, int n, int64_t count,
                                       TOut* __restrict__ y) {
    const int64_t quads = count / 4;
    for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < quads; q += (int64_t)gridDim.x * blockDim.x) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int i = 0; i < n; ++i) {
            const float4 v = reinterpret_cast<const float4*>(partials + (int64_t)i * count)[q];
            acc.x += v.x;
            acc.y += v.y;
            acc.z += v.z;
            acc.w += v.w;
        }
        TOut* o = y + 4 * q;
        o[0] = from_f32<TOut>(acc.x);
        o[1] = from_f32<TOut>(acc.y);
        o[2] = from_f32<TOut>(acc.z);
        o[3] = from_f32<TOut>(acc.w);
    }
}

int blocks_for(int64_t n, int threads) {
    int64_t b = (n + threads - 1) / threads;
    if (b > 148 * 16) b = 148 * 16;
    return b < 1 ? 1 : (int)b;
}

}  // namespace

cudaError_t launch_remap_experts(const int32_t* idx, int64_t S, int begin, int count, int32_t* local,
                                 cudaStream_t st) {
    if (S == 0) return cudaSuccess;
    trace_before("remap_experts", st);
    remap_experts_kernel<<<blocks_for(S, 256), 256, 0, st>>>(idx, S, begin, count, local);
    trace_after(st);
    return cudaGetLastError();
}

cudaError_t launch_reduce_partials(const float* partials, int n, int64_t count, bool bf16_out, void* y,
                                   cudaStream_t st) {
    if (count == 0) return cudaSuccess;
    trace_before("reduce_partials", st);
    if (bf16_out)
        reduce_partials_kernel<bf16><<<blocks_for(count / 4, 256), 256, 0, st>>>(partials, n, count, (bf16*)y);
    else
        reduce_partials_kernel<float><<<blocks_for(count / 4, 256), 256, 0, st>>>(partials, n, count, (float*)y);
    trace_after(st);
    return cudaGetLastError();
}

}  // namespace moe
