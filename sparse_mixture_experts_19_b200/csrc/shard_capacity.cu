// Capacity left for one token shard of a capacity-limited batch.
//
// "MoE稀疏架构是什么？从原理到落地的系统解读", section 三.2: an expert takes
// tokens up to its capacity and the rest are dropped.  Tokens are served in
// global token order, so when a batch is split into shards by tokens, shard r
// may keep for expert e only what shards 0..r-1 left of the capacity C:
//   capacity_left[e] = max(0, C - sum_{q < r} counts_q[e]),
// counts_q being shard q's per-expert counts before the cut.  The same
// arithmetic runs on the device (counts gathered into device memory, one
// thread per expert) and on the host (counts gathered on the host).
#include "common.cuh"

namespace moe {
namespace {

__host__ __device__ __forceinline__ int32_t left_for(int64_t C, const int32_t* counts, int shard, int E, int e) {
    int64_t used = 0;
    for (int q = 0; q < shard; ++q) used += counts[(int64_t)q * E + e];
    const int64_t left = C - used;
    return left > 0 ? (int32_t)left : 0;
}

__global__ void __launch_bounds__(256) shard_capacity_left_kernel(int64_t C, const int32_t* __restrict__ counts,
                                                                  int shard, int E, int32_t* __restrict__ out) {
    for (int e = threadIdx.x; e < E; e += blockDim.x) out[e] = left_for(C, counts, shard, E, e);
}

}  // namespace

cudaError_t launch_shard_capacity_left(int64_t C, const int32_t* counts, int n_shards, int shard, int E,
                                       int32_t* capacity_left, cudaStream_t st) {
    (void)n_shards;
    trace_before("shard_capacity_left", st);
    shard_capacity_left_kernel<<<1, 256, 0, st>>>(C, counts, shard, E, capacity_left);
    trace_after(st);
    return cudaGetLastError();
}

void shard_capacity_left_host(int64_t C, const int32_t* counts, int n_shards, int shard, int E,
                              int32_t* capacity_left) {
    (void)n_shards;
    for (int e = 0; e < E; ++e) capacity_left[e] = left_for(C, counts, shard, E, e);
}

}  // namespace moe
