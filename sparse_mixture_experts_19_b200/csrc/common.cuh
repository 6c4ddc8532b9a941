// Shared definitions of the MoE layer's CUDA path (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

typedef __nv_bfloat16 bf16;

constexpr int kMaxTopK = 32;     // k <= 8, or k == E <= 32 (dense case)
constexpr int kMaxExperts = 256;
constexpr int kPermuteChunk = 2048;  // slots per histogram chunk in moe_permute
constexpr int kWsAlign = 256;
constexpr int kGemmTileRows = 128;  // rows per tile of the tcgen05 grouped GEMMs
constexpr int64_t kNoAllocMaxSlots = 1 << 20;  // T*k limit of moe_permute_noalloc
constexpr int kDecodeMaxSlots = 8;             // T*k limit of the decode layer on bf16 experts
constexpr int kDecodeMaxSlotsMx = 32;          // T*k limit of the decode layer on MXFP4 experts
constexpr int kDecodeCounters = 2 + kDecodeMaxSlotsMx;  // decode layer: grid barrier + one per expert group
constexpr int kRouterMaxSplits = 8;            // reduction chunks of the tensor-core router

// Everything the kernels of one call need, carved out of the caller's workspace.
struct Plan {
    int64_t T, H, I, E, k, Is, S;  // S = T*k slots
    int64_t cap;                   // 0 = unlimited
    const int32_t* cap_left_arr;   // [E] device or null: capacity left per expert (token shards)
    float* importance;             // [E] device or null: router importance, added to
    bool bf16;
    bool drop_negative;            // expert index -1 = another shard's expert: dropped, not counted, no flag
    bool y_f32;                    // y is a float32 partial sum (expert shards), not the layer dtype
    int64_t nchunks;               // ceil(S / kPermuteChunk)
    int64_t h_rows;                // S + (Is ? T : 0)
    int64_t I_max;                 // max(I, Is)

    int32_t* flags;       // [16] device check flags (flags[0] = MOE_DEVFLAG_*)
    int32_t* topk_idx;    // [S]
    float* topk_w;        // [S]
    int32_t* chunk_base;  // [nchunks * E]
    int32_t* counts;      // [E]
    int32_t* dropped;     // [E]
    int32_t* offsets;     // [E + 2]: routed rows, offsets[E+1] = offsets[E] + shared rows
    int32_t* mtile_prefix;  // [E + 1]: prefix over experts of ceil(kept rows / 128)
    int32_t* mpair_prefix;  // [E + 1]: prefix over experts of ceil(kept rows / 256)
    int32_t* perm_rows;   // [S]
    int32_t* row_of;      // [S]
    void* xperm;          // [S, H] layer dtype: x rows in grouped order
    void* h;              // [S, I] + [T, Is] layer dtype: SwiGLU activations
    void* rows;           // [S + T, H] layer dtype: routing-weighted expert output rows
    float* rt_part;       // tensor-core router: [splits, T, E] float32 partial scores
    float* rt_xn2;        // [splits, T] squared norms of the x rows over each chunk
    float* rt_wn2;        // [splits, E] squared norms of the router rows over each chunk
    double* dec_scores;   // decode layer (S <= kDecodeMaxSlotsMx): [T, E] router scores
    unsigned int* dec_bar;  // decode layer: [kDecodeCounters] arrival counters
    size_t bytes;         // total workspace bytes
};

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(bf16 v) { return __bfloat162float(v); }
template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ bf16 from_f32<bf16>(float v) { return __float2bfloat16_rn(v); }

// silu(z) = z * sigmoid(z) = z / (1 + e^-z), float32.
__device__ __forceinline__ float silu_f32(float z) { return z / (1.0f + __expf(-z)); }

__device__ __forceinline__ void set_flag(int32_t* flags, int32_t bit) { atomicOr(flags, bit); }

// Capacity of expert e when cap > 0: the per-expert capacity left for this
// token shard when given (the batch's capacity minus the rows of e that
// earlier shards kept; capacity is served in global token order), else cap.
__device__ __forceinline__ int64_t cap_left(int64_t cap, const int32_t* cap_left_arr, int e) {
    const int64_t left = cap_left_arr ? (int64_t)cap_left_arr[e] : cap;
    return left > 0 ? left : 0;
}

// ---- launchers (defined in the .cu files; return the launch error) ------
// Router for the float32 layer (CUDA cores, float32 FMAs).
cudaError_t launch_router_simt(const Plan& p, const void* x, const void* router_w,
                               const float* router_b, int32_t* topk_idx, float* topk_w,
                               cudaStream_t st);
// Router for the bf16 layer (tcgen05; float32 TMEM scores, exact fp64
// rescoring of near-boundary experts).
cudaError_t launch_router_sm100(const Plan& p, const void* x, const void* router_w,
                                const float* router_b, int32_t* topk_idx, float* topk_w,
                                cudaStream_t st);
// Reduction chunks of the tensor-core router for hidden size H.
void router_splits(int64_t H, int* ns, int* kchunk);
// Router for few tokens: one CTA per token, exact fp64 scores.
cudaError_t launch_router_decode(const Plan& p, const void* x, const void* router_w,
                                 const float* router_b, int32_t* topk_idx, float* topk_w,
                                 cudaStream_t st);
// Scores of T*E*H at most this many multiply-adds go to the per-token router
// (its weight traffic, T*E*H*2 bytes from L2, stays small).
constexpr int64_t kDecodeRouterMaxMacs = int64_t(1) << 26;
// Decode layer (bf16, T*k <= kDecodeMaxSlots): routing (unless given), the
// expert FFNs and the weighted combine in one cooperative weight-streaming
// kernel, y written directly; also writes counts and dropped, and
// topk_idx_out when non-null.
bool decode_ffn_eligible(const Plan& p);
// The MXFP4 variant's size limit (T*k <= kDecodeMaxSlotsMx, shared memory).
bool decode_mxfp4_eligible(const Plan& p);
cudaError_t launch_decode_layer(const Plan& p, const void* x, const void* router_w, const float* router_b,
                                const int32_t* topk_idx_in, const float* topk_w_in, int32_t* topk_idx_out,
                                const void* w_gate, const void* w_up, const void* w_down, const void* ws_gate,
                                const void* ws_up, const void* ws_down, void* y, int32_t* counts,
                                int32_t* dropped, cudaStream_t st);
// The same with the routed experts in MXFP4 (no shared expert; H, I multiples
// of 32): mx = {gate blocks, gate scales, up blocks, up scales, down blocks,
// down scales}.
cudaError_t launch_decode_layer_mxfp4(const Plan& p, const void* x, const void* router_w, const float* router_b,
                                      int32_t* topk_idx_out, const uint8_t* const (&mx)[6], void* y, int32_t* counts,
                                      int32_t* dropped, cudaStream_t st);
// MXFP4 rows (blocks [rows, K/32, 16], scales [rows, K/32]; K a multiple of
// 32) -> bf16 rows [rows, K] at out (16-byte aligned), exact within bf16's range.
cudaError_t launch_mxfp4_dequant(const uint8_t* blocks, const uint8_t* scales, int64_t rows, int K, void* out,
                                 cudaStream_t st);
cudaError_t launch_permute(const Plan& p, const int32_t* topk_idx, int32_t* counts,
                           int32_t* offsets, int32_t* perm_rows, int32_t* row_of,
                           int32_t* dropped, cudaStream_t st);
// moe_permute with the scratch in a static device array; sizes.S <= kNoAllocMaxSlots.
cudaError_t launch_permute_noalloc(const Plan& sizes, const int32_t* topk_idx, int32_t* counts,
                                   int32_t* offsets, int32_t* perm_rows, int32_t* row_of,
                                   int32_t* dropped, cudaStream_t st);
// plan offsets [E+2] from a caller's offsets [E+1] (appends the shared rows).
cudaError_t launch_offsets_from_user(const Plan& p, const int32_t* offsets, cudaStream_t st);
// xperm rows built token by token from row_of [T, k] (x read once).
cudaError_t launch_scatter_x_rows(const Plan& p, const void* x, const int32_t* row_of, void* xperm,
                                  cudaStream_t st);
cudaError_t launch_gather_rows(const Plan& p, const void* x, const int32_t* perm_rows,
                               const int32_t* offsets, void* xperm, cudaStream_t st);
// Grouped expert GEMMs for all groups (routed + shared):
//   gate/up: h = silu(X W_g^T) * (X W_u^T), rounded to the layer dtype;
//   down:    mode 0 stores unweighted float32 rows h W_d^T to `out` [S + T, H];
//            mode 1 stores topk_w-weighted rows in the layer dtype to `out`
//            (shared rows with weight 1).
// float32 layer: CUDA cores (exact FMAs); bf16 layer: tcgen05 + TMEM + TMA.
cudaError_t launch_gateup_simt(const Plan& p, const void* xperm, const void* x,
                               const int32_t* offsets, const void* w_gate, const void* w_up,
                               const void* ws_gate, const void* ws_up, void* h, cudaStream_t st);
cudaError_t launch_down_simt(const Plan& p, const void* h, const int32_t* offsets,
                             const int32_t* perm_rows, const float* topk_w, const void* w_down,
                             const void* ws_down, int mode, void* out, cudaStream_t st);
cudaError_t launch_gateup_sm100(const Plan& p, const void* x, const void* w_gate, const void* w_up,
                                const void* ws_gate, const void* ws_up, cudaStream_t st);
cudaError_t launch_down_sm100(const Plan& p, const void* w_down, const void* ws_down, int mode,
                              void* out, cudaStream_t st);
// The same GEMMs with the routed experts' weights in MXFP4 (E2M1 code blocks
// [E, N, K/32, 16] and E8M0 scales [E, N, K/32], K = H for gate/up, I for
// down), converted to bf16 in shared memory: bf16 layer, no shared expert,
// H and I multiples of 32 and at most 3072, T*k at most 128 rows per expert
// (mx_gemm_eligible).
bool mx_gemm_eligible(const Plan& p);
cudaError_t launch_gateup_mx_sm100(const Plan& p, const uint8_t* gate_blocks, const uint8_t* gate_scales,
                                   const uint8_t* up_blocks, const uint8_t* up_scales, cudaStream_t st);
cudaError_t launch_down_mx_sm100(const Plan& p, const uint8_t* down_blocks, const uint8_t* down_scales, int mode,
                                 void* out, cudaStream_t st);
// y[t] = sum_j rows[row_of[t,j]] (j in order, dropped slots skipped) + rows[S + t]
// (shared), summed in float32 and rounded once to the layer dtype.
cudaError_t launch_combine_rows(const Plan& p, const void* rows, const int32_t* row_of, void* y,
                                cudaStream_t st);
// Stage API: y[t] = sum_j topk_w[t,j] * expert_out[row_of[t,j]] (+ shared row).
cudaError_t launch_combine(const Plan& p, const float* expert_out, const int32_t* row_of,
                           const float* topk_w, void* y, cudaStream_t st);

// Expert shards: topk_idx -> shard-local expert ids (expert - begin for
// experts in [begin, begin + count), else -1).
cudaError_t launch_remap_experts(const int32_t* idx, int64_t S, int begin, int count, int32_t* local,
                                 cudaStream_t st);
// y[t, h] = dtype(sum over i < n of partials[i][t][h]), float32, i in order.
cudaError_t launch_reduce_partials(const float* partials, int n, int64_t count, bool bf16_out, void* y,
                                   cudaStream_t st);

// capacity_left[e] = max(0, C - sum_{q < shard} counts[q][e]) for one token
// shard of a batch with capacity C (device kernel / host loop).
cudaError_t launch_shard_capacity_left(int64_t C, const int32_t* counts, int n_shards, int shard, int E,
                                       int32_t* capacity_left, cudaStream_t st);
void shard_capacity_left_host(int64_t C, const int32_t* counts, int n_shards, int shard, int E,
                              int32_t* capacity_left);

// Backward pass (bf16): extra workspace after the forward plan's bytes, and
// the whole pass (grouping of the given routing, then every gradient).
size_t backward_workspace_bytes(const Plan& p);
cudaError_t launch_backward(const Plan& p, void* bwd_ws, const void* x, const void* dy, const int32_t* idx,
                            const float* topk_w, const void* router_w, const void* w_gate, const void* w_up,
                            const void* w_down, const void* ws_gate, const void* ws_up, const void* ws_down,
                            float* dx, float* d_router_w, float* d_router_b, float* d_w_gate, float* d_w_up,
                            float* d_w_down, float* d_ws_gate, float* d_ws_up, float* d_ws_down, cudaStream_t st);

// Kernel-trace hooks (moe_abi.cu): bracket one launch with events.
void trace_before(const char* name, cudaStream_t st);
void trace_after(cudaStream_t st);

}  // namespace moe
