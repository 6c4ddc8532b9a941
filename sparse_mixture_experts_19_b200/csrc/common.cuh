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

// Everything the kernels of one call need, carved out of the caller's workspace.
struct Plan {
    int64_t T, H, I, E, k, Is, S;  // S = T*k slots
    int64_t cap;                   // 0 = unlimited
    bool bf16;
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
    int32_t* perm_rows;   // [S]
    int32_t* row_of;      // [S]
    void* xperm;          // [S, H] layer dtype: x rows in grouped order
    void* h;              // [h_rows, I_max] layer dtype: SwiGLU activations
    float* yacc;          // [T, H] float32 accumulator of the combine
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

// ---- launchers (defined in the .cu files; return the launch error) ------
cudaError_t launch_router_simt(const Plan& p, const void* x, const void* router_w,
                               const float* router_b, int32_t* topk_idx, float* topk_w,
                               float* yacc_zero, cudaStream_t st);
// tcgen05 router for the bf16 layer (scores in float32 TMEM accumulators).
cudaError_t launch_router_sm100(const Plan& p, const void* x, const void* router_w,
                                const float* router_b, int32_t* topk_idx, float* topk_w,
                                cudaStream_t st);
// dst[0..n) = 0 (float32, n a multiple of 4).
cudaError_t launch_zero_f32(float* dst, int64_t n, cudaStream_t st);
cudaError_t launch_permute(const Plan& p, const int32_t* topk_idx, int32_t* counts,
                           int32_t* offsets, int32_t* perm_rows, int32_t* row_of,
                           int32_t* dropped, cudaStream_t st);
// moe_permute with the scratch in a static device array; sizes.S <= kNoAllocMaxSlots.
cudaError_t launch_permute_noalloc(const Plan& sizes, const int32_t* topk_idx, int32_t* counts,
                                   int32_t* offsets, int32_t* perm_rows, int32_t* row_of,
                                   int32_t* dropped, cudaStream_t st);
// plan offsets [E+2] from a caller's offsets [E+1] (appends the shared rows).
cudaError_t launch_offsets_from_user(const Plan& p, const int32_t* offsets, cudaStream_t st);
cudaError_t launch_gather_rows(const Plan& p, const void* x, const int32_t* perm_rows,
                               const int32_t* offsets, void* xperm, cudaStream_t st);
// h = silu(X W_g^T) * (X W_u^T) for all groups (routed + shared).
cudaError_t launch_gateup_simt(const Plan& p, const void* xperm, const void* x,
                               const int32_t* offsets, const void* w_gate, const void* w_up,
                               const void* ws_gate, const void* ws_up, void* h, cudaStream_t st);
// out = h W_d^T: mode 0 stores float32 rows to `out`; mode 1 adds
// topk_w-weighted rows into yacc[token] (shared rows with weight 1).
cudaError_t launch_down_simt(const Plan& p, const void* h, const int32_t* offsets,
                             const int32_t* perm_rows, const float* topk_w, const void* w_down,
                             const void* ws_down, int mode, float* out, cudaStream_t st);
// tcgen05 grouped GEMMs (bf16): h = silu(X W_g^T) * (X W_u^T); out = h W_d^T
// (mode 0: float32 rows; mode 1: weighted atomic add into yacc[token]).
cudaError_t launch_gateup_sm100(const Plan& p, const void* x, const void* w_gate, const void* w_up,
                                const void* ws_gate, const void* ws_up, cudaStream_t st);
cudaError_t launch_down_sm100(const Plan& p, const void* w_down, const void* ws_down, int mode,
                              float* out, cudaStream_t st);
cudaError_t launch_finalize(const Plan& p, const float* yacc, void* y, cudaStream_t st);
cudaError_t launch_combine(const Plan& p, const float* expert_out, const int32_t* row_of,
                           const float* topk_w, void* y, cudaStream_t st);

// Kernel-trace hooks (moe_abi.cu): bracket one launch with events.
void trace_before(const char* name, cudaStream_t st);
void trace_after(cudaStream_t st);

}  // namespace moe
