// MXFP4 expert weights -> bf16, for moe_forward_mxfp4 above the decode
// kernel's sizes ("Mixture of Experts (MoEs) in Transformers", section From
// Dense to Sparse: gpt-oss ships its experts in mxfp4).  Every dequantized
// value e * 2^(s - 127) (e an E2M1 value, at most two significant bits) is
// exact in bf16 down to 2^-133, so the grouped GEMMs that follow see the
// weights exactly; only a value above the bf16 range (s >= 254 with |e| >= 2)
// becomes +-inf, and s = 255 gives NaN for its 32 elements.
//
// Bound by HBM: 17 bytes read and 64 bytes written per block of 32 elements.
// A thread converts 8 elements at a time (4 code bytes -> 16 bytes of bf16),
// four such chunks 32 apart with their loads issued together: a warp's loads
// then cover 128 contiguous bytes each and its stores 512.
#include <cuda_fp16.h>

#include <algorithm>

#include "common.cuh"
#include "mxfp4.cuh"
#include "tma_host.cuh"

namespace moe {
namespace {

constexpr int kDqUnroll = 4;  // chunks per thread in flight

__global__ void __launch_bounds__(256) mxfp4_dequant_kernel(const uint32_t* __restrict__ codes,
                                                            const uint8_t* __restrict__ scales, int64_t nchunk,
                                                            uint4* __restrict__ out) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x / 32);
    for (int64_t t = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32; t * 32 * kDqUnroll < nchunk;
         t += warps) {
        const int64_t c0 = t * 32 * kDqUnroll + lane;  // chunks c0, c0 + 32, ...
        uint32_t w[kDqUnroll], sb[kDqUnroll];
#pragma unroll
        for (int u = 0; u < kDqUnroll; ++u) {
            const int64_t c = c0 + 32 * u;
            w[u] = c < nchunk ? __ldcs(codes + c) : 0u;         // read once
            sb[u] = c < nchunk ? __ldcs(scales + c / 4) : 127u;  // four chunks per 32-element block
        }
#pragma unroll
        for (int u = 0; u < kDqUnroll; ++u) {
            const int64_t c = c0 + 32 * u;
            if (c >= nchunk) break;
            const float sc = e8m0_value(sb[u]);
            uint32_t h[4], o[4];
            e2m1x8_to_f16x2(w[u], h);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h[j]));
                const __nv_bfloat162 v = __floats2bfloat162_rn(f.x * sc, f.y * sc);
                o[j] = *reinterpret_cast<const uint32_t*>(&v);
            }
            out[c] = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
}

}  // namespace

cudaError_t launch_mxfp4_dequant(const uint8_t* blocks, const uint8_t* scales, int64_t rows, int K, void* out,
                                 cudaStream_t st) {
    if (K % 32 || rows < 0) return cudaErrorInvalidValue;
    const int64_t nchunk = rows * (K / 8);
    if (nchunk == 0) return cudaSuccess;
    const int64_t want = (nchunk + 256 * kDqUnroll - 1) / (256 * kDqUnroll);
    const int grid = (int)std::min<int64_t>(want, (int64_t)device_sm_count() * 8);
    trace_before("mxfp4_dequant", st);
    mxfp4_dequant_kernel<<<grid, 256, 0, st>>>(reinterpret_cast<const uint32_t*>(blocks), scales, nchunk,
                                               reinterpret_cast<uint4*>(out));
    trace_after(st);
    return cudaGetLastError();
}

}  // namespace moe
