// MXFP4 expert weights -> bf16, for moe_forward_mxfp4 above the decode
// kernel's sizes ("Mixture of Experts (MoEs) in Transformers", section From
// Dense to Sparse: gpt-oss ships its experts in mxfp4).  Every dequantized
// value e * 2^(s - 127) (e an E2M1 value, at most two significant bits) is
// exact in bf16 down to 2^-133, so the grouped GEMMs that follow see the
// weights exactly; only a value above the bf16 range (s >= 254 with |e| >= 2)
// becomes +-inf, and s = 255 gives NaN for its 32 elements.
//
// Bound by HBM: 17 bytes read and 64 bytes written per block of 32 elements.
// One thread per block; a warp's 32 blocks are consecutive, so its code
// loads, scale loads and stores each cover contiguous memory.
#include <cuda_fp16.h>

#include <algorithm>

#include "common.cuh"
#include "mxfp4.cuh"
#include "tma_host.cuh"

namespace moe {
namespace {

__global__ void __launch_bounds__(256) mxfp4_dequant_kernel(const uint4* __restrict__ codes,
                                                            const uint8_t* __restrict__ scales, int64_t nblk,
                                                            uint4* __restrict__ out) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < nblk; b += stride) {
        const uint4 c = __ldcs(codes + b);  // read once
        const float sc = e8m0_value(__ldcs(scales + b));
        const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            uint32_t h[4], o[4];
            e2m1x8_to_f16x2(cw[q], h);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h[j]));
                const __nv_bfloat162 v = __floats2bfloat162_rn(f.x * sc, f.y * sc);
                o[j] = *reinterpret_cast<const uint32_t*>(&v);
            }
            out[b * 4 + q] = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
}

}  // namespace

cudaError_t launch_mxfp4_dequant(const uint8_t* blocks, const uint8_t* scales, int64_t rows, int K, void* out,
                                 cudaStream_t st) {
    if (K % 32 || rows < 0) return cudaErrorInvalidValue;
    const int64_t nblk = rows * (K / 32);
    if (nblk == 0) return cudaSuccess;
    const int64_t want = (nblk + 255) / 256;
    const int grid = (int)std::min<int64_t>(want, (int64_t)device_sm_count() * 8);
    trace_before("mxfp4_dequant", st);
    mxfp4_dequant_kernel<<<grid, 256, 0, st>>>(reinterpret_cast<const uint4*>(blocks), scales, nblk,
                                               reinterpret_cast<uint4*>(out));
    trace_after(st);
    return cudaGetLastError();
}

}  // namespace moe
