// Host-side helpers shared by the tcgen05 kernels: TMA tensor-map encoding
// through the driver entry point (no link-time dependency on libcuda) and the
// SM count of the current device.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <mutex>

namespace moe {

inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// Rank-3 map of a bf16 tensor [depth][rows][inner] (inner contiguous) with
// box {box_inner, box_rows, 1} and the 128-byte swizzle; out-of-range
// elements of a box read as zero.  A map depends only on these arguments, so
// encoded maps are kept in a small process-wide cache.
inline bool make_map_bf16(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
                          uint64_t depth, uint32_t box_inner, uint32_t box_rows) {
    struct Entry {
        const void* base;
        uint64_t inner, rows, depth;
        uint32_t box_inner, box_rows;
        CUtensorMap map;
    };
    constexpr int kCache = 64;
    static Entry cache[kCache];
    static int used = 0, next = 0;
    static std::mutex mu;
    {
        std::lock_guard<std::mutex> lock(mu);
        for (int i = 0; i < used; ++i) {
            const Entry& c = cache[i];
            if (c.base == base && c.inner == inner && c.rows == rows && c.depth == depth &&
                c.box_inner == box_inner && c.box_rows == box_rows) {
                *m = c.map;
                return true;
            }
        }
    }
    auto fn = tensor_map_encoder();
    if (!fn) return false;
    cuuint64_t dims[3] = {inner, rows, depth};
    cuuint64_t strides[2] = {inner * 2, inner * rows * 2};
    cuuint32_t box[3] = {box_inner, box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    if (fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return false;
    std::lock_guard<std::mutex> lock(mu);
    Entry& c = cache[next];
    c = Entry{base, inner, rows, depth, box_inner, box_rows, *m};
    next = (next + 1) % kCache;
    if (used < kCache) ++used;
    return true;
}

// Rank-3 map of a byte tensor [depth][rows][inner] (inner contiguous, a
// multiple of 16 bytes) with box {box_inner, box_rows, 1}; box_inner = 128
// takes the 128-byte swizzle (16-byte chunk c of box row r at c ^ (r % 8)),
// other widths none (rows box_inner bytes apart).  Out-of-range bytes of a
// box read as zero.  Cached like make_map_bf16.
inline bool make_map_u8(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t depth,
                        uint32_t box_inner, uint32_t box_rows) {
    struct Entry {
        const void* base;
        uint64_t inner, rows, depth;
        uint32_t box_inner, box_rows;
        CUtensorMap map;
    };
    constexpr int kCache = 32;
    static Entry cache[kCache];
    static int used = 0, next = 0;
    static std::mutex mu;
    {
        std::lock_guard<std::mutex> lock(mu);
        for (int i = 0; i < used; ++i) {
            const Entry& c = cache[i];
            if (c.base == base && c.inner == inner && c.rows == rows && c.depth == depth &&
                c.box_inner == box_inner && c.box_rows == box_rows) {
                *m = c.map;
                return true;
            }
        }
    }
    auto fn = tensor_map_encoder();
    if (!fn) return false;
    cuuint64_t dims[3] = {inner, rows, depth};
    cuuint64_t strides[2] = {inner, inner * rows};
    cuuint32_t box[3] = {box_inner, box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    if (fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, box_inner == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return false;
    std::lock_guard<std::mutex> lock(mu);
    Entry& c = cache[next];
    c = Entry{base, inner, rows, depth, box_inner, box_rows, *m};
    next = (next + 1) % kCache;
    if (used < kCache) ++used;
    return true;
}

// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per kernel (by
// address), device and size.
template <typename Kernel>
inline cudaError_t ensure_smem_attr(Kernel kernel, size_t bytes) {
    struct Done {
        const void* fn;
        int dev;
        size_t bytes;
    };
    static Done done[64];
    static int n = 0;
    static std::mutex mu;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const void* fn = reinterpret_cast<const void*>(kernel);
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < n; ++i)
        if (done[i].fn == fn && done[i].dev == dev && done[i].bytes >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess && n < 64) done[n++] = Done{fn, dev, bytes};
    return e;
}

inline int device_sm_count() {
    static int count[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    if (!count[dev]) cudaDeviceGetAttribute(&count[dev], cudaDevAttrMultiProcessorCount, dev);
    return count[dev] > 0 ? count[dev] : 148;
}

}  // namespace moe
