// Grouping of (token, slot) pairs by expert, with capacity drop in token order.
//
// "Mixture of Experts (MoEs) in Transformers", section Expert Backend
// (grouped_mm sorts tokens by expert id and groups them); "MoE稀疏架构是什么？
// 从原理到落地的系统解读", section 三.2 (capacity-limited token dropping).
//
// Passes over the T*k slot ids (chunks of 2048), all bit-reproducible:
//   1. chunk histogram: hist[c][e] = pairs of expert e in slot chunk c;
//   2a. one block per expert: exclusive scan of hist[.][e] over the chunks
//      (in place), so base[c][e] = pairs of e in earlier chunks; the total
//      is counts[e];
//   2b. one block: capacity cut, dropped, and the exclusive scan over
//      experts -> offsets (and the GEMM schedulers' tile prefixes);
//   3. stable scatter: one block per chunk, each of its 8 warps walking a
//      256-slot segment in order, 32 slots at a time, ranking equal experts
//      inside a warp with __match_any_sync and across the block's warps
//      with per-warp counts; the rank of a pair is the number of earlier
//      slots of the same expert.  Slot order is token-major, hence ranks
//      follow ascending token order, and a pair is kept iff its rank < C.
#include <cuda.h>

#include <mutex>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kHistThreads = 256;
constexpr int kScanThreads = 256;  // >= kMaxExperts
constexpr int kScatterWarps = 8;                          // warps per chunk in the scatter
constexpr int kScatterSeg = kPermuteChunk / kScatterWarps;  // slots per warp segment
constexpr int kChunkScanThreads = 1024;

__global__ void __launch_bounds__(kHistThreads) permute_hist_kernel(
    const int32_t* __restrict__ idx, int64_t S, int E, int32_t* __restrict__ hist,
    int32_t* __restrict__ flags, bool drop_negative) {
    __shared__ int32_t h[kMaxExperts];
    for (int e = threadIdx.x; e < E; e += blockDim.x) h[e] = 0;
    __syncthreads();
    const int64_t s0 = (int64_t)blockIdx.x * kPermuteChunk;
    const int64_t s1 = min(S, s0 + kPermuteChunk);
    bool bad = false;
    for (int64_t s = s0 + threadIdx.x; s < s1; s += blockDim.x) {
        int e = idx[s];
        if (e >= 0 && e < E)
            atomicAdd(&h[e], 1);
        else if (!(drop_negative && e == -1))
            bad = true;
    }
    if (bad) set_flag(flags, MOE_DEVFLAG_BAD_EXPERT_INDEX);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) hist[(int64_t)blockIdx.x * E + e] = h[e];
}

// Inclusive scan over the 256 threads of the block (v of thread i -> sum of 0..i).
// Starts with a barrier: callers may still be reading `sm` from earlier work.
__device__ __forceinline__ int32_t block_scan_256(int32_t v, int32_t* sm) {
    const int i = threadIdx.x;
    __syncthreads();
    sm[i] = v;
    __syncthreads();
    for (int o = 1; o < kScanThreads; o <<= 1) {
        int32_t u = (i >= o) ? sm[i - o] : 0;
        __syncthreads();
        sm[i] += u;
        __syncthreads();
    }
    int32_t r = sm[i];
    __syncthreads();
    return r;
}

// Tiles of `rows_per_tile` rows per expert -> exclusive prefix prefix[0..E].
__device__ __forceinline__ void write_tile_prefix(int32_t kept, int E, int32_t* sm, int rows_per_tile,
                                                  int32_t* prefix) {
    const int e = threadIdx.x;
    int32_t mt = (e < E) ? (kept + rows_per_tile - 1) / rows_per_tile : 0;
    int32_t incl = block_scan_256(mt, sm);
    if (e < E) prefix[e] = incl - mt;
    if (e == E - 1) prefix[E] = incl;
}

// Both tile prefixes of the grouped GEMMs: 128-row tiles and 256-row CTA-pair tiles.
__device__ __forceinline__ void write_mtile_prefix(int32_t kept, int E, int32_t* sm, int32_t* mtile_prefix,
                                                   int32_t* mpair_prefix) {
    write_tile_prefix(kept, E, sm, kGemmTileRows, mtile_prefix);
    write_tile_prefix(kept, E, sm, 2 * kGemmTileRows, mpair_prefix);
}

// 2a. Block e: exclusive scan of hist[.][e] over the chunks, in place, in
// tiles of 1024 chunks with a carry; counts[e] = the total.
__global__ void __launch_bounds__(kChunkScanThreads) permute_scan_chunks_kernel(int32_t* __restrict__ hist,
                                                                                int64_t nchunks, int E,
                                                                                int32_t* __restrict__ counts) {
    __shared__ int32_t wsum[kChunkScanThreads / 32];
    const int e = blockIdx.x, warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    int32_t carry = 0;
    for (int64_t c0 = 0; c0 < nchunks; c0 += kChunkScanThreads) {
        const int64_t c = c0 + threadIdx.x;
        const int32_t v = c < nchunks ? hist[c * E + e] : 0;
        int32_t x = v;  // inclusive warp scan
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) wsum[warp] = x;
        __syncthreads();
        if (warp == 0) {
            int32_t w = wsum[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int32_t y = __shfl_up_sync(0xffffffffu, w, o);
                if (lane >= o) w += y;
            }
            wsum[lane] = w;  // inclusive over warps
        }
        __syncthreads();
        const int32_t incl = x + (warp > 0 ? wsum[warp - 1] : 0);
        if (c < nchunks) hist[c * E + e] = carry + incl - v;
        carry += wsum[kChunkScanThreads / 32 - 1];
        __syncthreads();  // wsum is rewritten by the next tile
    }
    if (threadIdx.x == 0) counts[e] = carry;
}

// 2b. One block: per-expert totals -> capacity cut, dropped, offsets, and
// the tile prefixes of the grouped GEMMs.
__global__ void __launch_bounds__(kScanThreads) permute_scan_experts_kernel(
    const int32_t* __restrict__ counts, int E, int64_t cap, const int32_t* __restrict__ cap_left_arr,
    int32_t* __restrict__ dropped, int32_t* offsets_out,
    int32_t* offsets_ws, int32_t* __restrict__ mtile_prefix, int32_t* __restrict__ mpair_prefix,
    int32_t shared_rows) {
    __shared__ int32_t sm[kScanThreads];
    const int e = threadIdx.x;
    const int32_t total = (e < E) ? counts[e] : 0;
    const int64_t cl = (cap > 0 && e < E) ? cap_left(cap, cap_left_arr, e) : 0;
    const int32_t kept = (cap > 0 && total > cl) ? (int32_t)cl : total;
    if (e < E) dropped[e] = total - kept;
    const int32_t incl = block_scan_256(kept, sm);
    // offsets_ws [E+2] feeds the GEMMs; offsets_out [E+1] is the caller's copy
    if (e < E) {
        offsets_ws[e] = incl - kept;
        offsets_out[e] = incl - kept;
    }
    if (e == E - 1) {
        offsets_ws[E] = incl;
        offsets_ws[E + 1] = incl + shared_rows;
        offsets_out[E] = incl;
    }
    write_mtile_prefix(kept, E, sm, mtile_prefix, mpair_prefix);
}

// 3. Block c scatters chunk c: warp w ranks the slots of its segment
// [c*2048 + w*256, +256) from base[c][e] plus the earlier warps' counts.
__global__ void __launch_bounds__(kScatterWarps * 32) permute_scatter_kernel(
    const int32_t* __restrict__ idx, int64_t S, int E, int64_t cap, const int32_t* __restrict__ cap_left_arr,
    const int32_t* __restrict__ base,
    const int32_t* __restrict__ offsets, int32_t* __restrict__ perm_rows, int32_t* __restrict__ row_of) {
    __shared__ int32_t run[kScatterWarps][kMaxExperts];
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int64_t c = blockIdx.x;
    const int64_t cs1 = min(S, (c + 1) * kPermuteChunk);
    const int64_t s0 = min(cs1, c * kPermuteChunk + (int64_t)warp * kScatterSeg);
    const int64_t s1 = min(cs1, s0 + kScatterSeg);
    for (int i = threadIdx.x; i < kScatterWarps * kMaxExperts; i += blockDim.x) (&run[0][0])[i] = 0;
    __syncthreads();
    const uint32_t lt = (1u << lane) - 1u;
    for (int64_t sb = s0; sb < s1; sb += 32) {  // counts of this warp's segment
        const int64_t s = sb + lane;
        const int ex = (s < s1) ? idx[s] : -1;
        const bool valid = (ex >= 0 && ex < E);
        const uint32_t peers = __match_any_sync(0xffffffffu, valid ? ex : -1);
        if (valid && (peers & lt) == 0) run[warp][ex] += __popc(peers);
        __syncwarp();
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {  // first rank of each warp's segment
        int32_t r = base[c * E + e];
        for (int w = 0; w < kScatterWarps; ++w) {
            const int32_t n = run[w][e];
            run[w][e] = r;
            r += n;
        }
    }
    __syncthreads();
    for (int64_t sb = s0; sb < s1; sb += 32) {
        const int64_t s = sb + lane;
        const int ex = (s < s1) ? idx[s] : -1;
        const bool valid = (ex >= 0 && ex < E);
        const uint32_t peers = __match_any_sync(0xffffffffu, valid ? ex : -1);
        int32_t rank = 0;
        if (valid) rank = run[warp][ex] + __popc(peers & lt);
        __syncwarp();
        if (valid && (peers & lt) == 0) run[warp][ex] += __popc(peers);  // lowest peer updates
        __syncwarp();
        if (s < s1) {
            if (valid && (cap <= 0 || rank < cap_left(cap, cap_left_arr, ex))) {
                const int32_t row = offsets[ex] + rank;
                perm_rows[row] = (int32_t)s;
                row_of[s] = row;
            } else {
                row_of[s] = -1;
            }
        }
    }
}

__global__ void permute_fill_tail_kernel(int32_t* __restrict__ perm_rows, int64_t S,
                                         const int32_t* __restrict__ offsets, int E) {
    const int64_t R = offsets[E];
    for (int64_t r = R + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; r < S;
         r += (int64_t)gridDim.x * blockDim.x)
        perm_rows[r] = -1;
}

// All of the grouping in one CTA when the slots fit one chunk (S <= 2048).
// Each of the 8 warps owns a contiguous segment of slots: it counts its
// segment per expert (warp match, no atomics), the counts give the totals,
// capacity cut and scans (as permute_scan_experts_kernel, with a single
// chunk) and each warp's first rank per expert (earlier segments' counts),
// then every warp scatters its segment in slot order while the threads past
// the kept rows mark the unused tail of perm_rows.  Same outputs, one launch.
constexpr int kSmallWarps = kScanThreads / 32;

__global__ void __launch_bounds__(kScanThreads) permute_small_kernel(
    const int32_t* __restrict__ idx, int S, int E, int64_t cap, const int32_t* __restrict__ cap_left_arr,
    int32_t* __restrict__ counts,
    int32_t* __restrict__ dropped, int32_t* offsets_out, int32_t* offsets_ws,
    int32_t* __restrict__ mtile_prefix, int32_t* __restrict__ mpair_prefix, int32_t shared_rows,
    int32_t* __restrict__ perm_rows, int32_t* __restrict__ row_of, int32_t* __restrict__ flags, bool drop_negative) {
    __shared__ int32_t wcount[kSmallWarps][kScanThreads];  // per warp segment, per expert
    __shared__ int32_t sm[kScanThreads];
    __shared__ int32_t off[kScanThreads + 1];
    __shared__ int32_t capl[kScanThreads];  // capacity left per expert (when cap > 0)
    const int e = threadIdx.x, warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    for (int w = 0; w < kSmallWarps; ++w) wcount[w][e] = 0;
    __syncthreads();
    const int seg = ((S + kSmallWarps - 1) / kSmallWarps + 31) / 32 * 32;
    const int s0 = min(S, warp * seg), s1 = min(S, s0 + seg);
    const uint32_t lt = (1u << lane) - 1u;
    bool bad = false;
    for (int sb = s0; sb < s1; sb += 32) {
        const int s = sb + lane;
        const int ex = (s < s1) ? idx[s] : -1;
        const bool valid = (ex >= 0 && ex < E);
        if (s < s1 && !valid && !(drop_negative && ex == -1)) bad = true;
        const uint32_t peers = __match_any_sync(0xffffffffu, valid ? ex : -1);
        if (valid && (peers & lt) == 0) wcount[warp][ex] += __popc(peers);
        __syncwarp();
    }
    if (bad) set_flag(flags, MOE_DEVFLAG_BAD_EXPERT_INDEX);
    __syncthreads();
    int32_t total = 0;
    for (int w = 0; w < kSmallWarps; ++w) {
        const int32_t c = (e < E) ? wcount[w][e] : 0;
        wcount[w][e] = total;  // first rank of warp w's segment in expert e
        total += c;
    }
    const int64_t cl = (cap > 0 && e < E) ? cap_left(cap, cap_left_arr, e) : 0;
    const int32_t kept = (cap > 0 && total > cl) ? (int32_t)cl : total;
    if (e < E) {
        counts[e] = total;
        dropped[e] = total - kept;
        capl[e] = (int32_t)cl;
    }
    const int32_t incl = block_scan_256(kept, sm);
    if (e < E) {
        off[e] = incl - kept;
        offsets_ws[e] = incl - kept;
        offsets_out[e] = incl - kept;
    }
    if (e == E - 1) {
        off[E] = incl;
        offsets_ws[E] = incl;
        offsets_ws[E + 1] = incl + shared_rows;
        offsets_out[E] = incl;
    }
    write_mtile_prefix(kept, E, sm, mtile_prefix, mpair_prefix);  // ends with a barrier
    const int R = off[E];
    for (int sb = s0; sb < s1; sb += 32) {
        const int s = sb + lane;
        const int ex = (s < s1) ? idx[s] : -1;
        const bool valid = (ex >= 0 && ex < E);
        const uint32_t peers = __match_any_sync(0xffffffffu, valid ? ex : -1);
        int32_t rank = 0;
        if (valid) rank = wcount[warp][ex] + __popc(peers & lt);
        __syncwarp();
        if (valid && (peers & lt) == 0) wcount[warp][ex] += __popc(peers);
        __syncwarp();
        if (s < s1) {
            if (valid && (cap <= 0 || rank < capl[ex])) {
                const int32_t row = off[ex] + rank;
                perm_rows[row] = s;
                row_of[s] = row;
            } else {
                row_of[s] = -1;
            }
        }
    }
    for (int r = R + (int)threadIdx.x; r < S; r += kScanThreads) perm_rows[r] = -1;
}

__global__ void __launch_bounds__(kScanThreads) offsets_from_user_kernel(
    const int32_t* __restrict__ user, int E, int32_t shared_rows, int32_t* __restrict__ ws_off,
    int32_t* __restrict__ mtile_prefix, int32_t* __restrict__ mpair_prefix) {
    __shared__ int32_t sm[kScanThreads];
    const int e = threadIdx.x;
    if (e <= E) ws_off[e] = user[e];
    if (e == 0) ws_off[E + 1] = user[E] + shared_rows;
    write_mtile_prefix(e < E ? user[e + 1] - user[e] : 0, E, sm, mtile_prefix, mpair_prefix);
}

}  // namespace

cudaError_t launch_offsets_from_user(const Plan& p, const int32_t* offsets, cudaStream_t st) {
    trace_before("offsets_from_user", st);
    offsets_from_user_kernel<<<1, kScanThreads, 0, st>>>(offsets, (int)p.E,
                                                         (int32_t)(p.Is > 0 ? p.T : 0), p.offsets,
                                                         p.mtile_prefix, p.mpair_prefix);
    trace_after(st);
    return cudaGetLastError();
}

cudaError_t launch_permute(const Plan& p, const int32_t* topk_idx, int32_t* counts,
                           int32_t* offsets, int32_t* perm_rows, int32_t* row_of,
                           int32_t* dropped, cudaStream_t st) {
    if (p.S == 0) {
        // nothing routed: all counts and offsets are zero
        cudaError_t e1 = cudaMemsetAsync(counts, 0, sizeof(int32_t) * p.E, st);
        if (e1 == cudaSuccess) e1 = cudaMemsetAsync(dropped, 0, sizeof(int32_t) * p.E, st);
        if (e1 == cudaSuccess) e1 = cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (p.E + 1), st);
        if (e1 == cudaSuccess && offsets != p.offsets)
            e1 = cudaMemsetAsync(p.offsets, 0, sizeof(int32_t) * (p.E + 1), st);
        if (e1 == cudaSuccess) {
            // offsets[E+1] = shared rows (T = 0 here, so also 0)
            e1 = cudaMemsetAsync(p.offsets + p.E, 0, sizeof(int32_t) * 2, st);
        }
        if (e1 == cudaSuccess) e1 = cudaMemsetAsync(p.mtile_prefix, 0, sizeof(int32_t) * (p.E + 1), st);
        if (e1 == cudaSuccess) e1 = cudaMemsetAsync(p.mpair_prefix, 0, sizeof(int32_t) * (p.E + 1), st);
        return e1;
    }
    const int E = (int)p.E;
    if (p.nchunks == 1) {
        trace_before("permute_small", st);
        permute_small_kernel<<<1, kScanThreads, 0, st>>>(topk_idx, (int)p.S, E, p.cap, p.cap_left_arr, counts, dropped, offsets,
                                                         p.offsets, p.mtile_prefix, p.mpair_prefix,
                                                         (int32_t)(p.Is > 0 ? p.T : 0), perm_rows, row_of, p.flags,
                                                         p.drop_negative);
        trace_after(st);
        return cudaGetLastError();
    }
    trace_before("permute_hist", st);
    permute_hist_kernel<<<(unsigned)p.nchunks, kHistThreads, 0, st>>>(topk_idx, p.S, E,
                                                                       p.chunk_base, p.flags, p.drop_negative);
    trace_after(st);
    trace_before("permute_scan_chunks", st);
    permute_scan_chunks_kernel<<<(unsigned)E, kChunkScanThreads, 0, st>>>(p.chunk_base, p.nchunks, E, counts);
    trace_after(st);
    trace_before("permute_scan", st);
    permute_scan_experts_kernel<<<1, kScanThreads, 0, st>>>(counts, E, p.cap, p.cap_left_arr, dropped, offsets, p.offsets,
                                                            p.mtile_prefix, p.mpair_prefix,
                                                            (int32_t)(p.Is > 0 ? p.T : 0));
    trace_after(st);
    trace_before("permute_scatter", st);
    permute_scatter_kernel<<<(unsigned)p.nchunks, kScatterWarps * 32, 0, st>>>(topk_idx, p.S, E, p.cap, p.cap_left_arr,
                                                                                p.chunk_base, p.offsets,
                                                                                perm_rows, row_of);
    trace_after(st);
    trace_before("permute_fill_tail", st);
    permute_fill_tail_kernel<<<64, 256, 0, st>>>(perm_rows, p.S, p.offsets, E);
    trace_after(st);
    return cudaGetLastError();
}


// ------------------------------------------------------------------------
// Allocation-free variant (moe_permute_noalloc).  Some callers cannot call
// cudaMalloc at the point where they group tokens: code running inside a
// framework's custom allocator or memory-pool callback, plugins whose host
// application owns every device allocation, and tight serving loops that
// forbid allocation after start-up.  For them the scratch of the grouping
// kernels (per-chunk histograms, the offsets copy and a flag word) lives in
// this fixed file-scope device array instead of a caller workspace.  A GPU
// holds the array from the moment this file's device code is loaded on it
// (its first grouping call of any entry point, or context creation when
// modules load eagerly) until the process exits.
namespace {

constexpr int64_t kNoAllocChunks = kNoAllocMaxSlots / kPermuteChunk;
constexpr int64_t kNoAllocInts = kNoAllocChunks * kMaxExperts + 3 * (kMaxExperts + 2) + 64;

static __device__ __align__(256) int32_t g_noalloc_scratch[kNoAllocInts];

// Device address of g_noalloc_scratch, looked up once per CUDA context (the
// context of the stream the call enqueues on, which is current on the
// calling thread as for any launch) and cached under that context's unique
// id: in host code the array's name is only a host-side stand-in, never a
// device address, and an address found in one context means nothing in
// another (after cudaDeviceReset the device gets a new primary context with
// a new id, and the address is looked up again).
typedef CUresult (*StreamGetCtxFn)(CUstream, CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

struct ScratchEntry {
    unsigned long long ctx_id;
    int32_t* ptr;
};
std::mutex g_noalloc_mu;
ScratchEntry g_noalloc_cache[64];
int g_noalloc_used = 0, g_noalloc_next = 0;

cudaError_t stream_context_id(cudaStream_t st, unsigned long long* id) {
    static StreamGetCtxFn get_ctx = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        // the entry points of the CUDA 12.0 ABI, whose signatures the
        // typedefs above spell out (a plain lookup would return the newest
        // version, e.g. the three-argument cuStreamGetCtx of CUDA 12.5)
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuStreamGetCtx", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_ctx = reinterpret_cast<StreamGetCtxFn>(p);
        p = nullptr;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(p);
    });
    if (!get_ctx || !get_id) return cudaErrorNotSupported;
    CUcontext ctx = nullptr;
    if (get_ctx(reinterpret_cast<CUstream>(st), &ctx) != CUDA_SUCCESS || !ctx) {
        // the default stream before the runtime bound a context to this
        // thread: cudaFree(nullptr) binds the device's primary context
        // (it frees and allocates nothing)
        cudaError_t e = cudaFree(nullptr);
        if (e != cudaSuccess) return e;
        if (get_ctx(reinterpret_cast<CUstream>(st), &ctx) != CUDA_SUCCESS || !ctx)
            return cudaErrorDeviceUninitialized;
    }
    if (get_id(ctx, id) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
    return cudaSuccess;
}

cudaError_t noalloc_scratch(cudaStream_t st, int32_t** out) {
    unsigned long long id = 0;
    cudaError_t e = stream_context_id(st, &id);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    for (int i = 0; i < g_noalloc_used; ++i)
        if (g_noalloc_cache[i].ctx_id == id) {
            *out = g_noalloc_cache[i].ptr;
            return cudaSuccess;
        }
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_noalloc_cache[g_noalloc_next] = ScratchEntry{id, static_cast<int32_t*>(ptr)};
    g_noalloc_next = (g_noalloc_next + 1) % 64;
    if (g_noalloc_used < 64) ++g_noalloc_used;
    *out = static_cast<int32_t*>(ptr);
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_permute_noalloc(const Plan& sizes, const int32_t* topk_idx, int32_t* counts,
                                   int32_t* offsets, int32_t* perm_rows, int32_t* row_of,
                                   int32_t* dropped, cudaStream_t st) {
    if (sizes.S > kNoAllocMaxSlots) return cudaErrorInvalidValue;
    int32_t* scratch = nullptr;
    cudaError_t e = noalloc_scratch(st, &scratch);
    if (e != cudaSuccess) return e;
    Plan p = sizes;
    p.chunk_base = scratch;                                 // [kNoAllocChunks * E]
    p.offsets = scratch + kNoAllocChunks * kMaxExperts;     // [E + 2]
    p.mtile_prefix = p.offsets + (kMaxExperts + 2);         // [E + 1]
    p.mpair_prefix = p.offsets + 2 * (kMaxExperts + 2);     // [E + 1]
    p.flags = p.offsets + 3 * (kMaxExperts + 2);            // flag word, cleared per call
    e = cudaMemsetAsync(p.flags, 0, sizeof(int32_t), st);
    if (e != cudaSuccess) return e;
    return launch_permute(p, topk_idx, counts, offsets, perm_rows, row_of, dropped, st);
}

}  // namespace moe
