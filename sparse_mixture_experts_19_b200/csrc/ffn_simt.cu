// Grouped expert FFN on CUDA cores, plus the row gather, the combine and the
// final cast.
//
// "Mixture of Experts (MoEs) in Transformers", section Expert Backend
// (grouped_mm: rows grouped by expert, one grouped GEMM), section Weight
// Loading Refactor (packed [E, out, in] expert tensors, gate/up/down).
// "MoE稀疏架构是什么？从原理到落地的系统解读", section 四 (weighted sum of the
// chosen experts' outputs).
//
// The GEMMs here serve the float32 layer (exact float32 FMAs, no TF32); the
// gather and the combines serve both dtypes.
// Groups: 0..E-1 are the routed experts, rows offsets[g]..offsets[g+1];
// group E is the shared expert (rows offsets[E]..offsets[E+1], i.e. token
// t = row - offsets[E], reading x directly).
#include "common.cuh"

namespace moe {
namespace {

constexpr int kBM = 64, kBN = 64, kBK = 16, kThreads = 256;

// m-tile -> (group, first row, rows).  offsets [E+2] are in shared memory.
__device__ __forceinline__ bool find_tile(const int32_t* off, int groups, int64_t mt, int& g,
                                          int64_t& row0, int& rows) {
    for (g = 0; g < groups; ++g) {
        int64_t n = off[g + 1] - off[g];
        int64_t tiles = (n + kBM - 1) / kBM;
        if (mt < tiles) {
            row0 = off[g] + mt * kBM;
            rows = (int)(n - mt * kBM < kBM ? n - mt * kBM : kBM);
            return true;
        }
        mt -= tiles;
    }
    return false;
}

template <typename TIn, bool kGateUp>
__global__ void __launch_bounds__(kThreads) grouped_ffn_simt_kernel(
    int64_t S, int64_t T, int E, int k, int H, int I, int Is, const int32_t* __restrict__ offsets,
    const TIn* __restrict__ a_routed,   // gate/up: xperm [S,H]; down: h [S,I]
    const TIn* __restrict__ a_shared,   // gate/up: x [T,H];     down: hs [T,Is]
    const TIn* __restrict__ w0, const TIn* __restrict__ w1,    // gate/up or down (w1 unused)
    const TIn* __restrict__ ws0, const TIn* __restrict__ ws1,  // shared expert weights
    TIn* __restrict__ h_out, TIn* __restrict__ hs_out,         // gate/up outputs
    const int32_t* __restrict__ perm_rows, const float* __restrict__ topk_w, int mode,
    void* __restrict__ out) {
    __shared__ int32_t off[kMaxExperts + 2];
    __shared__ __align__(16) float As[kBK][kBM];
    __shared__ __align__(16) float Bs[kGateUp ? 2 : 1][kBK][kBN];

    const int groups = E + (Is > 0 ? 1 : 0);
    for (int i = threadIdx.x; i < groups + 1; i += kThreads) off[i] = offsets[i];
    __syncthreads();
    int g, rows;
    int64_t row0;
    if (!find_tile(off, groups, blockIdx.x, g, row0, rows)) return;
    const bool shared = (g == E);
    // GEMM dims of this group: N outputs, K reduction
    const int N = kGateUp ? (shared ? Is : I) : H;
    const int K = kGateUp ? H : (shared ? Is : I);
    const int n0 = blockIdx.y * kBN;
    if (n0 >= N) return;

    const TIn* A = shared ? a_shared + (row0 - off[E]) * (int64_t)K : a_routed + row0 * (int64_t)K;
    const TIn* B0 = shared ? ws0 : w0 + (int64_t)g * N * K;
    const TIn* B1 = kGateUp ? (shared ? ws1 : w1 + (int64_t)g * N * K) : nullptr;

    const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
    float acc0[4][4] = {}, acc1[4][4] = {};

    const int lr = tid / 4, lk = (tid % 4) * 4;  // loader: row/col of 4 elements
    for (int k0 = 0; k0 < K; k0 += kBK) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            int kk = k0 + lk + q;
            As[lk + q][lr] = (lr < rows && kk < K) ? to_f32(A[(int64_t)lr * K + kk]) : 0.f;
            int n = n0 + lr;
            Bs[0][lk + q][lr] = (n < N && kk < K) ? to_f32(B0[(int64_t)n * K + kk]) : 0.f;
            if (kGateUp)
                Bs[kGateUp ? 1 : 0][lk + q][lr] =
                    (n < N && kk < K) ? to_f32(B1[(int64_t)n * K + kk]) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < kBK; ++kk) {
            float4 a = *reinterpret_cast<const float4*>(&As[kk][ty * 4]);
            float4 b0 = *reinterpret_cast<const float4*>(&Bs[0][kk][tx * 4]);
            float av[4] = {a.x, a.y, a.z, a.w}, bv0[4] = {b0.x, b0.y, b0.z, b0.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc0[i][j] = fmaf(av[i], bv0[j], acc0[i][j]);
            if (kGateUp) {
                float4 b1 = *reinterpret_cast<const float4*>(&Bs[kGateUp ? 1 : 0][kk][tx * 4]);
                float bv1[4] = {b1.x, b1.y, b1.z, b1.w};
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc1[i][j] = fmaf(av[i], bv1[j], acc1[i][j]);
            }
        }
        __syncthreads();
    }

#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int r = ty * 4 + i;
        if (r >= rows) continue;
        int64_t row = row0 + r;
        if (kGateUp) {
            TIn* dst = shared ? hs_out + (row - off[E]) * (int64_t)N : h_out + row * (int64_t)N;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                int n = n0 + tx * 4 + j;
                if (n < N) dst[n] = from_f32<TIn>(silu_f32(acc0[i][j]) * acc1[i][j]);
            }
        } else {
            // output row: grouped row, or S + token for the shared expert
            const int64_t orow = shared ? S + (row - off[E]) : row;
            if (mode == 0) {
                float* dst = static_cast<float*>(out) + orow * (int64_t)H;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    int n = n0 + tx * 4 + j;
                    if (n < N) dst[n] = acc0[i][j];
                }
            } else {
                const float w = shared ? 1.f : topk_w[perm_rows[row]];
                TIn* dst = static_cast<TIn*>(out) + orow * (int64_t)H;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    int n = n0 + tx * 4 + j;
                    if (n < N) dst[n] = from_f32<TIn>(w * acc0[i][j]);
                }
            }
        }
    }
}

// xperm[r] = x[perm_rows[r] / k] for r < offsets[E]; one warp per row, 16 B chunks.
__global__ void gather_rows_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ perm_rows,
                                   const int32_t* __restrict__ offsets, int E, int k,
                                   int64_t row_chunks, uint4* __restrict__ xperm) {
    const int64_t R = offsets[E];
    const int lane = threadIdx.x % 32;
    for (int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 32; r < R;
         r += (int64_t)gridDim.x * blockDim.x / 32) {
        const int64_t t = perm_rows[r] / k;
        const uint4* src = x + t * row_chunks;
        uint4* dst = xperm + r * row_chunks;
        for (int64_t c = lane; c < row_chunks; c += 32) dst[c] = src[c];
    }
}

// The same rows built token by token: xperm[row_of[t,j]] = x[t] for each kept
// slot (t, j).  One warp per token; each 16-byte chunk of x[t] is read once and
// stored k times (consecutive lanes: consecutive chunks of a row).  Reading x
// once matters when x is larger than L2: the row-by-row gather reads every x
// row k times, once per expert group sweeping the tokens.
__global__ void scatter_x_rows_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ row_of,
                                      int64_t T, int k, int64_t row_chunks, uint4* __restrict__ xperm) {
    const int lane = threadIdx.x % 32;
    for (int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 32; t < T;
         t += (int64_t)gridDim.x * blockDim.x / 32) {
        const int32_t my_row = lane < k ? row_of[t * k + lane] : -1;  // k <= 32
        const uint4* src = x + t * row_chunks;
        // every lane takes the same iterations (the shuffles need the whole warp)
        for (int64_t c0 = 0; c0 < row_chunks; c0 += 32) {
            const int64_t c = c0 + lane;
            const bool in = c < row_chunks;
            const uint4 v = in ? src[c] : make_uint4(0, 0, 0, 0);
            for (int j = 0; j < k; ++j) {
                const int32_t r = __shfl_sync(0xffffffffu, my_row, j);
                if (in && r >= 0) xperm[r * row_chunks + c] = v;
            }
        }
    }
}

// y[t] = sum_j rows[row_of[t,j]] (+ rows[S + t]); one thread per 16-byte chunk
// of a token's row, float32 sum in slot order, one rounding at the end.
template <typename TV, typename TOut>
__global__ void combine_rows_kernel(const TV* __restrict__ rows, const int32_t* __restrict__ row_of,
                                    int64_t T, int H, int k, int64_t S, int shared, TOut* __restrict__ y) {
    constexpr int V = 16 / sizeof(TV);
    const int chunks = H / V;
    const int64_t n = T * chunks;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = i / chunks;
        const int c = (int)(i % chunks);
        float acc[V];
#pragma unroll
        for (int v = 0; v < V; ++v) acc[v] = 0.f;
        auto add_row = [&](int64_t r) {
            uint4 q = *reinterpret_cast<const uint4*>(rows + r * H + (int64_t)c * V);
            const TV* e = reinterpret_cast<const TV*>(&q);
#pragma unroll
            for (int v = 0; v < V; ++v) acc[v] += to_f32(e[v]);
        };
        for (int j = 0; j < k; ++j) {
            const int32_t r = row_of[t * k + j];
            if (r >= 0) add_row(r);
        }
        if (shared) add_row(S + t);
        TOut* dst = y + t * H + (int64_t)c * V;
        if (sizeof(TOut) == sizeof(TV)) {
            uint4 o;
            TOut* ov = reinterpret_cast<TOut*>(&o);
#pragma unroll
            for (int v = 0; v < V; ++v) ov[v] = from_f32<TOut>(acc[v]);
            *reinterpret_cast<uint4*>(dst) = o;
        } else {
#pragma unroll
            for (int v = 0; v < V; ++v) dst[v] = from_f32<TOut>(acc[v]);
        }
    }
}

// y[t,h] = sum_j w[t,j] eo[row_of[t,j], h] (+ eo[S + t, h]), float32, j in order.
template <typename TOut>
__global__ void combine_kernel(const float* __restrict__ eo, const int32_t* __restrict__ row_of,
                               const float* __restrict__ topk_w, int64_t T, int H, int k,
                               int64_t S, int shared, TOut* __restrict__ y) {
    const int64_t n = T * (int64_t)H;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        int64_t t = i / H;
        int h = (int)(i % H);
        float acc = 0.f;
        for (int j = 0; j < k; ++j) {
            int32_t r = row_of[t * k + j];
            if (r >= 0) acc = fmaf(topk_w[t * k + j], eo[(int64_t)r * H + h], acc);
        }
        if (shared) acc += eo[(S + t) * H + h];
        y[i] = from_f32<TOut>(acc);
    }
}

int grid_for(int64_t n, int threads) {
    int64_t b = (n + threads - 1) / threads;
    if (b > 148 * 32) b = 148 * 32;
    return b < 1 ? 1 : (int)b;
}

}  // namespace

static dim3 ffn_grid(const Plan& p, int64_t n_max) {
    int64_t mt = (p.S + kBM - 1) / kBM + p.E + (p.Is > 0 ? (p.T + kBM - 1) / kBM : 0);
    return dim3((unsigned)mt, (unsigned)((n_max + kBN - 1) / kBN));
}

cudaError_t launch_gather_rows(const Plan& p, const void* x, const int32_t* perm_rows,
                               const int32_t* offsets, void* xperm, cudaStream_t st) {
    if (p.S == 0) return cudaSuccess;
    const int64_t chunks = p.H * (p.bf16 ? 2 : 4) / 16;
    trace_before("gather_rows", st);
    gather_rows_kernel<<<grid_for(p.S * 32, 256), 256, 0, st>>>(
        (const uint4*)x, perm_rows, offsets, (int)p.E, (int)p.k, chunks, (uint4*)xperm);
    trace_after(st);
    return cudaGetLastError();
}

cudaError_t launch_scatter_x_rows(const Plan& p, const void* x, const int32_t* row_of, void* xperm,
                                  cudaStream_t st) {
    if (p.S == 0) return cudaSuccess;
    const int64_t chunks = p.H * (p.bf16 ? 2 : 4) / 16;
    trace_before("gather_rows", st);
    scatter_x_rows_kernel<<<grid_for(p.T * 32, 256), 256, 0, st>>>((const uint4*)x, row_of, p.T, (int)p.k, chunks,
                                                                   (uint4*)xperm);
    trace_after(st);
    return cudaGetLastError();
}

cudaError_t launch_gateup_simt(const Plan& p, const void* xperm, const void* x,
                               const int32_t* offsets, const void* w_gate, const void* w_up,
                               const void* ws_gate, const void* ws_up, void* h, cudaStream_t st) {
    if (p.T == 0) return cudaSuccess;
    dim3 grid = ffn_grid(p, p.I_max);
    void* hs = (float*)h + p.S * p.I;
    trace_before("gateup_simt", st);
    grouped_ffn_simt_kernel<float, true><<<grid, kThreads, 0, st>>>(
        p.S, p.T, (int)p.E, (int)p.k, (int)p.H, (int)p.I, (int)p.Is, offsets, (const float*)xperm,
        (const float*)x, (const float*)w_gate, (const float*)w_up, (const float*)ws_gate,
        (const float*)ws_up, (float*)h, (float*)hs, nullptr, nullptr, 0, nullptr);
    trace_after(st);
    return cudaGetLastError();
}

cudaError_t launch_down_simt(const Plan& p, const void* h, const int32_t* offsets,
                             const int32_t* perm_rows, const float* topk_w, const void* w_down,
                             const void* ws_down, int mode, void* out, cudaStream_t st) {
    if (p.T == 0) return cudaSuccess;
    dim3 grid = ffn_grid(p, p.H);
    const void* hs = (const float*)h + p.S * p.I;
    trace_before(mode ? "down_simt_weighted" : "down_simt", st);
    grouped_ffn_simt_kernel<float, false><<<grid, kThreads, 0, st>>>(
        p.S, p.T, (int)p.E, (int)p.k, (int)p.H, (int)p.I, (int)p.Is, offsets, (const float*)h,
        (const float*)hs, (const float*)w_down, nullptr, (const float*)ws_down, nullptr, nullptr,
        nullptr, perm_rows, topk_w, mode, out);
    trace_after(st);
    return cudaGetLastError();
}

cudaError_t launch_combine_rows(const Plan& p, const void* rows, const int32_t* row_of, void* y,
                                cudaStream_t st) {
    const int64_t n = p.T * p.H / (p.bf16 ? 8 : 4);
    if (n == 0) return cudaSuccess;
    trace_before("combine_rows", st);
    if (p.bf16 && p.y_f32)
        combine_rows_kernel<bf16, float><<<grid_for(n, 256), 256, 0, st>>>(
            (const bf16*)rows, row_of, p.T, (int)p.H, (int)p.k, p.S, p.Is > 0, (float*)y);
    else if (p.bf16)
        combine_rows_kernel<bf16, bf16><<<grid_for(n, 256), 256, 0, st>>>(
            (const bf16*)rows, row_of, p.T, (int)p.H, (int)p.k, p.S, p.Is > 0, (bf16*)y);
    else
        combine_rows_kernel<float, float><<<grid_for(n, 256), 256, 0, st>>>(
            (const float*)rows, row_of, p.T, (int)p.H, (int)p.k, p.S, p.Is > 0, (float*)y);
    trace_after(st);
    return cudaGetLastError();
}

cudaError_t launch_combine(const Plan& p, const float* expert_out, const int32_t* row_of,
                           const float* topk_w, void* y, cudaStream_t st) {
    const int64_t n = p.T * p.H;
    if (n == 0) return cudaSuccess;
    trace_before("combine", st);
    if (p.bf16)
        combine_kernel<bf16><<<grid_for(n, 256), 256, 0, st>>>(
            expert_out, row_of, topk_w, p.T, (int)p.H, (int)p.k, p.S, p.Is > 0, (bf16*)y);
    else
        combine_kernel<float><<<grid_for(n, 256), 256, 0, st>>>(
            expert_out, row_of, topk_w, p.T, (int)p.H, (int)p.k, p.S, p.Is > 0, (float*)y);
    trace_after(st);
    return cudaGetLastError();
}

}  // namespace moe
