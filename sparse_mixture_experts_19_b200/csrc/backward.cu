// Backward pass of the layer (bf16): every gradient, given the upstream
// gradient dy and the forward's routing.
//
// "Mixture of Experts (MoEs) in Transformers", section Training MoEs with
// Transformers (grouped-GEMM training of the experts); "MoE稀疏架构是什么？
// 从原理到落地的系统解读", section 四 (the forward these gradients belong
// to: top-k, softmax over the k selected scores, weighted sum of the chosen
// SwiGLU experts).  For a kept pair (token t, expert e, weight w):
//   g = W_g x, u = W_u x, h = silu(g) u (rounded to bf16 as in the forward)
//   dA' = W_d^T dy,  dw = dA' . h,  da = w dA'
//   dg = da u silu'(g),  du = da silu(g)
//   dW_d += w dy h^T,  dW_g += dg x^T,  dW_u += du x^T,  dx += W_g^T dg + W_u^T du
// and for every selected pair of a token (kept or dropped; a dropped pair
// has dw = 0) the softmax over the selected scores:
//   dl_j = w_j (dw_j - sum_i w_i dw_i),  dW_r[e_j] += dl_j x,  db[e_j] += dl_j,
//   dx += dl_j W_r[e_j].
// The shared expert is one more expert with w = 1 on every token.
//
// Layout: the kept rows of each routed expert are gathered into a padded
// grouped layout (each expert's rows start on a multiple of 64 and its
// padding rows are zero), so that the weight gradients, which reduce over an
// expert's rows, read whole 64-row steps of that expert only.  The products
// run on the tensor cores (gemm_bwd_sm100.cu); the kernels here move rows,
// apply the SwiGLU and softmax derivatives, and sum each token's gradient
// rows in slot order (float32, no atomics).
#include "common.cuh"

namespace moe {

// The tensor-core products of the backward pass (gemm_bwd_sm100.cu).
cudaError_t launch_bwd_gu_recompute(const void* A, int64_t R, const int32_t* goff, int groups, const void* wg,
                                    const void* wu, int I, int H, float* out, int32_t* flags, cudaStream_t st);
cudaError_t launch_bwd_down_dgrad(const void* dY, int64_t R, const int32_t* goff, int groups, const void* wd, int I,
                                  int H, float* out, int32_t* flags, cudaStream_t st);
cudaError_t launch_bwd_gateup_dgrad(const void* dGU, int64_t R, const int32_t* goff, int groups, const void* wg,
                                    const void* wu, int I, int H, float* out, int32_t* flags, cudaStream_t st);
cudaError_t launch_bwd_wgrad(const void* A, int64_t RA, const void* B, int64_t RB, const int32_t* goff, int groups,
                             int M, int N, int m_split, float* out0, float* out1, const char* name, int32_t* flags,
                             cudaStream_t st);

namespace {

constexpr int kPad = 64;

__host__ __device__ __forceinline__ int64_t pad64(int64_t v) { return (v + kPad - 1) / kPad * kPad; }

// Padded group offsets: poff[e] = sum over e' < e of pad64(kept rows of e').
__global__ void __launch_bounds__(256) bwd_pad_offsets_kernel(const int32_t* __restrict__ off, int E,
                                                              int32_t* __restrict__ poff) {
    __shared__ int32_t sm[kMaxExperts + 1];
    const int e = threadIdx.x;
    if (e < E) sm[e] = (int32_t)pad64(off[e + 1] - off[e]);
    __syncthreads();
    if (threadIdx.x == 0) {
        int32_t acc = 0;
        for (int i = 0; i < E; ++i) {
            poff[i] = acc;
            acc += sm[i];
        }
        poff[E] = acc;
    }
}

// For every kept row r of expert e (grouped order): its padded row p; the
// maps padded row -> token (-1: padding) and slot, and slot -> padded row.
__global__ void bwd_row_maps_kernel(const int32_t* __restrict__ perm_rows, const int32_t* __restrict__ off,
                                    const int32_t* __restrict__ poff, const int32_t* __restrict__ idx, int E, int k,
                                    int64_t S, int32_t* __restrict__ prow_tok, int32_t* __restrict__ prow_slot,
                                    int32_t* __restrict__ slot_prow) {
    const int64_t R = off[E];
    for (int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; r < R; r += (int64_t)gridDim.x * blockDim.x) {
        const int32_t s = perm_rows[r];
        const int e = idx[s];
        const int64_t p = poff[e] + (r - off[e]);
        prow_tok[p] = s / k;
        prow_slot[p] = s;
        slot_prow[s] = (int32_t)p;
    }
}

// Xp[p] = x[tok], dYp[p] = dy[tok] for every padded row (zeros for padding);
// one warp per row, 16-byte chunks.
__global__ void bwd_gather_kernel(const uint4* __restrict__ x, const uint4* __restrict__ dy,
                                  const int32_t* __restrict__ prow_tok, const int32_t* __restrict__ poff, int E,
                                  int64_t chunks, uint4* __restrict__ xp, uint4* __restrict__ dyp) {
    const int lane = threadIdx.x % 32;
    const int64_t Rp = poff[E];
    for (int64_t p = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 32; p < Rp;
         p += (int64_t)gridDim.x * blockDim.x / 32) {
        const int32_t t = prow_tok[p];
        for (int64_t c = lane; c < chunks; c += 32) {
            const uint4 zero = make_uint4(0, 0, 0, 0);
            xp[p * chunks + c] = t >= 0 ? x[t * chunks + c] : zero;
            dyp[p * chunks + c] = t >= 0 ? dy[t * chunks + c] : zero;
        }
    }
}

__device__ __forceinline__ float sigmoid_f32(float z) { return 1.f / (1.f + __expf(-z)); }

// SwiGLU backward of one row: GU [2I] float32 (g | u), dA [I] float32,
// weight w -> dGU [2I] bf16 (dg | du), hw [I] bf16 (w h); returns dA . h.
// One warp, eight consecutive elements per lane and pass (I is a multiple of
// 8: 16-byte loads and stores); pad rows write zeros and return 0.
__device__ float swiglu_backward_row(const float* __restrict__ gu, const float* __restrict__ da_row, float w,
                                     int I, bf16* __restrict__ dgu, bf16* __restrict__ hw, bool pad) {
    const int lane = threadIdx.x % 32;
    float dot = 0.f;
    for (int i = lane * 8; i < I; i += 32 * 8) {
        uint4 o_dg, o_du, o_hw;
        if (pad) {
            o_dg = o_du = o_hw = make_uint4(0, 0, 0, 0);
        } else {
            float g[8], u[8], d[8];
            *reinterpret_cast<float4*>(g) = *reinterpret_cast<const float4*>(gu + i);
            *reinterpret_cast<float4*>(g + 4) = *reinterpret_cast<const float4*>(gu + i + 4);
            *reinterpret_cast<float4*>(u) = *reinterpret_cast<const float4*>(gu + I + i);
            *reinterpret_cast<float4*>(u + 4) = *reinterpret_cast<const float4*>(gu + I + i + 4);
            *reinterpret_cast<float4*>(d) = *reinterpret_cast<const float4*>(da_row + i);
            *reinterpret_cast<float4*>(d + 4) = *reinterpret_cast<const float4*>(da_row + i + 4);
            __nv_bfloat162 rg[4], ru[4], rh[4];
#pragma unroll
            for (int j = 0; j < 8; j += 2) {
                float vg[2], vu[2], vh[2];
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    const float gj = g[j + h2], uj = u[j + h2];
                    const float sg = sigmoid_f32(gj);
                    const float silu = gj * sg;
                    const float h = __bfloat162float(__float2bfloat16_rn(silu * uj));  // the forward's bf16 h
                    dot = fmaf(d[j + h2], h, dot);
                    const float da = w * d[j + h2];
                    vg[h2] = da * uj * sg * (1.f + gj * (1.f - sg));
                    vu[h2] = da * silu;
                    vh[h2] = w * h;
                }
                rg[j / 2] = __floats2bfloat162_rn(vg[0], vg[1]);
                ru[j / 2] = __floats2bfloat162_rn(vu[0], vu[1]);
                rh[j / 2] = __floats2bfloat162_rn(vh[0], vh[1]);
            }
            o_dg = *reinterpret_cast<const uint4*>(rg);
            o_du = *reinterpret_cast<const uint4*>(ru);
            o_hw = *reinterpret_cast<const uint4*>(rh);
        }
        *reinterpret_cast<uint4*>(dgu + i) = o_dg;
        *reinterpret_cast<uint4*>(dgu + I + i) = o_du;
        *reinterpret_cast<uint4*>(hw + i) = o_hw;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
    return dot;
}

// Routed rows: warp per padded row; dw of the row's slot to dw_slot.
__global__ void bwd_swiglu_routed_kernel(const float* __restrict__ GU, const float* __restrict__ dA,
                                         const int32_t* __restrict__ prow_slot, const float* __restrict__ topk_w,
                                         const int32_t* __restrict__ poff, int E, int I, bf16* __restrict__ dGU,
                                         bf16* __restrict__ hw, float* __restrict__ dw_slot) {
    const int lane = threadIdx.x % 32;
    const int64_t Rp = poff[E];
    for (int64_t p = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 32; p < Rp;
         p += (int64_t)gridDim.x * blockDim.x / 32) {
        const int32_t s = prow_slot[p];
        const float w = s >= 0 ? topk_w[s] : 0.f;
        const float dot = swiglu_backward_row(GU + p * 2 * I, dA + p * I, w, I, dGU + p * 2 * I, hw + p * I, s < 0);
        if (lane == 0 && s >= 0) dw_slot[s] = dot;
    }
}

// Shared-expert rows (weight 1): rows t < T, padding rows up to Tpad zeroed.
__global__ void bwd_swiglu_shared_kernel(const float* __restrict__ GU, const float* __restrict__ dA, int64_t T,
                                         int64_t Tpad, int Is, bf16* __restrict__ dGU, bf16* __restrict__ hw) {
    for (int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 32; t < Tpad;
         t += (int64_t)gridDim.x * blockDim.x / 32) {
        const bool pad = t >= T;
        swiglu_backward_row(GU + (pad ? 0 : t) * 2 * Is, dA + (pad ? 0 : t) * Is, 1.f, Is, dGU + t * 2 * Is,
                            hw + t * Is, pad);
    }
}

// Softmax over the selected scores, backward; one thread per token:
// dl_j = w_j (dw_j - sum_i w_i dw_i) (dw = 0 for a dropped pair), written to
// dl_slot, to dL32 [T, E] and to dL [T, Epad] bf16 (zeros elsewhere, set by
// the caller).
__global__ void bwd_softmax_kernel(const int32_t* __restrict__ idx, const float* __restrict__ topk_w,
                                   const float* __restrict__ dw_slot, int64_t T, int k, int E, int Epad,
                                   float* __restrict__ dl_slot, float* __restrict__ dL32, bf16* __restrict__ dL) {
    for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < T; t += (int64_t)gridDim.x * blockDim.x) {
        float sw = 0.f;
        for (int j = 0; j < k; ++j) sw = fmaf(topk_w[t * k + j], dw_slot[t * k + j], sw);
        for (int j = 0; j < k; ++j) {
            const int64_t s = t * k + j;
            const float dl = topk_w[s] * (dw_slot[s] - sw);
            dl_slot[s] = dl;
            const int e = idx[s];
            dL32[t * E + e] = dl;
            dL[t * Epad + e] = __float2bfloat16_rn(dl);
        }
    }
}

// db[e] = sum over tokens of dL32[t, e], in two passes of fixed order:
// block b sums its token range (thread e: column e, tokens in order; rows
// read whole) into part[b][e], then thread e adds the parts in block order.
constexpr int kBiasBlocks = 128;
__global__ void __launch_bounds__(256) bwd_bias_part_kernel(const float* __restrict__ dL32, int64_t T, int E,
                                                            float* __restrict__ part) {
    const int64_t t0 = T * blockIdx.x / gridDim.x, t1 = T * (blockIdx.x + 1) / gridDim.x;
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        float acc = 0.f;
        for (int64_t t = t0; t < t1; ++t) acc += dL32[t * E + e];
        part[(int64_t)blockIdx.x * E + e] = acc;
    }
}
__global__ void bwd_bias_kernel(const float* __restrict__ part, int nparts, int E, float* __restrict__ db) {
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= E) return;
    float acc = 0.f;
    for (int b = 0; b < nparts; ++b) acc += part[(int64_t)b * E + e];
    db[e] = acc;
}

// dx[t] = sum over kept slots j (in order) of dXp[p(s)], + dXs[t] (shared),
// + sum over selected j of dl_j W_r[e_j]; float32, one thread per 4 columns.
__global__ void bwd_dx_kernel(const float* __restrict__ dXp, const float* __restrict__ dXs,
                              const int32_t* __restrict__ slot_prow, const int32_t* __restrict__ idx,
                              const float* __restrict__ dl_slot, const bf16* __restrict__ router_w, int64_t T, int H,
                              int k, float* __restrict__ dx) {
    const int q4 = H / 4;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < T * q4; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = i / q4;
        const int c = (int)(i % q4) * 4;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j = 0; j < k; ++j) {
            const int32_t p = slot_prow[t * k + j];
            if (p < 0) continue;
            const float4 v = *reinterpret_cast<const float4*>(dXp + (int64_t)p * H + c);
            acc.x += v.x;
            acc.y += v.y;
            acc.z += v.z;
            acc.w += v.w;
        }
        if (dXs) {
            const float4 v = *reinterpret_cast<const float4*>(dXs + t * H + c);
            acc.x += v.x;
            acc.y += v.y;
            acc.z += v.z;
            acc.w += v.w;
        }
        for (int j = 0; j < k; ++j) {
            const float dl = dl_slot[t * k + j];
            const bf16* wr = router_w + (int64_t)idx[t * k + j] * H + c;
            acc.x = fmaf(dl, __bfloat162float(wr[0]), acc.x);
            acc.y = fmaf(dl, __bfloat162float(wr[1]), acc.y);
            acc.z = fmaf(dl, __bfloat162float(wr[2]), acc.z);
            acc.w = fmaf(dl, __bfloat162float(wr[3]), acc.w);
        }
        *reinterpret_cast<float4*>(dx + t * H + c) = acc;
    }
}

// Offsets of the one-group products: {0, T} (the shared expert's rows, the
// router's reduction over tokens) and {0, Tpad} (the shared expert's padded
// reduction).
__global__ void bwd_aux_offsets_kernel(int32_t* aux, int32_t T, int32_t Tpad) {
    if (threadIdx.x == 0) {
        aux[0] = 0;
        aux[1] = T;
        aux[2] = 0;
        aux[3] = Tpad;
    }
}

int blocks(int64_t n, int threads) {
    int64_t b = (n + threads - 1) / threads;
    if (b > 148 * 16) b = 148 * 16;
    return b < 1 ? 1 : (int)b;
}

}  // namespace

// Workspace of the backward pass (carved after the forward plan's pieces).
struct BwdPlan {
    int64_t Rp, Tpad, Epad;
    int32_t *poff, *prow_tok, *prow_slot, *slot_prow, *aux;
    bf16 *xp, *dyp, *dgu, *hw, *dgus, *hws, *dL;
    float *gu, *da, *dxp, *gus, *das, *dxs, *dw_slot, *dl_slot, *dL32, *dwr, *bias_part;
    size_t bytes;
};

static size_t bwd_plan(const Plan& p, void* base, BwdPlan* b) {
    b->Rp = p.S + kPad * p.E;  // at most 63 padding rows per expert
    b->Tpad = p.Is ? pad64(p.T) : 0;
    b->Epad = pad64(p.E);
    size_t off = 0;
    char* c = (char*)base;
    auto take = [&](size_t bytes) -> void* {
        void* r = c ? c + off : nullptr;
        off += (bytes + kWsAlign - 1) / kWsAlign * kWsAlign;
        return r;
    };
    const int64_t H = p.H, I = p.I, Is = p.Is, T = p.T, S = p.S;
    b->poff = (int32_t*)take(sizeof(int32_t) * (p.E + 1));
    b->aux = (int32_t*)take(sizeof(int32_t) * 4);
    b->prow_tok = (int32_t*)take(sizeof(int32_t) * b->Rp);
    b->prow_slot = (int32_t*)take(sizeof(int32_t) * b->Rp);
    b->slot_prow = (int32_t*)take(sizeof(int32_t) * S);
    b->xp = (bf16*)take(2 * b->Rp * H);
    b->dyp = (bf16*)take(2 * b->Rp * H);
    b->gu = (float*)take(4 * b->Rp * 2 * I);
    b->da = (float*)take(4 * b->Rp * I);
    b->dgu = (bf16*)take(2 * b->Rp * 2 * I);
    b->hw = (bf16*)take(2 * b->Rp * I);
    b->dxp = (float*)take(4 * b->Rp * H);
    b->gus = (float*)take(4 * T * 2 * Is);
    b->das = (float*)take(4 * T * Is);
    b->dgus = (bf16*)take(2 * b->Tpad * 2 * Is);
    b->hws = (bf16*)take(2 * b->Tpad * Is);
    b->dxs = (float*)take(Is ? 4 * T * H : 0);
    b->dw_slot = (float*)take(4 * S);
    b->dl_slot = (float*)take(4 * S);
    b->dL32 = (float*)take(4 * T * p.E);
    b->dL = (bf16*)take(2 * T * b->Epad);
    b->dwr = (float*)take(4 * b->Epad * H);
    b->bias_part = (float*)take(4 * kBiasBlocks * p.E);
    b->bytes = off;
    return off;
}

#define BWD_TRY(expr)                         \
    do {                                      \
        cudaError_t e_ = (expr);              \
        if (e_ != cudaSuccess) return e_;     \
    } while (0)

// The backward pass after moe_permute has grouped the routing (p.offsets,
// p.perm_rows, p.row_of of the plan).
static cudaError_t run_backward(const Plan& p, const BwdPlan& b, const void* x, const void* dy, const int32_t* idx,
                         const float* topk_w, const void* router_w, const void* w_gate, const void* w_up,
                         const void* w_down, const void* ws_gate, const void* ws_up, const void* ws_down, float* dx,
                         float* d_router_w, float* d_router_b, float* d_w_gate, float* d_w_up, float* d_w_down,
                         float* d_ws_gate, float* d_ws_up, float* d_ws_down, cudaStream_t st) {
    const int E = (int)p.E, k = (int)p.k, H = (int)p.H, I = (int)p.I, Is = (int)p.Is;
    const int64_t T = p.T, S = p.S;
    // padded layout of the kept rows
    trace_before("bwd_layout", st);
    bwd_pad_offsets_kernel<<<1, 256, 0, st>>>(p.offsets, E, b.poff);
    bwd_aux_offsets_kernel<<<1, 32, 0, st>>>(b.aux, (int32_t)T, (int32_t)b.Tpad);
    BWD_TRY(cudaMemsetAsync(b.prow_tok, 0xff, sizeof(int32_t) * b.Rp, st));
    BWD_TRY(cudaMemsetAsync(b.prow_slot, 0xff, sizeof(int32_t) * b.Rp, st));
    BWD_TRY(cudaMemsetAsync(b.slot_prow, 0xff, sizeof(int32_t) * S, st));
    bwd_row_maps_kernel<<<blocks(S, 256), 256, 0, st>>>(p.perm_rows, p.offsets, b.poff, idx, E, k, S, b.prow_tok,
                                                        b.prow_slot, b.slot_prow);
    bwd_gather_kernel<<<blocks(b.Rp * 32, 256), 256, 0, st>>>((const uint4*)x, (const uint4*)dy, b.prow_tok, b.poff,
                                                              E, H / 8, (uint4*)b.xp, (uint4*)b.dyp);
    trace_after(st);
    BWD_TRY(cudaGetLastError());
    // recomputed gate/up pre-activations, the down projection's input gradient
    BWD_TRY(launch_bwd_gu_recompute(b.xp, b.Rp, b.poff, E, w_gate, w_up, I, H, b.gu, p.flags, st));
    BWD_TRY(launch_bwd_down_dgrad(b.dyp, b.Rp, b.poff, E, w_down, I, H, b.da, p.flags, st));
    // SwiGLU backward, dw per slot (dropped slots keep dw = 0)
    BWD_TRY(cudaMemsetAsync(b.dw_slot, 0, sizeof(float) * S, st));
    trace_before("bwd_swiglu", st);
    bwd_swiglu_routed_kernel<<<blocks(b.Rp * 32, 256), 256, 0, st>>>(b.gu, b.da, b.prow_slot, topk_w, b.poff, E, I,
                                                                     b.dgu, b.hw, b.dw_slot);
    trace_after(st);
    BWD_TRY(cudaGetLastError());
    if (Is > 0) {
        // the shared expert: one group of all T tokens, read in place from x and dy
        BWD_TRY(launch_bwd_gu_recompute(x, T, b.aux, 1, ws_gate, ws_up, Is, H, b.gus, p.flags, st));
        BWD_TRY(launch_bwd_down_dgrad(dy, T, b.aux, 1, ws_down, Is, H, b.das, p.flags, st));
    }
    // softmax over the selected scores, router gradients
    BWD_TRY(cudaMemsetAsync(b.dL32, 0, sizeof(float) * T * E, st));
    BWD_TRY(cudaMemsetAsync(b.dL, 0, sizeof(bf16) * T * b.Epad, st));
    trace_before("bwd_softmax", st);
    bwd_softmax_kernel<<<blocks(T, 256), 256, 0, st>>>(idx, topk_w, b.dw_slot, T, k, E, (int)b.Epad, b.dl_slot,
                                                       b.dL32, b.dL);
    bwd_bias_part_kernel<<<kBiasBlocks, 256, 0, st>>>(b.dL32, T, E, b.bias_part);
    bwd_bias_kernel<<<(E + 255) / 256, 256, 0, st>>>(b.bias_part, kBiasBlocks, E, d_router_b);
    trace_after(st);
    BWD_TRY(cudaGetLastError());
    // the experts' input gradient rows, then dx
    BWD_TRY(launch_bwd_gateup_dgrad(b.dgu, b.Rp, b.poff, E, w_gate, w_up, I, H, b.dxp, p.flags, st));
    if (Is > 0) {
        trace_before("bwd_swiglu", st);
        bwd_swiglu_shared_kernel<<<blocks(b.Tpad * 32, 256), 256, 0, st>>>(b.gus, b.das, T, b.Tpad, Is, b.dgus,
                                                                            b.hws);
        trace_after(st);
        BWD_TRY(cudaGetLastError());
        BWD_TRY(launch_bwd_gateup_dgrad(b.dgus, b.Tpad, b.aux, 1, ws_gate, ws_up, Is, H, b.dxs, p.flags, st));
    }
    trace_before("bwd_dx", st);
    bwd_dx_kernel<<<blocks(T * H / 4, 256), 256, 0, st>>>(b.dxp, Is > 0 ? b.dxs : nullptr, b.slot_prow, idx,
                                                          b.dl_slot, (const bf16*)router_w, T, H, k, dx);
    trace_after(st);
    BWD_TRY(cudaGetLastError());
    // weight gradients: reductions over each expert's padded rows
    BWD_TRY(launch_bwd_wgrad(b.dgu, b.Rp, b.xp, b.Rp, b.poff, E, 2 * I, H, I, d_w_gate, d_w_up, "bwd_wgrad_gateup",
                             p.flags, st));
    BWD_TRY(launch_bwd_wgrad(b.dyp, b.Rp, b.hw, b.Rp, b.poff, E, H, I, 0, d_w_down, nullptr, "bwd_wgrad_down",
                             p.flags, st));
    if (Is > 0) {
        // x and dy have T rows: the reduction's padding rows past T read as zero
        BWD_TRY(launch_bwd_wgrad(b.dgus, b.Tpad, x, T, b.aux + 2, 1, 2 * Is, H, Is, d_ws_gate, d_ws_up,
                                 "bwd_wgrad_gateup", p.flags, st));
        BWD_TRY(launch_bwd_wgrad(dy, T, b.hws, b.Tpad, b.aux + 2, 1, H, Is, 0, d_ws_down, nullptr, "bwd_wgrad_down",
                                 p.flags, st));
    }
    // router weights: dW_r = dL^T x over all T tokens (one group)
    BWD_TRY(launch_bwd_wgrad(b.dL, T, x, T, b.aux, 1, (int)b.Epad, H, 0, b.dwr, nullptr, "bwd_wgrad_router", p.flags,
                             st));
    BWD_TRY(cudaMemcpyAsync(d_router_w, b.dwr, sizeof(float) * E * H, cudaMemcpyDeviceToDevice, st));
    return cudaSuccess;
}

size_t backward_workspace_bytes(const Plan& p) {
    BwdPlan b;
    return bwd_plan(p, nullptr, &b);
}

cudaError_t launch_backward(const Plan& p, void* bwd_ws, const void* x, const void* dy, const int32_t* idx,
                            const float* topk_w, const void* router_w, const void* w_gate, const void* w_up,
                            const void* w_down, const void* ws_gate, const void* ws_up, const void* ws_down,
                            float* dx, float* d_router_w, float* d_router_b, float* d_w_gate, float* d_w_up,
                            float* d_w_down, float* d_ws_gate, float* d_ws_up, float* d_ws_down, cudaStream_t st) {
    BwdPlan b;
    bwd_plan(p, bwd_ws, &b);
    cudaError_t e = launch_permute(p, idx, p.counts, p.offsets, p.perm_rows, p.row_of, p.dropped, st);
    if (e != cudaSuccess) return e;
    return run_backward(p, b, x, dy, idx, topk_w, router_w, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, dx,
                        d_router_w, d_router_b, d_w_gate, d_w_up, d_w_down, d_ws_gate, d_ws_up, d_ws_down, st);
}

}  // namespace moe
