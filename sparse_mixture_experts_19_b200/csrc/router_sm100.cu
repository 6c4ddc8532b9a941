// Router scores, top-k and softmax over the selected scores for many tokens
// (bf16 layer): tensor-core partial scores, then an exact selection.
//
// "MoE稀疏架构是什么？从原理到落地的系统解读", section 三.1 (a small linear
// router gives one score per expert) and section 四 (keep the k best scores,
// softmax over those k).  "模型的“分工的艺术”：MoE技术如何提升计算效率",
// section 1.1 (the gate is a linear layer, here with an optional bias).
//
// 1. router_partial_kernel (tcgen05): the reduction over H is split into
//    ns chunks (ns <= 8, chunks of at least 512, multiples of 64); CTA
//    (tile, c) computes 128 tokens x all E experts over chunk c in float32
//    TMEM (E padded to a multiple of 16; the padding rows of the weight box
//    read as zero) and writes the float32 partial scores P_c[t, e].  The MMA
//    warp's idle lanes also read every staged x row and router row from
//    shared memory for their squared norms over the chunk.  Two CTAs share
//    an SM, so one's drain of its partials overlaps the other's MMAs.
// 2. router_select_kernel (CUDA cores, 32 tokens per block): the partials
//    are summed in float32 in chunk order with the bias, the selection is
//    made certain against a bound on the difference from the exact scores,
//    the uncertain experts are rescored exactly, and the k selected experts
//    are ordered exactly.
//
// Bound.  Each partial score is a float32 tensor-core sum of at most
// n = 4 * ceil(chunk / 64) MMA steps of 16 exact bf16 products.  Model of the
// tensor core, assumed rather than documented: one kind::f16 step adds its 16
// products to the accumulator D with an error of at most 17 * 2^-23 * (|D| +
// sum |products|), which covers 16 float32 additions with round-toward-zero
// in any order and a multi-term adder that aligns every term to the largest
// and truncates below 24 bits of it.  Summed over the steps, a partial score
// differs from its exact value by at most c * sum_h |x_h w_h| over the chunk,
// c = 17 * 2^-23 * (n + 1), and sum_h |x_h w_h| <= ||x_c|| ||w_c|| (Cauchy-
// Schwarz on the chunk).  The partials and the bias are then added in
// float32, in chunk order; those ns additions add at most
// (ns + 1) 2^-24 (sum_c ||x_{t,c}|| max_e ||w_{e,c}|| + max_e |b_e|).  So for
// token t every score is within
//   delta_t = sum_c c * ||x_{t,c}|| * max_e ||w_{e,c}|| (+ the sum's term)
// of exact (norms from float32 sums of squares inflated by 1 + H 2^-22, and
// the whole by 1.001).  Splitting the reduction makes the bound ns times
// smaller than one float32 sum over all of H.
//   Selection: with s_k, s_{k+1} the k-th and (k+1)-th approximate scores,
// an expert above s_{k+1} + 2 delta is certainly selected and one below
// s_k - 2 delta certainly not; the experts in between (the band) are rescored
// exactly (bf16 products are exact in float32, summed in fp64) and the
// selection is completed from those exact scores, ties to the lower index.
//   Order: two selected experts more than 2 delta apart are in the right
// order; every selected expert with another within 2 delta gets its exact
// score, and the k are sorted with exact scores where both have one and
// approximate ones otherwise, which is the exact order.
//
// Importance (optional): each token's thread forms its softmax over all E
// approximate scores; a block sums its tokens' probabilities per expert in
// shared memory and adds them to the importance with one atomic add per
// expert and block.
#include <algorithm>

#include "common.cuh"
#include "sm100.cuh"
#include "tma_host.cuh"

namespace moe {
namespace {

using namespace sm100;

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kMaxStages = 6;
constexpr int kThreads = 192;
constexpr int kABytes = kBM * kBK * 2;
constexpr int kMinChunk = 512;

// Sum of squares of the 64 bf16 values of one 128-byte row of a swizzled
// shared-memory tile at shared address `row`; lane l reads its 16-byte
// chunks starting at chunk l % 8, so 32 lanes reading 32 rows at once touch
// every bank equally (the swizzle permutes chunks inside a row, which a sum
// of squares does not see).
__device__ __forceinline__ float row_sumsq(uint32_t row, int lane) {
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        uint4 v;
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                     : "r"(row + (uint32_t)(((i + lane) & 7) * 16)));
        const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 f = __bfloat1622float2(p[j]);
            s = fmaf(f.x, f.x, s);
            s = fmaf(f.y, f.y, s);
        }
    }
    return s;
}

// One CTA: tile `tile` of 128 tokens, chunk c of the reduction.
__global__ void __launch_bounds__(kThreads, 2) router_partial_kernel(
    const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW, int T, int H, int E, int Npad,
    int ns, int kchunk, int stages, uint32_t acc_cols, float* __restrict__ part, float* __restrict__ xn2,
    float* __restrict__ wn2, int32_t* flags) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int stage_bytes = kABytes + Npad * kBK * 2;  // a multiple of 1024
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + stages * stage_bytes);
    uint64_t* empty = full + kMaxStages;
    uint64_t* tfull = empty + kMaxStages;
    uint64_t* drain = tfull + 1;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int tile = blockIdx.x / ns, c = blockIdx.x % ns;
    const int k0 = c * kchunk, k1 = min(H, k0 + kchunk);
    const int nkb = (k1 - k0 + kBK - 1) / kBK;
    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 2);  // the MMAs' commit and the norm pass
        }
        mbar_init(tfull, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, acc_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_map(&tmX);
            tma_prefetch_map(&tmW);
            int kb = 0;
            for (; kb < nkb; ++kb) {
                const int s = kb % stages;
                const uint32_t ph = (kb / stages) & 1;
                if (!wait_or_abort(&empty[s], ph ^ 1, abort_flag, flags, MOE_DEVFLAG_WAIT_TIMEOUT)) break;
                uint8_t* sa = smem + s * stage_bytes;
                mbar_arrive_expect_tx(&full[s], stage_bytes);
                tma_load_3d(sa, &tmX, &full[s], k0 + kb * kBK, tile * kBM, 0);
                tma_load_3d(sa + kABytes, &tmW, &full[s], k0 + kb * kBK, 0, 0);
            }
            for (int j = (kb > stages ? kb - stages : 0); j < kb; ++j) drain_wait(&full[j % stages], (j / stages) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (lane 0) + norms (all lanes)
        const uint32_t idesc = idesc_bf16(kBM, Npad);
        float xsq[kBM / 32];
        float wsq[kMaxExperts / 32];
#pragma unroll
        for (int q = 0; q < kBM / 32; ++q) xsq[q] = 0.f;
#pragma unroll
        for (int i = 0; i < kMaxExperts / 32; ++i) wsq[i] = 0.f;
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb) {
            const int s = kb % stages;
            const uint32_t ph = (kb / stages) & 1;
            if (!wait_or_abort(&full[s], ph, abort_flag, flags, MOE_DEVFLAG_WAIT_TIMEOUT)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t a0 = smem_u32(smem + s * stage_bytes);
            const uint32_t b0 = a0 + kABytes;
            if (lane == 0) {
#pragma unroll
                for (int kk = 0; kk < kBK / 16; ++kk)
                    mma_bf16(tmem_base, desc_kmajor_sw128(a0 + kk * 32), desc_kmajor_sw128(b0 + kk * 32), idesc,
                             (kb | kk) != 0);
                mma_commit(&empty[s]);
            }
#pragma unroll
            for (int q = 0; q < kBM / 32; ++q) xsq[q] += row_sumsq(a0 + (uint32_t)(lane + 32 * q) * 128u, lane);
            if (tile == 0) {
#pragma unroll
                for (int i = 0; i < kMaxExperts / 32; ++i)
                    if (lane + 32 * i < Npad) wsq[i] += row_sumsq(b0 + (uint32_t)(lane + 32 * i) * 128u, lane);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }
        if (ok) {
            if (lane == 0) mma_commit(tfull);
#pragma unroll
            for (int q = 0; q < kBM / 32; ++q) {
                const int t = tile * kBM + lane + 32 * q;
                if (t < T) xn2[(int64_t)c * T + t] = xsq[q];
            }
            if (tile == 0) {
#pragma unroll
                for (int i = 0; i < kMaxExperts / 32; ++i)
                    if (lane + 32 * i < E) wn2[c * E + lane + 32 * i] = wsq[i];
            }
        }
        if (lane == 0) {
            // every MMA issued has finished before TMEM is freed
            mma_commit(drain);
            drain_wait(drain, 0);
        }
    } else {
        // ------------------------------------------------ epilogue warps 2..5: partials -> global
        const int q = warp & 3;
        const int t = tile * kBM + q * 32 + lane;
        if (wait_or_abort(tfull, 0, abort_flag, flags, MOE_DEVFLAG_WAIT_TIMEOUT)) {
            tc_fence_after();
            const uint32_t tq = tmem_base + ((uint32_t)(q * 32) << 16);
            float* dst = part + ((int64_t)c * T + t) * E;
            const bool vec = (E % 4) == 0;
            for (int c0 = 0; c0 < E; c0 += 64) {
                float v[64];
                tmem_ld64(tq + c0, v);  // columns past E (up to the allocation) are ignored
                if (t < T) {
                    if (vec) {
#pragma unroll
                        for (int i = 0; i < 64; i += 4)
                            if (c0 + i < E)
                                *reinterpret_cast<float4*>(dst + c0 + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
                    } else {
#pragma unroll
                        for (int i = 0; i < 64; ++i)
                            if (c0 + i < E) dst[c0 + i] = v[i];
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, acc_cols);
}

// Exact score x_t . W_r[e] in fp64 by one warp (bf16 products are exact in
// float32, summed in fp64); every lane gets the result.
__device__ __forceinline__ double exact_score(const bf16* x, const bf16* w, int64_t t, int e, int H, int lane) {
    const uint4* xr = reinterpret_cast<const uint4*>(x + t * H);
    const uint4* wr = reinterpret_cast<const uint4*>(w + (int64_t)e * H);
    const int nch = H / 8;
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
    for (int c = lane; c < nch; c += 128) {
        uint4 a[4], bq[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int cu = c + 32 * u;
            a[u] = cu < nch ? xr[cu] : make_uint4(0, 0, 0, 0);
            bq[u] = cu < nch ? wr[cu] : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&a[u]);
            const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&bq[u]);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 fa = __bfloat1622float2(pa[i]), fb = __bfloat1622float2(pb[i]);
                acc[u] += (double)__fmul_rn(fa.x, fb.x);
                acc[u] += (double)__fmul_rn(fa.y, fb.y);
            }
        }
    }
    double sum = (acc[0] + acc[1]) + (acc[2] + acc[3]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    return sum;
}

// float -> unsigned with the same order (-0 taken as +0, so that equal floats
// get equal keys), and back.
__device__ __forceinline__ unsigned ordered_key(float v) {
    const unsigned u = __float_as_uint(v == 0.f ? 0.f : v);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float from_ordered_key(unsigned k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// (a, ea) ranks before (b, eb): larger score, then lower expert index.
__device__ __forceinline__ bool ranks_before(float a, int ea, float b, int eb) {
    return a > b || (a == b && ea < eb);
}
__device__ __forceinline__ bool ranks_before(double a, int ea, double b, int eb) {
    return a > b || (a == b && ea < eb);
}

constexpr int kSelTokens = 32;                 // tokens per block of the selection kernel
constexpr int kSelThreads = 256;               // eight warps
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kSelTokPerWarp = kSelTokens / kSelWarps;  // tokens a warp scans
constexpr int kSeg = 32;                       // queue entries per warp and round (band members)
constexpr int kPendQ = 128;                    // queue entries per round for certain picks
constexpr int kQueue = kSelWarps * kSeg + kPendQ;

// Shared memory of the selection kernel: summed scores [32][E + 1] (the +1
// spreads a column over the banks), then the rescoring queue.
size_t select_smem_bytes(int E) {
    return sizeof(float) * kSelTokens * (E + 1) + (size_t)kQueue * (8 + 8 + 4) + 64;
}

// The token's scores summed from the chunks' partials into shared memory
// (float32, chunk order); then
//   scan (a warp per token, four tokens per warp at once): lane l holds the
//     scores of experts l, l + 32, ...; the kk best are picked in kk rounds
//     of warp arg-max (ties to the lower index); the importance adds its
//     softmax over all E scores here;
//   decision (a thread per token): the bound, the band, the certain picks
//     that need exact scores for the order;
//   rescoring (every warp): band members found by the token's warp (ballot
//     over 32 experts at a time) and the certain picks go through a queue
//     whose exact scores every warp computes;
//   finish (a thread per token): the band decided from exact scores, the k
//     ordered exactly, the softmax over the k.
// Every long loop runs across a warp's lanes: a thread walking a whole row
// of E scores alone spends most of its time waiting on its own dependent
// instructions.
template <int KMAX, int kNV>
__global__ void __launch_bounds__(kSelThreads) router_select_kernel(
    const float* __restrict__ part, const float* __restrict__ xn2, const float* __restrict__ wn2, int T, int H, int E,
    int k, int ns, float cH, const float* __restrict__ bias, const bf16* __restrict__ x,
    const bf16* __restrict__ wr, int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
    float* __restrict__ importance) {
    constexpr bool kDense = (KMAX == kMaxTopK);
    // kNV = ceil(E / 32): scores per lane in the scan
    extern __shared__ __align__(16) uint8_t sm_raw[];
    const int ld = E + 1;
    float* sc = reinterpret_cast<float*>(sm_raw);                          // [32][E + 1]
    int2* qp = reinterpret_cast<int2*>(sc + (size_t)kSelTokens * ld + 1);  // 16-byte aligned below
    qp = reinterpret_cast<int2*>((reinterpret_cast<uintptr_t>(qp) + 15) & ~uintptr_t(15));
    double* qs = reinterpret_cast<double*>(qp + kQueue);
    float* qa = reinterpret_cast<float*>(qs + kQueue);
    __shared__ float wmax[kRouterMaxSplits];
    __shared__ float bmax_s;
    __shared__ float s_tv[kSelTokens][KMAX + 1];  // the scan's picks per token
    __shared__ int s_te[kSelTokens][KMAX + 1];
    __shared__ float s_lo[kSelTokens], s_hi[kSelTokens];  // band of each token
    __shared__ int s_cur[kSelTokens];                     // next expert of the band scan (E: done)
    __shared__ int s_segn[kSelWarps];                     // band entries per warp segment
    __shared__ int s_pn;                                  // certain-pick entries
    __shared__ float s_imp[kMaxExperts];
    const int r = threadIdx.x, lane = r & 31, warp = r / 32;
    const int t0 = blockIdx.x * kSelTokens;
    const int rows = min(kSelTokens, T - t0);
    const float slack = 1.f + (float)H * 2.3841858e-7f;  // 1 + H 2^-22
    if (importance)
        for (int e = r; e < E; e += kSelThreads) s_imp[e] = 0.f;
    // per chunk the largest router-row norm (warp c), and the largest |bias|
    // (warp ns, or the last warp): lanes stride over the experts, so the
    // loads are in flight together
    for (int c = warp; c < ns; c += kSelWarps) {
        float m = 0.f;
        for (int e = lane; e < E; e += 32) m = fmaxf(m, wn2[c * E + e]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) wmax[c] = sqrtf(m * slack);
    }
    if (warp == min(ns, kSelWarps - 1)) {
        float m = 0.f;
        if (bias)
            for (int e = lane; e < E; e += 32) m = fmaxf(m, fabsf(bias[e]));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) bmax_s = m;
    }
    // summed scores, chunks added in order 0..ns-1 and then the bias; the
    // block's rows of each chunk are one contiguous run, and every chunk's
    // load of an element is issued before the first add, so each thread
    // keeps ns loads in flight (float4 ones when E is a multiple of 4)
    {
        const float* src = part + (int64_t)t0 * E;
        const int64_t cstride = (int64_t)T * E;
        if ((E & 3) == 0) {
            const int n4 = rows * E / 4;
            for (int i4 = r; i4 < n4; i4 += kSelThreads) {
                float4 v[kRouterMaxSplits];
#pragma unroll
                for (int c = 0; c < kRouterMaxSplits; ++c)
                    if (c < ns) v[c] = __ldg(reinterpret_cast<const float4*>(src + c * cstride) + i4);
                float4 a = v[0];
#pragma unroll
                for (int c = 1; c < kRouterMaxSplits; ++c)
                    if (c < ns) {
                        a.x += v[c].x;
                        a.y += v[c].y;
                        a.z += v[c].z;
                        a.w += v[c].w;
                    }
                const int rr = (4 * i4) / E, e = (4 * i4) % E;
                if (bias) {
                    a.x += bias[e];
                    a.y += bias[e + 1];
                    a.z += bias[e + 2];
                    a.w += bias[e + 3];
                }
                float* d = sc + rr * ld + e;
                d[0] = a.x;
                d[1] = a.y;
                d[2] = a.z;
                d[3] = a.w;
            }
        } else {
            for (int i = r; i < rows * E; i += kSelThreads) {
                float v[kRouterMaxSplits];
#pragma unroll
                for (int c = 0; c < kRouterMaxSplits; ++c)
                    if (c < ns) v[c] = __ldg(src + c * cstride + i);
                float a = v[0];
#pragma unroll
                for (int c = 1; c < kRouterMaxSplits; ++c)
                    if (c < ns) a += v[c];
                if (bias) a += bias[i % E];
                sc[(i / E) * ld + i % E] = a;
            }
        }
    }
    __syncthreads();
    const int kk = k < E ? k + 1 : k;  // picks of the scan: k, and the (k+1)-th unless k == E

    // ---------------------------------------------------------- scan
    // warp w takes tokens w, w + 8, w + 16, w + 24 together (independent
    // chains hide each other's latency)
    {
        float v[kSelTokPerWarp][kNV];
        float pv[kSelTokPerWarp], top[kSelTokPerWarp];
        int pe[kSelTokPerWarp];
#pragma unroll
        for (int u = 0; u < kSelTokPerWarp; ++u) {
            const int tt = warp + kSelWarps * u;
            const float* row = sc + min(tt, kSelTokens - 1) * ld;
#pragma unroll
            for (int i = 0; i < kNV; ++i) {
                const int e = lane + 32 * i;
                v[u][i] = (tt < rows && e < E) ? row[e] : -INFINITY;
            }
            pv[u] = INFINITY;
            pe[u] = -1;
            top[u] = -INFINITY;
        }
#pragma unroll 1
        for (int j = 0; j < kk; ++j) {
            float bv[kSelTokPerWarp];
            int be[kSelTokPerWarp];
#pragma unroll
            for (int u = 0; u < kSelTokPerWarp; ++u) {
                // this lane's best score ranking after the previous pick
                // (ascending experts: the first of equal scores is kept)
                bv[u] = -INFINITY;
                be[u] = 0x7fffffff;
#pragma unroll
                for (int i = 0; i < kNV; ++i) {
                    const int e = lane + 32 * i;
                    const float c = v[u][i];
                    const bool after = (c < pv[u]) || (c == pv[u] && e > pe[u]);
                    if (e < E && after && c > -INFINITY && (c > bv[u] || (c == bv[u] && e < be[u]))) {
                        bv[u] = c;
                        be[u] = e;
                    }
                }
            }
            // warp arg-max: the largest score (one max reduction over
            // order-preserving keys), then the lowest expert index among the
            // lanes holding it (one min reduction)
            unsigned key[kSelTokPerWarp], m[kSelTokPerWarp];
#pragma unroll
            for (int u = 0; u < kSelTokPerWarp; ++u) {
                key[u] = ordered_key(bv[u]);
                m[u] = __reduce_max_sync(0xffffffffu, key[u]);
            }
#pragma unroll
            for (int u = 0; u < kSelTokPerWarp; ++u) {
                be[u] = (int)__reduce_min_sync(0xffffffffu, key[u] == m[u] ? (unsigned)be[u] : 0xffffffffu);
                bv[u] = from_ordered_key(m[u]);
            }
#pragma unroll
            for (int u = 0; u < kSelTokPerWarp; ++u) {
                const int tt = warp + kSelWarps * u;
                pv[u] = bv[u];
                pe[u] = be[u];
                if (j == 0) top[u] = bv[u];
                if (lane == 0 && tt < kSelTokens) {
                    s_tv[tt][j] = bv[u];
                    s_te[tt][j] = be[u];
                }
            }
        }
        if (lane == 0)
#pragma unroll
            for (int u = 0; u < kSelTokPerWarp; ++u) {
                const int tt = warp + kSelWarps * u;
                for (int j = kk; j <= KMAX; ++j) {
                    s_tv[tt][j] = -INFINITY;
                    s_te[tt][j] = 0x7fffffff;
                }
            }
        if (importance) {
            // softmax over all E scores of the token, shifted by its largest
            // (the first pick), summed per expert over the block
#pragma unroll
            for (int u = 0; u < kSelTokPerWarp; ++u) {
                const int tt = warp + kSelWarps * u;
                if (tt >= rows) continue;
                const float m = top[u];
                float z = 0.f;
#pragma unroll
                for (int i = 0; i < kNV; ++i)
                    if (lane + 32 * i < E) z += __expf(v[u][i] - m);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
                const float inv = 1.0f / z;
#pragma unroll
                for (int i = 0; i < kNV; ++i)
                    if (lane + 32 * i < E) atomicAdd(&s_imp[lane + 32 * i], __expf(v[u][i] - m) * inv);
            }
        }
    }
    __syncthreads();
    if (importance) {
        for (int e = r; e < E; e += kSelThreads) atomicAdd(&importance[e], s_imp[e]);
    }
    // ---------------------------------------------------------- decision
    // thread r carries token t = t0 + r (r < rows)
    const int t = t0 + r;
    const bool own = r < rows;
    float tv[KMAX + 1];
    int te[KMAX + 1];
#pragma unroll
    for (int j = 0; j <= KMAX; ++j) {
        tv[j] = own ? s_tv[r][j] : -INFINITY;
        te[j] = own ? s_te[r][j] : 0x7fffffff;
    }
    // the bound on |approximate - exact score| for this token (file comment),
    // with the float32 sums of the chunks and the bias counted in
    float delta = 0.f, nsum = 0.f;
    if (own)
        for (int c = 0; c < ns; ++c) {
            const float a = sqrtf(xn2[(int64_t)c * T + t] * slack) * wmax[c];
            delta += cH * a;
            nsum += a;
        }
    const float u24 = 5.9604645e-8f;
    const float del2 = 2.f * 1.001f * (delta + (float)(ns + 1) * u24 * (nsum + bmax_s));
    float band_lo = 0.f, band_hi = 0.f;
    bool uncertain = false;
    int n_in = k;  // slots 0 .. n_in-1 hold certain picks
    if (!kDense && own && k < E) {
        float kth = 0.f, next = 0.f;
#pragma unroll
        for (int j = 0; j <= KMAX; ++j) {
            if (j == k - 1) kth = tv[j];
            if (j == k) next = tv[j];
        }
        if (kth - next <= del2) {
            uncertain = true;
            band_lo = kth - del2;
            band_hi = next + del2;
            n_in = 0;
#pragma unroll
            for (int j = 0; j < KMAX; ++j)
                if (j < k && tv[j] > band_hi) n_in = j + 1;
        }
    }
    if (r < kSelTokens) {
        s_lo[r] = band_lo;
        s_hi[r] = band_hi;
        s_cur[r] = uncertain ? 0 : E;
    }
    // the k selected: approximate fa, expert fe, exact fx where known (has_x)
    float fa[KMAX];
    int fe[KMAX];
    double fx[KMAX];
    uint32_t has_x = 0;
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
        fa[j] = tv[j];
        fe[j] = te[j];
        fx[j] = 0.0;
    }
    // order: two selected experts within 2 delta need exact scores.  Among
    // the certain picks (sorted) that is every pick with a neighbour within
    // 2 delta; the last certain pick is also compared with the best band
    // score, which bounds every band pick from above.  Band members are all
    // rescored, so one rescoring pass covers selection and order.
    uint32_t pend = 0;
    if (own) {
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            if (j + 1 < n_in && tv[j] - tv[j + 1] <= del2) pend |= 3u << j;
            if (uncertain && j == n_in - 1 && tv[j] - tv[j + 1] <= del2) pend |= 1u << j;
        }
    }
    // band: the best `need` members by exact score (ties to the lower index)
    const int need = k - n_in;
    double bv[KMAX];
    int be[KMAX];
    float ba[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
        bv[j] = -INFINITY;
        be[j] = 0x7fffffff;
        ba[j] = -INFINITY;
    }
    if (r == 0) s_pn = 0;
    __syncthreads();
    // ---------------------------------------------------------- rescoring
    constexpr int kCertain = 1 << 30;  // queue tag: a certain pick's rescoring
    while (__syncthreads_or(pend != 0 || (own && s_cur[r] < E))) {
        // band members of the warp's tokens, 32 experts per ballot, into the
        // warp's segment of the queue; a token whose next hits do not fit
        // resumes there next round (a segment holds one whole ballot)
        {
            int wn = 0;
            bool full = false;
#pragma unroll 1
            for (int u = 0; u < kSelTokPerWarp && !full; ++u) {
                const int tt = warp + kSelWarps * u;
                if (tt >= rows) break;
                int cur = s_cur[tt];
                if (cur >= E) continue;
                const float lo = s_lo[tt], hi = s_hi[tt];
                const float* row = sc + tt * ld;
                for (; cur < E; cur += 32) {
                    const int e = cur + lane;
                    const float sv = e < E ? row[e] : 0.f;
                    const bool hit = e < E && sv >= lo && sv <= hi;
                    const unsigned m = __ballot_sync(0xffffffffu, hit);
                    const int nh = __popc(m);
                    if (wn + nh > kSeg) {
                        full = true;
                        break;
                    }
                    if (hit) {
                        const int slot = warp * kSeg + wn + __popc(m & ((1u << lane) - 1u));
                        qp[slot] = make_int2(tt, e);
                        qa[slot] = sv;
                    }
                    wn += nh;
                }
                __syncwarp();
                if (lane == 0) s_cur[tt] = cur;  // >= E: done
            }
            if (lane == 0) s_segn[warp] = wn;
        }
        // certain picks that need exact scores for the order
        if (pend != 0) {
#pragma unroll
            for (int j = 0; j < KMAX; ++j)
                if ((pend >> j) & 1u) {
                    const int slot = atomicAdd(&s_pn, 1);
                    if (slot < kPendQ) {
                        qp[kSelWarps * kSeg + slot] = make_int2(r, te[j] | kCertain);
                        pend &= ~(1u << j);
                    }
                }
        }
        __syncthreads();
        // exact scores of every entry: the warps' segments in warp order, then
        // the certain picks
        const int npn = min(s_pn, kPendQ);
        int total = npn;
#pragma unroll
        for (int w = 0; w < kSelWarps; ++w) total += s_segn[w];
        for (int i = warp; i < total; i += kSelWarps) {
            int q = i, w = 0;
            while (w < kSelWarps && q >= s_segn[w]) {
                q -= s_segn[w];
                ++w;
            }
            const int slot = w * kSeg + q;  // w == kSelWarps: the certain picks
            const int2 pr = qp[slot];
            const int e = pr.y & ~kCertain;
            const double sd = exact_score(x, wr, t0 + pr.x, e, H, lane);
            if (lane == 0) qs[slot] = sd + (bias ? (double)bias[e] : 0.0);
        }
        __syncthreads();
        if (own) {
            // band members: only the segment of the warp that scanned token r
            const int w0 = r % kSelWarps;
            for (int q = 0; q < s_segn[w0]; ++q) {
                const int slot = w0 * kSeg + q;
                const int2 pr = qp[slot];
                if (pr.x != r) continue;
                double cv = qs[slot];
                int ce = pr.y;
                float ca = qa[slot];
#pragma unroll
                for (int j = 0; j < KMAX; ++j) {
                    if (j < need && (cv > bv[j] || (cv == bv[j] && ce < be[j]))) {
                        const double ov = bv[j];
                        const int oe = be[j];
                        const float oa = ba[j];
                        bv[j] = cv;
                        be[j] = ce;
                        ba[j] = ca;
                        cv = ov;
                        ce = oe;
                        ca = oa;
                    }
                }
            }
            for (int q = 0; q < npn; ++q) {
                const int slot = kSelWarps * kSeg + q;
                const int2 pr = qp[slot];
                if (pr.x != r) continue;
                const int e = pr.y & ~kCertain;
#pragma unroll
                for (int j = 0; j < KMAX; ++j)
                    if (j < n_in && fe[j] == e) {
                        fx[j] = qs[slot];
                        has_x |= 1u << j;
                    }
            }
        }
        if (r == 0) s_pn = 0;  // read above into npn; the next pushes follow the loop's barrier
    }
    if (!kDense && uncertain) {
        // move the band picks to slots n_in..k-1 (predicated shifts keep
        // every index static: registers, no stack)
#pragma unroll
        for (int sft = 0; sft < KMAX; ++sft)
            if (sft < n_in) {
#pragma unroll
                for (int j = KMAX - 1; j > 0; --j) {
                    bv[j] = bv[j - 1];
                    be[j] = be[j - 1];
                    ba[j] = ba[j - 1];
                }
            }
#pragma unroll
        for (int j = 0; j < KMAX; ++j)
            if (j >= n_in && j < k) {
                fa[j] = ba[j];
                fe[j] = be[j];
                fx[j] = bv[j];
                has_x |= 1u << j;
            }
    }
    // sort the k by (score desc, index asc): exact scores where both have
    // one, else approximate ones (more than 2 delta apart, in the right order)
#pragma unroll 1
    for (int pass = 0; pass + 1 < KMAX; ++pass) {
#pragma unroll
        for (int j = 0; j + 1 < KMAX; ++j) {
            if (j + 1 < k) {
                const bool both = ((has_x >> j) & (has_x >> (j + 1)) & 1u) != 0;
                const bool swap = both ? ranks_before(fx[j + 1], fe[j + 1], fx[j], fe[j])
                                       : ranks_before(fa[j + 1], fe[j + 1], fa[j], fe[j]);
                if (swap) {
                    const float ta = fa[j];
                    fa[j] = fa[j + 1];
                    fa[j + 1] = ta;
                    const int ti = fe[j];
                    fe[j] = fe[j + 1];
                    fe[j + 1] = ti;
                    const double tx = fx[j];
                    fx[j] = fx[j + 1];
                    fx[j + 1] = tx;
                    const uint32_t bj = (has_x >> j) & 1u, bj1 = (has_x >> (j + 1)) & 1u;
                    has_x = (has_x & ~(3u << j)) | (bj << (j + 1)) | (bj1 << j);
                }
            }
        }
    }
    if (own) {
        // softmax over the k selected; differences in fp64 where both scores are exact
        double sj[KMAX];
#pragma unroll
        for (int j = 0; j < KMAX; ++j) sj[j] = ((has_x >> j) & 1u) ? fx[j] : (double)fa[j];
        float z = 0.f;
#pragma unroll
        for (int j = 0; j < KMAX; ++j)
            if (j < k) z += expf((float)(sj[j] - sj[0]));
        const float inv = 1.0f / z;
#pragma unroll
        for (int j = 0; j < KMAX; ++j)
            if (j < k) {
                topk_idx[(int64_t)t * k + j] = fe[j] < E ? fe[j] : -1;
                topk_w[(int64_t)t * k + j] = expf((float)(sj[j] - sj[0])) * inv;
            }
    }
}

}  // namespace

void router_splits(int64_t H, int* ns, int* kchunk) {
    int n = (int)std::min<int64_t>(kRouterMaxSplits, std::max<int64_t>(1, (H + kMinChunk - 1) / kMinChunk));
    const int64_t ch = ((H + n - 1) / n + kBK - 1) / kBK * kBK;
    n = (int)((H + ch - 1) / ch);
    *ns = n;
    *kchunk = (int)ch;
}

cudaError_t launch_router_sm100(const Plan& p, const void* x, const void* router_w, const float* router_b,
                                int32_t* topk_idx, float* topk_w, cudaStream_t st) {
    if (p.T == 0) return cudaSuccess;
    const int E = (int)p.E;
    const int Npad = E <= 16 ? 16 : (E + 15) / 16 * 16;
    // accumulator width: a power of two >= Npad and >= 64, so that the
    // epilogue's 64-column TMEM reads stay inside the accumulator
    uint32_t cols = 64;
    while ((int)cols < Npad) cols <<= 1;
    CUtensorMap mx, mw;
    if (!make_map_bf16(&mx, x, p.H, p.T, 1, kBK, kBM) || !make_map_bf16(&mw, router_w, p.H, E, 1, kBK, Npad))
        return cudaErrorInvalidValue;
    int ns, kchunk;
    router_splits(p.H, &ns, &kchunk);
    const int stage_bytes = kABytes + Npad * kBK * 2;
    const size_t fixed = 1024 + 256;  // alignment slack + barrier block
    // a ring small enough for two CTAs per SM (and two accumulators in TMEM,
    // 2 x 256 columns at most): one CTA's drain of its partials overlaps the
    // other's loads and MMAs
    int stages = (int)((113 * 1024 - fixed) / stage_bytes);
    stages = std::max(2, std::min(stages, kMaxStages));
    stages = std::min(stages, (kchunk + kBK - 1) / kBK);
    const size_t smem = (size_t)stages * stage_bytes + fixed;
    const int ntiles = (int)((p.T + kBM - 1) / kBM);
    cudaError_t e = ensure_smem_attr(router_partial_kernel, smem);
    if (e != cudaSuccess) return e;
    trace_before("router_sm100", st);
    router_partial_kernel<<<(unsigned)(ntiles * ns), kThreads, smem, st>>>(mx, mw, (int)p.T, (int)p.H, E, Npad, ns,
                                                                          kchunk, stages, cols, p.rt_part, p.rt_xn2,
                                                                          p.rt_wn2, p.flags);
    trace_after(st);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // the bound's constant for the longest chunk: 4 MMA steps per 64 of reduction
    const float cH = 17.f * 1.1920929e-7f * (float)(4 * ((kchunk + kBK - 1) / kBK) + 1) * 1.01f;
    const size_t ssm = select_smem_bytes(E);
    const dim3 sgrid((unsigned)((p.T + kSelTokens - 1) / kSelTokens));
    trace_before("router_select", st);
    // top_k > 8 only as top_k == E <= 32; kNV covers E in 32-expert steps
    auto go = [&](auto kern) {
        cudaError_t r = ensure_smem_attr(kern, ssm);
        if (r == cudaSuccess)
            kern<<<sgrid, kSelThreads, ssm, st>>>(p.rt_part, p.rt_xn2, p.rt_wn2, (int)p.T, (int)p.H, E, (int)p.k, ns,
                                                  cH, router_b, (const bf16*)x, (const bf16*)router_w, topk_idx,
                                                  topk_w, p.importance);
        return r;
    };
    const int nv = (E + 31) / 32;
    if (p.k > 8)
        e = go(router_select_kernel<kMaxTopK, 1>);
    else if (nv <= 1)
        e = go(router_select_kernel<8, 1>);
    else if (nv <= 2)
        e = go(router_select_kernel<8, 2>);
    else if (nv <= 4)
        e = go(router_select_kernel<8, 4>);
    else
        e = go(router_select_kernel<8, 8>);
    trace_after(st);
    if (e == cudaSuccess) e = cudaGetLastError();
    return e;
}

}  // namespace moe
