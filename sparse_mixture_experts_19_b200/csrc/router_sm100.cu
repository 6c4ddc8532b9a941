// Router scores, top-k and softmax over the selected scores on the tensor
// cores (tcgen05, sm_100a), for the bf16 layer.
//
// "MoE稀疏架构是什么？从原理到落地的系统解读", section 三.1 (a small linear
// router gives one score per expert) and section 四 (keep the k best scores,
// softmax over those k).  "模型的“分工的艺术”：MoE技术如何提升计算效率",
// section 1.1 (the gate is a linear layer, here with an optional bias).
//
// A tile is 128 tokens x all E experts of x W_r^T, accumulated in float32 in
// TMEM (E padded to a multiple of 16; the padding rows of the weight box
// read as zero).  Persistent CTAs loop over token tiles: warp 0 streams x and
// W_r through a TMA ring of up to 8 stages, warp 1 issues the MMAs into one
// of two TMEM accumulators, warps 2-5 (one token per thread) drain the other
// one: bias, the k best in registers ordered by (score desc, index asc), and
// the softmax of those k.  The epilogue of one tile overlaps the loads and
// MMAs of the next.
//
// Exactness of the decision and of the order.  Tensor-core float32 sums
// differ from the exact scores; the epilogue bounds that difference for each
// token by
//   delta_t = c_H * ||x_t|| * max_e ||w_e|| + 2^-23 * (||x_t|| max_e ||w_e|| + max_e |b_e|),
// where ||x_t|| * ||w_e|| >= sum_h |x_th w_eh| (Cauchy-Schwarz) and
// c_H = 17 * 2^-23 * (number of MMA steps + 1).  The constant rests on a
// model of the tensor core, assumed rather than documented: one kind::f16
// step adds its 16 exact bf16 products to the float32 accumulator D with an
// error of at most 17 * 2^-23 * (|D| + sum |products|), which is what 16
// float32 additions with round-toward-zero can lose in any order, and what
// a multi-term adder that aligns every term to the largest and truncates
// below 24 bits of it can lose.  Summed over the steps, the error of a score
// is at most c_H * sum_h |x_th w_eh|; the last term covers the rounding of
// the bias addition.  The norms come from the MMA warp's idle lanes, which
// read every x stage (and, on the CTA's first tile, every router-weight
// stage) from shared memory after issuing its MMAs; they are summed in
// float32 and inflated by 1 + H * 2^-22 to stay upper bounds.
//   Selection: an expert whose approximate score exceeds the (k+1)-th
// approximate score by more than 2 delta is certainly selected, one below the
// k-th by more than 2 delta certainly not; the experts in between (the band)
// are rescored exactly in fp64 (bf16 products are exact) by warp-cooperative
// dot products and the selection is completed from those exact scores,
// ties to the lower index.
//   Order: two selected experts whose approximate scores are more than
// 2 delta apart are in the right order; every selected expert with another
// one within 2 delta gets its exact score too, and the k are sorted with
// exact scores where both have one (ties to the lower index) and
// approximate ones otherwise.  The result is the exact order.
//
// Importance (optional).  Before the accumulator is handed back, each thread
// forms its token's softmax over all E float32 scores, each warp sums the 32
// tokens' probabilities per expert by a reduce-scatter over its lanes (lane l
// ends with expert c0 + l of a 32-column block) and adds the sums to the
// importance in global memory: one atomic add per expert, warp and tile.
#include "common.cuh"
#include "sm100.cuh"
#include "tma_host.cuh"

namespace moe {
namespace {

using namespace sm100;

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kMaxStages = 8;
constexpr int kThreads = 192;
constexpr int kABytes = kBM * kBK * 2;
constexpr int kQueue = 512;  // exact-rescoring queue entries per CTA and tile

constexpr int kBRowsMax = kMaxExperts;  // router rows per stage at most (E padded to 16)

// Sum of squares of the 64 bf16 values of one 128-byte row of a swizzled
// shared-memory tile at shared address `row`; lane l reads its 16-byte
// chunks starting at chunk l % 8, so 32 lanes reading 32 rows at once touch
// every bank equally.
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

// (a, ea) ranks before (b, eb): larger score, then lower expert index.
__device__ __forceinline__ bool ranks_before(float a, int ea, float b, int eb) {
    return a > b || (a == b && ea < eb);
}

// Exact score x[t] . W_r[e] in fp64 (products of bf16 values are exact),
// computed by one warp: lane l takes the 8-element chunks l, l+32, ...; four
// chunks per lane are loaded before any is used, into four accumulators.
__device__ __forceinline__ double exact_score(const bf16* x, const bf16* w, int t, int e, int H, int lane) {
    const uint4* xr = reinterpret_cast<const uint4*>(x + (int64_t)t * H);
    const uint4* wr = reinterpret_cast<const uint4*>(w + (int64_t)e * H);
    const int nch = H / 8;
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
    for (int c = lane; c < nch; c += 128) {
        uint4 a[4], b[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int cu = c + 32 * u;
            a[u] = cu < nch ? xr[cu] : make_uint4(0, 0, 0, 0);
            b[u] = cu < nch ? wr[cu] : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&a[u]);
            const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&b[u]);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float2 fa = __bfloat1622float2(pa[i]), fb = __bfloat1622float2(pb[i]);
                acc[u] = fma((double)fa.x, (double)fb.x, acc[u]);
                acc[u] = fma((double)fa.y, (double)fb.y, acc[u]);
            }
        }
    }
    double sum = (acc[0] + acc[1]) + (acc[2] + acc[3]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    return sum;
}

// Reduction barriers over the 128 epilogue threads (named barrier 1).
__device__ __forceinline__ bool epilogue_all(bool pred) {
    uint32_t out;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, 1, 128, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(out)
        : "r"((uint32_t)pred)
        : "memory");
    return out != 0;
}

__device__ __forceinline__ bool epilogue_any(bool pred) {
    uint32_t out;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, 1, 128, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(out)
        : "r"((uint32_t)pred)
        : "memory");
    return out != 0;
}

__device__ __forceinline__ void epilogue_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// Column sums of a warp's 32 x 32 values (v[i] of lane l is row l, column i):
// five exchange steps, each halving the columns a lane keeps; afterwards v[0]
// of lane l holds the sum of column l over all 32 lanes.
__device__ __forceinline__ float warp_column_sum32(float (&v)[32], int lane) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < o; ++i) {
            const float send = upper ? v[i] : v[i + o];
            const float keep = upper ? v[i + o] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
    return v[0];
}

// KMAX: capacity of the per-thread selection (k <= KMAX).  KMAX = kMaxTopK
// serves only k == E (every expert selected), where no decision is uncertain.
template <int KMAX>
__global__ void __launch_bounds__(kThreads, 1) router_sm100_kernel(
    const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW, int T, int H, int E,
    int Npad, int k, int stages, uint32_t acc_cols, const float* __restrict__ bias,
    const bf16* __restrict__ x_rows, const bf16* __restrict__ wr_rows, int32_t* __restrict__ topk_idx,
    float* __restrict__ topk_w, float* __restrict__ importance, int32_t* flags) {
    constexpr bool kDense = (KMAX == kMaxTopK);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int stage_bytes = kABytes + Npad * kBK * 2;  // a multiple of 1024
    uint8_t* tail = smem + stages * stage_bytes;
    int2* qp = reinterpret_cast<int2*>(tail);                   // [kQueue] (row, expert)
    double* qs = reinterpret_cast<double*>(qp + kQueue);       // [kQueue] exact scores
    float* qa = reinterpret_cast<float*>(qs + kQueue);         // [kQueue] approximate scores
    uint8_t* misc = reinterpret_cast<uint8_t*>(qa + kQueue);   // 1024-aligned, 256 bytes
    uint64_t* full = reinterpret_cast<uint64_t*>(misc);        // [stages]
    uint64_t* empty = full + kMaxStages;
    uint64_t* tfull = empty + kMaxStages;
    uint64_t* tempty = tfull + 2;
    uint64_t* nready = tempty + 2;  // squared x norms of an accumulator's tile written
    uint64_t* drain = nready + 2;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    int* qn = reinterpret_cast<int*>(tmem_holder + 2);
    float* wmax2 = reinterpret_cast<float*>(tmem_holder + 3);  // max_e ||w_e||^2 (after the first tile)
    float* xnorm2 = reinterpret_cast<float*>(misc + 256);      // [2][128] ||x_t||^2 per accumulator
    float* bs = xnorm2 + 2 * kBM;                              // [E rounded up to 64], 16-byte aligned

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const bool has_bias = bias != nullptr;
    const int E64 = (E + 63) / 64 * 64;
    for (int e = threadIdx.x; e < E64; e += kThreads) bs[e] = (bias && e < E) ? bias[e] : 0.f;
    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 2);  // the MMAs' commit and the norm pass of the MMA warp
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&tfull[i], 1);
            mbar_init(&tempty[i], 128);
            mbar_init(&nready[i], 1);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        *wmax2 = 0.f;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, 2 * acc_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    const int ntiles = (T + kBM - 1) / kBM;
    const int nkb = (H + kBK - 1) / kBK;
    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_map(&tmX);
            tma_prefetch_map(&tmW);
            uint32_t it = 0;
            for (int tile = blockIdx.x; tile < ntiles && !*abort_flag; tile += gridDim.x) {
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const int s = it % stages;
                    const uint32_t ph = (it / stages) & 1;
                    if (!wait_or_abort(&empty[s], ph ^ 1, abort_flag, flags, MOE_DEVFLAG_WAIT_TIMEOUT)) break;
                    uint8_t* sa = smem + s * stage_bytes;
                    mbar_arrive_expect_tx(&full[s], stage_bytes);
                    tma_load_3d(sa, &tmX, &full[s], kb * kBK, tile * kBM, 0);
                    tma_load_3d(sa + kABytes, &tmW, &full[s], kb * kBK, 0, 0);
                }
            }
            for (uint32_t j = (it > (uint32_t)stages ? it - stages : 0); j < it; ++j)
                drain_wait(&full[j % stages], (j / stages) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (lane 0) + norms (all lanes)
        const uint32_t idesc = idesc_bf16(kBM, Npad);
        uint32_t it = 0, tc = 0;
        float wsq[kBRowsMax / 32];  // ||w_e||^2 of router rows lane + 32 i (first tile)
#pragma unroll
        for (int i = 0; i < kBRowsMax / 32; ++i) wsq[i] = 0.f;
        bool ok = true;
        for (int tile = blockIdx.x; tile < ntiles && ok && !*abort_flag; tile += gridDim.x, ++tc) {
            const uint32_t acc = tc & 1, aph = (tc >> 1) & 1;
            if (!wait_or_abort(&tempty[acc], aph ^ 1, abort_flag, flags, MOE_DEVFLAG_WAIT_TIMEOUT)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t d = tmem_base + acc * acc_cols;
            float xsq[kBM / 32];  // ||x_t||^2 of tile rows lane + 32 q
#pragma unroll
            for (int q = 0; q < kBM / 32; ++q) xsq[q] = 0.f;
            for (int kb = 0; kb < nkb; ++kb, ++it) {
                const int s = it % stages;
                const uint32_t ph = (it / stages) & 1;
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
                        mma_bf16(d, desc_kmajor_sw128(a0 + kk * 32), desc_kmajor_sw128(b0 + kk * 32), idesc,
                                 (kb | kk) != 0);
                    mma_commit(&empty[s]);
                }
                // squared norms of the stage's rows (128-byte rows, 16-byte
                // chunks permuted inside a row by the swizzle, which a sum of
                // squares does not see); lane l reads chunk (i + l) % 8 in
                // step i, so a warp's 32 loads spread over all banks
#pragma unroll
                for (int q = 0; q < kBM / 32; ++q) xsq[q] += row_sumsq(a0 + (uint32_t)(lane + 32 * q) * 128u, lane);
                if (tc == 0) {
#pragma unroll
                    for (int i = 0; i < kBRowsMax / 32; ++i)
                        if (lane + 32 * i < Npad) wsq[i] += row_sumsq(b0 + (uint32_t)(lane + 32 * i) * 128u, lane);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);
            }
            if (!ok) break;
            if (lane == 0) mma_commit(&tfull[acc]);
#pragma unroll
            for (int q = 0; q < kBM / 32; ++q) xnorm2[acc * kBM + lane + 32 * q] = xsq[q];
            if (tc == 0) {
                float m = 0.f;
#pragma unroll
                for (int i = 0; i < kBRowsMax / 32; ++i) m = fmaxf(m, wsq[i]);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                if (lane == 0) *wmax2 = m;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&nready[acc]);  // release: the norms above are visible to its waiters
        }
        if (lane == 0) {
            mma_commit(drain);
            drain_wait(drain, 0);
        }
    } else {
        // ------------------------------------------------ epilogue warps 2..5
        const int q = warp & 3;
        const int r = q * 32 + lane;  // token row of this thread within the tile
        const int ew = warp - 2;      // epilogue warp 0..3
        // the bound on |approximate - exact score| (see the file comment)
        const float u23 = 1.1920929e-7f;  // 2^-23
        const float cH = 17.f * u23 * (float)(4 * nkb + 1) * 1.01f;
        const float slack = 1.f + (float)H * 2.3841858e-7f;  // 1 + H 2^-22: float32 sums of squares as upper bounds
        float bmax = 0.f;
        for (int e = 0; e < E; ++e) bmax = fmaxf(bmax, fabsf(bs[e]));
        uint32_t tc = 0;
        for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++tc) {
            const uint32_t acc = tc & 1, aph = (tc >> 1) & 1;
            bool ready = wait_or_abort(&tfull[acc], aph, abort_flag, flags, MOE_DEVFLAG_WAIT_TIMEOUT);
            ready = ready && wait_or_abort(&nready[acc], aph, abort_flag, flags, MOE_DEVFLAG_WAIT_TIMEOUT);
            // all 128 epilogue threads take the same branch, so every named
            // barrier below is reached by all of them
            if (!epilogue_all(ready)) break;
            tc_fence_after();
            const int t = tile * kBM + r;
            const uint32_t tq = tmem_base + acc * acc_cols + ((uint32_t)(q * 32) << 16);
            // twice the bound: the width of the uncertain band on each side
            const float anorm = sqrtf(xnorm2[acc * kBM + r] * slack) * sqrtf(*wmax2 * slack);
            const float del2 = 2.f * 1.001f * (cH * anorm + u23 * (anorm + bmax));

            // pass 1: the k (+1) best approximate scores, picked in k (+1)
            // rounds; round j takes the best score ranking after the pick of
            // round j-1 in the order (score desc, index asc).  Branch-free
            // scans of the TMEM row, all state in registers.
            float tv[KMAX + 1];
            int te[KMAX + 1];
            const int kk = k < E ? k + 1 : k;
            float pv = INFINITY;
            int pe = -1;
#pragma unroll
            for (int j = 0; j <= KMAX; ++j) {
                // four independent running maxima (elements i % 4), merged at
                // the end; each keeps the lower index on ties because it
                // visits its elements in ascending index order
                float bv[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
                int be[4] = {0x7fffffff, 0x7fffffff, 0x7fffffff, 0x7fffffff};
                if (j < kk) {
                    for (int c0 = 0; c0 < E; c0 += 64) {
                        float v[64];
                        tmem_ld64(tq + c0, v);  // columns past E (up to the allocation) are ignored
                        if (j == 0 && has_bias) {
                            // round 0: the bias is added once and the biased
                            // scores are written back to TMEM for the later
                            // rounds and the band pass
#pragma unroll
                            for (int i = 0; i < 64; i += 4) {
                                const float4 b4 = *reinterpret_cast<const float4*>(bs + c0 + i);
                                v[i] += b4.x;
                                v[i + 1] += b4.y;
                                v[i + 2] += b4.z;
                                v[i + 3] += b4.w;
                            }
                            tmem_st64(tq + c0, v);
                        }
#pragma unroll
                        for (int i = 0; i < 64; ++i) {
                            const int e = c0 + i;
                            const float cv = v[i];
                            const bool after = (cv < pv) || (cv == pv && e > pe);
                            if (e < E && after && cv > bv[i & 3]) {
                                bv[i & 3] = cv;
                                be[i & 3] = e;
                            }
                        }
                    }
#pragma unroll
                    for (int c = 1; c < 4; ++c)
                        if (ranks_before(bv[c], be[c], bv[0], be[0])) {
                            bv[0] = bv[c];
                            be[0] = be[c];
                        }
                    pv = bv[0];
                    pe = be[0];
                }
                tv[j] = bv[0];
                te[j] = be[0];
            }

            // certainty of the decision
            float band_lo = 0.f, band_hi = 0.f;
            bool uncertain = false;
            int n_in = k;
            if (!kDense && t < T && k < E) {
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

            // final selection state: certain prefix + the best `need` band
            // members by exact score (ties to the lower index), with their
            // approximate scores
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
            // pass 2, in rounds of at most kQueue band members per tile: queue
            // them (scores re-read from TMEM), rescore them exactly with whole
            // warps, let each token take its own.  One round in practice.
            int cursor = uncertain ? 0 : E;  // next expert this thread still has to scan
            while (epilogue_any(cursor < E)) {
                if (threadIdx.x == 64) *qn = 0;
                epilogue_sync();
                if (__any_sync(0xffffffffu, cursor < E)) {
                    bool stop = false;
                    for (int c0 = 0; c0 < E; c0 += 32) {
                        float v[32];
                        tmem_ld32(tq + c0, v);
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            const int e = c0 + i;
                            if (!stop && e >= cursor && e < E) {
                                const float sv = v[i];  // biased already (round 0)
                                if (sv >= band_lo && sv <= band_hi) {
                                    const int slot = atomicAdd(qn, 1);
                                    if (slot < kQueue) {
                                        qp[slot] = make_int2(r, e);
                                        qa[slot] = sv;
                                    } else {
                                        stop = true;  // queue full: resume here next round
                                        cursor = e;
                                    }
                                }
                            }
                        }
                    }
                    if (!stop) cursor = E;
                }
                epilogue_sync();
                const int nq = min(*qn, kQueue);
                for (int i = ew; i < nq; i += 4) {
                    const int2 pr = qp[i];
                    const double sd = exact_score(x_rows, wr_rows, tile * kBM + pr.x, pr.y, H, lane);
                    if (lane == 0) qs[i] = sd + (double)bs[pr.y];
                }
                epilogue_sync();
                if (uncertain)
                    for (int i = 0; i < nq; ++i) {
                        const int2 pr = qp[i];
                        if (pr.x != r) continue;
                        // insert (qs[i], pr.y) into the `need` best, ties to the lower index
                        double cv = qs[i];
                        int ce = pr.y;
                        float ca = qa[i];
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
            }
            if (importance) {
                // token's softmax over all E scores (TMEM holds them biased),
                // shifted by the largest (tv[0]); rows past T add nothing.
                // The fast exponential (relative error ~1e-6 for arguments
                // down to -20) keeps this cheap; the statistic needs ~1e-4.
                __syncwarp();
                const float m = tv[0];
                float z = 0.f;
                for (int c0 = 0; c0 < E; c0 += 32) {
                    float v[32];
                    tmem_ld32(tq + c0, v);
#pragma unroll
                    for (int i = 0; i < 32; ++i) z += (c0 + i < E) ? __expf(v[i] - m) : 0.f;
                }
                const float inv = 1.0f / z;
                for (int c0 = 0; c0 < E; c0 += 32) {
                    float v[32];
                    tmem_ld32(tq + c0, v);
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = (t < T && c0 + i < E) ? __expf(v[i] - m) * inv : 0.f;
                    const float colsum = warp_column_sum32(v, lane);
                    if (c0 + lane < E) atomicAdd(&importance[c0 + lane], colsum);
                }
            }
            // the accumulator is no longer needed: hand it back to the MMA warp
            tc_fence_before();
            mbar_arrive(&tempty[acc]);

            // the k selected: approximate score fa, expert fe, exact score fx
            // where known (bit j of has_x)
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
            if (!kDense && uncertain) {
                // move the band picks to slots n_in..k-1: n_in predicated
                // right-shifts keep every index static (registers, no stack)
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
            // order: every selected expert with another selected one within
            // 2 delta (approximate scores) needs its exact score
            uint32_t pending = 0;
            if (t < T) {
#pragma unroll
                for (int i = 0; i < KMAX; ++i)
#pragma unroll
                    for (int j = i + 1; j < KMAX; ++j)
                        if (j < k && fabsf(fa[i] - fa[j]) <= del2) pending |= (1u << i) | (1u << j);
                pending &= ~has_x;
            }
            while (epilogue_any(pending != 0)) {
                if (threadIdx.x == 64) *qn = 0;
                epilogue_sync();
#pragma unroll
                for (int j = 0; j < KMAX; ++j)
                    if ((pending >> j) & 1u) {
                        const int slot = atomicAdd(qn, 1);
                        if (slot < kQueue) {
                            qp[slot] = make_int2(r, fe[j]);
                            pending &= ~(1u << j);
                        }
                    }
                epilogue_sync();
                const int nq = min(*qn, kQueue);
                for (int i = ew; i < nq; i += 4) {
                    const int2 pr = qp[i];
                    const double sd = exact_score(x_rows, wr_rows, tile * kBM + pr.x, pr.y, H, lane);
                    if (lane == 0) qs[i] = sd + (double)bs[pr.y];
                }
                epilogue_sync();
                for (int i = 0; i < nq; ++i) {
                    const int2 pr = qp[i];
                    if (pr.x != r) continue;
#pragma unroll
                    for (int j = 0; j < KMAX; ++j)
                        if (j < k && fe[j] == pr.y) {
                            fx[j] = qs[i];
                            has_x |= 1u << j;
                        }
                }
            }
            // sort the k by (score desc, index asc): exact scores where both
            // have one, else approximate ones (more than 2 delta apart, so in
            // the right order); every comparison gives the exact order
#pragma unroll 1
            for (int pass = 0; pass + 1 < KMAX; ++pass) {
#pragma unroll
                for (int j = 0; j + 1 < KMAX; ++j) {
                    if (j + 1 < k) {
                        const bool both = ((has_x >> j) & (has_x >> (j + 1)) & 1u) != 0;
                        const bool swap = both ? (fx[j + 1] > fx[j] || (fx[j + 1] == fx[j] && fe[j + 1] < fe[j]))
                                               : ranks_before(fa[j + 1], fe[j + 1], fa[j], fe[j]);
                        if (swap) {
                            const float ta = fa[j];
                            fa[j] = fa[j + 1];
                            fa[j + 1] = ta;
                            const int tei = fe[j];
                            fe[j] = fe[j + 1];
                            fe[j + 1] = tei;
                            const double tx = fx[j];
                            fx[j] = fx[j + 1];
                            fx[j + 1] = tx;
                            const uint32_t bj = (has_x >> j) & 1u, bj1 = (has_x >> (j + 1)) & 1u;
                            has_x = (has_x & ~(3u << j)) | (bj << (j + 1)) | (bj1 << j);
                        }
                    }
                }
            }
            if (t < T) {
                // softmax over the k selected; score differences taken in fp64
                // where both scores are exact
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
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, 2 * acc_cols);
}

}  // namespace

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
    const int stage_bytes = kABytes + Npad * kBK * 2;
    // alignment slack + queue (pairs, exact and approximate scores) + barrier
    // block (204 B used of 256) + squared x norms [2][128] + bias
    const size_t fixed = 1024 + (size_t)kQueue * 20 + 256 + sizeof(float) * 2 * kBM +
                         sizeof(float) * ((E + 63) / 64 * 64);
    int stages = (int)((227 * 1024 - fixed) / stage_bytes);
    stages = stages > kMaxStages ? kMaxStages : stages;
    const size_t smem = (size_t)stages * stage_bytes + fixed;
    const int ntiles = (int)((p.T + kBM - 1) / kBM);
    const dim3 grid((unsigned)(ntiles < device_sm_count() ? ntiles : device_sm_count()));
    cudaError_t e;
    trace_before("router_sm100", st);
    if (p.k <= 8) {
        e = ensure_smem_attr(router_sm100_kernel<8>, smem);
        if (e == cudaSuccess)
            router_sm100_kernel<8><<<grid, kThreads, smem, st>>>(mx, mw, (int)p.T, (int)p.H, E, Npad, (int)p.k,
                                                               stages, cols, router_b, (const bf16*)x,
                                                               (const bf16*)router_w, topk_idx, topk_w,
                                                               p.importance, p.flags);
    } else {
        e = ensure_smem_attr(router_sm100_kernel<kMaxTopK>, smem);
        if (e == cudaSuccess)
            router_sm100_kernel<kMaxTopK><<<grid, kThreads, smem, st>>>(
                mx, mw, (int)p.T, (int)p.H, E, Npad, (int)p.k, stages, cols, router_b, (const bf16*)x,
                (const bf16*)router_w, topk_idx, topk_w, p.importance, p.flags);
    }
    trace_after(st);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace moe
