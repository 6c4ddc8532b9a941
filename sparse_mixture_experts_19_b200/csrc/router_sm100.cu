// Router scores, top-k and softmax over the selected scores on the tensor
// cores (tcgen05, sm_100a), for the bf16 layer.
//
// "MoE稀疏架构是什么？从原理到落地的系统解读", section 三.1 (a small linear
// router gives one score per expert) and section 四 (keep the k best scores,
// softmax over those k).  "模型的“分工的艺术”：MoE技术如何提升计算效率",
// section 1.1 (the gate is a linear layer, here with an optional bias).
//
// One CTA scores 128 tokens against all E experts: the scores are one
// 128 x E tile of x W_r^T, accumulated in float32 in TMEM (E padded to a
// multiple of 16; the padding rows of the weight box read as zero).  Warp 0
// streams x and W_r through a 4-stage TMA ring, warp 1 issues the MMAs,
// warps 2-5 each own 32 tokens: a thread reads its token's E scores from
// TMEM, adds the bias, keeps the k best in registers ordered by (score
// descending, expert index ascending), and writes the softmax of those k.
#include "common.cuh"
#include "sm100.cuh"
#include "tma_host.cuh"

namespace moe {
namespace {

using namespace sm100;

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kStages = 4;
constexpr int kThreads = 192;
constexpr int kABytes = kBM * kBK * 2;

// (a, ea) ranks before (b, eb): larger score, then lower expert index.
__device__ __forceinline__ bool ranks_before(float a, int ea, float b, int eb) {
    return a > b || (a == b && ea < eb);
}

constexpr int kQueue = 2048;  // exact-rescoring queue entries per CTA

// Exact score x[t] . W_r[e] in fp64 (products of bf16 values are exact),
// computed by one warp: lane l takes the 8-element chunks l, l+32, ...
__device__ __forceinline__ double exact_score(const bf16* x, const bf16* w, int t, int e, int H, int lane) {
    const uint4* xr = reinterpret_cast<const uint4*>(x + (int64_t)t * H);
    const uint4* wr = reinterpret_cast<const uint4*>(w + (int64_t)e * H);
    double acc = 0.0;
    for (int c = lane; c < H / 8; c += 32) {
        uint4 a = xr[c], b = wr[c];
        const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&a);
        const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float2 fa = __bfloat1622float2(pa[i]), fb = __bfloat1622float2(pb[i]);
            acc = fma((double)fa.x, (double)fb.x, acc);
            acc = fma((double)fa.y, (double)fb.y, acc);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    return acc;
}

// The same exact score computed by one thread (fallback when the queue is full).
__device__ __noinline__ double exact_score_serial(const bf16* x, const bf16* w, int t, int e, int H) {
    double acc = 0.0;
    for (int h = 0; h < H; ++h)
        acc = fma((double)__bfloat162float(x[(int64_t)t * H + h]), (double)__bfloat162float(w[(int64_t)e * H + h]),
                  acc);
    return acc;
}

// AND of `pred` over the 128 epilogue threads (named barrier 1).
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

// KMAX: capacity of the per-thread selection (k <= KMAX).  KMAX = kMaxTopK
// serves only k == E (every expert selected), where no decision is uncertain.
template <int KMAX>
__global__ void __launch_bounds__(kThreads, 1) router_sm100_kernel(
    const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW, int T, int H, int E,
    int Npad, int k, uint32_t tmem_cols, const float* __restrict__ bias, const bf16* __restrict__ x_rows,
    const bf16* __restrict__ wr_rows, int32_t* __restrict__ topk_idx, float* __restrict__ topk_w, int32_t* flags) {
    constexpr bool kDense = (KMAX == kMaxTopK);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int stage_bytes = kABytes + Npad * kBK * 2;  // a multiple of 1024
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * stage_bytes);
    uint64_t* empty = full + kStages;
    uint64_t* acc_ready = empty + kStages;
    uint64_t* drain = acc_ready + 1;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);  // [2]: abort, queue length
    float* bs = reinterpret_cast<float*>(smem + kStages * stage_bytes + 128);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    for (int e = threadIdx.x; e < E; e += kThreads) bs[e] = bias ? bias[e] : 0.f;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_ready, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    const int t0 = blockIdx.x * kBM;
    const int nkb = (H + kBK - 1) / kBK;
    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_map(&tmX);
            tma_prefetch_map(&tmW);
            int kb = 0;
            for (; kb < nkb; ++kb) {
                const int s = kb % kStages;
                const uint32_t ph = (kb / kStages) & 1;
                if (!wait_or_abort(&empty[s], ph ^ 1, abort_flag, flags, MOE_DEVFLAG_WAIT_TIMEOUT)) break;
                uint8_t* sa = smem + s * stage_bytes;
                mbar_arrive_expect_tx(&full[s], stage_bytes);
                tma_load_3d(sa, &tmX, &full[s], kb * kBK, t0, 0);
                tma_load_3d(sa + kABytes, &tmW, &full[s], kb * kBK, 0, 0);
            }
            for (int j = (kb > kStages ? kb - kStages : 0); j < kb; ++j)
                drain_wait(&full[j % kStages], (j / kStages) & 1);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(kBM, Npad);
            bool ok = true;
            for (int kb = 0; kb < nkb; ++kb) {
                const int s = kb % kStages;
                const uint32_t ph = (kb / kStages) & 1;
                if (!wait_or_abort(&full[s], ph, abort_flag, flags, MOE_DEVFLAG_WAIT_TIMEOUT)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t a0 = smem_u32(smem + s * stage_bytes);
                const uint32_t b0 = a0 + kABytes;
#pragma unroll
                for (int kk = 0; kk < kBK / 16; ++kk)
                    mma_bf16(tmem_base, desc_kmajor_sw128(a0 + kk * 32), desc_kmajor_sw128(b0 + kk * 32), idesc,
                             (kb | kk) != 0);
                mma_commit(&empty[s]);
            }
            if (ok) mma_commit(acc_ready);
            mma_commit(drain);
            drain_wait(drain, 0);
        }
    } else {
        // ------------------------------------------------ epilogue warps 2..5
        const int q = warp & 3;
        const int r = q * 32 + lane;  // token row of this thread within the tile
        const int t = t0 + r;
        const int ew = warp - 2;      // epilogue warp 0..3
        const bool ready = wait_or_abort(acc_ready, 0, abort_flag, flags, MOE_DEVFLAG_WAIT_TIMEOUT);
        // all four epilogue warps take the same branch, so the named barriers
        // below are always reached by all 128 threads
        if (epilogue_all(ready)) {
            tc_fence_after();
            // Every MMA has completed, so the stage buffers are free: they hold
            // the tile's scores and the exact-rescoring queue from here on.
            float* sc = reinterpret_cast<float*>(smem);                 // [128][E+1]
            int2* qp = reinterpret_cast<int2*>(sc + kBM * (E + 1));      // [kQueue] (row, expert)
            double* qs = reinterpret_cast<double*>(qp + kQueue);        // [kQueue] exact scores
            int* qn = const_cast<int*>(abort_flag) + 1;                 // queue length
            float* srow = sc + r * (E + 1);
            const uint32_t tq = tmem_base + ((uint32_t)(q * 32) << 16);

            // pass 1: approximate scores (float32 tensor-core sums + bias), the
            // k+1 best in registers ordered by (score desc, index asc), and the
            // magnitude of the raw dot products for the error bound
            float tv[KMAX + 1];
            int te[KMAX + 1];
#pragma unroll
            for (int j = 0; j <= KMAX; ++j) {
                tv[j] = -INFINITY;
                te[j] = 0x7fffffff;
            }
            const int kk = k < E ? k + 1 : k;  // also track the (k+1)-th when it exists
            float kth_v = -INFINITY, amax = 0.f;
            int kth_e = 0x7fffffff;
            for (int c0 = 0; c0 < E; c0 += 32) {
                float v[32];
                tmem_ld32(tq + c0, v);
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int e = c0 + i;
                    if (e < E) {
                        amax = fmaxf(amax, fabsf(v[i]));
                        float cv = v[i] + bs[e];
                        srow[e] = cv;
                        int ce = e;
                        if (ranks_before(cv, ce, kth_v, kth_e)) {
#pragma unroll
                            for (int j = 0; j <= KMAX; ++j) {
                                if (j < kk && ranks_before(cv, ce, tv[j], te[j])) {
                                    float fv = tv[j];
                                    int fe = te[j];
                                    tv[j] = cv;
                                    te[j] = ce;
                                    cv = fv;
                                    ce = fe;
                                }
                            }
#pragma unroll
                            for (int j = 0; j <= KMAX; ++j)
                                if (j == kk - 1) {
                                    kth_v = tv[j];
                                    kth_e = te[j];
                                }
                        }
                    }
                }
            }

            // Decision certainty.  The tensor-core sums differ from the exact
            // ones by at most about one float32 ulp of the running sum per
            // 16-wide step; delta is 32x that bound.  With the k-th and (k+1)-th
            // approximate scores more than delta apart the selection is exact.
            // Otherwise the experts whose approximate score lies in the band
            // [s_k - delta, s_{k+1} + delta] are rescored exactly (fp64) and the
            // selection is completed from those exact scores.
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
                const float delta = 2.0f * (float)H * 1.1920929e-7f * fmaxf(amax, 1.0f);
                if (kth - next <= delta) {
                    uncertain = true;
                    band_lo = kth - delta;
                    band_hi = next + delta;
                    n_in = 0;
#pragma unroll
                    for (int j = 0; j < KMAX; ++j)
                        if (j < k && tv[j] > band_hi) n_in = j + 1;
                }
            }

            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (threadIdx.x == 64) *qn = 0;
            asm volatile("bar.sync 1, 128;" ::: "memory");
            bool overflow = false;
            if (uncertain) {
                for (int e = 0; e < E; ++e) {
                    const float sv = srow[e];
                    if (sv >= band_lo && sv <= band_hi) {
                        const int slot = atomicAdd(qn, 1);
                        if (slot < kQueue)
                            qp[slot] = make_int2(r, e);
                        else
                            overflow = true;
                    }
                }
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");
            const int nq = min(*qn, kQueue);
            // warp-cooperative exact rescoring: lanes split H in 8-element chunks
            for (int i = ew; i < nq; i += 4) {
                const int2 pr = qp[i];
                const double sd = exact_score(x_rows, wr_rows, t0 + pr.x, pr.y, H, lane);
                if (lane == 0) qs[i] = sd + (double)bs[pr.y];
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");

            // final selection: certain prefix (approximate order) + the best
            // `need` band members by exact score (ties to the lower index)
            float fv[KMAX];
            int fe[KMAX];
#pragma unroll
            for (int j = 0; j < KMAX; ++j) {
                fv[j] = tv[j];
                fe[j] = te[j];
            }
            if (!kDense && uncertain) {
                const int need = k - n_in;
                double bv[KMAX];
                int be[KMAX];
#pragma unroll
                for (int j = 0; j < KMAX; ++j) {
                    bv[j] = -INFINITY;
                    be[j] = 0x7fffffff;
                }
                auto offer = [&](double cv, int ce) {
#pragma unroll
                    for (int j = 0; j < KMAX; ++j) {
                        if (j < need && (cv > bv[j] || (cv == bv[j] && ce < be[j]))) {
                            double ov = bv[j];
                            int oe = be[j];
                            bv[j] = cv;
                            be[j] = ce;
                            cv = ov;
                            ce = oe;
                        }
                    }
                };
                for (int i = 0; i < nq; ++i) {
                    const int2 pr = qp[i];
                    if (pr.x == r) offer(qs[i], pr.y);
                }
                if (overflow) {
                    // queue full (pathological near-ties): rescore the rest here
                    for (int e = 0; e < E; ++e) {
                        const float sv = srow[e];
                        if (sv >= band_lo && sv <= band_hi) {
                            bool queued = false;
                            for (int i = 0; i < nq && !queued; ++i) queued = (qp[i].x == r && qp[i].y == e);
                            if (!queued) offer(exact_score_serial(x_rows, wr_rows, t, e, H) + (double)bs[e], e);
                        }
                    }
                }
#pragma unroll
                for (int j = 0; j < KMAX; ++j)
                    if (j >= n_in && j < k) {
#pragma unroll
                        for (int i = 0; i < KMAX; ++i)
                            if (i == j - n_in) {
                                fv[j] = (float)bv[i];
                                fe[j] = be[i];
                            }
                    }
            }
            if (t < T) {
                float m = -INFINITY;
#pragma unroll
                for (int j = 0; j < KMAX; ++j)
                    if (j < k) m = fmaxf(m, fv[j]);
                float z = 0.f;
#pragma unroll
                for (int j = 0; j < KMAX; ++j)
                    if (j < k) z += expf(fv[j] - m);
                const float inv = 1.0f / z;
#pragma unroll
                for (int j = 0; j < KMAX; ++j)
                    if (j < k) {
                        topk_idx[(int64_t)t * k + j] = fe[j] < E ? fe[j] : -1;
                        topk_w[(int64_t)t * k + j] = expf(fv[j] - m) * inv;
                    }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, tmem_cols);
}

}  // namespace

cudaError_t launch_router_sm100(const Plan& p, const void* x, const void* router_w, const float* router_b,
                                int32_t* topk_idx, float* topk_w, cudaStream_t st) {
    if (p.T == 0) return cudaSuccess;
    const int E = (int)p.E;
    const int Npad = E <= 16 ? 16 : (E + 15) / 16 * 16;
    uint32_t cols = 32;
    while ((int)cols < Npad) cols <<= 1;
    CUtensorMap mx, mw;
    if (!make_map_bf16(&mx, x, p.H, p.T, 1, kBK, kBM) || !make_map_bf16(&mw, router_w, p.H, E, 1, kBK, Npad))
        return cudaErrorInvalidValue;
    const size_t smem = kStages * (size_t)(kABytes + Npad * kBK * 2) + 1024 + 128 + sizeof(float) * E;
    const dim3 grid((unsigned)((p.T + kBM - 1) / kBM));
    cudaError_t e;
    trace_before("router_sm100", st);
    if (p.k <= 8) {
        e = cudaFuncSetAttribute(router_sm100_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e == cudaSuccess)
            router_sm100_kernel<8><<<grid, kThreads, smem, st>>>(mx, mw, (int)p.T, (int)p.H, E, Npad, (int)p.k, cols,
                                                               router_b, (const bf16*)x, (const bf16*)router_w,
                                                               topk_idx, topk_w, p.flags);
    } else {
        e = cudaFuncSetAttribute(router_sm100_kernel<kMaxTopK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
        if (e == cudaSuccess)
            router_sm100_kernel<kMaxTopK><<<grid, kThreads, smem, st>>>(mx, mw, (int)p.T, (int)p.H, E, Npad,
                                                                      (int)p.k, cols, router_b, (const bf16*)x,
                                                                      (const bf16*)router_w, topk_idx, topk_w,
                                                                      p.flags);
    }
    trace_after(st);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace moe
