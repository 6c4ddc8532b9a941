// Decode layer: the whole MoE layer for a handful of routed slots (T*k <= 8)
// in one cooperative persistent kernel.
//
// "MoE稀疏架构是什么？从原理到落地的系统解读", section 四: score every expert,
// keep the k best, softmax over those k, y = sum of w * FFN_e(x).  "Mixture of
// Experts (MoEs) in Transformers": with few tokens the layer's time is the
// bytes of the selected experts' weights (the gpt-oss-20b bandwidth estimate
// of section From Dense to Sparse).
//
// With one or two rows per expert a 128-row tensor-core tile would be almost
// all padding, so the layer is written as one read of the selected experts'
// weight rows, spread evenly over every SM.  One CTA per SM (512 threads),
// launched cooperatively so that all CTAs are resident and may wait for one
// another; each wait is bounded (about 2 s, then MOE_DEVFLAG_WAIT_TIMEOUT is
// set and the CTA skips the rest).
//
//   0. scores (when the routing is not given): the T*E router scores are
//      split over the CTAs (a CTA with few pairs splits each pair's H over
//      its warps), exact up to fp64 rounding (a product of two bf16 values
//      is exact in float32, and the products are summed in fp64); grid
//      barrier.
//   1. selection: every CTA reads the T*E scores and picks each token's k
//      best (score descending, ties to the lower index) with warp arg-max
//      rounds, then the softmax of those k; the same arithmetic in every
//      CTA gives every CTA the same plan: the slots grouped by expert, the
//      capacity cut in token order, the shared expert as one more group.
//   2. gate/up and down, overlapped.  Ten warps stream gate/up rows:
//      CTA c owns the intermediate rows i in [R c / G, R (c+1) / G) of
//      every group (R = I, or I_s for the shared expert), group by group,
//      each row's gate and up rows read with 16-byte loads (L2
//      evict-first) and dotted with the group's token vectors from shared
//      memory: h[slot][i] = bf16(silu(x.g) * (x.u)).  When the CTA's rows
//      of a group are written, the CTA publishes the group (a per-group
//      counter in global memory).  The other six warps take the down rows
//      group by group: once every CTA has published group g, they copy its
//      h rows into shared memory and dot them with the down rows of this
//      CTA's output columns j in [H c / G, H (c+1) / G), while the gate/up
//      warps stream the next groups.  So the down rows are read during the
//      gate/up stream instead of after it, and no grid barrier separates
//      the two.  The gate/up warps, done with their rows, prefetch the last
//      group's down rows of their CTA into L2 and then share that group's
//      columns with the down warps.
//   3. y[t][j] = bf16(sum over the token's slots in order of w * d, + the
//      shared expert's d): y is bit-reproducible without atomics.
#include <algorithm>

#include "common.cuh"
#include "mxfp4.cuh"
#include "sm100.cuh"
#include "tma_host.cuh"

namespace moe {
namespace {

using namespace sm100;

constexpr int kDlThreads = 512;
constexpr int kDlWarps = kDlThreads / 32;
constexpr int kDlMaxSlots = kDecodeMaxSlotsMx;     // slots of either variant
constexpr int kDlMaxGroups = kDlMaxSlots + 1;      // distinct routed experts + the shared one
constexpr int kDlBatch = 4;                        // token vectors per pass over a weight row
constexpr int kDlUnroll = 6;                       // 16-byte chunks per lane in flight, per row
constexpr int kDlMaxCols = 64;                     // output columns per CTA in phase 3 (H <= 64 * grid)
constexpr int kDlSmemMax = 200 * 1024;
constexpr int kDlDownWarps = 6;                      // warps on the down rows (a third of the bytes, and the waits)
constexpr int kDlUpWarps = kDlWarps - kDlDownWarps;  // warps on the gate/up rows

// Bytes of one group's h vectors in shared memory: a routed expert meets a
// token at most once, so a group has at most T vectors (the shared expert
// exactly T).
__host__ __device__ __forceinline__ int dl_hbytes(int T, int I, int Is) {
    const int r = I > Is ? I : Is;
    return (T * r * 2 + 15) / 16 * 16;
}

struct DlArgs {
    const bf16* x;
    const bf16* router_w;
    const float* router_b;
    const int32_t* idx_in;  // given routing (token shards), or null: routed here
    const float* w_in;
    int32_t* idx_out;       // optional [T, k]
    const bf16 *wg, *wu, *wd, *wsg, *wsu, *wsd;
    // MXFP4 experts: blocks [E, rows, K/32, 16] (two E2M1 codes per byte, the
    // lower element in the low nibble) and scales [E, rows, K/32] (E8M0)
    const uint8_t *mgb, *mgs, *mub, *mus, *mdb, *mds;
    bf16* h;   // [S, I] routed activations, slot order
    bf16* hs;  // [T, Is] shared-expert activations
    void* y;               // [T, H] bf16, or float32 partial sums (y_f32)
    bool y_f32;
    bool drop_negative;    // expert -1 = another shard's: dropped, not counted
    double* scores;        // [T, E] router scores
    unsigned int* bar;     // [1 + groups]: the grid barrier, then each group's publishing CTAs; zero at launch
    int32_t* counts;
    int32_t* dropped;
    int32_t* flags;
    int T, H, I, Is, E, k, S;
    int64_t cap;
    const int32_t* cap_left_arr;
};

struct DlPlan {
    int ng;
    int gexp[kDlMaxGroups];                  // expert id; E marks the shared expert
    int gcnt[kDlMaxGroups];                  // vectors of the group
    int gvec[kDlMaxGroups][kDlMaxSlots];     // routed: slot s; shared: token t
    int e_of[kDlMaxSlots];
    int kept[kDlMaxSlots];
    float wslot[kDlMaxSlots];
};

__device__ __forceinline__ unsigned int ld_acquire_u32(const unsigned int* p) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// All CTAs of the (cooperatively launched) grid meet here.  Bounded: after
// about 2 s the device flag MOE_DEVFLAG_WAIT_TIMEOUT is set and false returned.
__device__ bool grid_barrier(unsigned int* ctr, int32_t* flags, int* ok_s) {
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();  // this CTA's writes, before its arrival
        atomicAdd(ctr, 1u);
        const uint64_t t0 = global_ns();
        int ok = 1;
        while (ld_acquire_u32(ctr) < gridDim.x) {
            if (global_ns() - t0 > 2000000000ull) {
                atomicOr(flags, MOE_DEVFLAG_WAIT_TIMEOUT);
                ok = 0;
                break;
            }
            __nanosleep(100);
        }
        __threadfence();
        *ok_s = ok;
    }
    __syncthreads();
    return *ok_s != 0;
}

__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// 16-byte load of data read once: no L1 allocation, L2 policy `pol`.
__device__ __forceinline__ uint4 ld_stream(const void* ptr, uint64_t pol) {
    uint4 v;
    asm("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
        : "l"(ptr), "l"(pol));
    return v;
}

// Bytes [ptr, ptr + bytes) into L2 (16-byte aligned, a multiple of 16).
__device__ __forceinline__ void prefetch_l2(const void* ptr, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(ptr), "r"(bytes) : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

// acc += w . v over 8 bf16 pairs, as four packed float32x2 FMAs (even and
// odd elements in the two halves).
__device__ __forceinline__ void dot8(const uint4& w, const uint4& v, float2& acc) {
    const __nv_bfloat162* pw = reinterpret_cast<const __nv_bfloat162*>(&w);
    const __nv_bfloat162* pv = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) acc = __ffma2_rn(__bfloat1622float2(pw[i]), __bfloat1622float2(pv[i]), acc);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// d[r][n] = row_r . vec_n for NR weight rows of K8 16-byte chunks in global
// memory (streamed with policy pol) and NV vectors in shared memory; every
// lane ends with the warp's totals.
template <int NR, int NV>
__device__ __forceinline__ void row_dots(const uint4* const (&rows)[NR], int K8, const uint32_t (&vec)[kDlBatch],
                                         uint64_t pol, float (&d)[NR][kDlBatch]) {
    const int lane = threadIdx.x & 31;
    float2 acc[NR][NV];
#pragma unroll
    for (int r = 0; r < NR; ++r)
#pragma unroll
        for (int n = 0; n < NV; ++n) acc[r][n] = make_float2(0.f, 0.f);
    for (int c0 = lane; c0 < K8; c0 += 32 * kDlUnroll) {
        uint4 w[NR][kDlUnroll];
#pragma unroll
        for (int u = 0; u < kDlUnroll; ++u)
#pragma unroll
            for (int r = 0; r < NR; ++r)
                w[r][u] = (c0 + 32 * u < K8) ? ld_stream(rows[r] + c0 + 32 * u, pol) : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int u = 0; u < kDlUnroll; ++u) {
            const int c = c0 + 32 * u;
            if (c < K8) {
#pragma unroll
                for (int n = 0; n < NV; ++n) {
                    const uint4 v = lds128(vec[n] + (uint32_t)c * 16u);
#pragma unroll
                    for (int r = 0; r < NR; ++r) dot8(w[r][u], v, acc[r][n]);
                }
            }
        }
    }
#pragma unroll
    for (int r = 0; r < NR; ++r)
#pragma unroll
        for (int n = 0; n < NV; ++n) d[r][n] = warp_sum(acc[r][n].x + acc[r][n].y);
}

// d[r] = row_r . v for NR weight rows (streamed with policy pol) and one
// vector v read from L2 alongside them (a group with one vector: the loads
// of both are in flight together, and nothing is staged).
template <int NR>
__device__ __forceinline__ void row_dots_l2(const uint4* const (&rows)[NR], int K8, const uint4* v, uint64_t pol,
                                            float (&d)[NR][kDlBatch]) {
    const int lane = threadIdx.x & 31;
    float2 acc[NR];
#pragma unroll
    for (int r = 0; r < NR; ++r) acc[r] = make_float2(0.f, 0.f);
    for (int c0 = lane; c0 < K8; c0 += 32 * kDlUnroll) {
        uint4 w[NR][kDlUnroll], x[kDlUnroll];
#pragma unroll
        for (int u = 0; u < kDlUnroll; ++u) {
            const bool in = c0 + 32 * u < K8;
            x[u] = in ? __ldcg(v + c0 + 32 * u) : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int r = 0; r < NR; ++r) w[r][u] = in ? ld_stream(rows[r] + c0 + 32 * u, pol) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < kDlUnroll; ++u)
#pragma unroll
            for (int r = 0; r < NR; ++r) dot8(w[r][u], x[u], acc[r]);
    }
#pragma unroll
    for (int r = 0; r < NR; ++r) d[r][0] = warp_sum(acc[r].x + acc[r].y);
}

template <int NR>
__device__ __forceinline__ void row_dots_n(const uint4* const (&rows)[NR], int K8, const uint32_t (&vec)[kDlBatch],
                                           int nv, uint64_t pol, float (&d)[NR][kDlBatch]) {
    switch (nv) {
        case 1: row_dots<NR, 1>(rows, K8, vec, pol, d); break;
        case 2: row_dots<NR, 2>(rows, K8, vec, pol, d); break;
        case 3: row_dots<NR, 3>(rows, K8, vec, pol, d); break;
        default: row_dots<NR, 4>(rows, K8, vec, pol, d); break;
    }
}

// ------------------------------------------------------------- MXFP4 rows
// The OCP Microscaling v1.0 MXFP4 format: 32 elements share one E8M0 scale
// 2^(s - 127) (s = 255: NaN); each element is FP4 E2M1.  A 16-byte chunk of a
// row's codes is one block.  The block's dot product with a token vector is
// formed in f16 (the E2M1 values are exact in f16, the vector is staged as f16
// scaled by a power of two so that every product and the 32-term partial
// stays in range), then widened to float32, scaled by the block's 2^(s-127)
// and accumulated in float32.
constexpr int kMxUnroll = 4;  // blocks per lane in flight, per row

__device__ __forceinline__ uint32_t hfma2_u32(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// d[r][n] = row_r . vec_n for NR MXFP4 rows of nblk blocks (codes streamed
// with policy pol, scale bytes read alongside) and NV f16 vectors in shared
// memory (64 bytes per block); every lane ends with the warp's totals.
template <int NR, int NV>
__device__ __forceinline__ void row_dots_mx(const uint4* const (&codes)[NR], const uint8_t* const (&scl)[NR], int nblk,
                                            const uint32_t (&vec)[kDlBatch], uint64_t pol, float (&d)[NR][kDlBatch]) {
    const int lane = threadIdx.x & 31;
    float acc[NR][NV];
#pragma unroll
    for (int r = 0; r < NR; ++r)
#pragma unroll
        for (int n = 0; n < NV; ++n) acc[r][n] = 0.f;
    for (int b0 = lane; b0 < nblk; b0 += 32 * kMxUnroll) {
        uint4 w[NR][kMxUnroll];
        uint32_t sb[NR][kMxUnroll];
#pragma unroll
        for (int u = 0; u < kMxUnroll; ++u)
#pragma unroll
            for (int r = 0; r < NR; ++r) {
                const int b = b0 + 32 * u;
                w[r][u] = b < nblk ? ld_stream(codes[r] + b, pol) : make_uint4(0, 0, 0, 0);
                sb[r][u] = b < nblk ? (uint32_t)__ldg(scl[r] + b) : 127u;
            }
#pragma unroll
        for (int u = 0; u < kMxUnroll; ++u) {
            const int b = b0 + 32 * u;
            if (b < nblk) {
                // the block's 32 codes of each row as f16x2 pairs, once for
                // all token vectors
                uint32_t hw[NR][16];
#pragma unroll
                for (int r = 0; r < NR; ++r) {
                    const uint32_t cw[4] = {w[r][u].x, w[r][u].y, w[r][u].z, w[r][u].w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint32_t h4[4];
                        e2m1x8_to_f16x2(cw[q], h4);
#pragma unroll
                        for (int j = 0; j < 4; ++j) hw[r][4 * q + j] = h4[j];
                    }
                }
#pragma unroll
                for (int n = 0; n < NV; ++n) {
                    uint32_t xv[16];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint4 v = lds128(vec[n] + (uint32_t)b * 64u + (uint32_t)q * 16u);
                        xv[4 * q] = v.x;
                        xv[4 * q + 1] = v.y;
                        xv[4 * q + 2] = v.z;
                        xv[4 * q + 3] = v.w;
                    }
#pragma unroll
                    for (int r = 0; r < NR; ++r) {
                        // four independent f16x2 chains of four FMAs each
                        uint32_t p[4] = {0u, 0u, 0u, 0u};  // f16x2 zeros
#pragma unroll
                        for (int q = 0; q < 4; ++q)
#pragma unroll
                            for (int j = 0; j < 4; ++j) p[j] = hfma2_u32(hw[r][4 * q + j], xv[4 * q + j], p[j]);
                        const __half2 ph = __hadd2(__hadd2(*reinterpret_cast<const __half2*>(&p[0]),
                                                           *reinterpret_cast<const __half2*>(&p[1])),
                                                   __hadd2(*reinterpret_cast<const __half2*>(&p[2]),
                                                           *reinterpret_cast<const __half2*>(&p[3])));
                        const float part = __low2float(ph) + __high2float(ph);
                        acc[r][n] = fmaf(part, e8m0_value(sb[r][u]), acc[r][n]);
                    }
                }
            }
        }
    }
#pragma unroll
    for (int r = 0; r < NR; ++r)
#pragma unroll
        for (int n = 0; n < NV; ++n) d[r][n] = warp_sum(acc[r][n]);
}

template <int NR>
__device__ __forceinline__ void row_dots_mx_n(const uint4* const (&codes)[NR], const uint8_t* const (&scl)[NR],
                                              int nblk, const uint32_t (&vec)[kDlBatch], int nv, uint64_t pol,
                                              float (&d)[NR][kDlBatch]) {
    switch (nv) {
        case 1: row_dots_mx<NR, 1>(codes, scl, nblk, vec, pol, d); break;
        case 2: row_dots_mx<NR, 2>(codes, scl, nblk, vec, pol, d); break;
        case 3: row_dots_mx<NR, 3>(codes, scl, nblk, vec, pol, d); break;
        default: row_dots_mx<NR, 4>(codes, scl, nblk, vec, pol, d); break;
    }
}

// Power of two that brings a vector whose largest magnitude is m below 2^8
// (so that 32 products with E2M1 values, at most 6, stay inside f16).
__device__ __forceinline__ float f16_stage_scale(float m) {
    if (!(m > 0.f) || isinf(m)) return 1.f;
    int ex;
    frexpf(m, &ex);  // m in [2^(ex-1), 2^ex)
    return ldexpf(1.f, 8 - ex);
}

// Barrier of `n` threads of the CTA (named barrier `id`; id 0 = all threads).
__device__ __forceinline__ void named_sync(int id, int n) {
    if (id == 0)
        __syncthreads();
    else
        asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// n bf16 values at src -> f16 values * sc at dst (shared memory), by the
// nthr threads numbered tid = 0 .. nthr-1.
__device__ __forceinline__ void stage_f16(uint8_t* dst, const bf16* src, int n, float sc, bool l2_only, int tid,
                                          int nthr) {
    const uint4* s4 = reinterpret_cast<const uint4*>(src);
    uint4* d4 = reinterpret_cast<uint4*>(dst);
    for (int i = tid; i < n / 8; i += nthr) {
        const uint4 v = l2_only ? __ldcg(s4 + i) : __ldg(s4 + i);
        const uint32_t in[4] = {v.x, v.y, v.z, v.w};
        uint32_t out[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&in[j]));
            const __half2 hv = __floats2half2_rn(f.x * sc, f.y * sc);
            out[j] = *reinterpret_cast<const uint32_t*>(&hv);
        }
        d4[i] = make_uint4(out[0], out[1], out[2], out[3]);
    }
}

// Largest magnitude of n bf16 values, by the nthr threads (whole warps)
// numbered tid = 0 .. nthr-1 that meet at named barrier `bar`; every one of
// them gets it.
__device__ float group_absmax(const bf16* src, int n, bool l2_only, float* red, int tid, int nthr, int bar) {
    float m = 0.f;
    const uint4* s4 = reinterpret_cast<const uint4*>(src);
    for (int i = tid; i < n / 8; i += nthr) {
        const uint4 v = l2_only ? __ldcg(s4 + i) : __ldg(s4 + i);
        const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 f = __bfloat1622float2(p[j]);
            m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    named_sync(bar, nthr);
    if ((tid & 31) == 0) red[tid / 32] = m;
    named_sync(bar, nthr);
    float r = 0.f;
    for (int w = 0; w < nthr / 32; ++w) r = fmaxf(r, red[w]);
    return r;
}

// double -> unsigned 64-bit with the same order (-0 taken as +0, so that
// equal doubles get equal keys), and back.
__device__ __forceinline__ unsigned long long ordered_key64(double v) {
    const unsigned long long u = (unsigned long long)__double_as_longlong(v == 0.0 ? 0.0 : v);
    return (u >> 63) ? ~u : (u | (1ull << 63));
}
__device__ __forceinline__ double from_ordered_key64(unsigned long long k) {
    return __longlong_as_double((long long)((k >> 63) ? (k & ~(1ull << 63)) : ~k));
}

// Part of an exact score x[t] . W_r[e] in fp64: the 16-byte chunks
// [cb, ce) of the two rows, summed by one warp (every lane gets the sum).
__device__ __forceinline__ double exact_dot_part(const bf16* x, const bf16* w, int cb, int ce) {
    const int lane = threadIdx.x & 31;
    const uint4* xr = reinterpret_cast<const uint4*>(x);
    const uint4* wr = reinterpret_cast<const uint4*>(w);
    double acc[2] = {0.0, 0.0};
    for (int c0 = cb + lane; c0 < ce; c0 += 32 * kDlUnroll) {
        uint4 a[kDlUnroll], b[kDlUnroll];
#pragma unroll
        for (int u = 0; u < kDlUnroll; ++u) {
            const int c = c0 + 32 * u;
            a[u] = c < ce ? __ldg(xr + c) : make_uint4(0, 0, 0, 0);
            b[u] = c < ce ? __ldg(wr + c) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < kDlUnroll; ++u) {
            const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&a[u]);
            const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&b[u]);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 fa = __bfloat1622float2(pa[i]), fb = __bfloat1622float2(pb[i]);
                // products of bf16 values are exact in float32
                acc[u & 1] += (double)__fmul_rn(fa.x, fb.x);
                acc[u & 1] += (double)__fmul_rn(fa.y, fb.y);
            }
        }
    }
    double s = acc[0] + acc[1];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    return s;
}

// Phase 1 (thread 0 after the selection): kept slots grouped by expert with
// the capacity cut in token order (a token meets an expert at most once, so
// slot order is token order), then the shared expert as one more group.  An
// expert gets a group only when one of its slots is kept: an expert whose
// capacity is 0 (all of its slots dropped) streams no weights.
__device__ void build_groups(const DlArgs& a, DlPlan& pl) {
    int ng = 0;
    bool bad = false;
    for (int s = 0; s < a.S; ++s) {
        const int e = pl.e_of[s];
        pl.kept[s] = 0;
        if (e < 0 || e >= a.E) {
            if (!(a.drop_negative && e == -1)) bad = true;  // -1: another shard's expert
            continue;
        }
        int g = 0;
        while (g < ng && pl.gexp[g] != e) ++g;
        const int kept_so_far = g < ng ? pl.gcnt[g] : 0;
        if (a.cap > 0 && kept_so_far >= cap_left(a.cap, a.cap_left_arr, e)) continue;
        if (g == ng) {
            pl.gexp[ng] = e;
            pl.gcnt[ng] = 0;
            ++ng;
        }
        pl.gvec[g][pl.gcnt[g]++] = s;
        pl.kept[s] = 1;
    }
    if (a.Is > 0) {
        pl.gexp[ng] = a.E;
        pl.gcnt[ng] = a.T;
        for (int t = 0; t < a.T; ++t) pl.gvec[ng][t] = t;
        ++ng;
    }
    pl.ng = ng;
    if (bad && blockIdx.x == 0) set_flag(a.flags, MOE_DEVFLAG_BAD_EXPERT_INDEX);
}

template <bool kMx>
__global__ void __launch_bounds__(kDlThreads, 1) decode_layer_kernel(const DlArgs a) {
    extern __shared__ __align__(128) uint8_t dsm[];
    __shared__ DlPlan pl;
    __shared__ int ok_s;
    __shared__ float red[2 * kDlWarps];        // block reductions (the down warps use the second half)
    __shared__ float inv_sx[kDlMaxSlots];      // MXFP4: 1 / staging scale of each token vector
    __shared__ float inv_sh[kDlMaxSlots];      // MXFP4: 1 / staging scale of each h vector
    __shared__ double dpart[kDlWarps];         // parts of the router scores
    __shared__ int up_done[kDlMaxGroups];      // gate/up warps done with each group
    __shared__ int down_ok;
    __shared__ int last_state;  // the last group's h rows: 0 not yet staged, 1 staged, 2 abandoned
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int G = gridDim.x, c = blockIdx.x;
    const uint64_t pol_first = policy_evict_first();

    // ---------------------------------------------------------- routing
    if (!a.idx_in) {
        const int P = a.T * a.E, nch = a.H / 8;
        // CTA c scores the pairs p0 .. p1-1 (p = t E + e).  With at most one
        // pair per warp, each pair's H is split over kDlWarps / n warps and
        // their parts are added in slice order, so a score costs one pass
        // of its rows' loads instead of H / (32 * unroll) passes.
        const int p0 = (int)((int64_t)P * c / G), p1 = (int)((int64_t)P * (c + 1) / G);
        const int nd = p1 - p0;
        if (nd > 0 && nd <= kDlWarps) {
            const int spd = kDlWarps / nd;  // warps (slices) per pair
            const int di = warp / spd, si = warp % spd;
            if (di < nd) {
                const int p = p0 + di, t = p / a.E, e = p % a.E;
                const double s = exact_dot_part(a.x + (int64_t)t * a.H, a.router_w + (int64_t)e * a.H,
                                                (int)((int64_t)nch * si / spd), (int)((int64_t)nch * (si + 1) / spd));
                if (lane == 0) dpart[di * spd + si] = s;
            }
            __syncthreads();
            if (threadIdx.x < nd) {
                const int p = p0 + threadIdx.x;
                double s = 0.0;
                for (int q = 0; q < spd; ++q) s += dpart[threadIdx.x * spd + q];
                a.scores[p] = s + (a.router_b ? (double)a.router_b[p % a.E] : 0.0);
            }
        } else {
            for (int p = p0 + warp; p < p1; p += kDlWarps) {
                const int t = p / a.E, e = p % a.E;
                const double s = exact_dot_part(a.x + (int64_t)t * a.H, a.router_w + (int64_t)e * a.H, 0, nch);
                if (lane == 0) a.scores[p] = s + (a.router_b ? (double)a.router_b[e] : 0.0);
            }
        }
        if (!grid_barrier(&a.bar[0], a.flags, &ok_s)) return;
        // warp t selects token t: its E scores read once (lane l holds
        // experts l, l + 32, ...), then k rounds of warp arg-max, ties to the
        // lower index
        for (int t = warp; t < a.T; t += kDlWarps) {
            const double* sc = a.scores + (int64_t)t * a.E;
            double sv[kMaxExperts / 32];
#pragma unroll
            for (int i = 0; i < kMaxExperts / 32; ++i) {
                const int e = lane + 32 * i;
                sv[i] = e < a.E ? __ldcg(sc + e) : 0.0;
            }
            double pv = INFINITY;
            int pe = -1;
            double v0 = 0.0;
            float z = 0.f;
            for (int j = 0; j < a.k; ++j) {
                double bv = -INFINITY;
                int be = 0x7fffffff;
#pragma unroll
                for (int i = 0; i < kMaxExperts / 32; ++i) {
                    const int e = lane + 32 * i;
                    const double v = sv[i];
                    const bool after = (v < pv) || (v == pv && e > pe);
                    if (e < a.E && after && (v > bv || (v == bv && e < be))) {
                        bv = v;
                        be = e;
                    }
                }
                {
                    // warp arg-max over order-preserving 64-bit keys: the
                    // largest high word, then the largest low word among the
                    // lanes holding it, then the lowest expert index among
                    // the lanes holding both (single-instruction reductions)
                    const unsigned long long key = ordered_key64(bv);
                    const unsigned hi = (unsigned)(key >> 32), lo = (unsigned)key;
                    const unsigned mhi = __reduce_max_sync(0xffffffffu, hi);
                    const unsigned mlo = __reduce_max_sync(0xffffffffu, hi == mhi ? lo : 0u);
                    const bool top = hi == mhi && lo == mlo;
                    be = (int)__reduce_min_sync(0xffffffffu, top ? (unsigned)be : 0xffffffffu);
                    bv = from_ordered_key64(((unsigned long long)mhi << 32) | mlo);
                }
                if (j == 0) v0 = bv;
                pv = bv;
                pe = be;
                if (lane == 0) {
                    pl.e_of[t * a.k + j] = be;
                    pl.wslot[t * a.k + j] = expf((float)(bv - v0));  // normalised below
                }
                z += expf((float)(bv - v0));
            }
            if (lane == 0) {
                const float inv = 1.0f / z;
                for (int j = 0; j < a.k; ++j) {
                    pl.wslot[t * a.k + j] *= inv;
                    if (c == 0 && a.idx_out) a.idx_out[t * a.k + j] = pl.e_of[t * a.k + j];
                }
            }
        }
    } else if (threadIdx.x < a.S) {
        pl.e_of[threadIdx.x] = a.idx_in[threadIdx.x];
        pl.wslot[threadIdx.x] = a.w_in[threadIdx.x];
    }
    __syncthreads();
    if (threadIdx.x == 0) build_groups(a, pl);
    __syncthreads();
    if (c == 0) {
        // per-expert counts before the capacity cut, and the dropped slots
        for (int e = threadIdx.x; e < a.E; e += kDlThreads) {
            int n = 0;
            for (int s = 0; s < a.S; ++s) n += pl.e_of[s] == e;
            const int64_t cl = a.cap > 0 ? cap_left(a.cap, a.cap_left_arr, e) : 0;
            const int kept = (a.cap > 0 && n > cl) ? (int)cl : n;
            a.counts[e] = n;
            a.dropped[e] = n - kept;
        }
    }
    const int ng = pl.ng;
    if (ng == 0) {  // nothing kept and no shared expert: y = 0
        for (int64_t i = (int64_t)c * kDlThreads + threadIdx.x; i < (int64_t)a.T * a.H; i += (int64_t)G * kDlThreads) {
            if (a.y_f32)
                static_cast<float*>(a.y)[i] = 0.f;
            else
                static_cast<bf16*>(a.y)[i] = __float2bfloat16_rn(0.f);
        }
        return;
    }

    // ------------------------------------------- gate/up and down, overlapped
    // Shared memory: the token vectors x [T][H] (bf16, or f16 scaled for
    // MXFP4), one group's h vectors [n][R], the partial dots [cols][S + T].
    const int j0 = (int)((int64_t)a.H * c / G), j1 = (int)((int64_t)a.H * (c + 1) / G);
    const int cols = j1 - j0;  // this CTA's output columns
    const int P = a.S + a.T;   // partial columns: routed slots, then shared rows
    const uint32_t xs = smem_u32(dsm);
    const int xbytes = (a.T * a.H * 2 + 15) / 16 * 16;
    const uint32_t hsm = xs + (uint32_t)xbytes;
    float* part = reinterpret_cast<float*>(dsm + xbytes + dl_hbytes(a.T, a.I, a.Is));  // [cols][P]
    if (kMx) {
        // f16 copies of the token rows, each scaled by a power of two
        for (int t = 0; t < a.T; ++t) {
            const float sc = f16_stage_scale(group_absmax(a.x + (int64_t)t * a.H, a.H, false, red, threadIdx.x,
                                                          kDlThreads, 0));
            if (threadIdx.x == 0) inv_sx[t] = 1.f / sc;
            stage_f16(dsm + (int64_t)t * a.H * 2, a.x + (int64_t)t * a.H, a.H, sc, false, threadIdx.x, kDlThreads);
        }
    } else {
        const uint4* src = reinterpret_cast<const uint4*>(a.x);
        uint4* dst = reinterpret_cast<uint4*>(dsm);
        for (int i = threadIdx.x; i < a.T * a.H / 8; i += kDlThreads) dst[i] = __ldg(src + i);
    }
    if (threadIdx.x < kDlMaxGroups) up_done[threadIdx.x] = 0;
    if (threadIdx.x == 0) {
        down_ok = 1;
        last_state = 0;
    }
    __syncthreads();
    unsigned int* gdone = a.bar + 1;  // [group]: CTAs whose h rows of the group are written
    const uint64_t pol_dn = policy_evict_first();
    // Down items of group g (its h rows staged at hsm): column pairs q =
    // first, first + step, ... of this CTA's columns.  A warp takes two
    // adjacent columns at a time: their down rows share the group's h
    // vectors, and twice the loads are in flight per pass.
    constexpr int kCols = 2;
    const int cp = (cols + kCols - 1) / kCols;
    // bf16 groups of one vector read it from L2 in the dot products; the
    // others (and MXFP4, whose vectors are rescaled to f16) are staged in
    // shared memory first
    auto h_direct = [&](int g) { return !kMx && pl.gcnt[g] == 1; };
    auto down_items = [&](int g, int first, int step) {
        const bool sh = pl.gexp[g] == a.E;
        const int R = sh ? a.Is : a.I;
        for (int q = first; q < cp; q += step) {
            const int jl = kCols * q;
            const bool two = kCols == 2 && jl + 1 < cols;
            const uint4* rows[kCols];
            const uint8_t* scl[kCols];
#pragma unroll
            for (int r = 0; r < kCols; ++r) {
                const int j = j0 + jl + (two ? r : 0);
                const int64_t drow = (int64_t)pl.gexp[g] * a.H + j;
                rows[r] = kMx ? reinterpret_cast<const uint4*>(a.mdb + drow * (R / 2))
                              : reinterpret_cast<const uint4*>(sh ? a.wsd + (int64_t)j * R : a.wd + drow * R);
                scl[r] = kMx ? a.mds + drow * (R / 32) : nullptr;
            }
            for (int b = 0; b < pl.gcnt[g]; b += kDlBatch) {
                const int nv = min(kDlBatch, pl.gcnt[g] - b);
                uint32_t vec[kDlBatch];
#pragma unroll
                for (int n = 0; n < kDlBatch; ++n) vec[n] = hsm + (uint32_t)((b + min(n, nv - 1)) * R * 2);
                float d[kCols][kDlBatch];
                if (kMx)
                    row_dots_mx_n<kCols>(rows, scl, R / 32, vec, nv, pol_dn, d);
                else if (h_direct(g))  // the group's one h vector, read from L2
                    row_dots_l2<kCols>(rows, R / 8,
                                       reinterpret_cast<const uint4*>((sh ? a.hs : a.h) + (int64_t)pl.gvec[g][0] * R),
                                       pol_dn, d);
                else
                    row_dots_n<kCols>(rows, R / 8, vec, nv, pol_dn, d);
#pragma unroll
                for (int n = 0; n < kDlBatch; ++n)
                    if (lane == n && n < nv) {
                        const int id = pl.gvec[g][b + n];
                        const int col = sh ? a.S + id : id;
                        const float f = kMx ? inv_sh[id] : 1.f;
                        part[jl * P + col] = d[0][n] * f;
                        if (two) part[(jl + 1) * P + col] = d[kCols - 1][n] * f;
                    }
            }
        }
    };

    if (warp < kDlUpWarps) {
        // gate/up warps: this CTA's rows i in [R c / G, R (c+1) / G) of every
        // group, group-major, dealt round-robin over the warps across group
        // boundaries; a warp reports each group as done (the CTA's last warp
        // to report publishes the group to the grid), so no warp waits.
        const int K8 = a.H / 8;
        int base = 0;  // index of the group's first item in the CTA's list
        for (int g = 0; g < ng; ++g) {
            const bool sh = pl.gexp[g] == a.E;
            const int R = sh ? a.Is : a.I;
            const int i0 = (int)((int64_t)R * c / G), n_items = (int)((int64_t)R * (c + 1) / G) - i0;
            int q = warp - base % kDlUpWarps;
            if (q < 0) q += kDlUpWarps;
            for (; q < n_items; q += kDlUpWarps) {
                const int i = i0 + q;
                const int64_t row = sh ? (int64_t)i : (int64_t)pl.gexp[g] * a.I + i;
                const uint4* rows[2];
                const uint8_t* scl[2] = {nullptr, nullptr};
                if (kMx) {
                    rows[0] = reinterpret_cast<const uint4*>(a.mgb + row * (a.H / 2));
                    rows[1] = reinterpret_cast<const uint4*>(a.mub + row * (a.H / 2));
                    scl[0] = a.mgs + row * (a.H / 32);
                    scl[1] = a.mus + row * (a.H / 32);
                } else {
                    rows[0] = reinterpret_cast<const uint4*>((sh ? a.wsg : a.wg) + row * a.H);
                    rows[1] = reinterpret_cast<const uint4*>((sh ? a.wsu : a.wu) + row * a.H);
                }
                for (int b = 0; b < pl.gcnt[g]; b += kDlBatch) {
                    const int nv = min(kDlBatch, pl.gcnt[g] - b);
                    uint32_t vec[kDlBatch];
#pragma unroll
                    for (int n = 0; n < kDlBatch; ++n) {
                        const int id = pl.gvec[g][b + min(n, nv - 1)];
                        const int tok = sh ? id : id / a.k;
                        vec[n] = xs + (uint32_t)(tok * a.H * 2);
                    }
                    float d[2][kDlBatch];
                    if (kMx)
                        row_dots_mx_n<2>(rows, scl, a.H / 32, vec, nv, pol_first, d);
                    else
                        row_dots_n<2>(rows, K8, vec, nv, pol_first, d);
#pragma unroll
                    for (int n = 0; n < kDlBatch; ++n)
                        if (lane == n && n < nv) {
                            const int id = pl.gvec[g][b + n];
                            if (kMx) {
                                const float f = inv_sx[sh ? id : id / a.k];
                                d[0][n] *= f;
                                d[1][n] *= f;
                            }
                            const bf16 hv = __float2bfloat16_rn(silu_f32(d[0][n]) * d[1][n]);
                            if (sh)
                                a.hs[(int64_t)id * a.Is + i] = hv;
                            else
                                a.h[(int64_t)id * a.I + i] = hv;
                        }
                }
            }
            base += n_items;
            // this warp's rows of group g are written: report; the last of
            // the CTA's gate/up warps publishes the group
            __syncwarp();
            if (lane == 0) {
                __threadfence();  // this warp's h rows, before its report
                if (atomicAdd(&up_done[g], 1) == kDlUpWarps - 1) {
                    __threadfence();  // every report seen, before the publication
                    atomicAdd(&gdone[g], 1u);
                }
            }
        }
        // then the last group's down columns, with the down warps, once the
        // down warps have staged its h rows (bounded wait).  Meanwhile its
        // down rows of this CTA's columns (consecutive rows) go into L2, in
        // 2 KB prefetches dealt over the gate/up warps' lanes: a prefetch
        // holds its warp up, and these warps have nothing else to do; the
        // last group's dots then wait on L2 instead of HBM.
        if (cols > 0) {
            {
                const int g = ng - 1;
                const bool sh = pl.gexp[g] == a.E;
                const int R = sh ? a.Is : a.I;
                const uint8_t* base =
                    kMx ? a.mdb + ((int64_t)pl.gexp[g] * a.H + j0) * (R / 2)
                        : reinterpret_cast<const uint8_t*>(sh ? a.wsd + (int64_t)j0 * R
                                                              : a.wd + ((int64_t)pl.gexp[g] * a.H + j0) * R);
                const int64_t bytes = (int64_t)cols * R * 2 / (kMx ? 4 : 1);
                for (int64_t off = (int64_t)(warp * 32 + lane) * 2048; off < bytes; off += kDlUpWarps * 32 * 2048)
                    prefetch_l2(base + off, (uint32_t)std::min<int64_t>(2048, bytes - off));
            }
            int st = 0;
            const uint64_t t0 = global_ns();
            while ((st = *reinterpret_cast<volatile int*>(&last_state)) == 0) {
                if (global_ns() - t0 > 2000000000ull) {
                    if (lane == 0) atomicOr(a.flags, MOE_DEVFLAG_WAIT_TIMEOUT);
                    break;
                }
                __nanosleep(128);
            }
            __syncwarp();
            if (st == 1) down_items(ng - 1, warp, kDlWarps);
        }
    } else if (cols > 0) {
        // down warps: group by group, once every CTA has published the
        // group's h rows, those rows into shared memory and this CTA's
        // columns j of the group's down rows dotted with them
        const int dt = threadIdx.x - kDlUpWarps * 32, dw = warp - kDlUpWarps;
        constexpr int kDn = kDlDownWarps * 32;
        for (int g = 0; g < ng; ++g) {
            const bool sh = pl.gexp[g] == a.E;
            const int R = sh ? a.Is : a.I;
            if (dt == 0) {
                const uint64_t t0 = global_ns();
                int ok = 1;
                while (ld_acquire_u32(&gdone[g]) < (unsigned)G) {
                    if (global_ns() - t0 > 2000000000ull) {
                        atomicOr(a.flags, MOE_DEVFLAG_WAIT_TIMEOUT);
                        ok = 0;
                        break;
                    }
                    __nanosleep(64);
                }
                __threadfence();
                down_ok = ok;
            }
            named_sync(1, kDn);  // also: every down warp is done with group g-1's h
            if (!down_ok) break;
            for (int n = 0; n < (h_direct(g) ? 0 : pl.gcnt[g]); ++n) {
                const int id = pl.gvec[g][n];
                const bf16* hrow = sh ? a.hs + (int64_t)id * R : a.h + (int64_t)id * R;
                uint8_t* dst = dsm + xbytes + n * R * 2;
                if (kMx) {
                    // routed groups only (no shared expert in this format): slot id
                    const float sc = f16_stage_scale(group_absmax(hrow, R, true, red + kDlWarps, dt, kDn, 1));
                    if (dt == 0) inv_sh[id] = 1.f / sc;
                    stage_f16(dst, hrow, R, sc, true, dt, kDn);
                } else {
                    const uint4* src = reinterpret_cast<const uint4*>(hrow);
                    uint4* d4 = reinterpret_cast<uint4*>(dst);
                    for (int i = dt; i < R / 8; i += kDn) d4[i] = __ldcg(src + i);
                }
            }
            if (!h_direct(g)) named_sync(1, kDn);
            if (g + 1 < ng) {
                down_items(g, dw, kDlDownWarps);
            } else {
                // the last group: the gate/up warps are done with their rows
                // and share its columns (all sixteen warps)
                if (dt == 0) {
                    __threadfence_block();
                    *reinterpret_cast<volatile int*>(&last_state) = 1;
                }
                down_items(g, warp, kDlWarps);
            }
        }
        if (dt == 0 && !down_ok) *reinterpret_cast<volatile int*>(&last_state) = 2;  // release the helpers
    }
    __syncthreads();
    if (cols <= 0 || !down_ok) return;
    // y[t][j]: the token's kept slots in order, then the shared expert
    for (int q = threadIdx.x; q < a.T * cols; q += kDlThreads) {
        const int t = q / cols, jl = q % cols;
        const float* pr = part + jl * P;
        float acc = 0.f;
        for (int j = 0; j < a.k; ++j) {
            const int s = t * a.k + j;
            if (pl.kept[s]) acc = fmaf(pl.wslot[s], pr[s], acc);
        }
        if (a.Is > 0) acc += pr[a.S + t];
        const int64_t o = (int64_t)t * a.H + j0 + jl;
        if (a.y_f32)
            static_cast<float*>(a.y)[o] = acc;
        else
            static_cast<bf16*>(a.y)[o] = __float2bfloat16_rn(acc);
    }
}

// Shared memory: the x rows, one group's h rows, the partial dots
// [columns per CTA][S + T].
int64_t dl_smem_bytes(const Plan& p, int grid) {
    const int64_t xb = (p.T * p.H * 2 + 15) / 16 * 16;
    const int64_t cols = (p.H + grid - 1) / grid;
    return xb + dl_hbytes((int)p.T, (int)p.I, (int)p.Is) + cols * (p.S + p.T) * 4;
}

}  // namespace

namespace {
bool decode_fits(const Plan& p, int max_slots) {
    if (!p.bf16 || p.S < 1 || p.S > max_slots) return false;
    const int grid = device_sm_count();
    if ((p.H + grid - 1) / grid > kDlMaxCols) return false;
    return dl_smem_bytes(p, grid) <= kDlSmemMax;
}
}  // namespace

bool decode_ffn_eligible(const Plan& p) { return decode_fits(p, kDecodeMaxSlots); }
bool decode_mxfp4_eligible(const Plan& p) { return decode_fits(p, kDecodeMaxSlotsMx); }

namespace {

DlArgs base_args(const Plan& p, const void* x, const void* router_w, const float* router_b,
                 const int32_t* topk_idx_in, const float* topk_w_in, int32_t* topk_idx_out, void* y,
                 int32_t* counts, int32_t* dropped) {
    DlArgs a{};
    a.x = (const bf16*)x;
    a.router_w = (const bf16*)router_w;
    a.router_b = router_b;
    a.idx_in = topk_idx_in;
    a.w_in = topk_w_in;
    a.idx_out = topk_idx_out;
    a.h = (bf16*)p.h;
    a.hs = (bf16*)p.h + p.S * p.I;
    a.y = y;
    a.y_f32 = p.y_f32;
    a.drop_negative = p.drop_negative;
    a.scores = p.dec_scores;
    a.bar = p.dec_bar;
    a.counts = counts;
    a.dropped = dropped;
    a.flags = p.flags;
    a.T = (int)p.T;
    a.H = (int)p.H;
    a.I = (int)p.I;
    a.Is = (int)p.Is;
    a.E = (int)p.E;
    a.k = (int)p.k;
    a.S = (int)p.S;
    a.cap = p.cap;
    a.cap_left_arr = p.cap_left_arr;
    return a;
}

template <bool kMx>
cudaError_t launch_typed(const Plan& p, const DlArgs& a, const char* name, cudaStream_t st) {
    const int grid = device_sm_count();
    const size_t smem = (size_t)dl_smem_bytes(p, grid);
    cudaError_t e = ensure_smem_attr(decode_layer_kernel<kMx>, kDlSmemMax);
    if (e != cudaSuccess) return e;
    // the grid barrier and the group counters count arrivals from zero
    e = cudaMemsetAsync(p.dec_bar, 0, kDecodeCounters * sizeof(unsigned int), st);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid, 1, 1);
    cfg.blockDim = dim3(kDlThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    trace_before(name, st);
    e = cudaLaunchKernelEx(&cfg, decode_layer_kernel<kMx>, a);
    trace_after(st);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_layer(const Plan& p, const void* x, const void* router_w, const float* router_b,
                                const int32_t* topk_idx_in, const float* topk_w_in, int32_t* topk_idx_out,
                                const void* w_gate, const void* w_up, const void* w_down, const void* ws_gate,
                                const void* ws_up, const void* ws_down, void* y, int32_t* counts,
                                int32_t* dropped, cudaStream_t st) {
    if (!decode_ffn_eligible(p)) return cudaErrorInvalidValue;
    DlArgs a = base_args(p, x, router_w, router_b, topk_idx_in, topk_w_in, topk_idx_out, y, counts, dropped);
    a.wg = (const bf16*)w_gate;
    a.wu = (const bf16*)w_up;
    a.wd = (const bf16*)w_down;
    a.wsg = (const bf16*)ws_gate;
    a.wsu = (const bf16*)ws_up;
    a.wsd = (const bf16*)ws_down;
    return launch_typed<false>(p, a, "decode_layer", st);
}

cudaError_t launch_decode_layer_mxfp4(const Plan& p, const void* x, const void* router_w, const float* router_b,
                                      int32_t* topk_idx_out, const uint8_t* const (&mx)[6], void* y, int32_t* counts,
                                      int32_t* dropped, cudaStream_t st) {
    if (!decode_mxfp4_eligible(p) || p.Is > 0 || p.H % 32 || p.I % 32) return cudaErrorInvalidValue;
    DlArgs a = base_args(p, x, router_w, router_b, nullptr, nullptr, topk_idx_out, y, counts, dropped);
    a.mgb = mx[0];
    a.mgs = mx[1];
    a.mub = mx[2];
    a.mus = mx[3];
    a.mdb = mx[4];
    a.mds = mx[5];
    return launch_typed<true>(p, a, "decode_layer_mxfp4", st);
}

}  // namespace moe
