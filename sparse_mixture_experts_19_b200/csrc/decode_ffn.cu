// Decode FFN: the expert FFNs and the weighted combine for a handful of
// routed slots (T*k <= 8), as two weight-streaming kernels.
//
// "MoE稀疏架构是什么？从原理到落地的系统解读", section 四: y is the sum over
// the selected experts of w * FFN_e(x).  "Mixture of Experts (MoEs) in
// Transformers", section Expert Backend: with few tokens the layer's time is
// the bytes of the selected experts' weights.
//
// With one or two slots per expert a 128-row tensor-core tile would be
// almost all padding, so the layer is written as what it is: one read of the
// selected experts' weight rows.  Both kernels are persistent (one CTA per
// SM).  Warps 0-3 stream whole weight rows (contiguous 2*H or 2*I bytes)
// into a shared-memory ring with 1-D bulk copies (cp.async.bulk, completion
// counted on the stage's mbarrier).  W compute warps (8, or fewer when few
// rows fit) take the stages round-robin, each lane over 16-byte chunks of
// the row, against the token vectors (x rows, or h rows) of the CTA's
// experts that the compute warps first copy into shared memory next to the
// ring (float32 sums in packed f32x2 FMAs).  Each compute warp owns its own
// run of ring slots, filled in its stage order by one producer, so every
// wait is on the next phase of a slot that warp itself released (an mbarrier
// parity wait can only tell its phase from the one before).  Each CTA takes
// a contiguous range of stages: consecutive stages read consecutive DRAM
// pages and every SM streams the same number of bytes.
//
//   decode_gateup: stage (group, i) = rows W_g[e][i] and W_u[e][i];
//                  h[slot][i] = bf16(silu(x . W_g[e][i]) * (x . W_u[e][i])).
//   decode_down:   stage (group, hrow pair) = rows W_d[e][hrow], W_d[e][hrow+1]
//                  (one contiguous copy); the dot products with the group's h
//                  rows go to a float32 buffer [H, S + T]; after its last
//                  stage each warp counts its stages' arrivals per pair, and
//                  the warp bringing a pair's count to the number of experts
//                  writes
//                  y[t][hrow] = bf16(sum over j in slot order of
//                  w[t,j] * d(t,j), plus the shared expert's d(t)).
// The counters only order the work; every sum has a fixed order, so y is
// bit-reproducible.
#include <algorithm>

#include "common.cuh"
#include "sm100.cuh"
#include "tma_host.cuh"

namespace moe {
namespace {

using namespace sm100;

constexpr int kDecMaxGroups = kDecodeMaxSlots + 1;  // distinct routed experts + shared
constexpr int kDecProducers = 4;                    // warps 0-3 stream (lane 0 of each)
constexpr int kDecWarps = 8;                        // compute warps 4-11
constexpr int kDecThreads = 32 * (kDecProducers + kDecWarps);
constexpr int kDecSmemBytes = 220 * 1024;  // vectors + ring
constexpr int kDecVecRows = 4;             // token vectors staged in shared memory per CTA
constexpr int kDecMaxStages = 32;          // ring slots at most
constexpr int kDecBatch = 4;               // token vectors per pass over a weight row
constexpr int kDecDownRows = 2;            // W_d rows per down stage

// Ring geometry: W compute warps (1, 2, 4 or 8), each owning Rw consecutive
// slots.  Stage l goes to compute warp l % W, which takes its stages in
// order; its j-th stage (j = l / W) uses slot j % Rw of its run.  Producer
// p < NP = min(4, W) issues the stages l = p mod NP, so each compute warp's
// slots are always filled, in order, by the same producer thread.
struct Ring {
    int W, Rw;
    __device__ __forceinline__ int producers() const { return W < kDecProducers ? W : kDecProducers; }
    __device__ __forceinline__ int slot(int l) const { return (l % W) * Rw + (l / W) % Rw; }
    __device__ __forceinline__ uint32_t parity(int l) const { return ((l / W) / Rw) & 1; }
};

struct DecArgs {
    const bf16* x;
    const int32_t* idx;
    const float* w;
    const bf16 *wg, *wu, *wd, *wsg, *wsu, *wsd;
    bf16* h;   // [S, I] routed activations, slot order
    bf16* hs;  // [T, Is] shared-expert activations
    bf16* y;
    float* part;   // [H, P] partial dot products: column s (routed slot) or S + t (shared)
    int32_t* cnt;  // [H / 2] stage arrivals per hrow pair
    int32_t* counts;
    int32_t* dropped;
    int32_t* flags;
    int T, H, I, Is, E, k, S, P;
    int64_t cap;
    const int32_t* cap_left_arr;  // [E] or null: capacity left per expert (token shards)
    int vec_bytes;  // bytes of shared memory before the ring (multiple of 128)
};

// The slots grouped by expert, rebuilt by every CTA (S <= kDecodeMaxSlots).
struct DecPlan {
    int ng;
    int gexp[kDecMaxGroups];  // expert id; E marks the shared expert
    int gcnt[kDecMaxGroups];
    int gvec[kDecMaxGroups][kDecodeMaxSlots];  // routed: slot s; shared: token t
    int gpre[kDecMaxGroups + 1];               // prefix of rows per group (I or Is)
    int voff[kDecMaxGroups];                   // byte offset of the group's vectors in vec, or -1
    int e_of[kDecodeMaxSlots];
    int kept[kDecodeMaxSlots];
    float wslot[kDecodeMaxSlots];
};

// Capacity in token order: slot s = t*k + j of expert e is kept while fewer
// than cap_left(e) earlier slots of e were kept (a token meets an expert at
// most once, so slot order is token order).
__device__ void build_plan(const DecArgs& a, DecPlan& pl) {
    const int tid = threadIdx.x;
    if (tid < a.S) {
        pl.e_of[tid] = a.idx[tid];
        pl.wslot[tid] = a.w[tid];
    }
    __syncthreads();
    if (tid == 0) {
        int ng = 0;
        bool bad = false;
        for (int s = 0; s < a.S; ++s) {
            const int e = pl.e_of[s];
            pl.kept[s] = 0;
            if (e < 0 || e >= a.E) {
                bad = true;
                continue;
            }
            int g = 0;
            while (g < ng && pl.gexp[g] != e) ++g;
            if (g == ng) {
                pl.gexp[ng] = e;
                pl.gcnt[ng] = 0;
                ++ng;
            }
            if (a.cap > 0 && pl.gcnt[g] >= cap_left(a.cap, a.cap_left_arr, e)) continue;
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
        pl.gpre[0] = 0;
        for (int g = 0; g < ng; ++g) pl.gpre[g + 1] = pl.gpre[g] + (pl.gexp[g] == a.E ? a.Is : a.I);
        if (bad && blockIdx.x == 0) set_flag(a.flags, MOE_DEVFLAG_BAD_EXPERT_INDEX);
    }
    __syncthreads();
}

__device__ __forceinline__ void init_ring(const Ring& rg, uint64_t* full, uint64_t* empty, int* abort_s) {
    if (threadIdx.x == 0) {
        for (int r = 0; r < rg.W * rg.Rw; ++r) {
            mbar_init(&full[r], 1);
            mbar_init(&empty[r], 1);
        }
        *abort_s = 0;
        fence_mbar_init();
    }
}

// Barrier of the 8 compute warps only (the producer warps keep streaming).
__device__ __forceinline__ void compute_warps_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(32 * kDecWarps) : "memory");
}

// Copy `bytes` (a multiple of 16) from global to shared memory with the
// compute warps' threads.
__device__ __forceinline__ void copy_to_smem(uint8_t* dst, const void* src, int64_t bytes) {
    const uint4* s = reinterpret_cast<const uint4*>(src);
    uint4* d = reinterpret_cast<uint4*>(dst);
    for (int64_t i = threadIdx.x - 32 * kDecProducers; i < bytes / 16; i += 32 * kDecWarps) d[i] = s[i];
}

__device__ __forceinline__ void widen8(const uint4& q, float2 (&f)[4]) {
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
    for (int i = 0; i < 4; ++i) f[i] = __bfloat1622float2(p[i]);
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

// d[r][n] = sum_c W_r[c] * v_n[c] over K8 16-byte chunks, for NW weight rows
// in shared memory (row r at shared address w + r*K8*16) and NV vectors, in
// shared memory (kVecSmem: shared addresses vs[n]) or global memory (vg[n]);
// float32 (each lane keeps even and odd elements in the two halves of an
// f32x2 accumulator), summed over the warp: every lane ends with the totals.
// The loop has no branches, so the loads of several iterations are in flight
// together.
template <int NW, int NV, bool kVecSmem>
__device__ __forceinline__ void dots(uint32_t w, int K8, const uint32_t (&vs)[kDecBatch],
                                     const uint4* const (&vg)[kDecBatch], float (&d)[NW][kDecBatch]) {
    const int lane = threadIdx.x & 31;
    float2 acc[NW][NV];
#pragma unroll
    for (int r = 0; r < NW; ++r)
#pragma unroll
        for (int n = 0; n < NV; ++n) acc[r][n] = make_float2(0.f, 0.f);
#pragma unroll 4
    for (int c = lane; c < K8; c += 32) {
        uint4 wq[NW], xq[NV];
#pragma unroll
        for (int r = 0; r < NW; ++r) wq[r] = lds128(w + (uint32_t)(r * K8 + c) * 16u);
#pragma unroll
        for (int n = 0; n < NV; ++n) xq[n] = kVecSmem ? lds128(vs[n] + (uint32_t)c * 16u) : __ldg(vg[n] + c);
        float2 wf[NW][4];
#pragma unroll
        for (int r = 0; r < NW; ++r) widen8(wq[r], wf[r]);
#pragma unroll
        for (int n = 0; n < NV; ++n) {
            float2 xf[4];
            widen8(xq[n], xf);
#pragma unroll
            for (int r = 0; r < NW; ++r)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[r][n] = __ffma2_rn(xf[e], wf[r][e], acc[r][n]);
        }
    }
#pragma unroll
    for (int r = 0; r < NW; ++r)
#pragma unroll
        for (int n = 0; n < NV; ++n) {
            float t = acc[r][n].x + acc[r][n].y;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
            d[r][n] = t;
        }
}

template <int NW, bool kVecSmem>
__device__ __forceinline__ void dots_n(uint32_t w, int K8, const uint32_t (&vs)[kDecBatch],
                                       const uint4* const (&vg)[kDecBatch], int nv, float (&d)[NW][kDecBatch]) {
    switch (nv) {
        case 1: dots<NW, 1, kVecSmem>(w, K8, vs, vg, d); break;
        case 2: dots<NW, 2, kVecSmem>(w, K8, vs, vg, d); break;
        case 3: dots<NW, 3, kVecSmem>(w, K8, vs, vg, d); break;
        default: dots<NW, 4, kVecSmem>(w, K8, vs, vg, d); break;
    }
}

// dots for nv (1..4) vectors at byte offsets off[n]: from the shared-memory
// vector area (smem_base, a shared address) or from global memory (gbase).
template <int NW>
__device__ __forceinline__ void dots_at(uint32_t w, int K8, bool in_smem, uint32_t smem_base, const uint8_t* gbase,
                                        const int64_t (&off)[kDecBatch], int nv, float (&d)[NW][kDecBatch]) {
    uint32_t vs[kDecBatch];
    const uint4* vg[kDecBatch];
#pragma unroll
    for (int n = 0; n < kDecBatch; ++n) {
        vs[n] = smem_base + (uint32_t)off[n];
        vg[n] = reinterpret_cast<const uint4*>(gbase + off[n]);
    }
    if (in_smem)
        dots_n<NW, true>(w, K8, vs, vg, nv, d);
    else
        dots_n<NW, false>(w, K8, vs, vg, nv, d);
}

// Shared-memory offsets for the vectors of the groups in [ga, gb] (in order,
// while they fit in vec_bytes; the rest are read from L2).  vbytes(g) is the
// bytes of one vector of group g.  Thread 0; the caller synchronises.
template <typename F>
__device__ __forceinline__ void place_vectors(DecPlan& pl, int ga, int gb, int vec_bytes, F vbytes) {
    int64_t off = 0;
    for (int g = 0; g < pl.ng; ++g) pl.voff[g] = -1;
    for (int g = ga; g <= gb; ++g) {
        const int64_t bytes = (int64_t)pl.gcnt[g] * vbytes(g);
        if (off + bytes > vec_bytes) break;
        pl.voff[g] = (int)off;
        off += bytes;
    }
}

// Every lane waits on the stage's phase (bounded); false if any gave up.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          int32_t* flags) {
    const bool ok = wait_sleep_or_abort(bar, parity, abort_flag, flags);
    return __all_sync(0xffffffffu, ok);
}

// Producer p's exit: none of its bulk copies may still be in flight (bounded
// waits on the phases of its stages among the last W*Rw before `end`, the
// stage it stopped at).
__device__ __forceinline__ void drain_ring(uint64_t* full, int p, int end, const Ring& rg) {
    const int np = rg.producers();
    for (int l = p; l < end; l += np)
        if (l >= end - rg.W * rg.Rw) drain_wait(&full[rg.slot(l)], rg.parity(l));
}

__global__ void __launch_bounds__(kDecThreads, 1) decode_gateup_kernel(const DecArgs a, const Ring rg) {
    extern __shared__ __align__(128) uint8_t dsm[];
    uint8_t* vec = dsm;                 // x rows of this CTA's groups
    uint8_t* ring = dsm + a.vec_bytes;  // W*Rw slots of a gate row and an up row
    __shared__ DecPlan pl;
    __shared__ uint64_t full[kDecMaxStages], empty[kDecMaxStages];
    __shared__ int abort_s;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    build_plan(a, pl);
    if (blockIdx.x == 0) {
        // per-expert counts before capacity and the dropped slots
        for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
            int c = 0;
            for (int s = 0; s < a.S; ++s) c += pl.e_of[s] == e;
            const int64_t cl = a.cap > 0 ? cap_left(a.cap, a.cap_left_arr, e) : 0;
            const int kept = (a.cap > 0 && c > cl) ? (int)cl : c;
            a.counts[e] = c;
            a.dropped[e] = c - kept;
        }
    }
    // the down kernel's arrival counters start at zero
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < a.H / kDecDownRows;
         i += (int64_t)gridDim.x * blockDim.x)
        a.cnt[i] = 0;
    const int64_t N = pl.gpre[pl.ng];
    const int64_t q0 = N * blockIdx.x / gridDim.x, q1 = N * (blockIdx.x + 1) / gridDim.x;
    const int nq = (int)(q1 - q0);
    const uint32_t row_bytes = 2u * (uint32_t)a.H;
    const uint32_t slot_bytes = 2 * row_bytes;
    const int K8 = a.H / 8;
    if (threadIdx.x == 0) {
        int ga = 0, gb = -1;
        if (nq > 0) {
            while (q0 >= pl.gpre[ga + 1]) ++ga;
            gb = ga;
            while (q1 - 1 >= pl.gpre[gb + 1]) ++gb;
        }
        place_vectors(pl, ga, gb, a.vec_bytes, [&](int) { return (int64_t)row_bytes; });
    }
    init_ring(rg, full, empty, &abort_s);
    __syncthreads();
    volatile int* abort_flag = &abort_s;

    if (warp < kDecProducers) {
        if (lane == 0 && warp < rg.producers()) {
            int g = 0, l = warp;
            for (; l < nq; l += rg.producers()) {
                const int r = rg.slot(l);
                if (!wait_sleep_or_abort(&empty[r], rg.parity(l) ^ 1, abort_flag, a.flags)) break;
                const int64_t q = q0 + l;
                while (q >= pl.gpre[g + 1]) ++g;
                const int64_t i = q - pl.gpre[g];
                const int e = pl.gexp[g];
                const bf16* rgate = e < a.E ? a.wg + ((int64_t)e * a.I + i) * a.H : a.wsg + i * a.H;
                const bf16* rup = e < a.E ? a.wu + ((int64_t)e * a.I + i) * a.H : a.wsu + i * a.H;
                uint8_t* dst = ring + (size_t)r * slot_bytes;
                mbar_arrive_expect_tx(&full[r], slot_bytes);
                bulk_load(dst, rgate, row_bytes, &full[r]);
                bulk_load(dst + row_bytes, rup, row_bytes, &full[r]);
            }
            drain_ring(full, warp, min(l, nq), rg);
        }
        return;
    }
    // stage the x rows of this CTA's groups (one per slot of the group)
    for (int g = 0; g < pl.ng; ++g) {
        if (pl.voff[g] < 0) continue;
        const bool shared = pl.gexp[g] == a.E;
        for (int n = 0; n < pl.gcnt[g]; ++n) {
            const int id = pl.gvec[g][n];
            const int64_t tok = shared ? id : id / a.k;
            copy_to_smem(vec + pl.voff[g] + (int64_t)n * row_bytes, a.x + tok * a.H, row_bytes);
        }
    }
    compute_warps_sync();
    const int cw = warp - kDecProducers;  // compute warp 0..7
    if (cw >= rg.W) return;
    int g = 0;
    for (int l = cw; l < nq; l += rg.W) {
        const int r = rg.slot(l);
        if (!warp_wait(&full[r], rg.parity(l), abort_flag, a.flags)) break;
        const int64_t q = q0 + l;
        while (q >= pl.gpre[g + 1]) ++g;
        const int i = (int)(q - pl.gpre[g]);
        const bool shared = pl.gexp[g] == a.E;
        const uint32_t wrow = smem_u32(ring + (size_t)r * slot_bytes);
        const bool in_smem = pl.voff[g] >= 0;
        for (int b = 0; b < pl.gcnt[g]; b += kDecBatch) {
            const int nv = min(kDecBatch, pl.gcnt[g] - b);
            int64_t off[kDecBatch];  // byte offsets of the vectors in vec, or in x
            float d[2][kDecBatch];
#pragma unroll
            for (int n = 0; n < kDecBatch; ++n) {
                const int nn = b + min(n, nv - 1);
                const int id = pl.gvec[g][nn];
                off[n] = in_smem ? pl.voff[g] + (int64_t)nn * row_bytes : (shared ? id : id / a.k) * (int64_t)row_bytes;
            }
            dots_at<2>(wrow, K8, in_smem, smem_u32(vec), reinterpret_cast<const uint8_t*>(a.x), off, nv, d);
#pragma unroll
            for (int n = 0; n < kDecBatch; ++n) {
                if (lane == n && n < nv) {
                    const int id = pl.gvec[g][b + n];
                    const bf16 hv = __float2bfloat16_rn(silu_f32(d[0][n]) * d[1][n]);
                    if (shared)
                        a.hs[(int64_t)id * a.Is + i] = hv;
                    else
                        a.h[(int64_t)id * a.I + i] = hv;
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[r]);
    }
}

__global__ void __launch_bounds__(kDecThreads, 1) decode_down_kernel(const DecArgs a, const Ring rg) {
    extern __shared__ __align__(128) uint8_t dsm[];
    uint8_t* vec = dsm;                 // h rows of this CTA's groups
    uint8_t* ring = dsm + a.vec_bytes;  // W*Rw slots of kDecDownRows W_d rows
    __shared__ DecPlan pl;
    __shared__ uint64_t full[kDecMaxStages], empty[kDecMaxStages];
    __shared__ int abort_s;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    build_plan(a, pl);
    const int ng = pl.ng;
    if (ng == 0) {  // no kept slot and no shared expert: y = 0
        for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < (int64_t)a.T * a.H;
             i += (int64_t)gridDim.x * blockDim.x)
            a.y[i] = __float2bfloat16_rn(0.f);
        return;
    }
    // stages (group, hrow pair), group-major; this CTA's range and its groups
    const int npair = a.H / kDecDownRows;
    const int64_t N = (int64_t)ng * npair;
    const int64_t q0 = N * blockIdx.x / gridDim.x, q1 = N * (blockIdx.x + 1) / gridDim.x;
    const int nq = (int)(q1 - q0);
    if (threadIdx.x == 0) {
        const int ga = (int)(q0 / npair), gb = nq > 0 ? (int)((q1 - 1) / npair) : ga - 1;
        place_vectors(pl, ga, gb, a.vec_bytes, [&](int g) { return (int64_t)2 * (pl.gexp[g] == a.E ? a.Is : a.I); });
    }
    init_ring(rg, full, empty, &abort_s);
    __syncthreads();
    volatile int* abort_flag = &abort_s;
    const uint32_t slot_bytes = 2u * kDecDownRows * (uint32_t)max(a.I, a.Is);

    if (warp < kDecProducers) {
        if (lane == 0 && warp < rg.producers()) {
            int l = warp;
            for (; l < nq; l += rg.producers()) {
                const int r = rg.slot(l);
                if (!wait_sleep_or_abort(&empty[r], rg.parity(l) ^ 1, abort_flag, a.flags)) break;
                const int64_t q = q0 + l, hrow = (q % npair) * kDecDownRows;
                const int e = pl.gexp[q / npair];
                const bool shared = e == a.E;
                const bf16* src = shared ? a.wsd + hrow * a.Is : a.wd + ((int64_t)e * a.H + hrow) * a.I;
                const uint32_t bytes = 2u * kDecDownRows * (uint32_t)(shared ? a.Is : a.I);
                mbar_arrive_expect_tx(&full[r], bytes);
                bulk_load(ring + (size_t)r * slot_bytes, src, bytes, &full[r]);
            }
            drain_ring(full, warp, min(l, nq), rg);
        }
        return;
    }
    // stage the groups' h rows (each row is contiguous in h or hs)
    for (int g = 0; g < ng; ++g) {
        if (pl.voff[g] < 0) continue;
        const bool shared = pl.gexp[g] == a.E;
        const int K = shared ? a.Is : a.I;
        for (int n = 0; n < pl.gcnt[g]; ++n) {
            const int id = pl.gvec[g][n];
            copy_to_smem(vec + pl.voff[g] + (int64_t)n * K * 2, shared ? a.hs + (int64_t)id * K : a.h + (int64_t)id * K,
                         (int64_t)K * 2);
        }
    }
    compute_warps_sync();
    const int cw = warp - kDecProducers;  // compute warp 0..7
    if (cw >= rg.W) return;
    int done = cw;  // first stage of this warp not completed
    for (int l = cw; l < nq; l += rg.W) {
        const int r = rg.slot(l);
        if (!warp_wait(&full[r], rg.parity(l), abort_flag, a.flags)) break;
        const int64_t q = q0 + l, pair = q % npair, hrow = pair * kDecDownRows;
        const int g = (int)(q / npair);
        const bool shared = pl.gexp[g] == a.E;
        const int K = shared ? a.Is : a.I;
        const uint32_t wrow = smem_u32(ring + (size_t)r * slot_bytes);
        const bool in_smem = pl.voff[g] >= 0;
        for (int b = 0; b < pl.gcnt[g]; b += kDecBatch) {
            const int nv = min(kDecBatch, pl.gcnt[g] - b);
            int64_t off[kDecBatch];  // byte offsets of the vectors in vec, or in h / hs
            float d[kDecDownRows][kDecBatch];
#pragma unroll
            for (int n = 0; n < kDecBatch; ++n) {
                const int nn = b + min(n, nv - 1);
                off[n] = in_smem ? pl.voff[g] + (int64_t)nn * K * 2 : (int64_t)pl.gvec[g][nn] * K * 2;
            }
            dots_at<kDecDownRows>(wrow, K / 8, in_smem, smem_u32(vec),
                                  reinterpret_cast<const uint8_t*>(shared ? a.hs : a.h), off, nv, d);
#pragma unroll
            for (int n = 0; n < kDecBatch; ++n) {
                if (lane == n && n < nv) {
                    const int col = shared ? a.S + pl.gvec[g][b + n] : pl.gvec[g][b + n];
#pragma unroll
                    for (int rr = 0; rr < kDecDownRows; ++rr) a.part[(hrow + rr) * a.P + col] = d[rr][n];
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[r]);  // the dot products are done: the ring slot is free
        done = l + rg.W;
    }
    // Arrivals after the warp's last stage, behind one fence: the counters
    // only pick which stage's warp sums a pair (the one bringing its arrivals
    // to ng), so they need not delay the streaming loop.
    __threadfence();  // this warp's partials, before its arrivals
    __syncwarp();
    // 32 stages at a time, one arrival per lane, all in flight together; a
    // lane whose arrival completes a pair sums that pair's y entries itself.
    for (int l0 = cw; l0 < done; l0 += 32 * rg.W) {
        const int l = l0 + lane * rg.W;
        if (l >= done) continue;
        const int64_t q = q0 + l, pair = q % npair, hrow = pair * kDecDownRows;
        if (atomicAdd(&a.cnt[pair], 1) != ng - 1) continue;
        __threadfence();
        for (int q2 = 0; q2 < a.T * kDecDownRows; ++q2) {
            const int t = q2 / kDecDownRows;
            const int64_t hr = hrow + q2 % kDecDownRows;
            const float* pr = a.part + hr * a.P;
            float acc = 0.f;
            for (int j = 0; j < a.k; ++j) {
                const int s = t * a.k + j;
                if (pl.kept[s]) acc = fmaf(pl.wslot[s], __ldcg(pr + s), acc);
            }
            if (a.Is > 0) acc += __ldcg(pr + a.S + t);
            a.y[(int64_t)t * a.H + hr] = __float2bfloat16_rn(acc);
        }
    }
}

// Bytes of shared memory for staged token vectors: up to kDecVecRows vectors
// of the longer vector length (H for the gate/up kernel; max(I, Is) for the
// down kernel), never more than S + T of them.
int64_t vec_bytes_for(const Plan& p, int64_t vec_len) {
    const int64_t rows = std::min<int64_t>(kDecVecRows, p.S + (p.Is ? p.T : 0));
    return (rows * vec_len * 2 + 127) / 128 * 128;
}

// W*Rw ring slots of slot_bytes in what shared memory the vectors leave: 8
// compute warps when 8 slots fit, else 4, 2 or 1; Rw = slots / W.
Ring make_ring(int64_t slot_bytes, int64_t vec_bytes) {
    const int n = (int)std::min<int64_t>(kDecMaxStages,
                                         (kDecSmemBytes - vec_bytes) / std::max<int64_t>(slot_bytes, 1));
    const int W = n >= 8 ? 8 : n >= 4 ? 4 : n >= 2 ? 2 : 1;
    return Ring{W, std::max(n, 1) / W};
}

struct DecGeom {
    int64_t vec_gu, vec_dn, slot_gu, slot_dn;
    Ring gu, dn;
};

DecGeom geometry(const Plan& p) {
    DecGeom d;
    d.vec_gu = vec_bytes_for(p, p.H);
    d.vec_dn = vec_bytes_for(p, std::max(p.I, p.Is));
    d.slot_gu = 4 * p.H;
    d.slot_dn = 2 * kDecDownRows * std::max(p.I, p.Is);
    d.gu = make_ring(d.slot_gu, d.vec_gu);
    d.dn = make_ring(d.slot_dn, d.vec_dn);
    return d;
}

}  // namespace

bool decode_ffn_eligible(const Plan& p) {
    if (!p.bf16 || p.S < 1 || p.S > kDecodeMaxSlots || p.H % kDecDownRows) return false;
    const DecGeom d = geometry(p);
    return d.gu.W * d.gu.Rw >= 2 && d.dn.W * d.dn.Rw >= 2 &&
           d.vec_gu + d.gu.W * d.gu.Rw * d.slot_gu <= kDecSmemBytes &&
           d.vec_dn + d.dn.W * d.dn.Rw * d.slot_dn <= kDecSmemBytes;
}

cudaError_t launch_decode_ffn(const Plan& p, const void* x, const int32_t* topk_idx, const void* w_gate,
                              const void* w_up, const void* w_down, const void* ws_gate, const void* ws_up,
                              const void* ws_down, void* y, int32_t* counts, int32_t* dropped, cudaStream_t st) {
    if (!decode_ffn_eligible(p)) return cudaErrorInvalidValue;
    DecArgs a{};
    a.x = (const bf16*)x;
    a.idx = topk_idx;
    a.w = p.topk_w;
    a.wg = (const bf16*)w_gate;
    a.wu = (const bf16*)w_up;
    a.wd = (const bf16*)w_down;
    a.wsg = (const bf16*)ws_gate;
    a.wsu = (const bf16*)ws_up;
    a.wsd = (const bf16*)ws_down;
    a.h = (bf16*)p.h;
    a.hs = (bf16*)p.h + p.S * p.I;
    a.y = (bf16*)y;
    a.part = p.dec_part;
    a.cnt = p.dec_cnt;
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
    a.P = (int)(p.S + (p.Is ? p.T : 0));
    a.cap = p.cap;
    a.cap_left_arr = p.cap_left_arr;
    cudaError_t e = ensure_smem_attr(decode_gateup_kernel, kDecSmemBytes);
    if (e == cudaSuccess) e = ensure_smem_attr(decode_down_kernel, kDecSmemBytes);
    if (e != cudaSuccess) return e;
    const DecGeom d = geometry(p);
    const int grid = device_sm_count();
    a.vec_bytes = (int)d.vec_gu;
    trace_before("decode_gateup", st);
    decode_gateup_kernel<<<grid, kDecThreads, d.vec_gu + d.gu.W * d.gu.Rw * d.slot_gu, st>>>(a, d.gu);
    trace_after(st);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    a.vec_bytes = (int)d.vec_dn;
    trace_before("decode_down", st);
    decode_down_kernel<<<grid, kDecThreads, d.vec_dn + d.dn.W * d.dn.Rw * d.slot_dn, st>>>(a, d.dn);
    trace_after(st);
    return cudaGetLastError();
}

}  // namespace moe
