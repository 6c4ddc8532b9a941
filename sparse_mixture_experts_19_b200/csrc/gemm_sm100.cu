// Grouped expert GEMMs on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// "Mixture of Experts (MoEs) in Transformers", section Expert Backend: the
// grouped_mm backend sorts tokens by expert and runs one grouped GEMM;
// section Weight Loading Refactor: experts packed as [E, out, in] tensors.
// "MoE稀疏架构是什么？从原理到落地的系统解读", section 四: the output is the
// routing-weighted sum of the selected experts' outputs.
//
// Two kernels from one template:
//   gate/up:  h = silu(X W_g[e]^T) * (X W_u[e]^T), rounded to bf16.  One MMA
//             of N = 256 covers 128 gate rows and the 128 matching up rows,
//             so G and U of a tile land side by side in one TMEM accumulator
//             and the SwiGLU is applied in the epilogue.
//   down:     out = h W_d[e]^T; the epilogue multiplies row r by its routing
//             weight and stores it in bf16 at its grouped row (the combine
//             kernel then sums each token's rows), or stores unweighted
//             float32 rows (stage API).
//
// Groups: 0..E-1 routed experts (rows offsets[g]..offsets[g+1] of the
// grouped activations), group E the shared expert (token rows of x / hs).
// A tile is 128 rows x BN columns of one group.  Tiles of one group run in
// bands of gm row tiles: a band visits every weight column block, m-fastest
// inside each block, before the next band starts.  CTAs running side by side
// then share one weight slice through L2, and the band's activation rows
// (gm x 128 x K, about 32 MB) stay in L2 across the column blocks instead of
// being read from HBM once per block when a group has many rows.
//
// Persistent CTA per SM, 192 threads: warp 0 issues TMA loads into a 4-stage
// shared-memory ring, warp 1 issues tcgen05.mma (one thread) and owns the
// TMEM (2 accumulators x 256 columns, so the epilogue of one tile overlaps
// the main loop of the next), warps 2-5 drain TMEM (one 32-lane quadrant
// each).  Every wait is bounded; a timeout sets MOE_DEVFLAG_WAIT_TIMEOUT and
// the CTA unwinds and frees its TMEM.
#include <algorithm>

#include <cuda_fp16.h>

#include "common.cuh"
#include "mxfp4.cuh"
#include "sm100.cuh"
#include "tma_host.cuh"

namespace moe {
namespace {

using namespace sm100;

constexpr int kBM = 128;   // tile rows = MMA M
constexpr int kBK = 64;    // K per stage: one 128-byte swizzle atom of bf16
constexpr int kStages = 4;
constexpr int kBRows = 256;  // B rows per stage = MMA N
constexpr int kABytes = kBM * kBK * 2;
constexpr int kBBytes = kBRows * kBK * 2;
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kAccCols = 256;
constexpr int kTmemCols = 2 * kAccCols;
constexpr int kThreads = 192;
constexpr int kEpiThreads = 128;
constexpr uint32_t kIdesc = idesc_bf16(kBM, kBRows);
constexpr int kSmallRows = 32;                   // A box rows of a group's short tile
constexpr int kSmallABytes = kSmallRows * kBK * 2;

struct GemmArgs {
    const int32_t* offsets;       // [E+2]
    const int32_t* mtile_prefix;  // [E+1] prefix of ceil(rows_e / 128)
    int32_t* flags;
    int E, T, has_shared;
    int N, Ns;  // output columns (routed, shared)
    int K, Ks;  // reduction length (routed, shared)
    bf16* h;    // gate/up: [S, N] routed, [T, Ns] shared
    bf16* hs;
    const int32_t* perm_rows;  // down: row -> slot
    const float* topk_w;       // down: slot -> routing weight
    int k;
    float* out;  // down mode 0: unweighted float32 rows [S + T, N]
    bf16* rows;  // down mode 1: routing-weighted bf16 rows [S + T, N]
    int64_t S;
    int mode;
};

struct Tables {
    int32_t off[kMaxExperts + 2];
    int32_t mtp[kMaxExperts + 1];
};

// Epilogue staging buffers (4 warps x kEpiStageBytes) after the ring, the
// barriers (256 B) and the tables, 128-byte aligned.
constexpr size_t kEpiStageOff = (kStages * kStageBytes + 256 + sizeof(Tables) + 127) / 128 * 128;

struct Sched {
    int E, nb_r, nb_s, mt_s;
    int gm_r, gm_s;  // row tiles per band (routed, shared)
    int64_t routed_tiles, total;
};

// Row tiles per band: as many 128-row A tiles of length K as fit in about
// 32 MB of L2 (at least 8).
__host__ __device__ __forceinline__ int band_tiles(int K, int rows_per_tile) {
    const int64_t per = (int64_t)rows_per_tile * (K > 0 ? K : 1) * 2;
    const int64_t g = (32ll << 20) / per;
    return g < 8 ? 8 : (g > (1 << 20) ? (1 << 20) : (int)g);
}

// Position `local` of a group's tile list (mt row tiles x nb column blocks,
// bands of gm row tiles) -> (column block, row tile).
__device__ __forceinline__ void band_order(int64_t local, int mt, int nb, int gm, int& nbi, int& mb) {
    const int64_t band = local / ((int64_t)gm * nb);
    const int64_t rem = local - band * gm * nb;
    const int first = (int)band * gm;
    const int width = min(gm, mt - first);
    nbi = (int)(rem / width);
    mb = first + (int)(rem % width);
}

struct TileInfo {
    bool shared;
    int g, e;      // group, expert coordinate of the weight maps
    int arow;      // first row in the A tensor (grouped rows, or token for shared)
    int64_t row0;  // first row in grouped-row numbering (shared: offsets[E] + token)
    int rows, n0, N, K;
};

__device__ __forceinline__ void decode_tile(int64_t t, const Tables& tb, const Sched& sc,
                                            const GemmArgs& a, int BN, TileInfo& ti) {
    if (t < sc.routed_tiles) {
        const int q = (int)(t / sc.nb_r);
        int lo = 0, hi = sc.E - 1;  // largest g with mtp[g] <= q
        while (lo < hi) {
            int mid = (lo + hi + 1) >> 1;
            if (tb.mtp[mid] <= q)
                lo = mid;
            else
                hi = mid - 1;
        }
        const int g = lo;
        const int mt = tb.mtp[g + 1] - tb.mtp[g];
        const int64_t local = t - (int64_t)tb.mtp[g] * sc.nb_r;
        int nbi, mb;
        band_order(local, mt, sc.nb_r, sc.gm_r, nbi, mb);
        ti.shared = false;
        ti.g = ti.e = g;
        ti.row0 = tb.off[g] + (int64_t)mb * kBM;
        ti.arow = (int)ti.row0;
        const int64_t left = tb.off[g + 1] - ti.row0;
        ti.rows = left < kBM ? (int)left : kBM;
        ti.n0 = nbi * BN;
        ti.N = a.N;
        ti.K = a.K;
    } else {
        const int64_t local = t - sc.routed_tiles;
        int nbi, mb;
        band_order(local, sc.mt_s, sc.nb_s, sc.gm_s, nbi, mb);
        ti.shared = true;
        ti.g = sc.E;
        ti.e = 0;
        ti.arow = mb * kBM;
        ti.row0 = tb.off[sc.E] + ti.arow;
        ti.rows = min(kBM, a.T - ti.arow);
        ti.n0 = nbi * BN;
        ti.N = a.Ns;
        ti.K = a.Ks;
    }
}

// Coalesced epilogue stores (down GEMM).  Each epilogue warp owns a 4 KB shared-memory
// buffer holding its 32 rows x 64 bf16 columns (128 B per row), with 16-byte
// chunk c of row r at r*128 + ((c ^ (r % 8)) * 16): the row-wise writes (lane
// = row) and the column-wise reads (8 lanes per row) are both free of bank
// conflicts.  The global stores then cover 4 rows x 128 B per instruction
// instead of 32 rows x 16 B.
constexpr int kEpiStageBytes = 32 * 128;

__device__ __forceinline__ uint32_t stage_off(int r, int c) { return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4)); }

__device__ __forceinline__ void st_shared_v4(uint32_t addr, const uint4& v) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr)
                 : "memory");
    return v;
}

// The warp's staged 32 x 64 chunk -> global: row i of the warp goes to
// row_ptr(i) (nullptr: row not stored), columns col0 .. col0 + 63, of which
// only those < N are stored (N a multiple of 8).
template <typename RowPtr>
__device__ __forceinline__ void flush_stage(uint32_t stage, int lane, int col0, int N, RowPtr row_ptr) {
    __syncwarp();
    const int c = lane & 7;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int rr = i * 4 + (lane >> 3);
        const uint4 v = ld_shared_v4(stage + stage_off(rr, c));
        bf16* dst = row_ptr(rr);
        const int n = col0 + c * 8;
        if (dst && n < N) *reinterpret_cast<uint4*>(dst + n) = v;
    }
    __syncwarp();
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// Drain one accumulator: this thread owns row r of the tile (TMEM lane
// quadrant q).  gate/up: h = silu(G) * U in bf16; down: mode 1 weighted bf16
// rows, mode 0 unweighted float32 rows.  tcgen05.ld is warp-collective, so
// every lane loads and only rows < ti.rows store.
template <bool kGateUp, int BN>
__device__ __forceinline__ void epilogue_tile(const TileInfo& ti, const GemmArgs& a, uint32_t acc_base, int q,
                                              int r, uint32_t stage) {
    const uint32_t tq = acc_base + ((uint32_t)(q * 32) << 16);
    const int lane = r & 31;
    const bool valid = r < ti.rows;
    if (kGateUp) {
        // h rows are stored directly: this kernel is bound by shared-memory
        // bandwidth, which staging would add to (measured slower)
        bf16* dst = ti.shared ? a.hs + (int64_t)(ti.arow + r) * a.Ns : a.h + (ti.row0 + r) * (int64_t)a.N;
#pragma unroll 1
        for (int j0 = 0; j0 < BN; j0 += 32) {
            float g[32], u[32];
            tmem_ld32(tq + j0, g);
            tmem_ld32(tq + BN + j0, u);
            if (valid) {
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const int n = ti.n0 + j0 + v * 8;
                    if (n < ti.N) {
                        uint4 pk;
                        pk.x = pack_bf16x2(silu_f32(g[v * 8 + 0]) * u[v * 8 + 0], silu_f32(g[v * 8 + 1]) * u[v * 8 + 1]);
                        pk.y = pack_bf16x2(silu_f32(g[v * 8 + 2]) * u[v * 8 + 2], silu_f32(g[v * 8 + 3]) * u[v * 8 + 3]);
                        pk.z = pack_bf16x2(silu_f32(g[v * 8 + 4]) * u[v * 8 + 4], silu_f32(g[v * 8 + 5]) * u[v * 8 + 5]);
                        pk.w = pack_bf16x2(silu_f32(g[v * 8 + 6]) * u[v * 8 + 6], silu_f32(g[v * 8 + 7]) * u[v * 8 + 7]);
                        *reinterpret_cast<uint4*>(dst + n) = pk;
                    }
                }
            }
        }
    } else {
        // output row: grouped row, or S + token for the shared expert
        const int64_t orow = ti.shared ? a.S + ti.arow + r : ti.row0 + r;
        float w = 1.f;
        if (valid && a.mode == 1 && !ti.shared) w = a.topk_w[a.perm_rows[ti.row0 + r]];
        if (a.mode == 1) {
            auto row_ptr = [&](int i) -> bf16* {
                const int rr = q * 32 + i;
                if (rr >= ti.rows) return nullptr;
                const int64_t orr = ti.shared ? a.S + ti.arow + rr : ti.row0 + rr;
                return a.rows + orr * (int64_t)ti.N;
            };
#pragma unroll 1
            for (int j0 = 0; j0 < BN; j0 += 64) {
                float v[64];
                tmem_ld64(tq + j0, v);  // 64 columns per TMEM round trip
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    uint4 pk;
                    pk.x = pack_bf16x2(w * v[i * 8 + 0], w * v[i * 8 + 1]);
                    pk.y = pack_bf16x2(w * v[i * 8 + 2], w * v[i * 8 + 3]);
                    pk.z = pack_bf16x2(w * v[i * 8 + 4], w * v[i * 8 + 5]);
                    pk.w = pack_bf16x2(w * v[i * 8 + 6], w * v[i * 8 + 7]);
                    st_shared_v4(stage + stage_off(lane, i), pk);
                }
                flush_stage(stage, lane, ti.n0 + j0, ti.N, row_ptr);
            }
        } else {
            // unweighted float32 rows (stage API): direct stores
#pragma unroll 1
            for (int j0 = 0; j0 < BN; j0 += 64) {
                float v[64];
                tmem_ld64(tq + j0, v);
                if (valid) {
                    float* dst = a.out + orow * (int64_t)ti.N;
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int n = ti.n0 + j0 + i * 4;
                        if (n < ti.N)
                            *reinterpret_cast<float4*>(dst + n) =
                                make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
                    }
                }
            }
        }
    }
}

template <bool kGateUp>
__global__ void __launch_bounds__(kThreads, 1) grouped_gemm_sm100_kernel(
    const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmAs,
    const __grid_constant__ CUtensorMap tmB0, const __grid_constant__ CUtensorMap tmB1,
    const __grid_constant__ CUtensorMap tmBs0, const __grid_constant__ CUtensorMap tmBs1,
    const __grid_constant__ CUtensorMap tmAsm, const GemmArgs a) {
    constexpr int BN = kGateUp ? kBRows / 2 : kBRows;  // output columns per tile
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
    uint64_t* empty = full + kStages;
    uint64_t* tfull = empty + kStages;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;  // MMA completion before TMEM is freed
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    Tables* tb = reinterpret_cast<Tables*>(smem + kStages * kStageBytes + 256);
    const uint32_t epi_stage = smem_u32(smem + kEpiStageOff) + (uint32_t)(((threadIdx.x / 32) & 3) * kEpiStageBytes);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    for (int i = threadIdx.x; i < a.E + 2; i += kThreads) tb->off[i] = a.offsets[i];
    for (int i = threadIdx.x; i < a.E + 1; i += kThreads) tb->mtp[i] = a.mtile_prefix[i];
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&tfull[i], 1);
            mbar_init(&tempty[i], kEpiThreads);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_map(&tmA);
        tma_prefetch_map(&tmB0);
        if (kGateUp) tma_prefetch_map(&tmB1);
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    Sched sc;
    sc.E = a.E;
    sc.nb_r = (a.N + BN - 1) / BN;
    sc.nb_s = a.has_shared ? (a.Ns + BN - 1) / BN : 0;
    sc.mt_s = a.has_shared ? (a.T + kBM - 1) / kBM : 0;
    sc.gm_r = band_tiles(a.K, kBM);
    sc.gm_s = band_tiles(a.Ks, kBM);
    sc.routed_tiles = (int64_t)tb->mtp[a.E] * sc.nb_r;
    sc.total = sc.routed_tiles + (int64_t)sc.mt_s * sc.nb_s;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t it = 0;
            for (int64_t t = blockIdx.x; t < sc.total && !*abort_flag; t += gridDim.x) {
                TileInfo ti;
                decode_tile(t, *tb, sc, a, BN, ti);
                // a group's last rows: a tile of at most kSmallRows rows loads
                // only those (the MMA still covers 128 rows; the accumulator
                // rows past ti.rows are never stored)
                const bool small = !ti.shared && ti.rows <= kSmallRows;
                const CUtensorMap* mA = ti.shared ? &tmAs : (small ? &tmAsm : &tmA);
                const uint32_t stage_tx = small ? kStageBytes - kABytes + kSmallABytes : kStageBytes;
                const CUtensorMap* mB0 = ti.shared ? &tmBs0 : &tmB0;
                const CUtensorMap* mB1 = ti.shared ? &tmBs1 : &tmB1;
                const int nkb = (ti.K + kBK - 1) / kBK;
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const int s = it % kStages;
                    const uint32_t ph = (it / kStages) & 1;
                    if (!wait_or_abort(&empty[s], ph ^ 1, abort_flag, a.flags)) break;
                    uint8_t* sa = smem + s * kStageBytes;
                    uint8_t* sb = sa + kABytes;
                    mbar_arrive_expect_tx(&full[s], stage_tx);
                    // every map is rank 3 (activations have depth 1): the load's
                    // dimensionality must match the map's rank
                    tma_load_3d(sa, mA, &full[s], kb * kBK, ti.arow, 0);
                    if (kGateUp) {
                        tma_load_3d(sb, mB0, &full[s], kb * kBK, ti.n0, ti.e);
                        tma_load_3d(sb + kBBytes / 2, mB1, &full[s], kb * kBK, ti.n0, ti.e);
                    } else {
                        tma_load_3d(sb, mB0, &full[s], kb * kBK, ti.n0, ti.e);
                    }
                }
            }
            // Never leave with copies in flight: wait (bounded) for the last
            // stages issued.  In a normal run these phases completed already.
            for (uint32_t j = (it > (uint32_t)kStages ? it - kStages : 0); j < it; ++j)
                for (uint32_t i = 0; i < kWaitLimit && !mbar_try_wait(&full[j % kStages], (j / kStages) & 1); ++i) {
                }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            uint32_t it = 0, tc = 0;
            for (int64_t t = blockIdx.x; t < sc.total && !*abort_flag; t += gridDim.x, ++tc) {
                TileInfo ti;
                decode_tile(t, *tb, sc, a, BN, ti);
                const int nkb = (ti.K + kBK - 1) / kBK;
                const uint32_t acc = tc & 1, aph = (tc >> 1) & 1;
                if (!wait_or_abort(&tempty[acc], aph ^ 1, abort_flag, a.flags)) break;
                tc_fence_after();
                const uint32_t d = tmem_base + acc * kAccCols;
                bool ok = true;
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const int s = it % kStages;
                    const uint32_t ph = (it / kStages) & 1;
                    if (!wait_or_abort(&full[s], ph, abort_flag, a.flags)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(smem + s * kStageBytes);
                    const uint32_t b0 = a0 + kABytes;
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)
                        mma_bf16(d, desc_kmajor_sw128(a0 + kk * 32), desc_kmajor_sw128(b0 + kk * 32), kIdesc,
                                 (kb | kk) != 0);
                    mma_commit(&empty[s]);  // frees the stage once these MMAs finish
                }
                if (!ok) break;
                mma_commit(&tfull[acc]);  // accumulator ready for the epilogue
            }
            // every MMA issued has finished before TMEM can be freed
            mma_commit(drain);
            for (uint32_t i = 0; i < kWaitLimit && !mbar_try_wait(drain, 0); ++i) {
            }
        }
    } else {
        // ------------------------------------------------ epilogue warps 2..5
        const int q = warp & 3;  // TMEM lane quadrant this warp may access
        const int r = q * 32 + lane;
        uint32_t tc = 0;
        for (int64_t t = blockIdx.x; t < sc.total; t += gridDim.x, ++tc) {
            TileInfo ti;
            decode_tile(t, *tb, sc, a, BN, ti);
            const uint32_t acc = tc & 1, aph = (tc >> 1) & 1;
            if (!wait_or_abort(&tfull[acc], aph, abort_flag, a.flags)) break;
            tc_fence_after();
            epilogue_tile<kGateUp, BN>(ti, a, tmem_base + acc * kAccCols, q, r, epi_stage);
            tc_fence_before();
            mbar_arrive(&tempty[acc]);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

// ----------------------------------------------------------- CTA pairs
// The same grouped GEMM on CTA pairs (clusters of 2): a tile is 256 rows x
// BN of one group.  Each CTA stages its own 128 rows of A and 128 rows of B
// (gate/up: CTA0 the gate rows, CTA1 the matching up rows; down: the two
// halves of the 256 output columns), so a stage is 32 KB per CTA instead of
// 48 KB and the shared-memory traffic per CTA drops by a third.  The leader
// (rank 0) issues M = 256, N = 256 MMAs that read both CTAs' stages and write
// each CTA's 128-row half of the accumulator into that CTA's TMEM, so both
// CTAs drain their own half with the single-CTA epilogue.
constexpr int kPStages = 6;
constexpr int kPABytes = kBM * kBK * 2;         // 16 KB: this CTA's 128 rows of A
constexpr int kPBBytes = (kBRows / 2) * kBK * 2;  // 16 KB: this CTA's half of B
constexpr int kPStageBytes = kPABytes + kPBBytes;
constexpr uint32_t kPIdesc = idesc_bf16(2 * kBM, kBRows);

struct PairTables {
    int32_t off[kMaxExperts + 2];
    int32_t mpp[kMaxExperts + 1];  // prefix of 256-row pair tiles
};

constexpr size_t kPEpiStageOff = (kPStages * kPStageBytes + 256 + sizeof(PairTables) + 127) / 128 * 128;

// Pair tile t -> this CTA's (rank) half: rows row0 .. row0 + rows - 1 (rows may
// be <= 0 when the group ends inside the pair's first half).
__device__ __forceinline__ void decode_pair(int64_t t, const PairTables& tb, const Sched& sc, const GemmArgs& a,
                                            int BN, uint32_t rank, TileInfo& ti) {
    if (t < sc.routed_tiles) {
        const int q = (int)(t / sc.nb_r);
        int lo = 0, hi = sc.E - 1;  // largest g with mpp[g] <= q
        while (lo < hi) {
            int mid = (lo + hi + 1) >> 1;
            if (tb.mpp[mid] <= q)
                lo = mid;
            else
                hi = mid - 1;
        }
        const int g = lo;
        const int mt = tb.mpp[g + 1] - tb.mpp[g];
        const int64_t local = t - (int64_t)tb.mpp[g] * sc.nb_r;
        int nbi, mb;
        band_order(local, mt, sc.nb_r, sc.gm_r, nbi, mb);
        ti.shared = false;
        ti.g = ti.e = g;
        ti.row0 = tb.off[g] + (int64_t)mb * (2 * kBM) + rank * kBM;
        ti.arow = (int)ti.row0;
        const int64_t left = tb.off[g + 1] - ti.row0;
        ti.rows = left < kBM ? (int)left : kBM;
        ti.n0 = nbi * BN;
        ti.N = a.N;
        ti.K = a.K;
    } else {
        const int64_t local = t - sc.routed_tiles;
        int nbi, mb;
        band_order(local, sc.mt_s, sc.nb_s, sc.gm_s, nbi, mb);
        ti.shared = true;
        ti.g = sc.E;
        ti.e = 0;
        ti.arow = mb * (2 * kBM) + (int)rank * kBM;
        ti.row0 = tb.off[sc.E] + ti.arow;
        ti.rows = min(kBM, a.T - ti.arow);
        ti.n0 = nbi * BN;
        ti.N = a.Ns;
        ti.K = a.Ks;
    }
}

template <bool kGateUp>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1) grouped_gemm_pair_kernel(
    const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmAs,
    const __grid_constant__ CUtensorMap tmB0, const __grid_constant__ CUtensorMap tmB1,
    const __grid_constant__ CUtensorMap tmBs0, const __grid_constant__ CUtensorMap tmBs1,
    const GemmArgs a) {
    constexpr int BN = kGateUp ? kBRows / 2 : kBRows;  // output columns per tile
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kPStages * kPStageBytes);  // used in the leader
    uint64_t* empty = full + kPStages;
    uint64_t* tfull = empty + kPStages;
    uint64_t* tempty = tfull + 2;  // used in the leader: 4 epilogue warps x 2 CTAs
    uint64_t* drain = tempty + 2;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    PairTables* tb = reinterpret_cast<PairTables*>(smem + kPStages * kPStageBytes + 256);
    const uint32_t epi_stage = smem_u32(smem + kPEpiStageOff) + (uint32_t)(((threadIdx.x / 32) & 3) * kEpiStageBytes);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const uint32_t rank = cluster_ctarank();
    const bool leader = (rank == 0);
    for (int i = threadIdx.x; i < a.E + 2; i += kThreads) tb->off[i] = a.offsets[i];
    for (int i = threadIdx.x; i < a.E + 1; i += kThreads) tb->mpp[i] = a.mtile_prefix[i];
    if (threadIdx.x == 0) {
        for (int s = 0; s < kPStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&tfull[i], 1);
            mbar_init(&tempty[i], 2 * (kEpiThreads / 32));
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_holder, kTmemCols);
        tmem_relinquish_pair();
    }
    // both CTAs' barriers are initialised before any cross-CTA signal
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    Sched sc;
    sc.E = a.E;
    sc.nb_r = (a.N + BN - 1) / BN;
    sc.nb_s = a.has_shared ? (a.Ns + BN - 1) / BN : 0;
    sc.mt_s = a.has_shared ? (a.T + 2 * kBM - 1) / (2 * kBM) : 0;
    sc.gm_r = band_tiles(a.K, 2 * kBM);
    sc.gm_s = band_tiles(a.Ks, 2 * kBM);
    sc.routed_tiles = (int64_t)tb->mpp[a.E] * sc.nb_r;
    sc.total = sc.routed_tiles + (int64_t)sc.mt_s * sc.nb_s;
    const int64_t pair = blockIdx.x / 2, npairs = gridDim.x / 2;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer (both CTAs)
        if (lane == 0) {
            uint32_t it = 0;
            for (int64_t t = pair; t < sc.total && !*abort_flag; t += npairs) {
                TileInfo ti;
                decode_pair(t, *tb, sc, a, BN, rank, ti);
                const CUtensorMap* mA = ti.shared ? &tmAs : &tmA;
                const CUtensorMap* mB = kGateUp ? (ti.shared ? (rank ? &tmBs1 : &tmBs0) : (rank ? &tmB1 : &tmB0))
                                                : (ti.shared ? &tmBs0 : &tmB0);
                const int bcol = kGateUp ? ti.n0 : ti.n0 + (int)rank * (kBRows / 2);
                const int nkb = (ti.K + kBK - 1) / kBK;
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const int s = it % kPStages;
                    const uint32_t ph = (it / kPStages) & 1;
                    if (!wait_or_abort(&empty[s], ph ^ 1, abort_flag, a.flags)) break;
                    uint8_t* sa = smem + s * kPStageBytes;
                    if (leader) mbar_arrive_expect_tx(&full[s], 2 * kPStageBytes);
                    tma_load_3d_pair(sa, mA, &full[s], kb * kBK, ti.arow, 0);
                    tma_load_3d_pair(sa + kPABytes, mB, &full[s], kb * kBK, bcol, ti.e);
                }
            }
            // copies of both CTAs complete on the leader's barriers
            if (leader)
                for (uint32_t j = (it > (uint32_t)kPStages ? it - kPStages : 0); j < it; ++j)
                    drain_wait(&full[j % kPStages], (j / kPStages) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (leader)
        if (lane == 0 && leader) {
            uint32_t it = 0, tc = 0;
            for (int64_t t = pair; t < sc.total && !*abort_flag; t += npairs, ++tc) {
                TileInfo ti;
                decode_pair(t, *tb, sc, a, BN, rank, ti);
                const int nkb = (ti.K + kBK - 1) / kBK;
                const uint32_t acc = tc & 1, aph = (tc >> 1) & 1;
                if (!wait_or_abort(&tempty[acc], aph ^ 1, abort_flag, a.flags)) break;
                tc_fence_after();
                const uint32_t d = tmem_base + acc * kAccCols;
                bool ok = true;
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const int s = it % kPStages;
                    const uint32_t ph = (it / kPStages) & 1;
                    if (!wait_or_abort(&full[s], ph, abort_flag, a.flags)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(smem + s * kPStageBytes);
                    const uint32_t b0 = a0 + kPABytes;
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)
                        mma_bf16_pair(d, desc_kmajor_sw128(a0 + kk * 32), desc_kmajor_sw128(b0 + kk * 32), kPIdesc,
                                      (kb | kk) != 0);
                    mma_commit_pair(&empty[s], 0x3);  // frees the stage in both CTAs
                }
                if (!ok) break;
                mma_commit_pair(&tfull[acc], 0x3);  // both halves of the accumulator ready
            }
            mma_commit_pair(drain, 0x1);
            drain_wait(drain, 0);
        }
    } else {
        // ------------------------------------------------ epilogue warps 2..5 (both CTAs)
        const int q = warp & 3;
        const int r = q * 32 + lane;
        uint32_t tc = 0;
        for (int64_t t = pair; t < sc.total; t += npairs, ++tc) {
            TileInfo ti;
            decode_pair(t, *tb, sc, a, BN, rank, ti);
            const uint32_t acc = tc & 1, aph = (tc >> 1) & 1;
            if (!wait_or_abort(&tfull[acc], aph, abort_flag, a.flags)) break;
            tc_fence_after();
            epilogue_tile<kGateUp, BN>(ti, a, tmem_base + acc * kAccCols, q, r, epi_stage);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(&tempty[acc], 0);  // the leader's barrier
        }
    }

    if (*abort_flag && !leader) {
        // aborted: this CTA's copies complete on the leader's barriers; give
        // any still in flight time to land before shared memory is released
        for (int i = 0; i < 2000; ++i) __nanosleep(100);
    }
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    if (warp == 1) tmem_dealloc_pair(tmem_base, kTmemCols);
}

// ---------------------------------------------------- MXFP4 weights (B)
// The same grouped GEMMs with the expert weights in MXFP4 (E2M1 codes with
// one E8M0 scale per 32 along K).  The codes of a k-step (256 rows x 64 K =
// 8 KB, a quarter of the bf16 bytes) arrive by TMA into a ring of 8 slots;
// eight converter warps turn them into the bf16 B tile in shared memory, in
// the 128-byte-swizzled K-major layout the MMA reads (chunk c of row r at
// r*128 + ((c ^ r%8) * 16)), and the MMA runs as on bf16 weights.  Three
// rings, each as deep as it needs to be: A tiles (3 x 16 KB, TMA), converted
// B tiles (2 x 32 KB) and codes (2 x 32 KB, four k-steps of 256 rows x 32
// bytes per slot, so that a TMA row is a whole 128-byte line and the TMA
// unit is not held up by narrow rows ahead of the A copies): 64 KB of weight
// reads in flight per SM; a producer warp of its own refills a codes slot as
// soon as the converters have read it.  The conversion is integer
// work plus one bf16 multiply per two elements (see mx_chunk_to_bf16): the
// float conversion instructions run at a fraction of the ALU rate.  Every
// converted value e * 2^(s-127) is exact in bf16 (normal or subnormal;
// above bf16's range it becomes +-inf), so the products are those of the
// dequantized weights.  A tile's scale bytes (its
// rows x K/32, contiguous per 128 rows) are copied into shared memory when
// the tile starts; K <= 32 * kMxMaxScales.
constexpr int kMxAStages = 3;
constexpr int kMxBStages = 2;
constexpr int kMxGroupSteps = 4;                                // k-steps per codes copy (128-byte rows)
constexpr int kMxCStages = 2;
constexpr int kMxCodeBytes = kBRows * kBK / 2 * kMxGroupSteps;  // 32 KB of codes per slot
constexpr int kMxMaxScales = 96;                 // scale bytes per row a tile holds: K <= 3072
constexpr int kMxConvWarps = 8;
constexpr int kMxConvThreads = kMxConvWarps * 32;
constexpr int kMxCodeWarp = (kThreads + kMxConvThreads) / 32;  // the codes producer
constexpr int kMxThreads = kThreads + kMxConvThreads + 32;
constexpr size_t kMxBOff = (size_t)kMxAStages * kABytes;
constexpr size_t kMxCOff = kMxBOff + (size_t)kMxBStages * kBBytes;
constexpr size_t kMxBarOff = kMxCOff + (size_t)kMxCStages * kMxCodeBytes;
constexpr size_t kMxTablesOff = kMxBarOff + 512;
constexpr size_t kMxScaleOff = (kMxTablesOff + sizeof(Tables) + 127) / 128 * 128;
constexpr size_t kMxEpiStageOff = (kMxScaleOff + (size_t)kBRows * kMxMaxScales + 127) / 128 * 128;
constexpr size_t kMxSmemBytes = kMxEpiStageOff + 4 * kEpiStageBytes + 1024;
static_assert(kMxSmemBytes <= 227 * 1024, "MXFP4 GEMM shared memory");

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Named barrier of n threads that also returns whether every one of them
// passed v = true.
__device__ __forceinline__ bool named_and(int id, int n, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "barrier.cta.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

__device__ __forceinline__ uint32_t mul_bf16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Eight E2M1 codes (byte q: element 2q in the low nibble, 2q+1 in the high)
// with E8M0 scale byte s -> eight bf16 values e * 2^(s-127) in o[0..3].
// A nibble's sign bit moved to bit 15 and its three exponent/mantissa bits
// to bits 8..6 form the bf16 of e * 2^-126 exactly (exponent field 0 makes
// the codes 0 and 0.5 the subnormals 0 and 2^-127).  With one nibble per
// 16-bit lane, t * 0x1040 = (t << 12) | (t << 6) (the copies do not
// overlap), and the mask keeps bits 15 and 8..6 of each lane.  One rounding
// multiply by 2^(s-1) (two, by 2^126 then 2^(s-127), when 2^(s-1) exceeds
// bf16's range) then gives e * 2^(s-127), exact wherever bf16 holds it.
__device__ __forceinline__ void mx_chunk_to_bf16(uint32_t w, uint32_t s, uint32_t (&o)[4]) {
    const uint32_t lo = w & 0x0f0f0f0fu, hi = (w >> 4) & 0x0f0f0f0fu;
    uint32_t t[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        // byte q of lo and of hi into the two lanes, zeros (the sign of a
        // nibble byte) above them
        const uint32_t sel = (uint32_t)q | ((8u | q) << 4) | ((4u + q) << 8) | ((12u + q) << 12);
        t[q] = (prmt(lo, hi, sel) * 0x1040u) & 0x81c081c0u;
    }
    if (s <= 128u) {
        const uint32_t sc = (s + 126u) * 0x00800080u;  // 2^(s-1) in both lanes
#pragma unroll
        for (int q = 0; q < 4; ++q) o[q] = mul_bf16x2(t[q], sc);
    } else {
        const uint32_t sc = s == 255u ? 0x7fc07fc0u : s * 0x00800080u;  // NaN, or 2^(s-127)
#pragma unroll
        for (int q = 0; q < 4; ++q) o[q] = mul_bf16x2(mul_bf16x2(t[q], 0x7e807e80u), sc);  // x 2^126 first
    }
}

struct MxArgs {
    const uint8_t* sc0;  // scales of the B rows: gate / down [E, N, K/32]
    const uint8_t* sc1;  // up [E, N, K/32] (gate/up only)
    int keep_a;          // the A rows fit in L2: read them with evict_last, the codes with evict_first
};

// The k-steps of this CTA's tiles in order: (tile, k-step) of step `it`.
struct StepCursor {
    int64_t t;
    int kb, nkb;
    TileInfo ti;
};

__device__ __forceinline__ bool cursor_start(StepCursor& c, const Tables& tb, const Sched& sc, const GemmArgs& a,
                                             int BN) {
    c.t = blockIdx.x;
    c.kb = 0;
    if (c.t >= sc.total) return false;
    decode_tile(c.t, tb, sc, a, BN, c.ti);
    c.nkb = (c.ti.K + kBK - 1) / kBK;
    return true;
}

__device__ __forceinline__ bool cursor_next(StepCursor& c, const Tables& tb, const Sched& sc, const GemmArgs& a,
                                            int BN, int stride = 1) {
    c.kb += stride;
    if (c.kb < c.nkb) return true;
    c.t += gridDim.x;
    c.kb = 0;
    if (c.t >= sc.total) return false;
    decode_tile(c.t, tb, sc, a, BN, c.ti);
    c.nkb = (c.ti.K + kBK - 1) / kBK;
    return true;
}

template <bool kGateUp>
__global__ void __launch_bounds__(kMxThreads, 1) grouped_gemm_mx_kernel(
    const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmAsm,
    const __grid_constant__ CUtensorMap tmC0, const __grid_constant__ CUtensorMap tmC1, const GemmArgs a,
    const MxArgs mxa) {
    constexpr int BN = kGateUp ? kBRows / 2 : kBRows;
    extern __shared__ uint8_t smem_raw[];
    // aligned by pointer arithmetic, so that accesses through it stay shared-memory accesses
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t* afull = reinterpret_cast<uint64_t*>(smem + kMxBarOff);
    uint64_t* aempty = afull + kMxAStages;
    uint64_t* bfull = aempty + kMxAStages;   // converted B tile ready (converters)
    uint64_t* bempty = bfull + kMxBStages;   // B tile consumed (MMA)
    uint64_t* cfull = bempty + kMxBStages;   // codes landed (TMA)
    uint64_t* cempty = cfull + kMxCStages;   // codes slot read (converters)
    uint64_t* tfull = cempty + kMxCStages;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    Tables* tb = reinterpret_cast<Tables*>(smem + kMxTablesOff);
    uint8_t* sscale = smem + kMxScaleOff;
    const uint32_t epi_stage = smem_u32(smem + kMxEpiStageOff) + (uint32_t)(((threadIdx.x / 32) & 3) * kEpiStageBytes);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    for (int i = threadIdx.x; i < a.E + 2; i += kMxThreads) tb->off[i] = a.offsets[i];
    for (int i = threadIdx.x; i < a.E + 1; i += kMxThreads) tb->mtp[i] = a.mtile_prefix[i];
    if (threadIdx.x == 0) {
        for (int s = 0; s < kMxAStages; ++s) {
            mbar_init(&afull[s], 1);
            mbar_init(&aempty[s], 1);
        }
        for (int s = 0; s < kMxBStages; ++s) {
            mbar_init(&bfull[s], kMxConvWarps);  // one arrival per converter warp
            mbar_init(&bempty[s], 1);
        }
        for (int s = 0; s < kMxCStages; ++s) {
            mbar_init(&cfull[s], 1);
            mbar_init(&cempty[s], kMxConvWarps);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&tfull[i], 1);
            mbar_init(&tempty[i], kEpiThreads);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) tma_prefetch_map(&tmA);
    if (warp == kMxCodeWarp && lane == 0) {
        tma_prefetch_map(&tmC0);
        if (kGateUp) tma_prefetch_map(&tmC1);
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    Sched sc;
    sc.E = a.E;
    sc.nb_r = (a.N + BN - 1) / BN;
    sc.nb_s = 0;
    sc.mt_s = 0;
    sc.gm_r = band_tiles(a.K, kBM);
    sc.gm_s = 1;
    sc.routed_tiles = (int64_t)tb->mtp[a.E] * sc.nb_r;
    sc.total = sc.routed_tiles;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer of A
        if (lane == 0) {
            // A tiles are read once per column block: when they fit in L2
            // they are kept there ahead of the codes streaming past
            const uint64_t pol = mxa.keep_a ? l2_policy_evict_last() : 0;
            uint32_t it = 0;
            for (int64_t t = blockIdx.x; t < sc.total && !*abort_flag; t += gridDim.x) {
                TileInfo ti;
                decode_tile(t, *tb, sc, a, BN, ti);
                const bool small = ti.rows <= kSmallRows;
                const CUtensorMap* mA = small ? &tmAsm : &tmA;
                const uint32_t a_tx = small ? kSmallABytes : kABytes;
                const int nkb = (ti.K + kBK - 1) / kBK;
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const int s = it % kMxAStages;
                    const uint32_t ph = (it / kMxAStages) & 1;
                    if (!wait_or_abort(&aempty[s], ph ^ 1, abort_flag, a.flags)) break;
                    mbar_arrive_expect_tx(&afull[s], a_tx);
                    if (mxa.keep_a)
                        tma_load_3d_hint(smem + s * kABytes, mA, &afull[s], kb * kBK, ti.arow, 0, pol);
                    else
                        tma_load_3d(smem + s * kABytes, mA, &afull[s], kb * kBK, ti.arow, 0);
                }
            }
            // never leave with copies in flight (bounded waits)
            for (uint32_t j = (it > (uint32_t)kMxAStages ? it - kMxAStages : 0); j < it; ++j)
                for (uint32_t i = 0; i < kWaitLimit && !mbar_try_wait(&afull[j % kMxAStages], (j / kMxAStages) & 1);
                     ++i) {
                }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            uint32_t it = 0, tc = 0;
            for (int64_t t = blockIdx.x; t < sc.total && !*abort_flag; t += gridDim.x, ++tc) {
                TileInfo ti;
                decode_tile(t, *tb, sc, a, BN, ti);
                const int nkb = (ti.K + kBK - 1) / kBK;
                const uint32_t acc = tc & 1, aph = (tc >> 1) & 1;
                if (!wait_or_abort(&tempty[acc], aph ^ 1, abort_flag, a.flags)) break;
                tc_fence_after();
                const uint32_t d = tmem_base + acc * kAccCols;
                bool ok = true;
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const int sa = it % kMxAStages, sb = it % kMxBStages;
                    if (!wait_or_abort(&afull[sa], (it / kMxAStages) & 1, abort_flag, a.flags) ||
                        !wait_or_abort(&bfull[sb], (it / kMxBStages) & 1, abort_flag, a.flags)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(smem + sa * kABytes);
                    const uint32_t b0 = smem_u32(smem + kMxBOff + sb * kBBytes);
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)
                        mma_bf16(d, desc_kmajor_sw128(a0 + kk * 32), desc_kmajor_sw128(b0 + kk * 32), kIdesc,
                                 (kb | kk) != 0);
                    mma_commit(&aempty[sa]);
                    mma_commit(&bempty[sb]);
                }
                if (!ok) break;
                mma_commit(&tfull[acc]);
            }
            mma_commit(drain);
            for (uint32_t i = 0; i < kWaitLimit && !mbar_try_wait(drain, 0); ++i) {
            }
        }
    } else if (warp < kThreads / 32) {
        // ------------------------------------------------ epilogue warps 2..5
        const int q = warp & 3;
        const int r = q * 32 + lane;
        uint32_t tc = 0;
        for (int64_t t = blockIdx.x; t < sc.total; t += gridDim.x, ++tc) {
            TileInfo ti;
            decode_tile(t, *tb, sc, a, BN, ti);
            const uint32_t acc = tc & 1, aph = (tc >> 1) & 1;
            // a whole tile's wait: sleep in try_wait instead of taking issue
            // slots from the converters on the same schedulers
            if (!wait_sleep_or_abort(&tfull[acc], aph, abort_flag, a.flags)) break;
            tc_fence_after();
            epilogue_tile<kGateUp, BN>(ti, a, tmem_base + acc * kAccCols, q, r, epi_stage);
            tc_fence_before();
            mbar_arrive(&tempty[acc]);
        }
    } else if (warp == kMxCodeWarp) {
        // ------------------------------------------------ TMA producer of the codes
        if (lane == 0) {
            const uint64_t pol = l2_policy_evict_first();
            StepCursor c{};
            uint32_t it = 0;
            // one copy per group of kMxGroupSteps k-steps of a tile (it counts groups)
            for (bool more = cursor_start(c, *tb, sc, a, BN); more && !*abort_flag;
                 more = cursor_next(c, *tb, sc, a, BN, kMxGroupSteps), ++it) {
                const int s = it % kMxCStages;
                if (!wait_or_abort(&cempty[s], ((it / kMxCStages) & 1) ^ 1, abort_flag, a.flags)) break;
                uint8_t* dst = smem + kMxCOff + s * kMxCodeBytes;
                const int x = c.kb * (kBK / 2);  // byte column of the group's first k-step
                mbar_arrive_expect_tx(&cfull[s], kMxCodeBytes);
                if (mxa.keep_a) {  // each tile's codes are read once
                    tma_load_3d_hint(dst, &tmC0, &cfull[s], x, c.ti.n0, c.ti.e, pol);
                    if (kGateUp) tma_load_3d_hint(dst + kMxCodeBytes / 2, &tmC1, &cfull[s], x, c.ti.n0, c.ti.e, pol);
                } else {
                    tma_load_3d(dst, &tmC0, &cfull[s], x, c.ti.n0, c.ti.e);
                    if (kGateUp) tma_load_3d(dst + kMxCodeBytes / 2, &tmC1, &cfull[s], x, c.ti.n0, c.ti.e);
                }
            }
            // never leave with copies in flight (bounded waits)
            for (uint32_t j = (it > (uint32_t)kMxCStages ? it - kMxCStages : 0); j < it; ++j)
                for (uint32_t i = 0; i < kWaitLimit && !mbar_try_wait(&cfull[j % kMxCStages], (j / kMxCStages) & 1);
                     ++i) {
                }
        }
    } else {
        // ------------------------------------------------ converter warps 6..13
        // Thread ct converts chunk j = ct % 8 (8 elements) of rows r0 + 32 i, a
        // warp's four lane groups taking rows two apart (r0 % 8 = 0,2,4,6 or
        // 1,3,5,7), so that the swizzled code chunks they read fall in
        // different banks; a warp writes 4 rows x 128 bytes.
        const int ct = threadIdx.x - kThreads;
        const int cw_ = ct >> 5, j = ct & 7;
        const int r0 = (cw_ >> 1) * 8 + (cw_ & 1) + 2 * ((ct >> 3) & 3);
        const int nsb = a.K / 32;  // scale bytes per row
        // Each warp reports a step done with its own arrivals on bfull and
        // cempty, so the warps meet only when a tile starts (its scale
        // bytes).  After an abort every wait returns at once: the warps walk
        // the remaining steps without work and still meet at the same
        // barriers.
        uint32_t it = 0, gi = 0;  // k-steps, codes groups
        for (int64_t t = blockIdx.x; t < sc.total; t += gridDim.x) {
            TileInfo ti;
            decode_tile(t, *tb, sc, a, BN, ti);
            // the tile's scale bytes -> sscale[row][nsb] (rows past N left as
            // they are: their codes are zeros and their columns are not stored)
            named_and(2, kMxConvThreads, true);  // every converter is done with the previous tile's
            {
                // every load of the copy issued before its stores (one round
                // trip per tile, not one per word)
                constexpr int kHalf = kGateUp ? kBRows / 2 : kBRows;
                constexpr int kWords = kHalf * kMxMaxScales / 4 / kMxConvThreads;  // per thread and source
                const int bytes = min(kHalf, ti.N - ti.n0) * nsb;  // 32 | N - n0, so 4 | bytes
#pragma unroll
                for (int src = 0; src < (kGateUp ? 2 : 1); ++src) {
                    const uint8_t* g = (src ? mxa.sc1 : mxa.sc0) + ((int64_t)ti.e * ti.N + ti.n0) * nsb;
                    uint8_t* d = sscale + src * kHalf * nsb;
                    if (((uintptr_t)g & 3) == 0) {  // 32 | N and 128 | n0 keep g word-aligned if the array is
                        uint32_t v[kWords];
#pragma unroll
                        for (int u = 0; u < kWords; ++u) {
                            const int w = ct + u * kMxConvThreads;
                            v[u] = w < bytes / 4 ? __ldg(reinterpret_cast<const uint32_t*>(g) + w) : 0u;
                        }
#pragma unroll
                        for (int u = 0; u < kWords; ++u) {
                            const int w = ct + u * kMxConvThreads;
                            if (w < bytes / 4) reinterpret_cast<uint32_t*>(d)[w] = v[u];
                        }
                    } else {
                        for (int b = ct; b < bytes; b += kMxConvThreads) d[b] = __ldg(g + b);
                    }
                }
            }
            named_and(2, kMxConvThreads, true);
            const int nkb = (ti.K + kBK - 1) / kBK;
            for (int kb = 0; kb < nkb; ++kb, ++it) {
                const int cs = gi % kMxCStages, bs = it % kMxBStages, pos = kb % kMxGroupSteps;
                const bool got = (pos != 0 || wait_or_abort(&cfull[cs], (gi / kMxCStages) & 1, abort_flag, a.flags)) &&
                                 wait_or_abort(&bempty[bs], ((it / kMxBStages) & 1) ^ 1, abort_flag, a.flags);
                if (__all_sync(0xffffffffu, got)) {
                    // plain shared-memory accesses (the waits and barriers around
                    // them are compiler barriers): the 8 chunks' loads issue
                    // together instead of one chunk's chain after another
                    // word j of this k-step in row r (128-byte rows, the TMA's
                    // 128-byte swizzle: 16-byte chunk c at c ^ (r % 8); r % 8
                    // = r0 % 8 for every row of the thread)
                    const int byte = pos * (kBK / 2) + j * 4;
                    const uint32_t* cw = reinterpret_cast<const uint32_t*>(
                        smem + kMxCOff + cs * kMxCodeBytes + r0 * 128 + ((((byte >> 4) ^ (r0 & 7)) << 4) | (byte & 15)));
                    const int bi = kb * 2 + (j >> 2);  // this chunk's 32-element block along K
                    const uint8_t* ss = sscale + r0 * nsb + bi;
                    uint8_t* bst = smem + kMxBOff + bs * kBBytes;
                    uint32_t w[kBRows / 32], sv[kBRows / 32];
#pragma unroll
                    for (int i = 0; i < kBRows / 32; ++i) {
                        w[i] = cw[i * 32 * 32];  // 32 rows of 128 bytes further
                        sv[i] = bi < nsb ? ss[i * 32 * nsb] : 0u;  // a block past K: zero codes (TMA fill)
                    }
#pragma unroll
                    for (int i = 0; i < kBRows / 32; ++i) {
                        uint32_t o[4];
                        mx_chunk_to_bf16(w[i], sv[i], o);
                        *reinterpret_cast<uint4*>(bst + stage_off(r0 + 32 * i, j)) = make_uint4(o[0], o[1], o[2], o[3]);
                    }
                    fence_proxy_async_smem();  // these generic-proxy writes, before the MMA's async reads
                }
                __syncwarp();
                const bool group_end = pos == kMxGroupSteps - 1 || kb == nkb - 1;
                if (lane == 0) {  // this warp's rows of the step are written (and the group's codes read)
                    mbar_arrive(&bfull[bs]);
                    if (group_end) mbar_arrive(&cempty[cs]);
                }
                if (group_end) ++gi;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

// ------------------------------------------------------------------ host side
constexpr size_t kSmemBytes = kEpiStageOff + 4 * kEpiStageBytes + 1024;

template <bool kGateUp>
cudaError_t launch_grouped(const Plan& p, const CUtensorMap (&maps)[7], const GemmArgs& args,
                           cudaStream_t st) {
    constexpr int BN = kGateUp ? kBRows / 2 : kBRows;
    cudaError_t e = ensure_smem_attr(grouped_gemm_sm100_kernel<kGateUp>, kSmemBytes);
    if (e != cudaSuccess) return e;
    const int64_t nb_r = (args.N + BN - 1) / BN;
    const int64_t nb_s = args.has_shared ? (args.Ns + BN - 1) / BN : 0;
    const int64_t ub = ((p.S + kBM - 1) / kBM + p.E) * nb_r + ((p.T + kBM - 1) / kBM) * nb_s;
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(device_sm_count(), ub));
    grouped_gemm_sm100_kernel<kGateUp><<<grid, kThreads, kSmemBytes, st>>>(maps[0], maps[1], maps[2], maps[3],
                                                                         maps[4], maps[5], maps[6], args);
    return cudaGetLastError();
}

constexpr size_t kPSmemBytes = kPEpiStageOff + 4 * kEpiStageBytes + 1024;

template <bool kGateUp>
cudaError_t launch_grouped_pair(const Plan& p, const CUtensorMap (&maps)[7], const GemmArgs& args,
                                cudaStream_t st) {
    constexpr int BN = kGateUp ? kBRows / 2 : kBRows;
    cudaError_t e = ensure_smem_attr(grouped_gemm_pair_kernel<kGateUp>, kPSmemBytes);
    if (e != cudaSuccess) return e;
    const int64_t nb_r = (args.N + BN - 1) / BN;
    const int64_t nb_s = args.has_shared ? (args.Ns + BN - 1) / BN : 0;
    const int64_t ub = ((p.S + 2 * kBM - 1) / (2 * kBM) + p.E) * nb_r + ((p.T + 2 * kBM - 1) / (2 * kBM)) * nb_s;
    const int64_t pairs = std::max<int64_t>(1, std::min<int64_t>(device_sm_count() / 2, ub));
    grouped_gemm_pair_kernel<kGateUp><<<(unsigned)(2 * pairs), kThreads, kPSmemBytes, st>>>(
        maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], args);
    return cudaGetLastError();
}

// CTA pairs where they measured faster on B200: the down GEMM with a short
// reduction (I <= 1024) and groups large enough (>= 512 kept rows per routed
// expert on average) that 256-row tiles waste little.  Elsewhere single CTAs
// were as fast or faster: in a pair each SM's tensor core still reads all of
// B (its half from its own shared memory, the other half from the peer's),
// so shared-memory traffic drops only by about a sixth.
bool use_pairs(const Plan& p) { return p.I <= 1024 && p.S >= 512 * p.E; }

template <bool kGateUp>
cudaError_t launch_grouped_mx(const Plan& p, const CUtensorMap (&maps)[4], const GemmArgs& args, const MxArgs& mx,
                              cudaStream_t st) {
    constexpr int BN = kGateUp ? kBRows / 2 : kBRows;
    cudaError_t e = ensure_smem_attr(grouped_gemm_mx_kernel<kGateUp>, kMxSmemBytes);
    if (e != cudaSuccess) return e;
    const int64_t nb_r = (args.N + BN - 1) / BN;
    const int64_t ub = ((p.S + kBM - 1) / kBM + p.E) * nb_r;
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(device_sm_count(), ub));
    grouped_gemm_mx_kernel<kGateUp><<<grid, kMxThreads, kMxSmemBytes, st>>>(maps[0], maps[1], maps[2], maps[3],
                                                                            args, mx);
    return cudaGetLastError();
}

GemmArgs base_args(const Plan& p) {
    GemmArgs a{};
    a.offsets = p.offsets;
    a.mtile_prefix = p.mtile_prefix;
    a.flags = p.flags;
    a.E = (int)p.E;
    a.T = (int)p.T;
    a.has_shared = p.Is > 0;
    a.k = (int)p.k;
    a.S = p.S;
    return a;
}

}  // namespace

cudaError_t launch_gateup_sm100(const Plan& p, const void* x, const void* w_gate, const void* w_up,
                                const void* ws_gate, const void* ws_up, cudaStream_t st) {
    if (p.T == 0) return cudaSuccess;
    bf16* h = (bf16*)p.h;
    bf16* hs = h + p.S * p.I;
    CUtensorMap m[7];
    bool ok = make_map_bf16(&m[0], p.xperm, p.H, p.S, 1, kBK, kBM) &&
              make_map_bf16(&m[6], p.xperm, p.H, p.S, 1, kBK, kSmallRows) &&
              make_map_bf16(&m[2], w_gate, p.H, p.I, p.E, kBK, kBRows / 2) &&
              make_map_bf16(&m[3], w_up, p.H, p.I, p.E, kBK, kBRows / 2);
    if (ok && p.Is > 0)
        ok = make_map_bf16(&m[1], x, p.H, p.T, 1, kBK, kBM) && make_map_bf16(&m[4], ws_gate, p.H, p.Is, 1, kBK, kBRows / 2) &&
             make_map_bf16(&m[5], ws_up, p.H, p.Is, 1, kBK, kBRows / 2);
    else {
        m[1] = m[0];
        m[4] = m[2];
        m[5] = m[3];
    }
    if (!ok) return cudaErrorInvalidValue;
    GemmArgs a = base_args(p);
    a.N = (int)p.I;
    a.Ns = (int)p.Is;
    a.K = a.Ks = (int)p.H;
    a.h = h;
    a.hs = hs;
    trace_before("gateup_sm100", st);
    cudaError_t e = launch_grouped<true>(p, m, a, st);  // single CTAs (pairs measured no faster here)
    trace_after(st);
    return e;
}

cudaError_t launch_down_sm100(const Plan& p, const void* w_down, const void* ws_down, int mode, void* out,
                              cudaStream_t st) {
    if (p.T == 0) return cudaSuccess;
    const bf16* h = (const bf16*)p.h;
    const bf16* hs = h + p.S * p.I;
    CUtensorMap m[7];
    // a CTA pair stages half of the 256 output columns per CTA
    const bool pairs = use_pairs(p);
    const uint32_t brows = pairs ? kBRows / 2 : kBRows;
    bool ok = make_map_bf16(&m[0], h, p.I, p.S, 1, kBK, kBM) && make_map_bf16(&m[2], w_down, p.I, p.H, p.E, kBK, brows) &&
              make_map_bf16(&m[6], h, p.I, p.S, 1, kBK, kSmallRows);
    if (ok && p.Is > 0)
        ok = make_map_bf16(&m[1], hs, p.Is, p.T, 1, kBK, kBM) && make_map_bf16(&m[4], ws_down, p.Is, p.H, 1, kBK, brows);
    else {
        m[1] = m[0];
        m[4] = m[2];
    }
    m[3] = m[2];
    m[5] = m[4];
    if (!ok) return cudaErrorInvalidValue;
    GemmArgs a = base_args(p);
    a.N = a.Ns = (int)p.H;
    a.K = (int)p.I;
    a.Ks = (int)p.Is;
    a.perm_rows = p.perm_rows;
    a.topk_w = p.topk_w;
    a.out = mode == 0 ? (float*)out : nullptr;
    a.rows = mode == 1 ? (bf16*)out : nullptr;
    a.mode = mode;
    if (pairs) a.mtile_prefix = p.mpair_prefix;
    trace_before(mode ? "down_sm100_weighted" : "down_sm100", st);
    cudaError_t e = pairs ? launch_grouped_pair<false>(p, m, a, st) : launch_grouped<false>(p, m, a, st);
    trace_after(st);
    return e;
}

// Used where it is the faster path (measured at gpt-oss size): up to 128
// rows per expert on average.  With more rows the tiles turn compute-bound
// and the converters' integer work per k-step (about twice the MMA's time)
// decides, so one bf16 conversion of the weights followed by the bf16 GEMMs
// is faster there.
bool mx_gemm_eligible(const Plan& p) {
    return p.bf16 && p.Is == 0 && p.H % 32 == 0 && p.I % 32 == 0 && p.H / 32 <= kMxMaxScales &&
           p.I / 32 <= kMxMaxScales && p.S <= 128 * p.E;
}

cudaError_t launch_gateup_mx_sm100(const Plan& p, const uint8_t* gate_blocks, const uint8_t* gate_scales,
                                   const uint8_t* up_blocks, const uint8_t* up_scales, cudaStream_t st) {
    if (p.T == 0) return cudaSuccess;
    if (!mx_gemm_eligible(p)) return cudaErrorInvalidValue;
    CUtensorMap m[4];
    const bool ok = make_map_bf16(&m[0], p.xperm, p.H, p.S, 1, kBK, kBM) &&
                    make_map_bf16(&m[1], p.xperm, p.H, p.S, 1, kBK, kSmallRows) &&
                    make_map_u8(&m[2], gate_blocks, p.H / 2, p.I, p.E, kBK / 2 * kMxGroupSteps, kBRows / 2) &&
                    make_map_u8(&m[3], up_blocks, p.H / 2, p.I, p.E, kBK / 2 * kMxGroupSteps, kBRows / 2);
    if (!ok) return cudaErrorInvalidValue;
    GemmArgs a = base_args(p);
    a.N = (int)p.I;
    a.K = a.Ks = (int)p.H;
    a.h = (bf16*)p.h;
    a.hs = (bf16*)p.h + p.S * p.I;
    trace_before("gateup_mx_sm100", st);
    // A rows that fit in a quarter of L2 stay there across the column blocks
    const int keep_a = p.S * p.H * 2 <= (32ll << 20);
    cudaError_t e = launch_grouped_mx<true>(p, m, a, MxArgs{gate_scales, up_scales, keep_a}, st);
    trace_after(st);
    return e;
}

cudaError_t launch_down_mx_sm100(const Plan& p, const uint8_t* down_blocks, const uint8_t* down_scales, int mode,
                                 void* out, cudaStream_t st) {
    if (p.T == 0) return cudaSuccess;
    if (!mx_gemm_eligible(p)) return cudaErrorInvalidValue;
    CUtensorMap m[4];
    const bool ok = make_map_bf16(&m[0], p.h, p.I, p.S, 1, kBK, kBM) &&
                    make_map_bf16(&m[1], p.h, p.I, p.S, 1, kBK, kSmallRows) &&
                    make_map_u8(&m[2], down_blocks, p.I / 2, p.H, p.E, kBK / 2 * kMxGroupSteps, kBRows);
    if (!ok) return cudaErrorInvalidValue;
    m[3] = m[2];
    GemmArgs a = base_args(p);
    a.N = a.Ns = (int)p.H;
    a.K = (int)p.I;
    a.perm_rows = p.perm_rows;
    a.topk_w = p.topk_w;
    a.out = mode == 0 ? (float*)out : nullptr;
    a.rows = mode == 1 ? (bf16*)out : nullptr;
    a.mode = mode;
    trace_before(mode ? "down_mx_sm100_weighted" : "down_mx_sm100", st);
    const int keep_a = p.S * p.I * 2 <= (32ll << 20);
    cudaError_t e = launch_grouped_mx<false>(p, m, a, MxArgs{down_scales, nullptr, keep_a}, st);
    trace_after(st);
    return e;
}

}  // namespace moe
