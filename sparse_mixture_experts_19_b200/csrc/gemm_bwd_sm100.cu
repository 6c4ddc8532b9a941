// Grouped GEMMs of the layer's backward pass on the 5th-generation tensor
// cores (tcgen05, sm_100a).
//
// "Mixture of Experts (MoEs) in Transformers", section Training MoEs with
// Transformers: training runs the experts as grouped GEMMs in both
// directions.  The backward pass of a grouped expert layer needs, besides
// the forward's products, products whose reduction runs over the rows of an
// expert (the weight gradients) and products with the weights' other
// orientation (the input gradients).  Both are written here without copying
// any operand into another layout: an operand stored with its reduction
// dimension contiguous is K-major (as in the forward), one stored with its
// row (M) or column (N) dimension contiguous is MN-major, and the tensor
// core reads either from shared memory through the matching descriptor.
//
// One persistent kernel template, 128 x 256 output tiles, K in steps of 64,
// a 4-stage TMA ring, double-buffered TMEM accumulators, float32 output:
//   row groups (kgroups = 0): group g owns the rows [goff[g], goff[g+1]) of
//     A and multiplies them by B[g]; the forward-shaped products (the
//     recomputed gate/up activations, the down projection's input gradient,
//     the experts' input gradients);
//   K groups (kgroups = 1): group g reduces over the rows [goff[g],
//     goff[g+1]) of both (MN-major) operands, producing an M x N block per
//     group; the weight gradients.  A group with no rows writes zeros.
// Every wait is bounded (timeout -> MOE_DEVFLAG_WAIT_TIMEOUT); no multicast.
//
// MN-major tiles are loaded as 64 x 64 boxes (64 M or N elements, contiguous,
// by 64 k) with the 128-byte swizzle, side by side 8 KB apart: in the
// descriptor, 64 M/N elements further is 8 KB (leading byte offset) and
// 8 k further is 1 KB (stride byte offset).
#include <algorithm>

#include "common.cuh"
#include "sm100.cuh"
#include "tma_host.cuh"

namespace moe {
namespace {

using namespace sm100;

constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kBK = 64;
constexpr int kStages = 4;
constexpr int kABytes = kBM * kBK * 2;
constexpr int kBBytes = kBN * kBK * 2;
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kAccCols = kBN;
constexpr int kTmemCols = 2 * kAccCols;
constexpr int kThreads = 192;
constexpr int kEpiThreads = 128;
constexpr uint32_t kMnBox = 64 * kBK * 2;  // one 64 x 64 bf16 box of an MN-major tile (8 KB)
// Epilogue staging: each epilogue warp owns 4 KB for its 32 rows x 32 float32
// columns (128 B per row), 16-byte chunk c of row r at r * 128 + ((c ^ (r %
// 8)) * 16), so that both the row-wise writes (a lane per row) and the
// column-wise reads (8 lanes per row) are free of bank conflicts, and each
// global store instruction writes 4 rows x 128 contiguous bytes.
constexpr int kEpiStageBytes = 32 * 128;
constexpr size_t kEpiOff = (kStages * kStageBytes + 256 + 2 * (kMaxExperts + 2) * sizeof(int32_t) + 127) / 128 * 128;

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

struct BwdArgs {
    int groups;
    int kgroups;           // 1: groups split the reduction (weight gradients)
    const int32_t* goff;   // [groups + 1] device: row offsets (row groups) or reduction offsets (K groups)
    int M, N, K;           // K groups: M x N per group; row groups: N, K
    int n_split;           // > 0: output columns [0, n_split) from B0, [n_split, N) from B1 (at n - n_split)
    int k_split;           // > 0: reduction [0, k_split) from B0, then from B1; A's second part at column a_k1
    int a_k1;
    float* out0;           // row groups: out0 + row * ldo + col; K groups: out0 + g * m_split * N + m * N + col
    float* out1;           // K groups: rows m >= m_split go to out1 + g * (M - m_split) * N + (m - m_split) * N
    int ldo;
    int m_split;
    int32_t* flags;
};

struct Sched {
    int nb;        // column blocks
    int mt_k;      // K groups: row tiles per group
    int kb_fixed;  // row groups: reduction steps
    int nkb0;      // k_split > 0: reduction steps from B0
    int64_t total;
};

struct Tile {
    int g;
    int64_t row0;  // row groups: first row of A; K groups: first output row m
    int rows;      // valid rows of the tile
    int n0;        // first output column
    int nkb;       // reduction steps (0: the tile is zero)
    int64_t k0;    // K groups: first reduction row
};

// Row groups: tiles of group g are mt_g row tiles x nb column blocks,
// m-fastest within a column block (CTAs working side by side share B).
__device__ __forceinline__ void decode(int64_t t, const BwdArgs& a, const Sched& sc, const int32_t* tiles_pre,
                                       const int32_t* off, Tile& ti) {
    if (!a.kgroups) {
        int lo = 0, hi = a.groups - 1;  // largest g with tiles_pre[g] <= t / nb... over tiles
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if ((int64_t)tiles_pre[mid] * sc.nb <= t)
                lo = mid;
            else
                hi = mid - 1;
        }
        const int g = lo;
        const int mt = tiles_pre[g + 1] - tiles_pre[g];
        const int64_t local = t - (int64_t)tiles_pre[g] * sc.nb;
        const int nbi = (int)(local / mt), mb = (int)(local % mt);
        ti.g = g;
        ti.row0 = off[g] + (int64_t)mb * kBM;
        const int64_t left = off[g + 1] - ti.row0;
        ti.rows = left < kBM ? (int)left : kBM;
        ti.n0 = nbi * kBN;
        ti.nkb = sc.kb_fixed;
        ti.k0 = 0;
    } else {
        const int64_t per = (int64_t)sc.mt_k * sc.nb;
        const int g = (int)(t / per);
        const int64_t local = t - (int64_t)g * per;
        const int nbi = (int)(local / sc.mt_k), mb = (int)(local % sc.mt_k);
        ti.g = g;
        ti.row0 = (int64_t)mb * kBM;
        ti.rows = min(kBM, a.M - (int)ti.row0);
        ti.n0 = nbi * kBN;
        ti.k0 = off[g];
        ti.nkb = (int)((off[g + 1] - off[g] + kBK - 1) / kBK);
    }
}

// Output column of local tile column j (the B split maps tile columns of the
// second operand after the first's).
__device__ __forceinline__ int out_col(const BwdArgs& a, const Sched& sc, int n0) {
    if (a.n_split > 0) {
        const int nb0 = (a.n_split + kBN - 1) / kBN;
        const int nbi = n0 / kBN;
        return nbi < nb0 ? n0 : a.n_split + (nbi - nb0) * kBN;
    }
    return n0;
}

template <bool kAMN, bool kBMN>
__global__ void __launch_bounds__(kThreads, 1) bwd_gemm_kernel(
    const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
    const __grid_constant__ CUtensorMap tmB1, const BwdArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
    uint64_t* empty = full + kStages;
    uint64_t* tfull = empty + kStages;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    int32_t* off = reinterpret_cast<int32_t*>(smem + kStages * kStageBytes + 256);  // [groups + 1]
    int32_t* tiles_pre = off + (kMaxExperts + 2);                                    // [groups + 1]

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    for (int i = threadIdx.x; i <= a.groups; i += kThreads) off[i] = a.goff[i];
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
    if (warp == 1) {
        tmem_alloc(tmem_holder, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0) {
        // row groups: prefix of row tiles per group
        tiles_pre[0] = 0;
        for (int g = 0; g < a.groups; ++g)
            tiles_pre[g + 1] = tiles_pre[g] + (a.kgroups ? 0 : (off[g + 1] - off[g] + kBM - 1) / kBM);
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    Sched sc;
    sc.nb = a.n_split > 0 ? (a.n_split + kBN - 1) / kBN + (a.N - a.n_split + kBN - 1) / kBN : (a.N + kBN - 1) / kBN;
    sc.mt_k = (a.M + kBM - 1) / kBM;
    sc.nkb0 = a.k_split > 0 ? (a.k_split + kBK - 1) / kBK : 0;
    sc.kb_fixed = a.k_split > 0 ? sc.nkb0 + (a.K - a.k_split + kBK - 1) / kBK : (a.K + kBK - 1) / kBK;
    sc.total = a.kgroups ? (int64_t)a.groups * sc.mt_k * sc.nb : (int64_t)tiles_pre[a.groups] * sc.nb;
    constexpr uint32_t kIdesc = idesc_bf16_major(kBM, kBN, kAMN, kBMN);

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_map(&tmA);
            tma_prefetch_map(&tmB0);
            uint32_t it = 0;
            for (int64_t t = blockIdx.x; t < sc.total && !*abort_flag; t += gridDim.x) {
                Tile ti;
                decode(t, a, sc, tiles_pre, off, ti);
                // B coordinates: column block within B0 or B1
                const CUtensorMap* mB = &tmB0;
                int bn = ti.n0;
                if (a.n_split > 0) {
                    const int nb0 = (a.n_split + kBN - 1) / kBN;
                    if (ti.n0 / kBN >= nb0) {
                        mB = &tmB1;
                        bn = (ti.n0 / kBN - nb0) * kBN;
                    }
                }
                const int bz = a.kgroups ? 0 : ti.g;
                for (int kb = 0; kb < ti.nkb; ++kb, ++it) {
                    const int s = it % kStages;
                    const uint32_t ph = (it / kStages) & 1;
                    if (!wait_or_abort(&empty[s], ph ^ 1, abort_flag, a.flags)) break;
                    uint8_t* sa = smem + s * kStageBytes;
                    uint8_t* sb = sa + kABytes;
                    mbar_arrive_expect_tx(&full[s], kStageBytes);
                    // reduction coordinate of this step in A and in B
                    int ka = kb * kBK, kbB = kb * kBK;
                    const CUtensorMap* mBk = mB;
                    if (a.k_split > 0 && kb >= sc.nkb0) {
                        ka = a.a_k1 + (kb - sc.nkb0) * kBK;
                        kbB = (kb - sc.nkb0) * kBK;
                        mBk = &tmB1;
                    }
                    if (a.kgroups) {
                        ka += (int)ti.k0;
                        kbB += (int)ti.k0;
                    }
                    if (kAMN) {
                        tma_load_3d(sa, &tmA, &full[s], (int)ti.row0, ka, 0);
                        tma_load_3d(sa + kMnBox, &tmA, &full[s], (int)ti.row0 + 64, ka, 0);
                    } else {
                        tma_load_3d(sa, &tmA, &full[s], ka, (int)ti.row0, 0);
                    }
                    if (kBMN) {
#pragma unroll
                        for (int j = 0; j < kBN / 64; ++j)
                            tma_load_3d(sb + j * kMnBox, mBk, &full[s], bn + 64 * j, kbB, bz);
                    } else {
                        tma_load_3d(sb, mBk, &full[s], kbB, bn, bz);
                    }
                }
            }
            for (uint32_t j = (it > (uint32_t)kStages ? it - kStages : 0); j < it; ++j)
                drain_wait(&full[j % kStages], (j / kStages) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            uint32_t it = 0, tc = 0;
            for (int64_t t = blockIdx.x; t < sc.total && !*abort_flag; t += gridDim.x, ++tc) {
                Tile ti;
                decode(t, a, sc, tiles_pre, off, ti);
                const uint32_t acc = tc & 1, aph = (tc >> 1) & 1;
                if (!wait_or_abort(&tempty[acc], aph ^ 1, abort_flag, a.flags)) break;
                tc_fence_after();
                const uint32_t d = tmem_base + acc * kAccCols;
                bool ok = true;
                for (int kb = 0; kb < ti.nkb; ++kb, ++it) {
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
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        const uint64_t da = kAMN ? desc_mnmajor_sw128(a0 + kk * 2048, kMnBox, 1024)
                                                 : desc_kmajor_sw128(a0 + kk * 32);
                        const uint64_t db = kBMN ? desc_mnmajor_sw128(b0 + kk * 2048, kMnBox, 1024)
                                                 : desc_kmajor_sw128(b0 + kk * 32);
                        mma_bf16(d, da, db, kIdesc, (kb | kk) != 0);
                    }
                    mma_commit(&empty[s]);  // frees the stage once these MMAs finish
                }
                if (!ok) break;
                mma_commit(&tfull[acc]);  // a tile with no reduction steps arrives at once
            }
            mma_commit(drain);
            drain_wait(drain, 0);
        }
    } else {
        // ------------------------------------------------ epilogue warps 2..5
        const int q = warp & 3;
        const uint32_t stage = smem_u32(smem + kEpiOff) + (uint32_t)(q * kEpiStageBytes);
        uint32_t tc = 0;
        for (int64_t t = blockIdx.x; t < sc.total; t += gridDim.x, ++tc) {
            Tile ti;
            decode(t, a, sc, tiles_pre, off, ti);
            const uint32_t acc = tc & 1, aph = (tc >> 1) & 1;
            if (!wait_or_abort(&tfull[acc], aph, abort_flag, a.flags)) break;
            tc_fence_after();
            const uint32_t tq = tmem_base + acc * kAccCols + ((uint32_t)(q * 32) << 16);
            // the columns of this tile, and the output row of tile row m
            const int c0 = out_col(a, sc, ti.n0);
            const int ncols = (a.n_split > 0 ? (c0 < a.n_split ? a.n_split : a.N) : a.N) - c0;
            auto row_dst = [&](int m) -> float* {
                if (m >= ti.rows) return nullptr;
                if (!a.kgroups) return a.out0 + (ti.row0 + m) * (int64_t)a.ldo + c0;
                const int mm = (int)ti.row0 + m;
                return mm < a.m_split ? a.out0 + ((int64_t)ti.g * a.m_split + mm) * a.N + c0
                                      : a.out1 + ((int64_t)ti.g * (a.M - a.m_split) + (mm - a.m_split)) * a.N + c0;
            };
#pragma unroll 1
            for (int j0 = 0; j0 < kBN; j0 += 32) {
                float v[32];
                tmem_ld32(tq + j0, v);
                if (ti.nkb == 0) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = 0.f;
                }
                // this lane's row into the warp's stage, then 4 rows per store
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    st_shared_v4(stage + (uint32_t)(lane * 128 + ((c ^ (lane & 7)) << 4)),
                                 make_uint4(__float_as_uint(v[4 * c]), __float_as_uint(v[4 * c + 1]),
                                            __float_as_uint(v[4 * c + 2]), __float_as_uint(v[4 * c + 3])));
                __syncwarp();
                const int cc = lane & 7;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int rr = 4 * i + (lane >> 3);
                    const uint4 w = ld_shared_v4(stage + (uint32_t)(rr * 128 + ((cc ^ (rr & 7)) << 4)));
                    float* dst = row_dst(q * 32 + rr);
                    const int n = j0 + 4 * cc;
                    if (dst && n < ncols) *reinterpret_cast<uint4*>(dst + n) = w;
                }
                __syncwarp();
            }
            tc_fence_before();
            mbar_arrive(&tempty[acc]);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

constexpr size_t kSmemBytes = 1024 + kEpiOff + 4 * kEpiStageBytes;

// Rank-3 map of a bf16 tensor [depth][rows][inner]: K-major operands take
// 64 x box_rows boxes, MN-major ones 64 x 64 boxes (64 contiguous M/N
// elements by 64 reduction rows).
bool operand_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t depth, bool mn,
                 uint32_t box_rows) {
    return make_map_bf16(m, base, inner, rows, depth, 64, mn ? 64 : box_rows);
}

template <bool kAMN, bool kBMN>
cudaError_t launch_bwd(const CUtensorMap& mA, const CUtensorMap& mB0, const CUtensorMap& mB1, const BwdArgs& args,
                       int64_t tiles_bound, const char* name, cudaStream_t st) {
    cudaError_t e = ensure_smem_attr(bwd_gemm_kernel<kAMN, kBMN>, kSmemBytes);
    if (e != cudaSuccess) return e;
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(device_sm_count(), tiles_bound));
    trace_before(name, st);
    bwd_gemm_kernel<kAMN, kBMN><<<grid, kThreads, kSmemBytes, st>>>(mA, mB0, mB1, args);
    trace_after(st);
    return cudaGetLastError();
}

}  // namespace

// ---------------------------------------------------------------- launchers
// Every operand is bf16, row-major; output float32.

// out[rows, 2I] = A_rows . [W_g[g] ; W_u[g]]^T: the gate and up
// pre-activations of each group's rows (A [R, H] K-major, W [G, I, H]).
cudaError_t launch_bwd_gu_recompute(const void* A, int64_t R, const int32_t* goff, int groups, const void* wg,
                                    const void* wu, int I, int H, float* out, int32_t* flags, cudaStream_t st) {
    CUtensorMap mA, mB0, mB1;
    if (!operand_map(&mA, A, H, R, 1, false, kBM) || !operand_map(&mB0, wg, H, I, groups, false, kBN) ||
        !operand_map(&mB1, wu, H, I, groups, false, kBN))
        return cudaErrorInvalidValue;
    BwdArgs a{};
    a.groups = groups;
    a.goff = goff;
    a.N = 2 * I;
    a.K = H;
    a.n_split = I;
    a.out0 = out;
    a.ldo = 2 * I;
    a.flags = flags;
    const int64_t bound = ((R + kBM - 1) / kBM + groups) * (2 * ((I + kBN - 1) / kBN));
    return launch_bwd<false, false>(mA, mB0, mB1, a, bound, "bwd_gu_recompute", st);
}

// out[rows, I] = dY_rows . W_d[g]: the down projection's input gradient
// (dY [R, H] K-major; W_d [G, H, I] read MN-major: reduction over H).
cudaError_t launch_bwd_down_dgrad(const void* dY, int64_t R, const int32_t* goff, int groups, const void* wd, int I,
                                  int H, float* out, int32_t* flags, cudaStream_t st) {
    CUtensorMap mA, mB;
    if (!operand_map(&mA, dY, H, R, 1, false, kBM) || !operand_map(&mB, wd, I, H, groups, true, kBN))
        return cudaErrorInvalidValue;
    BwdArgs a{};
    a.groups = groups;
    a.goff = goff;
    a.N = I;
    a.K = H;
    a.out0 = out;
    a.ldo = I;
    a.flags = flags;
    const int64_t bound = ((R + kBM - 1) / kBM + groups) * ((I + kBN - 1) / kBN);
    return launch_bwd<false, true>(mA, mB, mB, a, bound, "bwd_down_dgrad", st);
}

// out[rows, H] = dGU_rows[:, :I] . W_g[g] + dGU_rows[:, I:] . W_u[g]: the
// experts' input gradient (dGU [R, 2I] K-major; W [G, I, H] MN-major).
cudaError_t launch_bwd_gateup_dgrad(const void* dGU, int64_t R, const int32_t* goff, int groups, const void* wg,
                                    const void* wu, int I, int H, float* out, int32_t* flags, cudaStream_t st) {
    CUtensorMap mA, mB0, mB1;
    if (!operand_map(&mA, dGU, 2 * I, R, 1, false, kBM) || !operand_map(&mB0, wg, H, I, groups, true, kBN) ||
        !operand_map(&mB1, wu, H, I, groups, true, kBN))
        return cudaErrorInvalidValue;
    BwdArgs a{};
    a.groups = groups;
    a.goff = goff;
    a.N = H;
    a.K = 2 * I;
    a.k_split = I;
    a.a_k1 = I;
    a.out0 = out;
    a.ldo = H;
    a.flags = flags;
    const int64_t bound = ((R + kBM - 1) / kBM + groups) * ((H + kBN - 1) / kBN);
    return launch_bwd<false, true>(mA, mB0, mB1, a, bound, "bwd_gateup_dgrad", st);
}

// Weight gradient per group: out[g] (M x N) = sum over the group's rows of
// A_row^T B_row (A [RA, M], B [RB, N], both read MN-major; goff 64-aligned
// reduction ranges whose padding rows are zero or past the tensor's rows,
// which read as zero).  Rows m >= m_split of the result go to out1 (the
// gate/up split of one product).
cudaError_t launch_bwd_wgrad(const void* A, int64_t RA, const void* B, int64_t RB, const int32_t* goff, int groups,
                             int M, int N, int m_split, float* out0, float* out1, const char* name, int32_t* flags,
                             cudaStream_t st) {
    CUtensorMap mA, mB;
    if (!operand_map(&mA, A, M, RA, 1, true, 64) || !operand_map(&mB, B, N, RB, 1, true, 64))
        return cudaErrorInvalidValue;
    BwdArgs a{};
    a.groups = groups;
    a.kgroups = 1;
    a.goff = goff;
    a.M = M;
    a.N = N;
    a.out0 = out0;
    a.out1 = out1 ? out1 : out0;
    a.m_split = m_split > 0 ? m_split : M;
    a.flags = flags;
    const int64_t bound = (int64_t)groups * ((M + kBM - 1) / kBM) * ((N + kBN - 1) / kBN);
    return launch_bwd<true, true>(mA, mB, mB, a, bound, name, st);
}

}  // namespace moe
