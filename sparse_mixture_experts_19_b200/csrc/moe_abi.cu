// Host side of the C ABI declared in include/moe.h: argument checks,
// workspace carving, launch sequencing, status codes and kernel tracing.
// No entry point allocates device memory or synchronises, except
// moe_get_device_status (documented to wait) and moe_trace_end.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <vector>

#include "common.cuh"

namespace moe {

// ------------------------------------------------------------------ errors
static thread_local char g_last_error[256] = "";

static moe_status_t fail(moe_status_t st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
    return st;
}

static moe_status_t cuda_fail(cudaError_t e, const char* where) {
    return fail(MOE_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

// ----------------------------------------------------------------- tracing
namespace {
struct TraceState {
    bool on = false;
    int max = 0;
    int n = 0;
    bool open = false;  // a launch has been started and not yet closed
    char only[64] = {};  // trace only kernels whose name contains this ("" = all)
    std::vector<const char*> names;
    std::vector<cudaEvent_t> ev;
};
TraceState g_trace;
}  // namespace

// Inside a stream capture an event is recorded by an external event-record
// node, so that replays of the graph record it.
static cudaError_t trace_record(cudaEvent_t ev, cudaStream_t st) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
        return cudaEventRecordWithFlags(ev, st, cudaEventRecordExternal);
    return cudaEventRecord(ev, st);
}

void trace_before(const char* name, cudaStream_t st) {
    if (!g_trace.on || g_trace.n >= g_trace.max) return;
    if (g_trace.only[0] && !strstr(name, g_trace.only)) return;
    if (trace_record(g_trace.ev[2 * g_trace.n], st) != cudaSuccess) return;
    g_trace.names[g_trace.n] = name;
    g_trace.open = true;
}

void trace_after(cudaStream_t st) {
    if (!g_trace.on || !g_trace.open) return;
    g_trace.open = false;
    if (trace_record(g_trace.ev[2 * g_trace.n + 1], st) == cudaSuccess) g_trace.n++;
}

// --------------------------------------------------------------- the plan
static moe_status_t check_config(const moe_config_t* c) {
    if (!c) return fail(MOE_ERR_INVALID_ARG, "cfg is NULL");
    if (c->T < 0) return fail(MOE_ERR_INVALID_ARG, "T = %d < 0", c->T);
    if (c->H < 8 || c->H % 8) return fail(MOE_ERR_INVALID_ARG, "H = %d must be a positive multiple of 8", c->H);
    if (c->I < 8 || c->I % 8) return fail(MOE_ERR_INVALID_ARG, "I = %d must be a positive multiple of 8", c->I);
    if (c->E < 1 || c->E > kMaxExperts) return fail(MOE_ERR_INVALID_ARG, "E = %d outside 1..%d", c->E, kMaxExperts);
    bool k_ok = (c->top_k >= 1 && c->top_k <= c->E && c->top_k <= 8) || (c->top_k == c->E && c->E <= kMaxTopK);
    if (!k_ok) return fail(MOE_ERR_INVALID_ARG, "top_k = %d must be in 1..min(E,8), or equal E <= 32", c->top_k);
    if (c->I_shared < 0 || c->I_shared % 8) return fail(MOE_ERR_INVALID_ARG, "I_shared = %d must be 0 or a positive multiple of 8", c->I_shared);
    if (c->dtype != MOE_F32 && c->dtype != MOE_BF16) return fail(MOE_ERR_INVALID_ARG, "dtype = %d unknown", c->dtype);
    if (!isfinite(c->capacity_factor)) return fail(MOE_ERR_INVALID_ARG, "capacity_factor is not finite");
    if ((int64_t)c->T * c->top_k > INT32_MAX / 2) return fail(MOE_ERR_UNSUPPORTED, "T * top_k too large");
    return MOE_OK;
}

// C = ceil(cf * T * k / E).  cf arrives as float32, whose rounding (about
// 6e-8 relative) can lift an exact integer just above itself (0.8f * 2400 / 8
// = 240.0000029): the ceiling is taken after removing a relative 1e-6, far
// below any fractional part a real configuration produces.
static int64_t capacity_of(const moe_config_t* c) {
    if (c->capacity_factor <= 0.f) return 0;
    const double v = (double)c->capacity_factor * (double)c->T * (double)c->top_k / (double)c->E;
    const double C = ceil(v - 1e-6 * (v > 1.0 ? v : 1.0));
    return C < 1.0 ? 1 : (int64_t)C;
}

static size_t align_up(size_t v) { return (v + kWsAlign - 1) / kWsAlign * kWsAlign; }

// Fills the plan; with ws == nullptr only sizes are computed.
static void make_plan(const moe_config_t* c, void* ws, Plan* p) {
    p->T = c->T;
    p->H = c->H;
    p->I = c->I;
    p->E = c->E;
    p->k = c->top_k;
    p->Is = c->I_shared;
    p->S = p->T * p->k;
    p->cap = capacity_of(c);
    p->cap_left_arr = nullptr;
    p->importance = nullptr;
    p->bf16 = (c->dtype == MOE_BF16);
    p->drop_negative = false;
    p->y_f32 = false;
    p->nchunks = (p->S + kPermuteChunk - 1) / kPermuteChunk;
    p->h_rows = p->S + (p->Is ? p->T : 0);
    p->I_max = p->I > p->Is ? p->I : p->Is;
    const size_t elt = p->bf16 ? 2 : 4;
    size_t off = 0;
    char* base = (char*)ws;
    auto take = [&](size_t bytes) -> void* {
        void* r = base ? base + off : nullptr;
        off += align_up(bytes);
        return r;
    };
    p->flags = (int32_t*)take(64);
    p->topk_idx = (int32_t*)take(sizeof(int32_t) * p->S);
    p->topk_w = (float*)take(sizeof(float) * p->S);
    p->chunk_base = (int32_t*)take(sizeof(int32_t) * p->nchunks * p->E);
    p->counts = (int32_t*)take(sizeof(int32_t) * p->E);
    p->dropped = (int32_t*)take(sizeof(int32_t) * p->E);
    p->offsets = (int32_t*)take(sizeof(int32_t) * (p->E + 2));
    p->mtile_prefix = (int32_t*)take(sizeof(int32_t) * (p->E + 1));
    p->mpair_prefix = (int32_t*)take(sizeof(int32_t) * (p->E + 1));
    p->perm_rows = (int32_t*)take(sizeof(int32_t) * p->S);
    p->row_of = (int32_t*)take(sizeof(int32_t) * p->S);
    p->xperm = take(elt * p->S * p->H);
    p->h = take(elt * (p->S * p->I + p->T * p->Is));
    p->rows = take(elt * (p->S + (p->Is ? p->T : 0)) * p->H);
    const bool tc_router = p->bf16 && p->T * p->E * p->H > kDecodeRouterMaxMacs;
    p->rt_part = (float*)take(tc_router ? sizeof(float) * kRouterMaxSplits * p->T * p->E : 0);
    p->rt_xn2 = (float*)take(tc_router ? sizeof(float) * kRouterMaxSplits * p->T : 0);
    p->rt_wn2 = (float*)take(tc_router ? sizeof(float) * kRouterMaxSplits * p->E : 0);
    const bool dec = p->S <= kDecodeMaxSlotsMx;
    p->dec_scores = (double*)take(dec ? sizeof(double) * p->T * p->E : 0);
    p->dec_bar = (unsigned int*)take(dec ? kDecodeCounters * sizeof(unsigned int) : 0);
    p->bytes = off;
}

static moe_status_t plan_for(const moe_config_t* c, void* ws, size_t ws_bytes, Plan* p) {
    moe_status_t st = check_config(c);
    if (st != MOE_OK) return st;
    make_plan(c, nullptr, p);
    if (!ws) return fail(MOE_ERR_WORKSPACE, "workspace is NULL");
    if ((uintptr_t)ws % kWsAlign) return fail(MOE_ERR_WORKSPACE, "workspace not %d-byte aligned", kWsAlign);
    if (ws_bytes < p->bytes)
        return fail(MOE_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, p->bytes);
    make_plan(c, ws, p);
    return MOE_OK;
}

static bool aligned16(const void* ptr) { return ((uintptr_t)ptr & 15) == 0; }

#define REQUIRE_PTR(ptr)                                                                    \
    do {                                                                                    \
        if (!(ptr)) return fail(MOE_ERR_INVALID_ARG, "%s is NULL", #ptr);                   \
        if (!aligned16(ptr)) return fail(MOE_ERR_INVALID_ARG, "%s is not 16-byte aligned", #ptr); \
    } while (0)

#define OPTIONAL_PTR(ptr)                                                                   \
    do {                                                                                    \
        if ((ptr) && !aligned16(ptr)) return fail(MOE_ERR_INVALID_ARG, "%s is not 16-byte aligned", #ptr); \
    } while (0)

#define CUDA_TRY(expr, where)                           \
    do {                                                \
        cudaError_t e_ = (expr);                        \
        if (e_ != cudaSuccess) return cuda_fail(e_, where); \
    } while (0)

static moe_status_t check_shared(const Plan& p, const void* a, const void* b, const void* c) {
    if (p.Is > 0) {
        REQUIRE_PTR(a);
        REQUIRE_PTR(b);
        REQUIRE_PTR(c);
    }
    return MOE_OK;
}

// Router choice by size: few tokens -> per-token exact router; otherwise the
// tensor-core router (bf16) or the CUDA-core float32 router.
static cudaError_t run_router(const Plan& p, const void* x, const void* router_w, const float* router_b,
                              int32_t* idx, float* w, cudaStream_t st) {
    if (p.T * p.E * p.H <= kDecodeRouterMaxMacs) return launch_router_decode(p, x, router_w, router_b, idx, w, st);
    if (p.bf16) return launch_router_sm100(p, x, router_w, router_b, idx, w, st);
    return launch_router_simt(p, x, router_w, router_b, idx, w, st);
}

// The grouped FFN of moe_forward / moe_grouped_ffn, after routing and grouping.
// row_of (slot -> grouped row, or -1) when known: the x rows are then built
// token by token, reading x once; else row by row from perm_rows.
static moe_status_t run_ffn(const Plan& p, const void* x, const void* w_gate, const void* w_up,
                            const void* w_down, const void* ws_gate, const void* ws_up,
                            const void* ws_down, int mode, void* out, const int32_t* row_of, cudaStream_t st) {
    if (row_of)
        CUDA_TRY(launch_scatter_x_rows(p, x, row_of, p.xperm, st), "gather_rows");
    else
        CUDA_TRY(launch_gather_rows(p, x, p.perm_rows, p.offsets, p.xperm, st), "gather_rows");
    if (p.bf16) {
        // bf16: tensor cores (tcgen05 + TMEM + TMA)
        CUDA_TRY(launch_gateup_sm100(p, x, w_gate, w_up, ws_gate, ws_up, st), "gateup");
        CUDA_TRY(launch_down_sm100(p, w_down, ws_down, mode, out, st), "down");
    } else {
        // float32: exact float32 FMAs on CUDA cores (tensor cores would round the inputs)
        CUDA_TRY(launch_gateup_simt(p, p.xperm, x, p.offsets, w_gate, w_up, ws_gate, ws_up, p.h, st),
                 "gateup");
        CUDA_TRY(launch_down_simt(p, p.h, p.offsets, p.perm_rows, p.topk_w, w_down, ws_down, mode, out, st),
                 "down");
    }
    return MOE_OK;
}

}  // namespace moe

using namespace moe;

extern "C" {

size_t moe_workspace_size(const moe_config_t* cfg) {
    if (check_config(cfg) != MOE_OK) return 0;
    Plan p;
    make_plan(cfg, nullptr, &p);
    return p.bytes;
}

int64_t moe_capacity(const moe_config_t* cfg) {
    if (check_config(cfg) != MOE_OK) return -1;
    return capacity_of(cfg);
}

moe_status_t moe_route(const moe_config_t* cfg, const void* x, const void* router_w,
                       const float* router_b, int32_t* topk_idx, float* topk_w, void* ws,
                       size_t ws_bytes, moe_stream_t stream) {
    Plan p;
    moe_status_t s = plan_for(cfg, ws, ws_bytes, &p);
    if (s != MOE_OK) return s;
    if (p.T == 0) return MOE_OK;
    REQUIRE_PTR(x);
    REQUIRE_PTR(router_w);
    OPTIONAL_PTR(router_b);
    REQUIRE_PTR(topk_idx);
    REQUIRE_PTR(topk_w);
    cudaStream_t st = (cudaStream_t)stream;
    CUDA_TRY(run_router(p, x, router_w, router_b, topk_idx, topk_w, st), "router");
    return MOE_OK;
}

moe_status_t moe_route_importance(const moe_config_t* cfg, const void* x, const void* router_w,
                                  const float* router_b, int32_t* topk_idx, float* topk_w, float* importance,
                                  void* ws, size_t ws_bytes, moe_stream_t stream) {
    Plan p;
    moe_status_t s = plan_for(cfg, ws, ws_bytes, &p);
    if (s != MOE_OK) return s;
    REQUIRE_PTR(importance);
    if (p.T == 0) return MOE_OK;
    REQUIRE_PTR(x);
    REQUIRE_PTR(router_w);
    OPTIONAL_PTR(router_b);
    REQUIRE_PTR(topk_idx);
    REQUIRE_PTR(topk_w);
    p.importance = importance;
    cudaStream_t st = (cudaStream_t)stream;
    CUDA_TRY(run_router(p, x, router_w, router_b, topk_idx, topk_w, st), "router");
    return MOE_OK;
}

moe_status_t moe_permute(const moe_config_t* cfg, const int32_t* topk_idx, int32_t* counts,
                         int32_t* offsets, int32_t* perm_rows, int32_t* row_of, int32_t* dropped,
                         void* ws, size_t ws_bytes, moe_stream_t stream) {
    Plan p;
    moe_status_t s = plan_for(cfg, ws, ws_bytes, &p);
    if (s != MOE_OK) return s;
    REQUIRE_PTR(counts);
    REQUIRE_PTR(offsets);
    REQUIRE_PTR(dropped);
    if (p.S > 0) {
        REQUIRE_PTR(topk_idx);
        REQUIRE_PTR(perm_rows);
        REQUIRE_PTR(row_of);
    }
    cudaStream_t st = (cudaStream_t)stream;
    CUDA_TRY(launch_permute(p, topk_idx, counts, offsets, perm_rows, row_of, dropped, st), "permute");
    return MOE_OK;
}

moe_status_t moe_permute_noalloc(const moe_config_t* cfg, const int32_t* topk_idx, int32_t* counts,
                                 int32_t* offsets, int32_t* perm_rows, int32_t* row_of,
                                 int32_t* dropped, moe_stream_t stream) {
    moe_status_t s = check_config(cfg);
    if (s != MOE_OK) return s;
    Plan p;
    make_plan(cfg, nullptr, &p);  // sizes only: this entry point takes no workspace
    if (p.S > kNoAllocMaxSlots)
        return fail(MOE_ERR_UNSUPPORTED,
                    "moe_permute_noalloc handles at most %lld slots (T*top_k) in its static scratch; "
                    "got %lld, use moe_permute with a workspace",
                    (long long)kNoAllocMaxSlots, (long long)p.S);
    REQUIRE_PTR(counts);
    REQUIRE_PTR(offsets);
    REQUIRE_PTR(dropped);
    if (p.S > 0) {
        REQUIRE_PTR(topk_idx);
        REQUIRE_PTR(perm_rows);
        REQUIRE_PTR(row_of);
    }
    CUDA_TRY(launch_permute_noalloc(p, topk_idx, counts, offsets, perm_rows, row_of, dropped,
                                    (cudaStream_t)stream),
             "permute_noalloc");
    return MOE_OK;
}

moe_status_t moe_grouped_ffn(const moe_config_t* cfg, const void* x, const int32_t* perm_rows,
                             const int32_t* offsets, const void* w_gate, const void* w_up,
                             const void* w_down, const void* ws_gate, const void* ws_up,
                             const void* ws_down, float* expert_out, void* ws, size_t ws_bytes,
                             moe_stream_t stream) {
    Plan p;
    moe_status_t s = plan_for(cfg, ws, ws_bytes, &p);
    if (s != MOE_OK) return s;
    if (p.T == 0) return MOE_OK;
    REQUIRE_PTR(x);
    REQUIRE_PTR(perm_rows);
    REQUIRE_PTR(offsets);
    REQUIRE_PTR(w_gate);
    REQUIRE_PTR(w_up);
    REQUIRE_PTR(w_down);
    REQUIRE_PTR(expert_out);
    if ((s = check_shared(p, ws_gate, ws_up, ws_down)) != MOE_OK) return s;
    cudaStream_t st = (cudaStream_t)stream;
    // the grouped kernels read the plan's copies of perm_rows and offsets [E+2]
    CUDA_TRY(launch_offsets_from_user(p, offsets, st), "offsets");
    CUDA_TRY(cudaMemcpyAsync(p.perm_rows, perm_rows, sizeof(int32_t) * p.S, cudaMemcpyDeviceToDevice, st),
             "perm_rows copy");
    return run_ffn(p, x, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, 0, expert_out, nullptr, st);
}

moe_status_t moe_combine(const moe_config_t* cfg, const float* expert_out, const int32_t* row_of,
                         const float* topk_w, void* y, void* ws, size_t ws_bytes,
                         moe_stream_t stream) {
    Plan p;
    moe_status_t s = plan_for(cfg, ws, ws_bytes, &p);
    if (s != MOE_OK) return s;
    if (p.T == 0) return MOE_OK;
    REQUIRE_PTR(expert_out);
    REQUIRE_PTR(row_of);
    REQUIRE_PTR(topk_w);
    REQUIRE_PTR(y);
    CUDA_TRY(launch_combine(p, expert_out, row_of, topk_w, y, (cudaStream_t)stream), "combine");
    return MOE_OK;
}

}  // extern "C"

// Everything after routing: grouping (with a per-expert capacity for a token
// shard, when given), the expert FFNs and the combine.
static moe_status_t forward_after_routing(Plan& p, const void* x, const int32_t* idx, const void* w_gate,
                                          const void* w_up, const void* w_down, const void* ws_gate,
                                          const void* ws_up, const void* ws_down, void* y, int32_t* counts,
                                          int32_t* dropped, cudaStream_t st) {
    if (decode_ffn_eligible(p)) {
        // few slots: the weight-streaming decode layer, no grouped rows
        CUDA_TRY(launch_decode_layer(p, x, nullptr, nullptr, idx, p.topk_w, nullptr, w_gate, w_up, w_down, ws_gate,
                                     ws_up, ws_down, y, counts, dropped, st),
                 "decode_layer");
        return MOE_OK;
    }
    CUDA_TRY(launch_permute(p, idx, counts, p.offsets, p.perm_rows, p.row_of, dropped, st), "permute");
    moe_status_t s = run_ffn(p, x, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, 1, p.rows, p.row_of, st);
    if (s != MOE_OK) return s;
    CUDA_TRY(launch_combine_rows(p, p.rows, p.row_of, y, st), "combine_rows");
    return MOE_OK;
}

extern "C" {

moe_status_t moe_forward(const moe_config_t* cfg, const void* x, const void* router_w,
                         const float* router_b, const void* w_gate, const void* w_up,
                         const void* w_down, const void* ws_gate, const void* ws_up,
                         const void* ws_down, void* y, int32_t* topk_idx_out, int32_t* counts_out,
                         int32_t* dropped_out, void* ws, size_t ws_bytes, moe_stream_t stream) {
    Plan p;
    moe_status_t s = plan_for(cfg, ws, ws_bytes, &p);
    if (s != MOE_OK) return s;
    OPTIONAL_PTR(topk_idx_out);
    OPTIONAL_PTR(counts_out);
    OPTIONAL_PTR(dropped_out);
    cudaStream_t st = (cudaStream_t)stream;
    if (p.T == 0) {
        if (counts_out) CUDA_TRY(cudaMemsetAsync(counts_out, 0, sizeof(int32_t) * p.E, st), "memset");
        if (dropped_out) CUDA_TRY(cudaMemsetAsync(dropped_out, 0, sizeof(int32_t) * p.E, st), "memset");
        return MOE_OK;
    }
    REQUIRE_PTR(x);
    REQUIRE_PTR(router_w);
    OPTIONAL_PTR(router_b);
    REQUIRE_PTR(w_gate);
    REQUIRE_PTR(w_up);
    REQUIRE_PTR(w_down);
    REQUIRE_PTR(y);
    if ((s = check_shared(p, ws_gate, ws_up, ws_down)) != MOE_OK) return s;

    int32_t* idx = topk_idx_out ? topk_idx_out : p.topk_idx;
    int32_t* counts = counts_out ? counts_out : p.counts;
    int32_t* dropped = dropped_out ? dropped_out : p.dropped;
    if (decode_ffn_eligible(p)) {
        // few slots: routing, expert FFNs and combine in one decode kernel
        CUDA_TRY(launch_decode_layer(p, x, router_w, router_b, nullptr, nullptr, topk_idx_out, w_gate, w_up, w_down,
                                     ws_gate, ws_up, ws_down, y, counts, dropped, st),
                 "decode_layer");
        return MOE_OK;
    }
    CUDA_TRY(run_router(p, x, router_w, router_b, idx, p.topk_w, st), "router");
    return forward_after_routing(p, x, idx, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, y, counts, dropped, st);
}

moe_status_t moe_forward_routed(const moe_config_t* cfg, const void* x, const int32_t* topk_idx,
                                const float* topk_w, const int32_t* capacity_left, const void* w_gate,
                                const void* w_up, const void* w_down, const void* ws_gate, const void* ws_up,
                                const void* ws_down, void* y, int32_t* counts_out, int32_t* dropped_out,
                                void* ws, size_t ws_bytes, moe_stream_t stream) {
    Plan p;
    moe_status_t s = plan_for(cfg, ws, ws_bytes, &p);
    if (s != MOE_OK) return s;
    OPTIONAL_PTR(capacity_left);
    OPTIONAL_PTR(counts_out);
    OPTIONAL_PTR(dropped_out);
    cudaStream_t st = (cudaStream_t)stream;
    if (p.T == 0) {
        if (counts_out) CUDA_TRY(cudaMemsetAsync(counts_out, 0, sizeof(int32_t) * p.E, st), "memset");
        if (dropped_out) CUDA_TRY(cudaMemsetAsync(dropped_out, 0, sizeof(int32_t) * p.E, st), "memset");
        return MOE_OK;
    }
    REQUIRE_PTR(x);
    REQUIRE_PTR(topk_idx);
    REQUIRE_PTR(topk_w);
    REQUIRE_PTR(w_gate);
    REQUIRE_PTR(w_up);
    REQUIRE_PTR(w_down);
    REQUIRE_PTR(y);
    if ((s = check_shared(p, ws_gate, ws_up, ws_down)) != MOE_OK) return s;
    p.topk_w = const_cast<float*>(topk_w);  // read only on this path
    if (capacity_left) {
        p.cap_left_arr = capacity_left;  // the shard's capacities replace cfg's
        p.cap = INT32_MAX;               // marks the layer as capped
    }
    int32_t* counts = counts_out ? counts_out : p.counts;
    int32_t* dropped = dropped_out ? dropped_out : p.dropped;
    return forward_after_routing(p, x, topk_idx, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, y, counts, dropped,
                                 st);
}

static moe_status_t check_shard_args(const moe_config_t* cfg, const int32_t* counts, int32_t n_shards,
                                     int32_t shard, const int32_t* out, int64_t* C) {
    moe_status_t s = check_config(cfg);
    if (s != MOE_OK) return s;
    *C = capacity_of(cfg);
    if (*C <= 0) return fail(MOE_ERR_INVALID_ARG, "the batch has no capacity limit (capacity_factor <= 0)");
    if (n_shards < 1) return fail(MOE_ERR_INVALID_ARG, "n_shards = %d < 1", n_shards);
    if (shard < 0 || shard >= n_shards)
        return fail(MOE_ERR_INVALID_ARG, "shard = %d outside [0, %d)", shard, n_shards);
    if (!counts) return fail(MOE_ERR_INVALID_ARG, "counts_per_shard is NULL");
    if (!out) return fail(MOE_ERR_INVALID_ARG, "capacity_left is NULL");
    return MOE_OK;
}

moe_status_t moe_shard_capacity_left(const moe_config_t* cfg, const int32_t* counts_per_shard, int32_t n_shards,
                                     int32_t shard, int32_t* capacity_left, moe_stream_t stream) {
    int64_t C = 0;
    moe_status_t s = check_shard_args(cfg, counts_per_shard, n_shards, shard, capacity_left, &C);
    if (s != MOE_OK) return s;
    CUDA_TRY(launch_shard_capacity_left(C, counts_per_shard, n_shards, shard, cfg->E, capacity_left,
                                        (cudaStream_t)stream),
             "shard_capacity_left");
    return MOE_OK;
}

moe_status_t moe_shard_capacity_left_host(const moe_config_t* cfg, const int32_t* counts_per_shard,
                                          int32_t n_shards, int32_t shard, int32_t* capacity_left) {
    int64_t C = 0;
    moe_status_t s = check_shard_args(cfg, counts_per_shard, n_shards, shard, capacity_left, &C);
    if (s != MOE_OK) return s;
    shard_capacity_left_host(C, counts_per_shard, n_shards, shard, cfg->E, capacity_left);
    return MOE_OK;
}

// Load-balance penalties in fp64 from importance [E] and load [E] (host
// arrays): KL from uniform to the mean gate probability, std(importance) +
// std(load) (unbiased), and E * sum f_e P_e.  Sums run in expert order.
moe_status_t moe_balance_losses(int32_t E, int64_t T, const float* importance, const int32_t* load,
                                double* out) {
    if (E < 2) return fail(MOE_ERR_INVALID_ARG, "E = %d: the penalties need at least 2 experts", E);
    if (T <= 0) return fail(MOE_ERR_INVALID_ARG, "T = %lld must be positive", (long long)T);
    if (!importance || !load || !out) return fail(MOE_ERR_INVALID_ARG, "importance, load and out are required");
    const double inv_e = 1.0 / E, tt = (double)T;
    double kl = 0.0, sum_i = 0.0, sum_l = 0.0, sw = 0.0;
    for (int e = 0; e < E; ++e) {
        const double q = (double)importance[e] / tt;
        kl += inv_e * (log(inv_e) - log(q + 1e-8));
        sum_i += importance[e];
        sum_l += load[e];
        sw += ((double)load[e] / tt) * q;
    }
    const double mi = sum_i / E, ml = sum_l / E;
    double vi = 0.0, vl = 0.0;
    for (int e = 0; e < E; ++e) {
        const double di = importance[e] - mi, dl = load[e] - ml;
        vi += di * di;
        vl += dl * dl;
    }
    out[0] = kl / E;
    out[1] = sqrt(vi / (E - 1)) + sqrt(vl / (E - 1));
    out[2] = E * sw;
    return MOE_OK;
}

moe_status_t moe_forward_expert_shard(const moe_config_t* cfg, const void* x, const int32_t* topk_idx,
                                      const float* topk_w, int32_t expert_begin, int32_t expert_count,
                                      const void* w_gate, const void* w_up, const void* w_down, const void* ws_gate,
                                      const void* ws_up, const void* ws_down, float* y_partial, int32_t* counts_out,
                                      int32_t* dropped_out, void* ws, size_t ws_bytes, moe_stream_t stream) {
    moe_status_t s = check_config(cfg);
    if (s != MOE_OK) return s;
    if (expert_count < 1 || expert_begin < 0 || (int64_t)expert_begin + expert_count > cfg->E)
        return fail(MOE_ERR_INVALID_ARG, "experts [%d, %d + %d) outside [0, %d)", expert_begin, expert_begin,
                    expert_count, cfg->E);
    if (ws_gate && cfg->I_shared == 0)
        return fail(MOE_ERR_INVALID_ARG, "shared-expert weights given but I_shared = 0");
    // the shard's plan: its experts only, the shared expert where its weights
    // are given, the batch's capacity
    moe_config_t local = *cfg;
    local.E = expert_count;
    local.I_shared = ws_gate ? cfg->I_shared : 0;
    Plan p;
    make_plan(&local, nullptr, &p);
    if (!ws) return fail(MOE_ERR_WORKSPACE, "workspace is NULL");
    if ((uintptr_t)ws % kWsAlign) return fail(MOE_ERR_WORKSPACE, "workspace not %d-byte aligned", kWsAlign);
    if (ws_bytes < p.bytes) return fail(MOE_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, p.bytes);
    make_plan(&local, ws, &p);
    p.cap = capacity_of(cfg);
    p.drop_negative = true;
    p.y_f32 = true;
    OPTIONAL_PTR(counts_out);
    OPTIONAL_PTR(dropped_out);
    cudaStream_t st = (cudaStream_t)stream;
    if (p.T == 0) {
        if (counts_out) CUDA_TRY(cudaMemsetAsync(counts_out, 0, sizeof(int32_t) * p.E, st), "memset");
        if (dropped_out) CUDA_TRY(cudaMemsetAsync(dropped_out, 0, sizeof(int32_t) * p.E, st), "memset");
        return MOE_OK;
    }
    REQUIRE_PTR(x);
    REQUIRE_PTR(topk_idx);
    REQUIRE_PTR(topk_w);
    REQUIRE_PTR(w_gate);
    REQUIRE_PTR(w_up);
    REQUIRE_PTR(w_down);
    REQUIRE_PTR(y_partial);
    if ((s = check_shared(p, ws_gate, ws_up, ws_down)) != MOE_OK) return s;
    CUDA_TRY(launch_remap_experts(topk_idx, p.S, expert_begin, expert_count, p.topk_idx, st), "remap_experts");
    p.topk_w = const_cast<float*>(topk_w);  // read only on this path
    int32_t* counts = counts_out ? counts_out : p.counts;
    int32_t* dropped = dropped_out ? dropped_out : p.dropped;
    return forward_after_routing(p, x, p.topk_idx, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, y_partial, counts,
                                 dropped, st);
}

// Bytes of the bf16 copies of the gate, up and down weights that the MXFP4
// dequantizing path makes in the workspace after moe_forward's own scratch;
// 0 when the decode kernel or the MXFP4 GEMMs serve the size.
static size_t mxfp4_dequant_bytes(const Plan& p) {
    if (p.T == 0 || decode_mxfp4_eligible(p) || mx_gemm_eligible(p)) return 0;
    return align_up((size_t)3 * p.E * p.H * p.I * 2);
}

size_t moe_mxfp4_workspace_size(const moe_config_t* cfg) {
    if (check_config(cfg) != MOE_OK) return 0;
    Plan p;
    make_plan(cfg, nullptr, &p);
    return p.bytes + mxfp4_dequant_bytes(p);
}

moe_status_t moe_forward_mxfp4(const moe_config_t* cfg, const void* x, const void* router_w, const float* router_b,
                               const uint8_t* w_gate_blocks, const uint8_t* w_gate_scales, const uint8_t* w_up_blocks,
                               const uint8_t* w_up_scales, const uint8_t* w_down_blocks, const uint8_t* w_down_scales,
                               void* y, int32_t* topk_idx_out, int32_t* counts_out, int32_t* dropped_out, void* ws,
                               size_t ws_bytes, moe_stream_t stream) {
    Plan p;
    moe_status_t s = plan_for(cfg, ws, ws_bytes, &p);
    if (s != MOE_OK) return s;
    if (!p.bf16) return fail(MOE_ERR_UNSUPPORTED, "moe_forward_mxfp4 takes bf16 activations (dtype MOE_BF16)");
    if (p.Is > 0) return fail(MOE_ERR_UNSUPPORTED, "moe_forward_mxfp4 has no shared expert (I_shared must be 0)");
    if (p.H % 32 || p.I % 32) return fail(MOE_ERR_INVALID_ARG, "H and I must be multiples of 32 (MXFP4 blocks)");
    OPTIONAL_PTR(topk_idx_out);
    OPTIONAL_PTR(counts_out);
    OPTIONAL_PTR(dropped_out);
    cudaStream_t st = (cudaStream_t)stream;
    if (p.T == 0) {
        if (counts_out) CUDA_TRY(cudaMemsetAsync(counts_out, 0, sizeof(int32_t) * p.E, st), "memset");
        if (dropped_out) CUDA_TRY(cudaMemsetAsync(dropped_out, 0, sizeof(int32_t) * p.E, st), "memset");
        return MOE_OK;
    }
    const size_t dq_bytes = mxfp4_dequant_bytes(p);
    if (ws_bytes < p.bytes + dq_bytes)
        return fail(MOE_ERR_WORKSPACE,
                    "moe_forward_mxfp4 with %lld routed slots dequantizes the experts into the workspace: it needs "
                    "moe_mxfp4_workspace_size(cfg) = %zu bytes, got %zu",
                    (long long)p.S, p.bytes + dq_bytes, ws_bytes);
    REQUIRE_PTR(x);
    REQUIRE_PTR(router_w);
    OPTIONAL_PTR(router_b);
    REQUIRE_PTR(w_gate_blocks);
    REQUIRE_PTR(w_up_blocks);
    REQUIRE_PTR(w_down_blocks);
    if (!w_gate_scales || !w_up_scales || !w_down_scales)
        return fail(MOE_ERR_INVALID_ARG, "the three scale arrays are required");
    REQUIRE_PTR(y);
    const uint8_t* mx[6] = {w_gate_blocks, w_gate_scales, w_up_blocks, w_up_scales, w_down_blocks, w_down_scales};
    int32_t* counts = counts_out ? counts_out : p.counts;
    int32_t* dropped = dropped_out ? dropped_out : p.dropped;
    if (decode_mxfp4_eligible(p)) {
        // decode sizes: routing, the expert FFNs on the MXFP4 rows and the
        // combine in one weight-streaming kernel
        CUDA_TRY(launch_decode_layer_mxfp4(p, x, router_w, router_b, topk_idx_out, mx, y, counts, dropped, st),
                 "decode_layer_mxfp4");
        return MOE_OK;
    }
    int32_t* idx = topk_idx_out ? topk_idx_out : p.topk_idx;
    if (dq_bytes == 0) {
        // moe_forward's tile path with grouped GEMMs that read the MXFP4
        // codes and convert them to bf16 in shared memory
        CUDA_TRY(run_router(p, x, router_w, router_b, idx, p.topk_w, st), "router");
        CUDA_TRY(launch_permute(p, idx, counts, p.offsets, p.perm_rows, p.row_of, dropped, st), "permute");
        CUDA_TRY(launch_scatter_x_rows(p, x, p.row_of, p.xperm, st), "gather_rows");
        CUDA_TRY(launch_gateup_mx_sm100(p, mx[0], mx[1], mx[2], mx[3], st), "gateup_mx");
        CUDA_TRY(launch_down_mx_sm100(p, mx[4], mx[5], 1, p.rows, st), "down_mx");
        CUDA_TRY(launch_combine_rows(p, p.rows, p.row_of, y, st), "combine_rows");
        return MOE_OK;
    }
    // H or I above the MXFP4 GEMMs' limit: the weights dequantized (exactly)
    // to bf16 in the workspace, then moe_forward's routing, grouping, tcgen05
    // grouped GEMMs and combine
    bf16* wg = reinterpret_cast<bf16*>(static_cast<uint8_t*>(ws) + p.bytes);
    bf16* wu = wg + p.E * p.I * p.H;
    bf16* wd = wu + p.E * p.I * p.H;
    CUDA_TRY(launch_mxfp4_dequant(mx[0], mx[1], p.E * p.I, (int)p.H, wg, st), "mxfp4_dequant");
    CUDA_TRY(launch_mxfp4_dequant(mx[2], mx[3], p.E * p.I, (int)p.H, wu, st), "mxfp4_dequant");
    CUDA_TRY(launch_mxfp4_dequant(mx[4], mx[5], p.E * p.H, (int)p.I, wd, st), "mxfp4_dequant");
    CUDA_TRY(run_router(p, x, router_w, router_b, idx, p.topk_w, st), "router");
    return forward_after_routing(p, x, idx, wg, wu, wd, nullptr, nullptr, nullptr, y, counts, dropped, st);
}

moe_status_t moe_reduce_partials(const moe_config_t* cfg, const float* partials, int32_t n, void* y,
                                 moe_stream_t stream) {
    moe_status_t s = check_config(cfg);
    if (s != MOE_OK) return s;
    if (n < 1) return fail(MOE_ERR_INVALID_ARG, "n = %d < 1", n);
    if ((int64_t)cfg->T * cfg->H == 0) return MOE_OK;
    REQUIRE_PTR(partials);
    REQUIRE_PTR(y);
    CUDA_TRY(launch_reduce_partials(partials, n, (int64_t)cfg->T * cfg->H, cfg->dtype == MOE_BF16, y,
                                    (cudaStream_t)stream),
             "reduce_partials");
    return MOE_OK;
}

size_t moe_backward_workspace_size(const moe_config_t* cfg) {
    if (check_config(cfg) != MOE_OK) return 0;
    Plan p;
    make_plan(cfg, nullptr, &p);
    return p.bytes + backward_workspace_bytes(p);
}

moe_status_t moe_backward(const moe_config_t* cfg, const void* x, const void* dy, const int32_t* topk_idx,
                          const float* topk_w, const void* router_w, const void* w_gate, const void* w_up,
                          const void* w_down, const void* ws_gate, const void* ws_up, const void* ws_down, float* dx,
                          float* d_router_w, float* d_router_b, float* d_w_gate, float* d_w_up, float* d_w_down,
                          float* d_ws_gate, float* d_ws_up, float* d_ws_down, void* ws, size_t ws_bytes,
                          moe_stream_t stream) {
    moe_status_t s = check_config(cfg);
    if (s != MOE_OK) return s;
    if (cfg->dtype != MOE_BF16) return fail(MOE_ERR_UNSUPPORTED, "moe_backward takes the bf16 layer (MOE_BF16)");
    Plan p;
    make_plan(cfg, nullptr, &p);
    const size_t need = p.bytes + backward_workspace_bytes(p);
    if (!ws) return fail(MOE_ERR_WORKSPACE, "workspace is NULL");
    if ((uintptr_t)ws % kWsAlign) return fail(MOE_ERR_WORKSPACE, "workspace not %d-byte aligned", kWsAlign);
    if (ws_bytes < need)
        return fail(MOE_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu (moe_backward_workspace_size)", ws_bytes,
                    need);
    make_plan(cfg, ws, &p);
    if (p.T == 0) return MOE_OK;
    REQUIRE_PTR(x);
    REQUIRE_PTR(dy);
    REQUIRE_PTR(topk_idx);
    REQUIRE_PTR(topk_w);
    REQUIRE_PTR(router_w);
    REQUIRE_PTR(w_gate);
    REQUIRE_PTR(w_up);
    REQUIRE_PTR(w_down);
    REQUIRE_PTR(dx);
    REQUIRE_PTR(d_router_w);
    REQUIRE_PTR(d_router_b);
    REQUIRE_PTR(d_w_gate);
    REQUIRE_PTR(d_w_up);
    REQUIRE_PTR(d_w_down);
    if ((s = check_shared(p, ws_gate, ws_up, ws_down)) != MOE_OK) return s;
    if ((s = check_shared(p, d_ws_gate, d_ws_up, d_ws_down)) != MOE_OK) return s;
    CUDA_TRY(launch_backward(p, (char*)ws + p.bytes, x, dy, topk_idx, topk_w, router_w, w_gate, w_up, w_down, ws_gate,
                             ws_up, ws_down, dx, d_router_w, d_router_b, d_w_gate, d_w_up, d_w_down, d_ws_gate,
                             d_ws_up, d_ws_down, (cudaStream_t)stream),
             "backward");
    return MOE_OK;
}

moe_status_t moe_get_device_status(const moe_config_t* cfg, void* ws, size_t ws_bytes,
                                   moe_stream_t stream, int32_t* flags_out) {
    Plan p;
    moe_status_t s = plan_for(cfg, ws, ws_bytes, &p);
    if (s != MOE_OK) return s;
    cudaStream_t st = (cudaStream_t)stream;
    int32_t flags = 0;
    CUDA_TRY(cudaMemcpyAsync(&flags, p.flags, sizeof(int32_t), cudaMemcpyDeviceToHost, st), "flags read");
    CUDA_TRY(cudaStreamSynchronize(st), "stream sync");
    CUDA_TRY(cudaMemsetAsync(p.flags, 0, sizeof(int32_t), st), "flags clear");
    CUDA_TRY(cudaStreamSynchronize(st), "stream sync");
    if (flags_out) *flags_out = flags;
    if (flags) return fail(MOE_ERR_DEVICE_CHECK, "device check flags 0x%x", flags);
    return MOE_OK;
}

const char* moe_status_string(moe_status_t status) {
    switch (status) {
        case MOE_OK: return "MOE_OK";
        case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
        case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
        case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
        case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
        case MOE_ERR_DEVICE_CHECK: return "MOE_ERR_DEVICE_CHECK";
    }
    return "MOE_ERR_UNKNOWN";
}

const char* moe_last_error(void) { return g_last_error; }

moe_status_t moe_trace_begin(int32_t max_launches, const char* only) {
    if (max_launches <= 0) return fail(MOE_ERR_INVALID_ARG, "max_launches = %d", max_launches);
    if (g_trace.on) return fail(MOE_ERR_INVALID_ARG, "tracing already on");
    g_trace = TraceState();
    if (only) {
        strncpy(g_trace.only, only, sizeof(g_trace.only) - 1);
        g_trace.only[sizeof(g_trace.only) - 1] = 0;
    }
    g_trace.ev.resize(2 * (size_t)max_launches);
    g_trace.names.resize(max_launches);
    for (auto& e : g_trace.ev)
        if (cudaEventCreate(&e) != cudaSuccess) {
            for (auto& f : g_trace.ev)
                if (f) cudaEventDestroy(f);
            g_trace = TraceState();
            return fail(MOE_ERR_CUDA, "cudaEventCreate failed");
        }
    g_trace.max = max_launches;
    g_trace.on = true;
    return MOE_OK;
}

moe_status_t moe_trace_end(moe_trace_record_t* records, int32_t max_records, int32_t* n_records) {
    if (!g_trace.on) return fail(MOE_ERR_INVALID_ARG, "tracing is off");
    moe_status_t st = MOE_OK;
    int n = g_trace.n;
    if (n > 0 && cudaEventSynchronize(g_trace.ev[2 * n - 1]) != cudaSuccess)
        st = fail(MOE_ERR_CUDA, "cudaEventSynchronize failed");
    int w = 0;
    for (int i = 0; i < n && st == MOE_OK && records && w < max_records; ++i, ++w) {
        float ms = 0.f;
        cudaEventElapsedTime(&ms, g_trace.ev[2 * i], g_trace.ev[2 * i + 1]);
        records[w].name = g_trace.names[i];
        records[w].ms = ms;
    }
    if (n_records) *n_records = w;
    for (auto& e : g_trace.ev) cudaEventDestroy(e);
    g_trace = TraceState();
    return st;
}

}  // extern "C"
