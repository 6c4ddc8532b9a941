/*
 * moe.h -- C ABI of the B200 (sm_100a) routed Mixture-of-Experts FFN layer.
 *
 * The layer computes, for every token t of x [T, H]:
 *
 *   l[t, e]  = x[t] . router_w[e] + router_b[e]                 (router scores)
 *   S_t      = the top_k experts by score (ties: lower index)     (selection)
 *   w[t, j]  = softmax over the top_k selected scores            (gating)
 *   y[t]     = sum_{j kept} w[t,j] * FFN_{S_t[j]}(x[t])  (+ shared FFN(x[t]))
 *   FFN_e(v) = W_down[e] (silu(W_gate[e] v) * (W_up[e] v))         (SwiGLU)
 *
 * Sources (page title, section):
 *   "MoE稀疏架构是什么？从原理到落地的系统解读", section 四 (one forward pass:
 *     router scores, top-k, softmax over the chosen scores, weighted sum of
 *     the chosen experts; unchosen experts are not evaluated); section 三.1
 *     (the router is a small linear layer); section 三.2 (capacity-limited
 *     token dropping).
 *   "Mixture of Experts (MoEs) in Transformers", section Weight Loading
 *     Refactor (all experts packed in one [E, out, in] tensor; gate = w1,
 *     up = w3, down = w2), section Expert Backend (grouped_mm: tokens sorted
 *     and grouped by expert id, then one grouped GEMM).
 *   "模型的“分工的艺术”：MoE技术如何提升计算效率", section 3.1 (expert capacity).
 *
 * Readings where the pages are silent: ties go to the lower expert index;
 * the expert FFN is SwiGLU without biases; capacity C = ceil(cf * T * k / E)
 * (taken with a relative tolerance of 1e-6, so that the float32 rounding of
 * cf does not lift an exact integer to the next one)
 * with tokens served in ascending token order, a dropped (token, expert)
 * pair contributes nothing and the token's other weights are not
 * renormalised; a shared expert (I_shared > 0) is always applied with
 * weight 1.
 *
 * Conventions for every entry point below
 *   - All tensor pointers are DEVICE pointers owned by the caller, row-major
 *     and contiguous, 16-byte aligned.  The library never allocates, frees
 *     or synchronises inside a compute call and keeps no pointer after the
 *     call returns.  Work is enqueued on `stream` in stream order.
 *   - dtype MOE_BF16: x, router_w, expert weights and y are bfloat16;
 *     MOE_F32: all of them float32.  router_b, topk_w are always float32.
 *   - Layouts: x, y [T, H]; router_w [E, H]; router_b [E];
 *     w_gate, w_up [E, I, H]; w_down [E, H, I];
 *     ws_gate, ws_up [I_shared, H]; ws_down [H, I_shared];
 *     topk_idx int32 [T, top_k]; topk_w float32 [T, top_k].
 *   - Slot id s = t * top_k + j names the j-th choice of token t.
 *   - `ws` is scratch device memory of at least moe_workspace_size(cfg)
 *     bytes, 256-byte aligned; its contents are undefined between calls,
 *     except that device-side check flags persist until
 *     moe_get_device_status() reads and clears them.  A new workspace must
 *     start zeroed (or be cleared by one moe_get_device_status() call) for
 *     those flags to mean anything.  Calls that share one workspace must be
 *     ordered on the GPU (the same stream, or joined).
 *   - Errors in arguments, shapes or alignment return synchronously, before
 *     anything is enqueued.  A failed launch returns MOE_ERR_CUDA.
 *     Data-dependent faults found on the device (an expert index out of
 *     range fed to moe_permute) set a flag in `ws` and the offending entry
 *     is skipped; moe_get_device_status() reports them.  No kernel traps.
 *   - moe_last_error() gives a one-line reason for the last failure of the
 *     calling thread.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* moe_stream_t; /* same object as cudaStream_t */

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,  /* null pointer, bad shape, misaligned pointer */
    MOE_ERR_UNSUPPORTED = 2,  /* valid but outside this build's limits       */
    MOE_ERR_WORKSPACE = 3,    /* ws too small or misaligned                  */
    MOE_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed        */
    MOE_ERR_DEVICE_CHECK = 5  /* a device-side check fired (see status)      */
} moe_status_t;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype_t;

typedef struct {
    int32_t T;               /* tokens, >= 0 (0 is a valid no-op)             */
    int32_t H;               /* hidden size, multiple of 8                     */
    int32_t I;               /* expert intermediate size, multiple of 8        */
    int32_t E;               /* routed experts, 1..256                         */
    int32_t top_k;           /* 1..min(E, 8), or top_k == E when E <= 32       */
    int32_t I_shared;        /* shared expert intermediate size, 0 = none      */
    float capacity_factor;   /* <= 0: unlimited; else C = ceil(cf*T*top_k/E)   */
    int32_t dtype;           /* moe_dtype_t                                    */
} moe_config_t;

/* Device-side check flags reported by moe_get_device_status(). */
#define MOE_DEVFLAG_BAD_EXPERT_INDEX 0x1 /* moe_permute saw idx < 0 or >= E    */
#define MOE_DEVFLAG_WAIT_TIMEOUT 0x2     /* a bounded device wait gave up      */

/* Bytes of workspace every entry point below needs for `cfg`; 0 if the
 * configuration is invalid (moe_last_error() says why). */
size_t moe_workspace_size(const moe_config_t* cfg);

/* Per-expert capacity C for cfg (0 = unlimited). */
int64_t moe_capacity(const moe_config_t* cfg);

/*
 * moe_route -- router scores, top-k selection and softmax over the
 * selected scores ("MoE稀疏架构是什么？从原理到落地的系统解读", sections 三.1
 * and 四).  Scores are never rounded to bf16.  bf16 with T*E*H > 2^26:
 * float32 tensor-core sums, and the experts near a token's k-th/(k+1)-th
 * boundary are rescored exactly in fp64 before the choice.  Otherwise
 * (few tokens): every score exact up to fp64 rounding (bf16 products are
 * exact in float32).  float32 layer with many tokens: float32 FMAs.
 *   x [T,H], router_w [E,H], router_b [E] float32 or NULL
 *   -> topk_idx [T,top_k] int32: chosen experts, score descending, ties to
 *      the lower index; topk_w [T,top_k] float32: softmax of those scores.
 */
moe_status_t moe_route(const moe_config_t* cfg, const void* x, const void* router_w,
                       const float* router_b, int32_t* topk_idx, float* topk_w, void* ws,
                       size_t ws_bytes, moe_stream_t stream);

/*
 * moe_route_importance -- moe_route plus the router statistic that the
 * load-balance penalties start from ("2026年人工智能MoE混合专家模型入门指南",
 * the MoE layer's importance = softmax probabilities summed over tokens;
 * "模型的“分工的艺术”：MoE技术如何提升计算效率", section 3.1, mean gate
 * probability per expert = importance / T).  topk_idx and topk_w are those
 * of moe_route, bit for bit.
 *   importance [E] float32, device, 16-byte aligned, required: ADDED to
 *   (the caller zeroes it, or keeps summing over batches):
 *   importance[e] += sum over tokens t of exp(s[t,e] - m_t) / sum_e' exp(s[t,e'] - m_t),
 *   s the router scores with bias, m_t the token's largest score.  The
 *   probabilities come from the scores moe_route computes (float32
 *   tensor-core sums on the tensor-core path; exact scores on the few-token
 *   path) and are summed with float32 atomic adds, so the order of the sum,
 *   and its last bits, vary from run to run.  With T = 0 nothing is added.
 * The top-k counts, the other statistic, come from moe_permute (counts) or
 * moe_forward (counts_out).  Errors: as moe_route, and importance NULL or
 * misaligned is MOE_ERR_INVALID_ARG.
 */
moe_status_t moe_route_importance(const moe_config_t* cfg, const void* x, const void* router_w,
                                  const float* router_b, int32_t* topk_idx, float* topk_w, float* importance,
                                  void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * moe_permute -- group (token, slot) pairs by expert, with capacity drop in
 * token order ("Mixture of Experts (MoEs) in Transformers", section Expert
 * Backend: grouped_mm sorts tokens by expert id; "MoE稀疏架构是什么？…",
 * section 三.2: capacity-limited dropping).
 *   topk_idx [T,top_k] int32 ->
 *   counts [E]      pairs per expert before the capacity cut
 *   dropped [E]     pairs per expert beyond the capacity
 *   offsets [E+1]   first kept row of each expert; offsets[E] = kept rows R
 *   perm_rows [T*top_k]  slot id of each row; an expert's rows in ascending
 *                   token order; entries >= R are set to -1
 *   row_of [T*top_k]     row of each slot, -1 if dropped
 * Every output is a pure function of topk_idx (bit-reproducible).
 * An index outside [0, E) sets MOE_DEVFLAG_BAD_EXPERT_INDEX and the slot is
 * treated as dropped without being counted.
 */
moe_status_t moe_permute(const moe_config_t* cfg, const int32_t* topk_idx, int32_t* counts,
                         int32_t* offsets, int32_t* perm_rows, int32_t* row_of, int32_t* dropped,
                         void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * moe_permute_noalloc -- moe_permute for callers that cannot allocate
 * device memory: code running inside an allocator or memory-pool callback,
 * plugins whose host application owns every device allocation, serving
 * loops that forbid allocation after start-up.  The pages have no
 * counterpart of this entry point; it only changes where the scratch lives.
 *   Same arguments, outputs and bit-exact results as moe_permute, without
 *   `ws`: the grouping kernels' scratch (about 520 KB) is a fixed array in
 *   the library's device memory.  A GPU holds that array from the moment
 *   the library's grouping code is loaded on it (the first grouping call of
 *   any entry point on that device, or context creation when CUDA loads
 *   modules eagerly) until the process exits.
 *   Set-up: the first call on each device (each CUDA context) loads that
 *   code if it is not loaded yet, which itself takes device memory, and
 *   looks up the array's device address.  Make that first call at
 *   start-up, outside any allocator callback and before any stream capture;
 *   every later call in the same context allocates nothing (no cudaMalloc,
 *   no allocating library routine).  After cudaDeviceReset the next call is
 *   a first call again.
 *   Limit: T * top_k <= 1048576 slots (E <= 256 as everywhere); larger
 *   inputs return MOE_ERR_UNSUPPORTED before anything is enqueued.
 *   Every call on a device shares the one array, which keeps the last
 *   call's contents; calls that overlap on the GPU (concurrent streams)
 *   race and give wrong results, so order them.  An expert index outside
 *   [0, E) is skipped as in moe_permute but not reported: there is no
 *   workspace to hold the flag.
 */
moe_status_t moe_permute_noalloc(const moe_config_t* cfg, const int32_t* topk_idx, int32_t* counts,
                                 int32_t* offsets, int32_t* perm_rows, int32_t* row_of,
                                 int32_t* dropped, moe_stream_t stream);

/*
 * moe_grouped_ffn -- every kept row through its expert's SwiGLU FFN, as
 * grouped GEMMs over the rows of each expert ("Mixture of Experts (MoEs) in
 * Transformers", section Expert Backend, grouped_mm).
 *   x [T,H]; perm_rows, offsets as produced by moe_permute;
 *   w_gate, w_up [E,I,H]; w_down [E,H,I]; shared weights or NULLs;
 *   -> expert_out float32 [T*top_k + (I_shared ? T : 0), H]:
 *      row r < offsets[E] holds FFN_e(x[perm_rows[r] / top_k]) (unweighted);
 *      row T*top_k + t holds the shared expert's FFN(x[t]).
 *      Rows in [offsets[E], T*top_k) are left untouched.
 * Intermediate activations are rounded to the layer dtype (bf16 for
 * MOE_BF16) between the two GEMMs; accumulation is float32.
 */
moe_status_t moe_grouped_ffn(const moe_config_t* cfg, const void* x, const int32_t* perm_rows,
                             const int32_t* offsets, const void* w_gate, const void* w_up,
                             const void* w_down, const void* ws_gate, const void* ws_up,
                             const void* ws_down, float* expert_out, void* ws, size_t ws_bytes,
                             moe_stream_t stream);

/*
 * moe_combine -- weighted un-permute ("MoE稀疏架构是什么？…", section 四:
 * the output is the weight-scaled sum of the chosen experts' outputs).
 *   y[t] = sum_{j : row_of[t,j] >= 0} topk_w[t,j] * expert_out[row_of[t,j]]
 *          + (I_shared ? expert_out[T*top_k + t] : 0),  summed in float32
 *   in order j = 0..top_k-1 then the shared row, rounded once to the dtype.
 */
moe_status_t moe_combine(const moe_config_t* cfg, const float* expert_out, const int32_t* row_of,
                         const float* topk_w, void* y, void* ws, size_t ws_bytes,
                         moe_stream_t stream);

/*
 * moe_forward -- the whole layer, the C form of the pages' moe_forward(x,
 * experts, router, top_k) ("MoE稀疏架构是什么？…", section 四): route,
 * group, grouped gate/up GEMM with the SwiGLU fused in its epilogue, grouped
 * down GEMM with the routing-weight scale fused in its epilogue (each kept
 * row's w * FFN_e(x) stored in the layer dtype), then the un-permute: each
 * token's rows summed in float32 in slot order (then the shared row) and
 * rounded once to the layer dtype.
 *   y [T,H] (layer dtype).  Optional outputs (NULL to skip): topk_idx_out
 *   [T,top_k] int32, counts_out [E] and dropped_out [E] int32.
 * With T*top_k <= 8 (bf16) no rows are grouped: one cooperative
 * weight-streaming kernel reads each selected expert's weight rows once and
 * sums each token's k weighted FFN outputs (then the shared expert's) in
 * float32 in slot order, rounded once; the routed outputs are not rounded to
 * bf16 before that sum.
 * y is bit-reproducible for given inputs (fixed summation order; the only
 * atomics are arrival counters that pick which warp does a fixed-order sum).
 */
moe_status_t moe_forward(const moe_config_t* cfg, const void* x, const void* router_w,
                         const float* router_b, const void* w_gate, const void* w_up,
                         const void* w_down, const void* ws_gate, const void* ws_up,
                         const void* ws_down, void* y, int32_t* topk_idx_out, int32_t* counts_out,
                         int32_t* dropped_out, void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * moe_forward_routed -- the layer after routing, for one shard of a batch's
 * tokens ("MoE稀疏架构是什么？…", section 三.2: capacity-limited dropping).
 * Capacity is served in global token order, so a shard's capacity for an
 * expert is what the earlier shards left of it.
 *   x [T,H] (this shard's tokens); topk_idx [T,top_k] int32 and topk_w
 *   [T,top_k] float32 as moe_route produces them; capacity_left [E] int32 or
 *   NULL.  With capacity_left, a slot of expert e is kept iff fewer than
 *   capacity_left[e] earlier slots of e in this shard were kept, and
 *   cfg->capacity_factor is not used.  For shard r of a batch with capacity
 *   C: capacity_left[e] = max(0, C - sum over shards q < r of counts_q[e]),
 *   counts_q being shard q's counts (gathered from every shard).  NULL: the
 *   capacity of cfg applies, as in moe_forward.
 *   -> y [T,H], and optionally counts_out / dropped_out [E] for this shard.
 * With capacity_left NULL and the routing of moe_route, y equals
 * moe_forward's bit for bit.
 */
moe_status_t moe_forward_routed(const moe_config_t* cfg, const void* x, const int32_t* topk_idx,
                                const float* topk_w, const int32_t* capacity_left, const void* w_gate,
                                const void* w_up, const void* w_down, const void* ws_gate, const void* ws_up,
                                const void* ws_down, void* y, int32_t* counts_out, int32_t* dropped_out,
                                void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * moe_shard_capacity_left -- per-expert capacity left for one token shard of
 * a capacity-limited batch ("MoE稀疏架构是什么？…", section 三.2: an expert
 * takes tokens up to its capacity and drops the rest; capacity is served in
 * global token order, so a shard gets what the earlier shards left of it).
 *   cfg describes the WHOLE batch: cfg->T is the tokens of all shards
 *   together, so C = moe_capacity(cfg), which must be > 0.
 *   counts_per_shard [n_shards, E] int32, device: every shard's per-expert
 *   counts before the capacity cut (moe_permute counts, or moe_forward_routed
 *   counts_out with capacity_left NULL), gathered from all shards, shards in
 *   token order.
 *   -> capacity_left [E] int32, device:
 *      capacity_left[e] = max(0, C - sum over shards q < shard of counts_q[e]),
 *   the argument moe_forward_routed takes for that shard.  One small kernel
 *   on `stream`; the counts never leave the device.
 * Errors: no capacity (cfg->capacity_factor <= 0), n_shards < 1 or shard
 * outside [0, n_shards) -> MOE_ERR_INVALID_ARG, before anything is enqueued.
 */
moe_status_t moe_shard_capacity_left(const moe_config_t* cfg, const int32_t* counts_per_shard, int32_t n_shards,
                                     int32_t shard, int32_t* capacity_left, moe_stream_t stream);

/* moe_shard_capacity_left on HOST arrays (counts gathered on the host, e.g.
 * by a CPU process group): same arguments and result, computed on the
 * calling thread, no CUDA call. */
moe_status_t moe_shard_capacity_left_host(const moe_config_t* cfg, const int32_t* counts_per_shard,
                                          int32_t n_shards, int32_t shard, int32_t* capacity_left);

/*
 * moe_balance_losses -- the load-balance penalties from the two per-expert
 * router statistics, on HOST arrays (2*E numbers; no CUDA call), in fp64:
 *   q_e = importance[e] / T (mean gate probability),
 *   out[0] kl     = (1/E) sum_e (1/E) (log(1/E) - log(q_e + 1e-8)):
 *                   KL from uniform to the mean gate probability, the batch
 *                   mean over the E-vector ("模型的“分工的艺术”：MoE技术如何
 *                   提升计算效率", section 3.1);
 *   out[1] std    = std(importance) + std(load), unbiased (divisor E - 1)
 *                   ("2026年人工智能MoE混合专家模型入门指南", the MoE layer's
 *                   load-balance loss; the page's load, a count of positive
 *                   dense-softmax probabilities, is T for every expert, so
 *                   the top-k counts stand in for it);
 *   out[2] switch = E * sum_e (load[e] / T) * q_e, the Switch-Transformer
 *                   form (fraction of tokens routed to e times its mean gate
 *                   probability).
 *   importance [E] float32 (from moe_route_importance), load [E] int32 (the
 *   top-k counts from moe_permute or moe_forward), T the tokens they cover.
 * Errors: E < 2, T <= 0 or a NULL pointer -> MOE_ERR_INVALID_ARG.
 */
moe_status_t moe_balance_losses(int32_t E, int64_t T, const float* importance, const int32_t* load,
                                double* out);

/*
 * moe_forward_expert_shard -- this device's share of the layer under expert
 * parallelism ("Mixture of Experts (MoEs) in Transformers", section Expert
 * Parallelism: each device holds a slice of the experts along their first
 * dimension; the router's global expert indices are remapped to local ones,
 * experts the device does not hold are left out, and the devices' partial
 * outputs are summed with an all-reduce).
 *   cfg describes the whole layer: E all experts, the batch's T tokens and
 *   capacity factor (capacity is per expert and global: C = moe_capacity(cfg),
 *   served in token order over all T tokens, which every shard sees).
 *   x [T,H]; topk_idx [T,top_k] int32 and topk_w [T,top_k] float32 as
 *   moe_route produces them for the whole layer (replicated routing).
 *   This shard holds experts [expert_begin, expert_begin + expert_count):
 *   w_gate, w_up [expert_count, I, H], w_down [expert_count, H, I].
 *   ws_gate, ws_up, ws_down: the shared expert's weights on exactly one
 *   shard (cfg->I_shared > 0), NULL on the others.
 *   -> y_partial [T,H] float32: sum over this shard's kept (token, expert)
 *      pairs of w * FFN_e(x[t]) in slot order (+ the shared expert's FFN
 *      where its weights are given), each pair's output rounded to the layer
 *      dtype as in moe_forward; counts_out / dropped_out [expert_count]
 *      (nullable): the shard's experts' counts before the capacity cut and
 *      dropped pairs.
 * The sum of all shards' y_partial, rounded once (moe_reduce_partials after
 * an all-reduce of y_partial, or on the stacked partials of one device), is
 * the layer's output up to float32 summation order.  Workspace:
 * moe_workspace_size(cfg) bytes suffice.  Errors as moe_forward_routed, and
 * an expert range outside [0, E) is MOE_ERR_INVALID_ARG.
 */
moe_status_t moe_forward_expert_shard(const moe_config_t* cfg, const void* x, const int32_t* topk_idx,
                                      const float* topk_w, int32_t expert_begin, int32_t expert_count,
                                      const void* w_gate, const void* w_up, const void* w_down, const void* ws_gate,
                                      const void* ws_up, const void* ws_down, float* y_partial, int32_t* counts_out,
                                      int32_t* dropped_out, void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * moe_mxfp4_workspace_size -- bytes of workspace moe_forward_mxfp4 needs for
 * cfg: moe_workspace_size(cfg), plus the bf16 copies of the expert weights
 * (3*E*H*I*2 bytes, 256-aligned) when the size takes the converting path
 * (more than 128 rows per expert, or H or I above 3072).  0 for an invalid
 * cfg (see moe_last_error).
 */
size_t moe_mxfp4_workspace_size(const moe_config_t* cfg);

/*
 * moe_forward_mxfp4 -- moe_forward with the routed experts' weights in the
 * MXFP4 format of the OCP Microscaling (MX) v1.0 specification
 * ("Mixture of Experts (MoEs) in Transformers", section From Dense to
 * Sparse: the gpt-oss generation speed is set by the bytes of the active
 * parameters, and native mxfp4 kernels would raise it further).  An element
 * is FP4 E2M1 (sign, 2 exponent bits with bias 1, 1 mantissa bit); each
 * block of 32 elements along the reduction dimension shares one E8M0 scale
 * byte s standing for 2^(s - 127) (s = 255: NaN).  Storage order (the pages
 * give none): two codes per byte, the element with the lower index in the
 * low nibble; a row's blocks are contiguous.
 *   w_gate_blocks, w_up_blocks [E, I, H/32, 16] uint8; w_gate_scales,
 *   w_up_scales [E, I, H/32] uint8; w_down_blocks [E, H, I/32, 16],
 *   w_down_scales [E, H, I/32].  Blocks 16-byte aligned; scales any alignment.
 *   x, router_w, y bf16 (cfg->dtype MOE_BF16); the router is moe_forward's.
 * The weights are used exactly (every dequantized value is exact in float32).
 * On the decode kernel each block's 32 products are summed in f16 with the
 * token vector scaled by a power of two into f16's range, and the blocks'
 * sums in float32; on the tile paths the tensor cores multiply the bf16
 * activations by the weights converted to bf16 and accumulate in float32.
 * h is rounded to bf16 between the two projections as in moe_forward.
 * Three paths by size.  T * top_k <= 32 (gpt-oss-sized layers up to T = 8)
 * with the decode kernel's shared memory within 200 KB (the token vectors,
 * T*H*2 bytes, one expert's h vectors, T*I*2 bytes, and the partial dots):
 * one weight-streaming kernel reads the MXFP4 rows themselves.  Up to 128
 * rows per expert on average (T * top_k <= 128 * E) with H and I <= 3072:
 * moe_forward's tile path with grouped GEMMs that read the codes and scales
 * and convert them to bf16 in shared memory.  Both take a workspace of
 * moe_workspace_size(cfg).  Otherwise the gate, up and down weights are
 * converted to bf16 into the workspace after moe_forward's scratch, then
 * moe_forward's tile path runs on them; the workspace must hold
 * moe_mxfp4_workspace_size(cfg) bytes (3*E*H*I*2 more), else
 * MOE_ERR_WORKSPACE.  Every path uses each dequantized value e * 2^(s-127)
 * exactly (bf16 holds it down to 2^-133; above bf16's range it becomes
 * +-inf).  No shared expert (I_shared = 0), H and I multiples of 32;
 * otherwise MOE_ERR_UNSUPPORTED / MOE_ERR_INVALID_ARG.
 * Every error is returned before anything is enqueued.  Outputs and errors
 * otherwise as moe_forward.
 */
moe_status_t moe_forward_mxfp4(const moe_config_t* cfg, const void* x, const void* router_w, const float* router_b,
                               const uint8_t* w_gate_blocks, const uint8_t* w_gate_scales, const uint8_t* w_up_blocks,
                               const uint8_t* w_up_scales, const uint8_t* w_down_blocks, const uint8_t* w_down_scales,
                               void* y, int32_t* topk_idx_out, int32_t* counts_out, int32_t* dropped_out, void* ws,
                               size_t ws_bytes, moe_stream_t stream);

/*
 * moe_reduce_partials -- y = sum over i < n of partials[i], float32 in order
 * i = 0..n-1, rounded once to the layer dtype: the last step of an
 * expert-parallel layer (n = 1 after an all-reduce of the partial outputs).
 *   partials [n, T, H] float32, y [T, H] layer dtype (cfg->dtype), device.
 */
moe_status_t moe_reduce_partials(const moe_config_t* cfg, const float* partials, int32_t n, void* y,
                                 moe_stream_t stream);

/*
 * moe_backward -- every gradient of the layer for an upstream gradient dy
 * (the training use of the grouped-GEMM backend, "Mixture of Experts (MoEs)
 * in Transformers", section Training MoEs with Transformers), bf16 layer.
 * For a kept (token t, expert e) pair with weight w, g = W_gate[e] x,
 * u = W_up[e] x, h = silu(g) u (bf16 as in the forward):
 *   dW_down[e] += w dy h^T;  da = w W_down[e]^T dy;  dw = (W_down[e]^T dy) . h
 *   dW_gate[e] += (da u silu'(g)) x^T;  dW_up[e] += (da silu(g)) x^T
 *   dx += W_gate[e]^T (da u silu'(g)) + W_up[e]^T (da silu(g))
 * and through the softmax over the selected scores (every selected pair; a
 * pair the capacity dropped has dw = 0): dl_j = w_j (dw_j - sum_i w_i dw_i),
 * d_router_w[e_j] += dl_j x, d_router_b[e_j] += dl_j, dx += dl_j router_w[e_j].
 * The shared expert (I_shared > 0) is one more expert with w = 1.  The top-k
 * selection and the capacity cut carry no gradient.
 *   x, dy [T,H] bf16; topk_idx [T,top_k] int32 and topk_w [T,top_k] float32
 *   as moe_route gave them for this forward; router_w and the expert weights
 *   as in moe_forward.
 *   -> float32, written (not accumulated into): dx [T,H], d_router_w [E,H],
 *      d_router_b [E], d_w_gate, d_w_up [E,I,H], d_w_down [E,H,I], and with a
 *      shared expert d_ws_gate, d_ws_up [I_shared,H], d_ws_down [H,I_shared]
 *      (NULL otherwise).  Experts with no kept rows get exact zeros.
 * The products run as tcgen05 grouped GEMMs: the weight gradients reduce
 * over each expert's rows (operands read MN-major from shared memory), the
 * input gradients use the weights in their other orientation without a
 * copy.  ws: moe_backward_workspace_size(cfg) bytes.  Errors as moe_forward;
 * the float32 layer is MOE_ERR_UNSUPPORTED.
 */
size_t moe_backward_workspace_size(const moe_config_t* cfg);
moe_status_t moe_backward(const moe_config_t* cfg, const void* x, const void* dy, const int32_t* topk_idx,
                          const float* topk_w, const void* router_w, const void* w_gate, const void* w_up,
                          const void* w_down, const void* ws_gate, const void* ws_up, const void* ws_down, float* dx,
                          float* d_router_w, float* d_router_b, float* d_w_gate, float* d_w_up, float* d_w_down,
                          float* d_ws_gate, float* d_ws_up, float* d_ws_down, void* ws, size_t ws_bytes,
                          moe_stream_t stream);

/* Waits for `stream`, then returns the device check flags (MOE_DEVFLAG_*)
 * accumulated in `ws` since the last call and clears them.  Returns
 * MOE_ERR_DEVICE_CHECK if any flag was set, MOE_OK otherwise. */
moe_status_t moe_get_device_status(const moe_config_t* cfg, void* ws, size_t ws_bytes,
                                   moe_stream_t stream, int32_t* flags_out);

/* Static strings; never NULL. */
const char* moe_status_string(moe_status_t status);
const char* moe_last_error(void);

/*
 * Kernel tracing (for measurement).  While tracing is on, every kernel the
 * library enqueues whose name contains `only` (every kernel if `only` is
 * NULL or empty) is bracketed by two CUDA events on its stream; up to
 * `max_launches` launches are recorded.  moe_trace_end() waits for the
 * recorded events, writes for each launch its kernel name and its duration
 * in milliseconds, and turns tracing off.  Host-side only; no device
 * memory is allocated.  Not thread-safe: one tracing session at a time.
 * Calls enqueued while their stream is being captured into a CUDA graph are
 * traced through external event-record nodes: end the session after one
 * replay of that graph to read the launches' times.
 */
typedef struct {
    const char* name; /* static string */
    float ms;
} moe_trace_record_t;

moe_status_t moe_trace_begin(int32_t max_launches, const char* only);
moe_status_t moe_trace_end(moe_trace_record_t* records, int32_t max_records, int32_t* n_records);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
