/*
 * CPU oracle for the forward pass of a top-k routed MoE FFN layer.
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the tests, the smoke check
 * and the benchmark's CPU-baseline leg may load this library.  It shares no
 * code with the CUDA path.
 *
 * Everything is computed in double precision on the exact values of the
 * float32 / bfloat16 inputs, token by token, in the order the method states:
 *
 *   score -> select top-k -> softmax over the selected -> weighted sum of
 *   the selected experts' FFN outputs.
 *
 * Sources (page title, section):
 *   [P3] "MoE稀疏架构是什么？从原理到落地的系统解读", section 四 (how one forward
 *        pass works): a router gives one score per expert, the top-k scores
 *        are kept, those k scores are normalised with a softmax, and the
 *        output is the softmax-weighted sum of the k chosen experts applied
 *        to the token; experts that were not chosen are never evaluated.
 *        Section 三.1: the router is a small linear layer.
 *        Section 三.2: capacity-constrained token dropping.
 *   [P2] "Mixture of Experts (MoEs) in Transformers", section Weight Loading
 *        Refactor: experts are packed as [E, out, in] tensors; each expert
 *        is a small feed-forward network with gate (w1), up (w3) and down
 *        (w2) projections.  Section Expert Backend: tokens grouped by expert
 *        id for the grouped GEMM (the grouped order is what oracle_permute
 *        emits).
 *   [P4] "模型的“分工的艺术”：MoE技术如何提升计算效率", section 3.1: an expert
 *        has a maximum number of tokens it takes (expert capacity).
 *
 * Readings where the pages are silent (each is a stated choice):
 *   - Ties between equal scores go to the lower expert index.
 *   - The expert FFN is SwiGLU without biases:
 *       FFN_e(x) = W_down[e] (silu(W_gate[e] x) * (W_up[e] x)),
 *       silu(z) = z / (1 + exp(-z)).
 *   - Capacity C = ceil(cf * T * k / E); tokens are served in ascending
 *     token order, so (t, e) is kept iff fewer than C earlier tokens were
 *     kept for e.  A dropped pair contributes nothing; the remaining weights
 *     of that token are not renormalised.
 *   - The optional shared expert is always applied with weight 1.
 *
 * dtype codes: 0 = float32 arrays, 1 = bfloat16 bit patterns (uint16).
 * Weight layouts (row-major): router_w [E,H]; w_gate, w_up [E,I,H];
 * w_down [E,H,I]; shared ws_gate, ws_up [Is,H]; ws_down [H,Is].
 * Return value of every entry point: 0 on success, negative on bad input.
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static inline double bf16_to_double(uint16_t v) {
    uint32_t u = (uint32_t)v << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Widen n elements starting at element offset `off` of a typed array. */
static void load_row(const void* base, int dtype, int64_t off, int64_t n, double* out) {
    if (dtype == 0) {
        const float* p = (const float*)base + off;
        for (int64_t i = 0; i < n; ++i) out[i] = (double)p[i];
    } else {
        const uint16_t* p = (const uint16_t*)base + off;
        for (int64_t i = 0; i < n; ++i) out[i] = bf16_to_double(p[i]);
    }
}

/* sum_i a[i] * w[off + i] in double (w widened exactly). */
static double dot_row(const double* a, const void* w, int dtype, int64_t off, int64_t n) {
    double s = 0.0;
    if (dtype == 0) {
        const float* p = (const float*)w + off;
#pragma omp simd reduction(+ : s)
        for (int64_t i = 0; i < n; ++i) s += a[i] * (double)p[i];
    } else {
        const uint16_t* p = (const uint16_t*)w + off;
#pragma omp simd reduction(+ : s)
        for (int64_t i = 0; i < n; ++i) {
            uint32_t u = (uint32_t)p[i] << 16;
            float f;
            memcpy(&f, &u, 4);
            s += a[i] * (double)f;
        }
    }
    return s;
}

/* Threads the OpenMP regions of this library use. */
int oracle_threads(void) { return omp_get_max_threads(); }

static double silu(double z) { return z / (1.0 + exp(-z)); }

/*
 * Router scores and top-k selection with softmax over the selected ([P3]
 * sections 三.1 and 四).
 *   logits[t,e] = sum_h x[t,h] * router_w[e,h] + b[e]   (b nullable)
 *   topk_idx[t, 0..k-1]: the k largest logits, ordered by logit descending,
 *                        then expert index ascending.
 *   topk_w[t, j] = exp(l_j - l_max) / sum_{i in S} exp(l_i - l_max).
 * logits_out [T,E] is optional.
 */
int oracle_route(int64_t T, int H, int E, int k, int dtype, const void* x, const void* router_w,
                 const float* b, double* logits_out, int32_t* topk_idx, double* topk_w) {
    if (T < 0 || H <= 0 || E <= 0 || k <= 0 || k > E || (dtype != 0 && dtype != 1)) return -1;
    int rc = 0;
#pragma omp parallel
    {
        double* xr = (double*)malloc(sizeof(double) * (size_t)H);
        double* l = (double*)malloc(sizeof(double) * (size_t)E);
        unsigned char* taken = (unsigned char*)malloc((size_t)E);
        if (!xr || !l || !taken) {
#pragma omp atomic write
            rc = -2;
        }
#pragma omp for schedule(static)
        for (int64_t t = 0; t < T; ++t) {
            if (!xr || !l || !taken) continue;
            {
                load_row(x, dtype, t * (int64_t)H, H, xr);
                for (int e = 0; e < E; ++e) {
                    l[e] = dot_row(xr, router_w, dtype, (int64_t)e * H, H);
                    if (b) l[e] += (double)b[e];
                    taken[e] = 0;
                }
                if (logits_out) memcpy(logits_out + t * (int64_t)E, l, sizeof(double) * (size_t)E);
                /* select: repeated arg-max; the strict '>' keeps the lower index on ties */
                for (int j = 0; j < k; ++j) {
                    int best = -1;
                    for (int e = 0; e < E; ++e)
                        if (!taken[e] && (best < 0 || l[e] > l[best])) best = e;
                    taken[best] = 1;
                    topk_idx[t * k + j] = best;
                }
                /* softmax over the k selected scores; the first is the largest */
                double m = l[topk_idx[t * k]], z = 0.0;
                for (int j = 0; j < k; ++j) z += exp(l[topk_idx[t * k + j]] - m);
                for (int j = 0; j < k; ++j) topk_w[t * k + j] = exp(l[topk_idx[t * k + j]] - m) / z;
            }
        }
        free(xr);
        free(l);
        free(taken);
    }
    return rc;
}

/*
 * Grouping of (token, slot) pairs by expert ([P2] section Expert Backend),
 * with capacity-limited token dropping in token order ([P3] section 三.2,
 * [P4] section 3.1).
 *   counts[e]     number of (t, j) with topk_idx[t,j] == e, before capacity.
 *   dropped[e]    pairs of expert e beyond the capacity (0 when capacity <= 0).
 *   offsets[e]    first row of expert e; offsets[E] = number of kept rows.
 *   perm_rows[r]  slot id s = t*k + j of row r; rows of one expert are in
 *                 ascending token order.  Entries past offsets[E] are -1.
 *   row_of[s]     row of slot s, or -1 if the pair was dropped.
 */
int oracle_permute(int64_t T, int k, int E, int64_t capacity, const int32_t* topk_idx,
                   int32_t* counts, int32_t* offsets, int32_t* perm_rows, int32_t* row_of,
                   int32_t* dropped) {
    if (T < 0 || k <= 0 || E <= 0) return -1;
    int64_t S = T * (int64_t)k;
    int64_t* kept = (int64_t*)calloc((size_t)E, sizeof(int64_t));
    int64_t* fill = (int64_t*)calloc((size_t)E, sizeof(int64_t));
    if (!kept || !fill) {
        free(kept);
        free(fill);
        return -2;
    }
    for (int e = 0; e < E; ++e) counts[e] = dropped[e] = 0;
    for (int64_t s = 0; s < S; ++s) {
        int e = topk_idx[s];
        if (e < 0 || e >= E) {
            free(kept);
            free(fill);
            return -3;
        }
        counts[e]++;
    }
    /* pass 1: which pairs are kept (tokens in ascending order) */
    for (int64_t t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            int e = topk_idx[t * k + j];
            if (capacity > 0 && kept[e] >= capacity) {
                dropped[e]++;
                row_of[t * k + j] = -1;
            } else {
                kept[e]++;
                row_of[t * k + j] = -2; /* kept, row assigned below */
            }
        }
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + (int32_t)kept[e];
    for (int64_t r = 0; r < S; ++r) perm_rows[r] = -1;
    /* pass 2: rows of an expert in ascending token order */
    for (int64_t t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            int64_t s = t * k + j;
            if (row_of[s] == -1) continue;
            int e = topk_idx[s];
            int64_t r = offsets[e] + fill[e]++;
            row_of[s] = (int32_t)r;
            perm_rows[r] = (int32_t)s;
        }
    free(kept);
    free(fill);
    return 0;
}

/*
 * Output rows of the layer for a list of tokens ([P3] section 四):
 *   y[t] = sum_{j : pair (t,j) kept} topk_w[t,j] * FFN_{topk_idx[t,j]}(x[t])
 *          + FFN_shared(x[t])            (when Is > 0)
 * row_of (nullable) marks dropped pairs with -1.  tok (nullable) lists the
 * n tokens to evaluate (else tokens 0..n-1).  y_out is [n, H] double.
 */
int oracle_moe_tokens(int64_t T, int H, int I, int E, int k, int Is, int dtype, const void* x,
                      const void* w_gate, const void* w_up, const void* w_down,
                      const void* ws_gate, const void* ws_up, const void* ws_down,
                      const int32_t* topk_idx, const double* topk_w, const int32_t* row_of,
                      int64_t n, const int32_t* tok, double* y_out) {
    if (T < 0 || H <= 0 || I <= 0 || E <= 0 || k <= 0 || Is < 0 || n < 0) return -1;
    if (Is > 0 && (!ws_gate || !ws_up || !ws_down)) return -1;
    int rc = 0;
    int imax = I > Is ? I : Is;
#pragma omp parallel
    {
        double* xr = (double*)malloc(sizeof(double) * (size_t)H);
        double* a = (double*)malloc(sizeof(double) * (size_t)imax);
        if (!xr || !a) {
#pragma omp atomic write
            rc = -2;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t q = 0; q < n; ++q) {
            if (!xr || !a) continue;
            {
                int64_t t = tok ? tok[q] : q;
                double* y = y_out + q * (int64_t)H;
                for (int h = 0; h < H; ++h) y[h] = 0.0;
                if (t < 0 || t >= T) continue;
                load_row(x, dtype, t * (int64_t)H, H, xr);
                for (int j = 0; j < k; ++j) {
                    int64_t s = t * k + j;
                    if (row_of && row_of[s] < 0) continue; /* dropped: contributes 0 */
                    int64_t e = topk_idx[s];
                    double w = topk_w[s];
                    for (int i = 0; i < I; ++i) {
                        double g = dot_row(xr, w_gate, dtype, (e * I + i) * (int64_t)H, H);
                        double u = dot_row(xr, w_up, dtype, (e * I + i) * (int64_t)H, H);
                        a[i] = silu(g) * u;
                    }
                    for (int h = 0; h < H; ++h)
                        y[h] += w * dot_row(a, w_down, dtype, (e * H + h) * (int64_t)I, I);
                }
                if (Is > 0) {
                    for (int i = 0; i < Is; ++i) {
                        double g = dot_row(xr, ws_gate, dtype, (int64_t)i * H, H);
                        double u = dot_row(xr, ws_up, dtype, (int64_t)i * H, H);
                        a[i] = silu(g) * u;
                    }
                    for (int h = 0; h < H; ++h) y[h] += dot_row(a, ws_down, dtype, (int64_t)h * Is, Is);
                }
            }
        }
        free(xr);
        free(a);
    }
    return rc;
}

/*
 * Backward pass of the layer, given the upstream gradient dy [T,H] (fp64),
 * for the forward that oracle_route / oracle_permute / oracle_moe_tokens
 * define (the training use of the grouped-GEMM backend, "Mixture of Experts
 * (MoEs) in Transformers", section Training MoEs with Transformers).  Every
 * formula is the chain rule through the forward's steps, in fp64 on the
 * exact input values:
 *   kept pair (t, j) with expert e, weight w:
 *     g = W_gate[e] x, u = W_up[e] x, a = silu(g) * u, o = W_down[e] a
 *     dw_j = dy . o                         (dropped pairs: dw_j = 0)
 *     da = w * W_down[e]^T dy
 *     dg = da * u * silu'(g),  silu'(z) = s(z) (1 + z (1 - s(z))), s = sigmoid
 *     du = da * silu(g)
 *     dW_down[e] += w * dy a^T,  dW_gate[e] += dg x^T,  dW_up[e] += du x^T
 *     dx += W_gate[e]^T dg + W_up[e]^T du
 *   softmax over the selected scores (every selected pair, kept or not):
 *     dl_j = w_j (dw_j - sum_i w_i dw_i)
 *     dW_router[e_j] += dl_j x,  db[e_j] += dl_j,  dx += dl_j W_router[e_j]
 *   shared expert: the same with w = 1, always kept.
 * The selection itself (top-k) and the capacity cut are piecewise constant:
 * no gradient flows through them.
 * Outputs (all fp64, written, not accumulated into): dx [T,H], d_router_w
 * [E,H], d_router_b [E], d_w_gate, d_w_up [E,I,H], d_w_down [E,H,I] and,
 * when Is > 0, d_ws_gate, d_ws_up [Is,H], d_ws_down [H,Is].
 */
int oracle_moe_backward(int64_t T, int H, int I, int E, int k, int Is, int dtype, const void* x,
                        const void* router_w, const void* w_gate, const void* w_up, const void* w_down,
                        const void* ws_gate, const void* ws_up, const void* ws_down, const int32_t* topk_idx,
                        const double* topk_w, const int32_t* row_of, const double* dy, double* dx,
                        double* d_router_w, double* d_router_b, double* d_w_gate, double* d_w_up,
                        double* d_w_down, double* d_ws_gate, double* d_ws_up, double* d_ws_down) {
    if (T < 0 || H <= 0 || I <= 0 || E <= 0 || k <= 0 || Is < 0) return -1;
    if (Is > 0 && (!ws_gate || !ws_up || !ws_down || !d_ws_gate || !d_ws_up || !d_ws_down)) return -1;
    const int64_t S = T * (int64_t)k;
    /* per slot: a (activation), dg, du, and the token's dl */
    double* A = (double*)calloc((size_t)S * I, sizeof(double));
    double* DG = (double*)calloc((size_t)S * I, sizeof(double));
    double* DU = (double*)calloc((size_t)S * I, sizeof(double));
    double* DL = (double*)calloc((size_t)S, sizeof(double));
    double* AS = Is > 0 ? (double*)calloc((size_t)T * Is, sizeof(double)) : NULL;
    double* DGS = Is > 0 ? (double*)calloc((size_t)T * Is, sizeof(double)) : NULL;
    double* DUS = Is > 0 ? (double*)calloc((size_t)T * Is, sizeof(double)) : NULL;
    int rc = 0;
    if (!A || !DG || !DU || !DL || (Is > 0 && (!AS || !DGS || !DUS))) rc = -2;
    int imax = I > Is ? I : Is;
    /* phase 1, per token: slot quantities, dl, and dx */
    if (rc == 0) {
#pragma omp parallel
        {
            double* xr = (double*)malloc(sizeof(double) * (size_t)H);
            double* g = (double*)malloc(sizeof(double) * (size_t)imax);
            double* u = (double*)malloc(sizeof(double) * (size_t)imax);
            double* dw = (double*)malloc(sizeof(double) * (size_t)(k > 0 ? k : 1));
            double* col = (double*)malloc(sizeof(double) * (size_t)(H > imax ? H : imax));
            if (!xr || !g || !u || !dw || !col) {
#pragma omp atomic write
                rc = -2;
            }
#pragma omp for schedule(dynamic, 1)
            for (int64_t t = 0; t < T; ++t) {
                if (!xr || !g || !u || !dw || !col) continue;
                load_row(x, dtype, t * (int64_t)H, H, xr);
                const double* dyt = dy + t * (int64_t)H;
                double* dxt = dx + t * (int64_t)H;
                for (int h = 0; h < H; ++h) dxt[h] = 0.0;
                for (int j = 0; j < k; ++j) {
                    const int64_t s = t * k + j;
                    dw[j] = 0.0;
                    if (row_of && row_of[s] < 0) continue; /* dropped: no output, no gradient */
                    const int64_t e = topk_idx[s];
                    const double w = topk_w[s];
                    double* a = A + s * (int64_t)I;
                    for (int i = 0; i < I; ++i) {
                        g[i] = dot_row(xr, w_gate, dtype, (e * I + i) * (int64_t)H, H);
                        u[i] = dot_row(xr, w_up, dtype, (e * I + i) * (int64_t)H, H);
                        a[i] = silu(g[i]) * u[i];
                    }
                    /* da' = W_down[e]^T dy (unweighted); dw = da' . a = dy . o */
                    for (int i = 0; i < I; ++i) col[i] = 0.0;
                    for (int h = 0; h < H; ++h) {
                        for (int i = 0; i < I; ++i) {
                            double v;
                            load_row(w_down, dtype, (e * H + h) * (int64_t)I + i, 1, &v);
                            col[i] += v * dyt[h];
                        }
                    }
                    double d = 0.0;
                    for (int i = 0; i < I; ++i) d += col[i] * a[i];
                    dw[j] = d;
                    double* dg = DG + s * (int64_t)I;
                    double* du = DU + s * (int64_t)I;
                    for (int i = 0; i < I; ++i) {
                        const double da = w * col[i];
                        const double sg = 1.0 / (1.0 + exp(-g[i]));
                        dg[i] = da * u[i] * sg * (1.0 + g[i] * (1.0 - sg));
                        du[i] = da * g[i] * sg;
                    }
                    for (int h = 0; h < H; ++h) {
                        double acc = 0.0;
                        for (int i = 0; i < I; ++i) {
                            double vg, vu;
                            load_row(w_gate, dtype, (e * I + i) * (int64_t)H + h, 1, &vg);
                            load_row(w_up, dtype, (e * I + i) * (int64_t)H + h, 1, &vu);
                            acc += vg * dg[i] + vu * du[i];
                        }
                        dxt[h] += acc;
                    }
                }
                /* softmax over the selected scores */
                double sw = 0.0;
                for (int j = 0; j < k; ++j) sw += topk_w[t * k + j] * dw[j];
                for (int j = 0; j < k; ++j) {
                    const int64_t s = t * k + j;
                    DL[s] = topk_w[s] * (dw[j] - sw);
                    double* wr = col;
                    load_row(router_w, dtype, (int64_t)topk_idx[s] * H, H, wr);
                    for (int h = 0; h < H; ++h) dxt[h] += DL[s] * wr[h];
                }
                if (Is > 0) {
                    double* as = AS + t * (int64_t)Is;
                    double* dgs = DGS + t * (int64_t)Is;
                    double* dus = DUS + t * (int64_t)Is;
                    for (int i = 0; i < Is; ++i) {
                        g[i] = dot_row(xr, ws_gate, dtype, (int64_t)i * H, H);
                        u[i] = dot_row(xr, ws_up, dtype, (int64_t)i * H, H);
                        as[i] = silu(g[i]) * u[i];
                        double c = 0.0;
                        for (int h = 0; h < H; ++h) {
                            double v;
                            load_row(ws_down, dtype, (int64_t)h * Is + i, 1, &v);
                            c += v * dyt[h];
                        }
                        const double sg = 1.0 / (1.0 + exp(-g[i]));
                        dgs[i] = c * u[i] * sg * (1.0 + g[i] * (1.0 - sg));
                        dus[i] = c * g[i] * sg;
                    }
                    for (int h = 0; h < H; ++h) {
                        double acc = 0.0;
                        for (int i = 0; i < Is; ++i) {
                            double vg, vu;
                            load_row(ws_gate, dtype, (int64_t)i * H + h, 1, &vg);
                            load_row(ws_up, dtype, (int64_t)i * H + h, 1, &vu);
                            acc += vg * dgs[i] + vu * dus[i];
                        }
                        dxt[h] += acc;
                    }
                }
            }
            free(xr);
            free(g);
            free(u);
            free(dw);
            free(col);
        }
    }
    /* phase 2, per expert: weight gradients (and the router's) */
    if (rc == 0) {
#pragma omp parallel
        {
            double* xr = (double*)malloc(sizeof(double) * (size_t)H);
            if (!xr) {
#pragma omp atomic write
                rc = -2;
            }
#pragma omp for schedule(dynamic, 1)
            for (int e = 0; e < E; ++e) {
                if (!xr) continue;
                double* dWg = d_w_gate + (int64_t)e * I * H;
                double* dWu = d_w_up + (int64_t)e * I * H;
                double* dWd = d_w_down + (int64_t)e * H * I;
                double* dWr = d_router_w + (int64_t)e * H;
                for (int64_t q = 0; q < (int64_t)I * H; ++q) dWg[q] = dWu[q] = dWd[q] = 0.0;
                for (int h = 0; h < H; ++h) dWr[h] = 0.0;
                d_router_b[e] = 0.0;
                for (int64_t t = 0; t < T; ++t)
                    for (int j = 0; j < k; ++j) {
                        const int64_t s = t * k + j;
                        if (topk_idx[s] != e) continue;
                        load_row(x, dtype, t * (int64_t)H, H, xr);
                        for (int h = 0; h < H; ++h) dWr[h] += DL[s] * xr[h];
                        d_router_b[e] += DL[s];
                        if (row_of && row_of[s] < 0) continue;
                        const double w = topk_w[s];
                        const double* a = A + s * (int64_t)I;
                        const double* dg = DG + s * (int64_t)I;
                        const double* du = DU + s * (int64_t)I;
                        const double* dyt = dy + t * (int64_t)H;
                        for (int i = 0; i < I; ++i)
                            for (int h = 0; h < H; ++h) {
                                dWg[(int64_t)i * H + h] += dg[i] * xr[h];
                                dWu[(int64_t)i * H + h] += du[i] * xr[h];
                            }
                        for (int h = 0; h < H; ++h)
                            for (int i = 0; i < I; ++i) dWd[(int64_t)h * I + i] += w * dyt[h] * a[i];
                    }
            }
            free(xr);
        }
        if (Is > 0) {
            for (int64_t q = 0; q < (int64_t)Is * H; ++q) d_ws_gate[q] = d_ws_up[q] = d_ws_down[q] = 0.0;
            double* xr = (double*)malloc(sizeof(double) * (size_t)H);
            if (!xr) rc = -2;
            for (int64_t t = 0; t < T && xr; ++t) {
                load_row(x, dtype, t * (int64_t)H, H, xr);
                const double* as = AS + t * (int64_t)Is;
                const double* dgs = DGS + t * (int64_t)Is;
                const double* dus = DUS + t * (int64_t)Is;
                const double* dyt = dy + t * (int64_t)H;
                for (int i = 0; i < Is; ++i)
                    for (int h = 0; h < H; ++h) {
                        d_ws_gate[(int64_t)i * H + h] += dgs[i] * xr[h];
                        d_ws_up[(int64_t)i * H + h] += dus[i] * xr[h];
                    }
                for (int h = 0; h < H; ++h)
                    for (int i = 0; i < Is; ++i) d_ws_down[(int64_t)h * Is + i] += dyt[h] * as[i];
            }
            free(xr);
        }
    }
    free(A);
    free(DG);
    free(DU);
    free(DL);
    free(AS);
    free(DGS);
    free(DUS);
    return rc;
}
