/*
 * Plain, slow CPU oracle for the routed sigmoid top-k MoE FFN.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header, table or helper with
 * the CUDA library; it is written from the definitions on the source pages:
 *
 *   [P1] mlx-native 0.13.0, src/ops/dense_matmul_id_auto.rs
 *        (DenseMatmulIdShape, DenseMatmulIdInputLayout, routing profiles,
 *        expected_dispatches: Direct/Grouped matmul-by-expert-id)
 *   [P2] cortiq-engine 0.7.7, src/mimo_moe.rs
 *        (module doc: "top-8, sigmoid + selection-bias routing";
 *        Dynamic::run combine weights p[e]/wsum; tests::exact_moe, tests::rel)
 *   [P3] hf2q 0.1.1, src/inference/spec_decode/eagle3/forward.rs
 *        (Phase E4b.8 SwiGLU MLP: down(silu(gate(x)) * up(x)), no bias)
 *   [P5] hf2q, src/inference/models/qwen35/dense_ffn_arena.rs
 *        (MoeFfnArena: ids/weights/gate_all/up_all/h_all/y_all, then the
 *        weighted reduce over slots; the shared expert's buffers sh_logit
 *        [seq, 1], a_s and b_s [seq, m_sh], h_s [seq, m_sh])
 *
 * Every floating-point result is accumulated in double over bf16-valued
 * inputs (bf16 widened exactly), in the plain order of the definition.
 *
 * Parity pins: every function here is pinned by tests that do not re-type
 * its formula (closed forms, brute force, invariants, special cases that
 * reduce to numpy's dense matmul); see the test suite's oracle tests.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* bf16 bit pattern -> exact double. */
static double bf16_to_f64(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round a float to the nearest bf16 (ties to even); NaN stays NaN. */
static double round_to_bf16(double v) {
    float f = (float)v;
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu)) return v;
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    u &= 0xffff0000u;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* The activation as a down projection that multiplies in fp16 sees it: a
 * rounded to f32, scaled by 2^-4 (exact), rounded to fp16 (ties to even),
 * scaled back.  Values past the fp16 range become infinite. */
static double round_to_fp16_scaled(double v) {
    const float f = (float)v * 0.0625f;
    const _Float16 h = (_Float16)f;
    return (double)h * 16.0;
}

/* ------------------------------------------------------------------------
 * Routing [P2 module doc; Dynamic::run; test model config "router_sigmoid",
 * "norm_topk_prob"; mlp.expert_bias].
 *
 *   s[e]   = sigmoid(logit[e])            (f64 math, rounded once to f32)
 *   key[e] = s[e] + bias[e]               (f32 add; bias only selects)
 *   ids    = the top_k experts by key, descending; the lower index wins a tie
 *   w[j]   = s[ids[j]] / sum_j s[ids[j]]  (f64, slot order, stored as f32)
 *
 * Readings where the pages are silent: NaN keys sort as -inf, -0 as +0; the
 * selection is a full stable sort of all experts (not a partial heap).
 * ------------------------------------------------------------------------ */
typedef struct { float key; int32_t idx; } key_idx;

static int key_idx_cmp(const void *pa, const void *pb) {
    const key_idx *a = (const key_idx *)pa, *b = (const key_idx *)pb;
    if (a->key > b->key) return -1;
    if (a->key < b->key) return 1;
    return (a->idx < b->idx) ? -1 : (a->idx > b->idx);
}

static float canonical_key(float k) {
    if (isnan(k)) return -INFINITY;
    if (k == 0.0f) return 0.0f;
    return k;
}

float oracle_sigmoid_f32(float logit) {
    return (float)(1.0 / (1.0 + exp(-(double)logit)));
}

void oracle_route(const float *logits, const float *bias, int32_t m, int32_t n_experts,
                  int32_t top_k, int32_t *ids, float *weights, float *scores) {
#pragma omp parallel
    {
        key_idx *order = (key_idx *)malloc(sizeof(key_idx) * (size_t)n_experts);
        float *s = (float *)malloc(sizeof(float) * (size_t)n_experts);
#pragma omp for schedule(static)
        for (int32_t t = 0; t < m; ++t) {
            const float *lg = logits + (size_t)t * n_experts;
            for (int32_t e = 0; e < n_experts; ++e) {
                s[e] = oracle_sigmoid_f32(lg[e]);
                float key = s[e] + (bias ? bias[e] : 0.0f);
                order[e].key = canonical_key(key);
                order[e].idx = e;
                if (scores) scores[(size_t)t * n_experts + e] = s[e];
            }
            qsort(order, (size_t)n_experts, sizeof(key_idx), key_idx_cmp);
            double wsum = 0.0;
            for (int32_t j = 0; j < top_k; ++j) wsum += (double)s[order[j].idx];
            for (int32_t j = 0; j < top_k; ++j) {
                ids[(size_t)t * top_k + j] = order[j].idx;
                weights[(size_t)t * top_k + j] = (float)((double)s[order[j].idx] / wsum);
            }
        }
        free(order);
        free(s);
    }
}

/* Router projection [cortiq-engine 0.7.7, src/mimo_moe.rs test model tensor
 * mlp.gate.weight [NE, HS]; hf2q qwen35 dense_ffn_arena.rs logits buffer
 * [seq, num_experts]]: logits[t, e] = sum_c W_router[e, c] * x[t, c], f64. */
void oracle_router_logits(const uint16_t *x, const uint16_t *W_router, double *logits,
                          int32_t m, int32_t hidden, int32_t n_experts) {
#pragma omp parallel for schedule(static)
    for (int32_t t = 0; t < m; ++t) {
        const uint16_t *xt = x + (size_t)t * hidden;
        for (int32_t e = 0; e < n_experts; ++e) {
            const uint16_t *we = W_router + (size_t)e * hidden;
            double acc = 0.0;
            for (int32_t c = 0; c < hidden; ++c) acc += bf16_to_f64(we[c]) * bf16_to_f64(xt[c]);
            logits[(size_t)t * n_experts + e] = acc;
        }
    }
}

/* Combine weights for ids fixed by the caller [P2 Dynamic::run builds
 * mix[e] = p[e] / wsum over the picks; the bank frame then takes "forced"
 * picks and "preweighted" mixes].  w[j] = s[ids[j]] / sum_j s[ids[j]] with
 * s the f32-rounded sigmoid of the logit, f64 sum in slot order. */
void oracle_route_weights(const float *logits, const int32_t *ids, int32_t m,
                          int32_t n_experts, int32_t top_k, float *weights) {
#pragma omp parallel for schedule(static)
    for (int32_t t = 0; t < m; ++t) {
        const float *lg = logits + (size_t)t * n_experts;
        double wsum = 0.0;
        for (int32_t j = 0; j < top_k; ++j)
            wsum += (double)oracle_sigmoid_f32(lg[ids[(size_t)t * top_k + j]]);
        for (int32_t j = 0; j < top_k; ++j) {
            const double s = (double)oracle_sigmoid_f32(lg[ids[(size_t)t * top_k + j]]);
            weights[(size_t)t * top_k + j] = (float)(s / wsum);
        }
    }
}

/* ------------------------------------------------------------------------
 * Expert map [P1 expected_dispatches: the Grouped route's
 * "dense_matmul_id_map_distinct" pass; DenseMatmulIdScratch].
 *
 * Routed row r = t*top_k + j.  counts[e] = #rows routed to e; offsets is the
 * exclusive prefix sum (offsets[E] = m*top_k); perm lists the rows of expert
 * 0, then expert 1, ..., each group in ascending r (a stable counting sort);
 * inv_perm[perm[p]] = p.  Returns -1 if an id is out of range, else 0.
 * ------------------------------------------------------------------------ */
int oracle_expert_map(const int32_t *ids, int32_t m, int32_t top_k, int32_t n_experts,
                      int32_t *counts, int32_t *offsets, int32_t *perm, int32_t *inv_perm) {
    const int64_t rows = (int64_t)m * top_k;
    for (int32_t e = 0; e < n_experts; ++e) counts[e] = 0;
    for (int64_t r = 0; r < rows; ++r) {
        if (ids[r] < 0 || ids[r] >= n_experts) return -1;
        counts[ids[r]] += 1;
    }
    offsets[0] = 0;
    for (int32_t e = 0; e < n_experts; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int32_t *fill = (int32_t *)malloc(sizeof(int32_t) * (size_t)n_experts);
    for (int32_t e = 0; e < n_experts; ++e) fill[e] = offsets[e];
    for (int64_t r = 0; r < rows; ++r) {
        int32_t p = fill[ids[r]]++;
        perm[p] = (int32_t)r;
        inv_perm[r] = p;
    }
    free(fill);
    return 0;
}

/* ------------------------------------------------------------------------
 * matmul by expert id [P1 DenseMatmulIdShape / expected_dispatches, Direct
 * route: one output row per (token, slot)].
 *
 *   y[t, j, c] = sum_i W[ids[t,j], c, i] * x_row(t, j)[i]
 *   x_row = x[t]       (layout 0, SharedPerToken: x is [m, k])
 *         = x[t, j]    (layout 1, Slotted: x is [m, top_k, k])
 * W is [E, n, k] (row-major, k contiguous).  Output y is [m, top_k, n] f64.
 * ------------------------------------------------------------------------ */
void oracle_matmul_id(const uint16_t *x, const int32_t *ids, const uint16_t *W, double *y,
                      int32_t m, int32_t n, int32_t k, int32_t top_k, int32_t n_experts,
                      int32_t layout) {
    (void)n_experts;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < (int64_t)m * top_k; ++r) {
        const int64_t t = r / top_k;
        const uint16_t *xr = x + (size_t)(layout == 0 ? t : r) * k;
        const uint16_t *We = W + (size_t)ids[r] * n * k;
        for (int32_t c = 0; c < n; ++c) {
            double acc = 0.0;
            for (int32_t i = 0; i < k; ++i)
                acc += bf16_to_f64(We[(size_t)c * k + i]) * bf16_to_f64(xr[i]);
            y[(size_t)r * n + c] = acc;
        }
    }
}

/* ------------------------------------------------------------------------
 * Routed SwiGLU MoE FFN [P2 tests::exact_moe; P3 Phase E4b.8 SwiGLU MLP;
 * P5 MoeFfnArena dataflow].  For each requested token t:
 *
 *   for slot j (in slot order), e = ids[t, j]:
 *     g[i] = sum_c W_gate[e, i, c] * x_row[c]
 *     u[i] = sum_c W_up[e, i, c]   * x_row[c]
 *     a[i] = g[i] / (1 + exp(-g[i])) * u[i]          (silu(g) * u)
 *     d[h] = sum_i W_down[e, h, i] * a[i]
 *     y[t, h] += weights[t, j] * d[h]
 *
 * act_mode 0 keeps a[] unrounded (the pages' definition); act_mode 1 rounds
 * a[] to f32 then bf16 (what a plain bf16 down projection would see), used
 * only to show why the GPU keeps more than bf16 of the activation; act_mode 2
 * rounds it as an fp16 down projection with a 2^-4 scale does
 * (round_to_fp16_scaled), a reading of the precision P5 leaves to the
 * implementation (its h_all buffer is f32).
 * W_gate/W_up are [E, inter, hidden], W_down is [E, hidden, inter].
 * tokens (nullable => 0..m-1) selects n_tokens rows; y is [n_tokens, hidden].
 * ------------------------------------------------------------------------ */
void oracle_ffn(const uint16_t *x, const int32_t *ids, const float *weights,
                const uint16_t *W_gate, const uint16_t *W_up, const uint16_t *W_down,
                double *y, int32_t m, int32_t hidden, int32_t inter, int32_t top_k,
                int32_t n_experts, int32_t layout, int32_t act_mode,
                const int32_t *tokens, int32_t n_tokens) {
    (void)m;
    (void)n_experts;
#pragma omp parallel
    {
        double *a = (double *)malloc(sizeof(double) * (size_t)inter);
#pragma omp for schedule(dynamic, 1)
        for (int32_t q = 0; q < n_tokens; ++q) {
            const int64_t t = tokens ? tokens[q] : q;
            double *yt = y + (size_t)q * hidden;
            for (int32_t h = 0; h < hidden; ++h) yt[h] = 0.0;
            for (int32_t j = 0; j < top_k; ++j) {
                const int64_t r = t * top_k + j;
                const int32_t e = ids[r];
                const uint16_t *xr = x + (size_t)(layout == 0 ? t : r) * hidden;
                const uint16_t *Wg = W_gate + (size_t)e * inter * hidden;
                const uint16_t *Wu = W_up + (size_t)e * inter * hidden;
                const uint16_t *Wd = W_down + (size_t)e * hidden * inter;
                for (int32_t i = 0; i < inter; ++i) {
                    double g = 0.0, u = 0.0;
                    for (int32_t c = 0; c < hidden; ++c) {
                        const double xv = bf16_to_f64(xr[c]);
                        g += bf16_to_f64(Wg[(size_t)i * hidden + c]) * xv;
                        u += bf16_to_f64(Wu[(size_t)i * hidden + c]) * xv;
                    }
                    a[i] = g / (1.0 + exp(-g)) * u;
                    if (act_mode == 1) a[i] = round_to_bf16(a[i]);
                    else if (act_mode == 2) a[i] = round_to_fp16_scaled(a[i]);
                }
                const double w = (double)weights[r];
                for (int32_t h = 0; h < hidden; ++h) {
                    double d = 0.0;
                    for (int32_t i = 0; i < inter; ++i)
                        d += bf16_to_f64(Wd[(size_t)h * inter + i]) * a[i];
                    yt[h] += w * d;
                }
            }
        }
        free(a);
    }
}

/* ------------------------------------------------------------------------
 * Routed FFN plus a shared expert [P5 MoeFfnArena: sh_logit [seq, 1] is the
 * shared expert's gate input logit, a_s / b_s [seq, m_sh] its gate and up
 * outputs, h_s = silu_mul(a_s, b_s) its intermediate].  The page gives the
 * buffers, not the formula; the reading taken here (the plainest one the
 * shapes support, and the routed path's own gate function):
 *
 *   sh_logit[t] = w_sh . x[t]                         (w_sh: [hidden])
 *   a_s = W_sh_gate x[t],  b_s = W_sh_up x[t]          ([inter_sh, hidden])
 *   h_s = silu(a_s) * b_s
 *   y[t] = routed y[t] + sigmoid(sh_logit[t]) * (W_sh_down h_s)
 *
 * added after the routed slots.  x is one row per token (layout 0).
 * act_mode as in oracle_ffn, for both parts.
 */
void oracle_ffn_shared(const uint16_t *x, const int32_t *ids, const float *weights,
                       const uint16_t *W_gate, const uint16_t *W_up, const uint16_t *W_down,
                       const uint16_t *w_sh, const uint16_t *W_sh_gate,
                       const uint16_t *W_sh_up, const uint16_t *W_sh_down, double *y,
                       int32_t m, int32_t hidden, int32_t inter, int32_t inter_sh,
                       int32_t top_k, int32_t n_experts, int32_t act_mode,
                       const int32_t *tokens, int32_t n_tokens) {
    oracle_ffn(x, ids, weights, W_gate, W_up, W_down, y, m, hidden, inter, top_k, n_experts, 0,
               act_mode, tokens, n_tokens);
#pragma omp parallel
    {
        double *h_s = (double *)malloc(sizeof(double) * (size_t)inter_sh);
#pragma omp for schedule(dynamic, 1)
        for (int32_t q = 0; q < n_tokens; ++q) {
            const int64_t t = tokens ? tokens[q] : q;
            const uint16_t *xt = x + (size_t)t * hidden;
            double logit = 0.0;
            for (int32_t c = 0; c < hidden; ++c) logit += bf16_to_f64(w_sh[c]) * bf16_to_f64(xt[c]);
            const double gate = 1.0 / (1.0 + exp(-logit));
            for (int32_t i = 0; i < inter_sh; ++i) {
                double a_s = 0.0, b_s = 0.0;
                for (int32_t c = 0; c < hidden; ++c) {
                    a_s += bf16_to_f64(W_sh_gate[(size_t)i * hidden + c]) * bf16_to_f64(xt[c]);
                    b_s += bf16_to_f64(W_sh_up[(size_t)i * hidden + c]) * bf16_to_f64(xt[c]);
                }
                h_s[i] = a_s / (1.0 + exp(-a_s)) * b_s;
                if (act_mode == 1) h_s[i] = round_to_bf16(h_s[i]);
                else if (act_mode == 2) h_s[i] = round_to_fp16_scaled(h_s[i]);
            }
            double *yt = y + (size_t)q * hidden;
            for (int32_t h = 0; h < hidden; ++h) {
                double d_s = 0.0;
                for (int32_t i = 0; i < inter_sh; ++i)
                    d_s += bf16_to_f64(W_sh_down[(size_t)h * inter_sh + i]) * h_s[i];
                yt[h] += gate * d_s;
            }
        }
        free(h_s);
    }
}
