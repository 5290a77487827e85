/*
 * CPU oracle for the fine-grained MoE layer forward -- TEST INFRASTRUCTURE ONLY.
 *
 * Only the test suite, the smoke check and the benchmark's CPU-baseline leg
 * may load this library.  The CUDA library never links or calls it, and it
 * shares no code, header or table with the CUDA library.
 *
 * Plain, slow, obviously correct: every dot product is a straight loop with
 * an fp64 accumulator, token by token, in the order the pages state the
 * method.  OpenMP only splits the independent tokens across threads.
 *
 * Page titles used in citations:
 *   [FusionLLM]  "FusionLLM：融合 MLA、GDN 与 MoE 的高效混合架构大模型训练框架"
 *   [Arch]       "大模型工程（一）：Transformer 到 MoE"
 *   [Explainer]  "开源混合架构大模型技术解析"
 *
 * What is computed (one token x of length d):
 *   1. router logits    l[e] = sum_c W_router[e,c] * x[c]
 *        (bias-free linear router g(x) = W_g x: [Arch] "MoE 数学：路由、容量与
 *         平衡详解"; gate Linear without bias in the MoEBlock listing of [Arch]
 *         "混合专家：更多参数，相同 FLOPs")
 *   2. gate scores      s[e] = 1 / (1 + exp(-l[e]))
 *        (bias-free sigmoid gating: [FusionLLM] "混合专家（MoE）")
 *   3. group limit      the E experts form n_group equal groups of consecutive
 *        indices; a group's score is the max score inside it; the topk_group
 *        groups with the largest group score are kept (ties: lower group
 *        index) and all other experts are masked out
 *        (group-limited routing: [FusionLLM] "混合专家（MoE）"; the page gives
 *         no formula, the max-of-group reading is ours)
 *   4. top-k            the k largest unmasked scores (ties: lower expert
 *        index), listed in descending score order
 *        (fixed-k top-k: [Arch] "MoE 数学：路由、容量与平衡详解"; [Explainer]
 *         "四、工作原理：稀疏激活如何运行")
 *   5. normalise        w_j = s[idx_j] / sum_j' s[idx_j']
 *        (gate weights over the chosen experts sum to one)
 *   6. experts          for each selected expert e:
 *        g = W_gate_up[e, 0:I] x,  u = W_gate_up[e, I:2I] x,
 *        h = silu(g) * u with silu(g) = g * sigmoid(g)  (SwiGLU: [Arch]
 *        "变了什么，为什么变", item 3),  y += w_j * (W_down[e] h)
 *        (weighted sum over the chosen experts only: MoEBlock listing in
 *         [Arch]; moe_layer pseudocode in [Explainer] section 四)
 *   7. shared experts   y += sum_s W_down_s (silu(W_gate_s x) * (W_up_s x)),
 *        unweighted, for every token (n_shared_experts in the config YAML of
 *        [FusionLLM] "模型配置与规模"; always-on shared experts in [Arch]
 *        "Mixtral、Qwen3-MoE 与 DeepSeek-V3 架构对比")
 *
 * Gating variants (the pages' other gates, selected by score_func and bias):
 *   score_func 0  the FusionLLM gate above (sigmoid scores, weights s / sum s)
 *   score_func 1  softmax over the chosen experts ([Arch] "MoE 数学：路由、容量
 *                 与平衡详解" and the MoEBlock listing: top-k of the router
 *                 logits, weights = softmax of those k logits)
 *   bias b[E]     selection-only expert bias ([Arch], the aux-loss-free
 *                 balancing of DeepSeek-V3 in "MoE 数学" and "Mixtral、Qwen3-MoE
 *                 与 DeepSeek-V3 架构对比"): the group limit and the top-k
 *                 compare gate score + b_e (gate score = s_e for score_func 0,
 *                 l_e for 1); the weights use the unbiased gate scores.
 *
 * Inputs are read as the exact values handed to the GPU: fp32, or bf16 bit
 * patterns widened to fp32 (a bf16 value is the top 16 bits of an fp32).
 * Nothing is rounded to bf16 inside the oracle; h stays fp64.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { OR_F32 = 0, OR_BF16 = 1, OR_F64 = 2 };

/* Widen element i of an fp32, bf16 or fp64 array to double (fp64 inputs
 * serve the finite-difference checks of the backward). */
static inline double elem(const void *p, int dt, size_t i) {
    if (dt == OR_F64) return ((const double *)p)[i];
    if (dt == OR_F32) return (double)((const float *)p)[i];
    uint32_t bits = ((uint32_t)((const uint16_t *)p)[i]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* sum_c a[off + c] * v[c], c < n, fp64 accumulate.  a is fp32, bf16 or fp64; v is fp64. */
static double dot_row(const void *a, int dt, size_t off, const double *v, int n) {
    double acc = 0.0;
    if (dt == OR_F64) {
        const double *r = (const double *)a + off;
        for (int c = 0; c < n; ++c) acc += r[c] * v[c];
    } else if (dt == OR_F32) {
        const float *r = (const float *)a + off;
        for (int c = 0; c < n; ++c) acc += (double)r[c] * v[c];
    } else {
        const uint16_t *r = (const uint16_t *)a + off;
        for (int c = 0; c < n; ++c) {
            uint32_t bits = ((uint32_t)r[c]) << 16;
            float f;
            memcpy(&f, &bits, sizeof f);
            acc += (double)f * v[c];
        }
    }
    return acc;
}

static double sigmoid(double z) { return 1.0 / (1.0 + exp(-z)); }

int oracle_check_args(int T, int d, int E, int k, int G, int TG) {
    if (T < 0 || d <= 0 || E <= 0 || k <= 0 || G <= 0 || TG <= 0) return -1;
    if (E % G != 0) return -1;
    if (TG > G) return -1;
    if (k > E || k > TG * (E / G)) return -1;
    return 0;
}

/* Routing weights of the experts idx[0..k) from the gate scores g[E]. */
static void gate_weights(const double *g, const int32_t *idx, int k, int score_func,
                         double *w) {
    if (score_func == 0) {
        double sum = 0.0;
        for (int j = 0; j < k; ++j) sum += g[idx[j]];
        for (int j = 0; j < k; ++j) w[j] = g[idx[j]] / sum;
    } else {
        double m = g[idx[0]];
        for (int j = 1; j < k; ++j)
            if (g[idx[j]] > m) m = g[idx[j]];
        double sum = 0.0;
        for (int j = 0; j < k; ++j) sum += exp(g[idx[j]] - m);
        for (int j = 0; j < k; ++j) w[j] = exp(g[idx[j]] - m) / sum;
    }
}

/*
 * Steps 1-5 for one token.  g: [E] gate scores (out), s: [E] selection keys
 * (out; gate score + bias).  Writes idx[k], w[k], and the two decision gaps
 * used to flag near-ties:
 *   gap_e = key of the k-th chosen expert minus the best key not chosen among
 *           the experts of the kept groups (+inf when there is none),
 *   gap_g = group key of the TG-th kept group minus the best key of a
 *           dropped group (+inf when every group is kept).
 */
static void route_token(const double *xt, const void *Wr, int dt, int d, int E, int k,
                        int G, int TG, int score_func, const double *bias, double *g,
                        double *s, int32_t *idx, double *w, double *gap_e, double *gap_g) {
    int gsz = E / G;
    for (int e = 0; e < E; ++e) {
        double l = dot_row(Wr, dt, (size_t)e * d, xt, d);
        g[e] = score_func == 0 ? sigmoid(l) : l;
        s[e] = g[e] + (bias ? bias[e] : 0.0);
    }

    /* group scores and the kept groups */
    double *gs = (double *)malloc(sizeof(double) * G);
    char *gkeep = (char *)calloc(G, 1);
    for (int g = 0; g < G; ++g) {
        double m = s[g * gsz];
        for (int e = g * gsz + 1; e < (g + 1) * gsz; ++e)
            if (s[e] > m) m = s[e];
        gs[g] = m;
    }
    double last_kept_g = INFINITY;
    for (int r = 0; r < TG; ++r) {
        int best = -1;
        for (int g = 0; g < G; ++g)
            if (!gkeep[g] && (best < 0 || gs[g] > gs[best])) best = g;
        gkeep[best] = 1;
        last_kept_g = gs[best];
    }
    double best_dropped_g = -INFINITY;
    for (int g = 0; g < G; ++g)
        if (!gkeep[g] && gs[g] > best_dropped_g) best_dropped_g = gs[g];
    *gap_g = (TG < G) ? last_kept_g - best_dropped_g : INFINITY;

    /* top-k inside the kept groups */
    char *taken = (char *)calloc(E, 1);
    for (int j = 0; j < k; ++j) {
        int best = -1;
        for (int e = 0; e < E; ++e) {
            if (!gkeep[e / gsz] || taken[e]) continue;
            if (best < 0 || s[e] > s[best]) best = e;
        }
        taken[best] = 1;
        idx[j] = best;
    }
    double best_left = -INFINITY;
    int n_left = 0;
    for (int e = 0; e < E; ++e) {
        if (!gkeep[e / gsz] || taken[e]) continue;
        ++n_left;
        if (s[e] > best_left) best_left = s[e];
    }
    *gap_e = n_left ? s[idx[k - 1]] - best_left : INFINITY;
    gate_weights(g, idx, k, score_func, w);
    free(gs);
    free(gkeep);
    free(taken);
}

static void load_row(const void *x, int dt, size_t off, int d, double *out) {
    for (int c = 0; c < d; ++c) out[c] = elem(x, dt, off + c);
}

/*
 * Routing only (steps 1-5) for all T tokens.  score_func / bias: the gating
 * variant (bias [E] nullable).  idx [T,k] int32, w [T,k] fp64, scores [T,E]
 * fp64 selection keys (nullable), gap_e / gap_g [T] fp64 (nullable).
 * Returns 0, or -1 on invalid arguments.
 */
int oracle_route(const void *x, const void *Wr, int dt, int T, int d, int E, int k, int G,
                 int TG, int score_func, const double *bias, int32_t *idx, double *w,
                 double *scores, double *gap_e, double *gap_g, int nthreads) {
    if (oracle_check_args(T, d, E, k, G, TG) || score_func < 0 || score_func > 1) return -1;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel
#endif
    {
        double *xt = (double *)malloc(sizeof(double) * d);
        double *g = (double *)malloc(sizeof(double) * E);
        double *s = (double *)malloc(sizeof(double) * E);
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 16)
#endif
        for (int t = 0; t < T; ++t) {
            double ge, gg;
            load_row(x, dt, (size_t)t * d, d, xt);
            route_token(xt, Wr, dt, d, E, k, G, TG, score_func, bias, g, s, idx + (size_t)t * k,
                        w + (size_t)t * k, &ge, &gg);
            if (scores) memcpy(scores + (size_t)t * E, s, sizeof(double) * E);
            if (gap_e) gap_e[t] = ge;
            if (gap_g) gap_g[t] = gg;
        }
        free(xt);
        free(g);
        free(s);
    }
    return 0;
}

/* y[0:d] += coef * W_dn h, where row c of W_dn starts at dn_off + c*row_len and
 * h has n entries placed at column col0 of that row. */
static void add_down(const void *Wdn, int dt, size_t dn_off, size_t row_len, int col0,
                     const double *h, int n, double coef, int d, double *y) {
    for (int c = 0; c < d; ++c)
        y[c] += coef * dot_row(Wdn, dt, dn_off + (size_t)c * row_len + col0, h, n);
}

/* h[i] = silu(W[g_row0+i] x) * (W[u_row0+i] x), i < n. */
static void swiglu_hidden(const void *Wgu, int dt, size_t base, size_t g_row0, size_t u_row0,
                          const double *xt, int d, int n, double *h) {
    for (int i = 0; i < n; ++i) {
        double g = dot_row(Wgu, dt, base + (g_row0 + i) * (size_t)d, xt, d);
        double u = dot_row(Wgu, dt, base + (u_row0 + i) * (size_t)d, xt, d);
        h[i] = g * sigmoid(g) * u;
    }
}

/*
 * Full layer forward (steps 1-7) for the tokens listed in `tokens` (n_tok of
 * them, indices into x).  y [n_tok, d] fp64.  When forced_idx [n_tok, k] is
 * given, that expert set is used instead of the oracle's own top-k; the
 * weights are still the oracle's scores of those experts, normalised.
 * idx_out [n_tok,k] and w_out [n_tok,k] (nullable) receive the set and weights
 * used.  W_shared may be NULL only when S == 0.  Returns 0, or -1.
 */
int oracle_forward(const void *x, const void *Wr, const void *Wgu, const void *Wd,
                   const void *Wsh, int dt, int T, int d, int E, int k, int G, int TG, int I,
                   int S, int score_func, const double *bias, const int32_t *tokens, int n_tok,
                   const int32_t *forced_idx, double *y, int32_t *idx_out, double *w_out,
                   int nthreads) {
    if (oracle_check_args(T, d, E, k, G, TG) || I <= 0 || S < 0) return -1;
    if (score_func < 0 || score_func > 1) return -1;
    if (S > 0 && !Wsh) return -1;
    for (int n = 0; n < n_tok; ++n)
        if (tokens[n] < 0 || tokens[n] >= T) return -1;
    if (forced_idx)
        for (int n = 0; n < n_tok * k; ++n)
            if (forced_idx[n] < 0 || forced_idx[n] >= E) return -1;
    int SI = S * I;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel
#endif
    {
        double *xt = (double *)malloc(sizeof(double) * d);
        double *g = (double *)malloc(sizeof(double) * E);
        double *s = (double *)malloc(sizeof(double) * E);
        double *h = (double *)malloc(sizeof(double) * (I > SI ? I : SI) + 8);
        int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * k);
        double *w = (double *)malloc(sizeof(double) * k);
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
        for (int n = 0; n < n_tok; ++n) {
            int t = tokens[n];
            double ge, gg, *yt = y + (size_t)n * d;
            load_row(x, dt, (size_t)t * d, d, xt);
            route_token(xt, Wr, dt, d, E, k, G, TG, score_func, bias, g, s, idx, w, &ge, &gg);
            if (forced_idx) {
                for (int j = 0; j < k; ++j) idx[j] = forced_idx[(size_t)n * k + j];
                gate_weights(g, idx, k, score_func, w);
            }
            for (int c = 0; c < d; ++c) yt[c] = 0.0;
            for (int j = 0; j < k; ++j) {
                int e = idx[j];
                size_t gu_base = (size_t)e * 2 * I * d;
                swiglu_hidden(Wgu, dt, gu_base, 0, (size_t)I, xt, d, I, h);
                add_down(Wd, dt, (size_t)e * d * I, (size_t)I, 0, h, I, w[j], d, yt);
            }
            for (int sh = 0; sh < S; ++sh) {
                /* shared expert sh: gate rows sh*I.., up rows SI + sh*I.. of the
                 * gate_up block; down columns sh*I.. of the [d, SI] block */
                swiglu_hidden(Wsh, dt, 0, (size_t)sh * I, (size_t)SI + (size_t)sh * I, xt, d,
                              I, h);
                add_down(Wsh, dt, (size_t)2 * SI * d, (size_t)SI, sh * I, h, I, 1.0, d, yt);
            }
            if (idx_out) memcpy(idx_out + (size_t)n * k, idx, sizeof(int32_t) * k);
            if (w_out) memcpy(w_out + (size_t)n * k, w, sizeof(double) * k);
        }
        free(xt);
        free(g);
        free(s);
        free(h);
        free(idx);
        free(w);
    }
    return 0;
}

/*
 * ---------------------------------------------------------------------------
 * Backward of the layer (training; the training use of the layer is the
 * pretraining setup of [FusionLLM]).  For a scalar loss L with a given
 * upstream gradient dy [T, d] = dL/dy, the chain rule through steps 1-7 gives,
 * token by token (e_j the chosen experts, o_j = W_down[e_j] h_j the expert's
 * unweighted output):
 *
 *   a_j = dL/dw_j = dy . o_j,   abar = sum_j w_j a_j
 *   gate, score_func 0: w_j = s_j / S with S = sum_j s_j, so
 *                       dL/ds_j = (a_j - abar) / S and
 *                       dL/dl_j = dL/ds_j * s_j * (1 - s_j)
 *   gate, score_func 1: w = softmax of the chosen logits, so
 *                       dL/dl_j = w_j * (a_j - abar)
 *        Only the chosen experts' scores enter the weights; the selection is
 *        piecewise constant and passes no gradient; a selection bias only
 *        moves the selection.  Logits of experts not chosen get 0.
 *   router:  dW_router[e] += dL/dl_e * x,   dx += sum_j dL/dl_j * W_router[e_j]
 *   expert e_j (weight w_j; a shared expert has weight 1):
 *            do = w_j dy,  dh = W_down^T do,  dW_down += do h^T,
 *            dg = dh * u * silu'(g),  du = dh * silu(g),
 *            silu(g) = g sigmoid(g),  silu'(g) = sigmoid(g) (1 + g (1 - sigmoid(g))),
 *            dW_gate += dg x^T,  dW_up += du x^T,
 *            dx += W_gate^T dg + W_up^T du
 *
 * Phase 1 handles each token on its own (in parallel) and keeps per chosen
 * slot (t, j) the vectors dg|du and h; phase 2 forms every weight-gradient row
 * as a sum over tokens in token order (one thread per row), so the result
 * does not depend on the thread count.
 */

/* Per-token inputs and outputs of the backward. */
typedef struct {
    const void *x, *Wr, *Wgu, *Wd, *Wsh, *dy;
    int dt, T, d, E, k, G, TG, I, S, score_func;
    const double *bias;
} bwd_args;

/* Routing of token t (idx, w, the chosen experts' gate scores gsel) with an
 * optional forced set. */
static void bwd_route(const bwd_args *A, const double *xt, const int32_t *forced, double *g,
                      double *s, int32_t *idx, double *w, double *gsel) {
    double ge, gg;
    route_token(xt, A->Wr, A->dt, A->d, A->E, A->k, A->G, A->TG, A->score_func, A->bias, g, s,
                idx, w, &ge, &gg);
    if (forced) {
        for (int j = 0; j < A->k; ++j) idx[j] = forced[j];
        gate_weights(g, idx, A->k, A->score_func, w);
    }
    for (int j = 0; j < A->k; ++j) gsel[j] = g[idx[j]];
}

/* One SwiGLU expert's backward for one token.  The expert's gate rows start at
 * element gu_base + g_row0 * d of Wgu, its up rows at gu_base + u_row0 * d;
 * its down matrix has rows of length dn_len starting at dn_base, the expert's
 * columns from col0.  coef: the expert's weight.  Writes h [n], dgu [2n]
 * (dg then du) and, when dx_acc is given, adds W_gate^T dg + W_up^T du to it.
 * Returns a = dy . (W_down h) (the unweighted output against dy). */
static double expert_backward(const void *Wgu, const void *Wdn, int dt, size_t gu_base,
                              size_t g_row0, size_t u_row0, size_t dn_base, size_t dn_len,
                              int col0, const double *xt, const double *dyt, int d, int n,
                              double coef, double *h, double *dgu, double *dx_acc) {
    double a = 0.0;
    for (int i = 0; i < n; ++i) {
        double g = dot_row(Wgu, dt, gu_base + (g_row0 + i) * (size_t)d, xt, d);
        double u = dot_row(Wgu, dt, gu_base + (u_row0 + i) * (size_t)d, xt, d);
        double sg = sigmoid(g);
        h[i] = g * sg * u;
        /* dh_i = coef * sum_c W_down[c, col0 + i] dy[c] */
        double q = 0.0;
        for (int c = 0; c < d; ++c) q += elem(Wdn, dt, dn_base + (size_t)c * dn_len + col0 + i) * dyt[c];
        double dh = coef * q;
        dgu[i] = dh * u * sg * (1.0 + g * (1.0 - sg));
        dgu[n + i] = dh * g * sg;
    }
    /* a = dy . o with o = W_down h, the plain definition */
    for (int c = 0; c < d; ++c)
        a += dyt[c] * dot_row(Wdn, dt, dn_base + (size_t)c * dn_len + col0, h, n);
    if (dx_acc) {
        for (int i = 0; i < n; ++i) {
            size_t gr = gu_base + (g_row0 + i) * (size_t)d, ur = gu_base + (u_row0 + i) * (size_t)d;
            for (int c = 0; c < d; ++c)
                dx_acc[c] += dgu[i] * elem(Wgu, dt, gr + c) + dgu[n + i] * elem(Wgu, dt, ur + c);
        }
    }
    return a;
}

/* d L / d l for the chosen experts of one token from a_j, w_j and the chosen
 * gate scores gsel_j (sigmoid scores for score_func 0, logits for 1). */
static void router_grad(int score_func, int k, const double *a, const double *w,
                        const double *gsel, double *dl) {
    double abar = 0.0, S = 0.0;
    for (int j = 0; j < k; ++j) abar += w[j] * a[j];
    for (int j = 0; j < k; ++j) S += gsel[j];
    for (int j = 0; j < k; ++j) {
        if (score_func == 0)
            dl[j] = (a[j] - abar) / S * gsel[j] * (1.0 - gsel[j]);
        else
            dl[j] = w[j] * (a[j] - abar);
    }
}

/* Phase 1 for token t: dx row (when dx_t is given), dl [k], and per chosen
 * slot j: h_slots [k, I] and dgu_slots [k, 2I]; shared experts: h_sh [SI] and
 * dgu_sh [2SI] (skipped when h_sh is NULL; dx_t then lacks their part). */
static void token_backward(const bwd_args *A, int t, const int32_t *forced, double *xt,
                           double *dyt, int32_t *idx, double *w, double *dl, double *h_slots,
                           double *dgu_slots, double *h_sh, double *dgu_sh, double *dx_t) {
    const int d = A->d, k = A->k, I = A->I, S = A->S, E = A->E;
    const int SI = S * I;
    double *g = (double *)malloc(sizeof(double) * E);
    double *s = (double *)malloc(sizeof(double) * E);
    double *a = (double *)malloc(sizeof(double) * k);
    double *gsel = (double *)malloc(sizeof(double) * k);
    load_row(A->x, A->dt, (size_t)t * d, d, xt);
    load_row(A->dy, A->dt, (size_t)t * d, d, dyt);
    bwd_route(A, xt, forced, g, s, idx, w, gsel);
    if (dx_t)
        for (int c = 0; c < d; ++c) dx_t[c] = 0.0;
    for (int j = 0; j < k; ++j) {
        int e = idx[j];
        a[j] = expert_backward(A->Wgu, A->Wd, A->dt, (size_t)e * 2 * I * d, 0, (size_t)I,
                               (size_t)e * d * I, (size_t)I, 0, xt, dyt, d, I, w[j],
                               h_slots + (size_t)j * I, dgu_slots + (size_t)j * 2 * I, dx_t);
    }
    router_grad(A->score_func, k, a, w, gsel, dl);
    if (dx_t)
        for (int j = 0; j < k; ++j) {
            size_t r = (size_t)idx[j] * d;
            for (int c = 0; c < d; ++c) dx_t[c] += dl[j] * elem(A->Wr, A->dt, r + c);
        }
    /* shared expert sh: gate rows sh*I.., up rows SI + sh*I.. of the gate_up
     * block, down columns sh*I.. of the [d, SI] block; weight 1 */
    for (int sh = 0; sh < (h_sh ? S : 0); ++sh) {
        double *hh = (double *)malloc(sizeof(double) * I);
        double *dd = (double *)malloc(sizeof(double) * 2 * I);
        expert_backward(A->Wsh, A->Wsh, A->dt, 0, (size_t)sh * I, (size_t)SI + (size_t)sh * I,
                        (size_t)2 * SI * d, (size_t)SI, sh * I, xt, dyt, d, I, 1.0, hh, dd, dx_t);
        for (int i = 0; i < I; ++i) {
            h_sh[sh * I + i] = hh[i];
            dgu_sh[sh * I + i] = dd[i];
            dgu_sh[SI + sh * I + i] = dd[I + i];
        }
        free(hh);
        free(dd);
    }
    free(g);
    free(s);
    free(a);
    free(gsel);
}

static int bwd_check(const bwd_args *A, const int32_t *forced) {
    if (oracle_check_args(A->T, A->d, A->E, A->k, A->G, A->TG) || A->I <= 0 || A->S < 0) return -1;
    if (A->score_func < 0 || A->score_func > 1) return -1;
    if (A->S > 0 && !A->Wsh) return -1;
    if (!A->dy) return -1;
    if (forced)
        for (size_t n = 0; n < (size_t)A->T * A->k; ++n)
            if (forced[n] < 0 || forced[n] >= A->E) return -1;
    return 0;
}

/*
 * Full backward for all T tokens.  dy [T,d] in the dtype of x.  forced_idx
 * [T,k] (nullable): expert sets to use in place of the oracle's own top-k
 * (weights still from the oracle's scores).  Outputs, fp64, in the layouts of
 * the forward's tensors: dx [T,d], dWr [E,d], dWgu [E,2I,d], dWd [E,d,I],
 * dWsh [2SI*d + d*SI] (gate_up block then down block; nullable when S == 0),
 * idx_out [T,k] and dl_out [T,k] (dL/dlogit of the chosen experts; both
 * nullable).  Returns 0, or -1 on invalid arguments.
 */
int oracle_backward(const void *x, const void *Wr, const void *Wgu, const void *Wd,
                    const void *Wsh, int dt, int T, int d, int E, int k, int G, int TG, int I,
                    int S, int score_func, const double *bias, const int32_t *forced_idx,
                    const void *dy, double *dx, double *dWr, double *dWgu, double *dWd,
                    double *dWsh, int32_t *idx_out, double *dl_out, int nthreads) {
    bwd_args A = {x, Wr, Wgu, Wd, Wsh, dy, dt, T, d, E, k, G, TG, I, S, score_func, bias};
    if (bwd_check(&A, forced_idx)) return -1;
    const int SI = S * I;
    const size_t Tk = (size_t)T * k;
    int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * (Tk + 1));
    double *w = (double *)malloc(sizeof(double) * (Tk + 1));
    double *dl = (double *)malloc(sizeof(double) * (Tk + 1));
    double *hs = (double *)malloc(sizeof(double) * (Tk * I + 1));
    double *dgus = (double *)malloc(sizeof(double) * (Tk * 2 * I + 1));
    double *hsh = (double *)malloc(sizeof(double) * ((size_t)T * SI + 1));
    double *dgush = (double *)malloc(sizeof(double) * ((size_t)T * 2 * SI + 1));
    double *xs = (double *)malloc(sizeof(double) * ((size_t)T * d + 1));
    double *dys = (double *)malloc(sizeof(double) * ((size_t)T * d + 1));
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
    /* phase 1: token by token */
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int t = 0; t < T; ++t)
        token_backward(&A, t, forced_idx ? forced_idx + (size_t)t * k : NULL, xs + (size_t)t * d,
                       dys + (size_t)t * d, idx + (size_t)t * k, w + (size_t)t * k,
                       dl + (size_t)t * k, hs + (size_t)t * k * I, dgus + (size_t)t * k * 2 * I,
                       hsh + (size_t)t * SI, dgush + (size_t)t * 2 * SI, dx + (size_t)t * d);

    /* phase 2: weight-gradient rows, each a sum over tokens in token order */
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int e = 0; e < E; ++e) {
        double *row = dWr + (size_t)e * d;
        for (int c = 0; c < d; ++c) row[c] = 0.0;
        for (size_t n = 0; n < Tk; ++n)
            if (idx[n] == e) {
                const double *xt = xs + (n / k) * d;
                for (int c = 0; c < d; ++c) row[c] += dl[n] * xt[c];
            }
    }
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 4)
#endif
    for (long er = 0; er < (long)E * 2 * I; ++er) {
        const int e = (int)(er / (2 * I)), r = (int)(er % (2 * I));
        double *row = dWgu + (size_t)er * d;
        for (int c = 0; c < d; ++c) row[c] = 0.0;
        for (size_t n = 0; n < Tk; ++n)
            if (idx[n] == e) {
                const double v = dgus[n * 2 * I + r];
                const double *xt = xs + (n / k) * d;
                for (int c = 0; c < d; ++c) row[c] += v * xt[c];
            }
    }
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 4)
#endif
    for (long ec = 0; ec < (long)E * d; ++ec) {
        const int e = (int)(ec / d), c = (int)(ec % d);
        double *row = dWd + (size_t)ec * I;
        for (int i = 0; i < I; ++i) row[i] = 0.0;
        for (size_t n = 0; n < Tk; ++n)
            if (idx[n] == e) {
                const double v = w[n] * dys[(n / k) * d + c];
                const double *hn = hs + n * I;
                for (int i = 0; i < I; ++i) row[i] += v * hn[i];
            }
    }
    if (S > 0 && dWsh) {
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 4)
#endif
        for (int r = 0; r < 2 * SI; ++r) {
            double *row = dWsh + (size_t)r * d;
            for (int c = 0; c < d; ++c) row[c] = 0.0;
            for (int t = 0; t < T; ++t) {
                const double v = dgush[(size_t)t * 2 * SI + r];
                const double *xt = xs + (size_t)t * d;
                for (int c = 0; c < d; ++c) row[c] += v * xt[c];
            }
        }
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 4)
#endif
        for (int c = 0; c < d; ++c) {
            double *row = dWsh + (size_t)2 * SI * d + (size_t)c * SI;
            for (int i = 0; i < SI; ++i) row[i] = 0.0;
            for (int t = 0; t < T; ++t) {
                const double v = dys[(size_t)t * d + c];
                const double *hn = hsh + (size_t)t * SI;
                for (int i = 0; i < SI; ++i) row[i] += v * hn[i];
            }
        }
    }
    if (idx_out) memcpy(idx_out, idx, sizeof(int32_t) * Tk);
    if (dl_out) memcpy(dl_out, dl, sizeof(double) * Tk);
    free(idx);
    free(w);
    free(dl);
    free(hs);
    free(dgus);
    free(hsh);
    free(dgush);
    free(xs);
    free(dys);
    return 0;
}

/* dg (which 0) or du (which 1) of feature i of one SwiGLU expert for one
 * token; expert located as in expert_backward. */
static double swiglu_grad_entry(const void *Wgu, const void *Wdn, int dt, size_t gu_base,
                                size_t g_row0, size_t u_row0, size_t dn_base, size_t dn_len,
                                int col0, const double *xt, const double *dyt, int d, int i,
                                double coef, int which) {
    double g = dot_row(Wgu, dt, gu_base + (g_row0 + i) * (size_t)d, xt, d);
    double u = dot_row(Wgu, dt, gu_base + (u_row0 + i) * (size_t)d, xt, d);
    double sg = sigmoid(g);
    double q = 0.0;
    for (int c = 0; c < d; ++c) q += elem(Wdn, dt, dn_base + (size_t)c * dn_len + col0 + i) * dyt[c];
    double dh = coef * q;
    return which == 0 ? dh * u * sg * (1.0 + g * (1.0 - sg)) : dh * g * sg;
}

/*
 * Selected entries of the backward at any batch size, each computed on its
 * own with the arithmetic of oracle_backward: dx rows of the tokens
 * dx_tokens[n_dx] (into dx_rows [n_dx, d]), and weight-gradient rows
 * wsel[2 n] = (tensor, row) into wrows [n_w, ld]:
 *   0  dW_router row e            (d values)
 *   1  dW_gate_up row e * 2I + r  (d values)
 *   2  dW_down row e * d + c      (I values)
 *   3  dW_shared gate_up row r    (d values)
 *   4  dW_shared down row c       (SI values)
 * Every sum over tokens runs in token order.  Returns 0, or -1.
 */
int oracle_backward_rows(const void *x, const void *Wr, const void *Wgu, const void *Wd,
                         const void *Wsh, int dt, int T, int d, int E, int k, int G, int TG,
                         int I, int S, int score_func, const double *bias,
                         const int32_t *forced_idx, const void *dy, const int32_t *dx_tokens,
                         int n_dx, double *dx_rows, const int32_t *wsel, int n_w, double *wrows,
                         int ld, int nthreads) {
    bwd_args A = {x, Wr, Wgu, Wd, Wsh, dy, dt, T, d, E, k, G, TG, I, S, score_func, bias};
    if (bwd_check(&A, forced_idx)) return -1;
    const int SI = S * I;
    const size_t Tk = (size_t)T * k;
    for (int n = 0; n < n_dx; ++n)
        if (dx_tokens[n] < 0 || dx_tokens[n] >= T) return -1;
    for (int n = 0; n < n_w; ++n) {
        const int ten = wsel[2 * n], r = wsel[2 * n + 1];
        const long lim = ten == 0 ? E : ten == 1 ? (long)E * 2 * I : ten == 2 ? (long)E * d
                         : ten == 3 ? 2L * SI : ten == 4 ? d : 0;
        const int len = ten == 2 ? I : ten == 4 ? SI : d;
        if (r < 0 || r >= lim || len > ld || ((ten == 3 || ten == 4) && S == 0)) return -1;
    }
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
    /* routing of every token (the sets decide which tokens reach each row) */
    int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * (Tk + 1));
    double *w = (double *)malloc(sizeof(double) * (Tk + 1));
    double *vals = (double *)malloc(sizeof(double) * (Tk + 1));
#ifdef _OPENMP
#pragma omp parallel
#endif
    {
        double *xt = (double *)malloc(sizeof(double) * d);
        double *g = (double *)malloc(sizeof(double) * E);
        double *sc = (double *)malloc(sizeof(double) * E);
        double *gsel = (double *)malloc(sizeof(double) * k);
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 16)
#endif
        for (int t = 0; t < T; ++t) {
            load_row(x, dt, (size_t)t * d, d, xt);
            bwd_route(&A, xt, forced_idx ? forced_idx + (size_t)t * k : NULL, g, sc,
                      idx + (size_t)t * k, w + (size_t)t * k, gsel);
        }
        free(xt);
        free(g);
        free(sc);
        free(gsel);
    }
    /* dx rows: the whole per-token backward */
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int n = 0; n < n_dx; ++n) {
        double *xt = (double *)malloc(sizeof(double) * d), *dyt = (double *)malloc(sizeof(double) * d);
        int32_t *ii = (int32_t *)malloc(sizeof(int32_t) * k);
        double *ww = (double *)malloc(sizeof(double) * k), *dl = (double *)malloc(sizeof(double) * k);
        double *hs = (double *)malloc(sizeof(double) * (size_t)k * I);
        double *dg = (double *)malloc(sizeof(double) * (size_t)k * 2 * I);
        double *hsh = (double *)malloc(sizeof(double) * (SI + 1));
        double *dgsh = (double *)malloc(sizeof(double) * (2 * SI + 1));
        const int t = dx_tokens[n];
        token_backward(&A, t, forced_idx ? forced_idx + (size_t)t * k : NULL, xt, dyt, ii, ww, dl,
                       hs, dg, hsh, dgsh, dx_rows + (size_t)n * d);
        free(xt); free(dyt); free(ii); free(ww); free(dl); free(hs); free(dg); free(hsh); free(dgsh);
    }
    /* weight-gradient rows */
    for (int q = 0; q < n_w; ++q) {
        const int ten = wsel[2 * q], r = wsel[2 * q + 1];
        double *row = wrows + (size_t)q * ld;
        const int len = ten == 2 ? I : ten == 4 ? SI : d;
        for (int c = 0; c < len; ++c) row[c] = 0.0;
        const int e = ten == 0 ? r : ten == 1 ? r / (2 * I) : ten == 2 ? r / d : -1;
        /* the slots (routed rows: those of expert e, in token order) or tokens
         * (shared rows) that reach this row */
        const size_t nall = (ten <= 2) ? Tk : (size_t)T;
        size_t *list = (size_t *)malloc(sizeof(size_t) * (nall + 1));
        size_t nl = 0;
        for (size_t n = 0; n < nall; ++n)
            if (ten > 2 || idx[n] == e) list[nl++] = n;
        const int vlen = ten == 2 ? I : ten == 4 ? SI : 0;
        double *vecs = vlen ? (double *)malloc(sizeof(double) * (nl * vlen + 1)) : NULL;
        /* per listed slot or token: the scalar (and vector) this row needs, in
         * parallel; then the ordered sum */
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 8)
#endif
        for (size_t m = 0; m < nl; ++m) {
            const size_t n = list[m];
            const int t = (ten <= 2) ? (int)(n / k) : (int)n;
            double *xt = (double *)malloc(sizeof(double) * d), *dyt = (double *)malloc(sizeof(double) * d);
            load_row(x, dt, (size_t)t * d, d, xt);
            load_row(dy, dt, (size_t)t * d, d, dyt);
            if (ten == 0) {
                /* dL/dl of this slot needs the token's whole routed backward */
                int32_t *ii = (int32_t *)malloc(sizeof(int32_t) * k);
                double *ww = (double *)malloc(sizeof(double) * k), *dl = (double *)malloc(sizeof(double) * k);
                double *hs = (double *)malloc(sizeof(double) * (size_t)k * I);
                double *dg = (double *)malloc(sizeof(double) * (size_t)k * 2 * I);
                token_backward(&A, t, forced_idx ? forced_idx + (size_t)t * k : NULL, xt, dyt, ii,
                               ww, dl, hs, dg, NULL, NULL, NULL);
                vals[m] = dl[n % k];
                free(ii); free(ww); free(dl); free(hs); free(dg);
            } else if (ten == 1) {
                const int rr = r % (2 * I);
                vals[m] = swiglu_grad_entry(Wgu, Wd, dt, (size_t)e * 2 * I * d, 0, (size_t)I,
                                            (size_t)e * d * I, (size_t)I, 0, xt, dyt, d, rr % I,
                                            w[n], rr >= I);
            } else if (ten == 2) {
                swiglu_hidden(Wgu, dt, (size_t)e * 2 * I * d, 0, (size_t)I, xt, d, I,
                              vecs + m * I);
                vals[m] = w[n] * dyt[r % d];
            } else if (ten == 3) {
                vals[m] = swiglu_grad_entry(Wsh, Wsh, dt, 0, 0, (size_t)SI, (size_t)2 * SI * d,
                                            (size_t)SI, 0, xt, dyt, d, r % SI, 1.0, r >= SI);
            } else {
                for (int sh = 0; sh < S; ++sh)
                    swiglu_hidden(Wsh, dt, 0, (size_t)sh * I, (size_t)SI + (size_t)sh * I, xt, d,
                                  I, vecs + m * SI + (size_t)sh * I);
                vals[m] = dyt[r];
            }
            free(xt);
            free(dyt);
        }
        for (size_t m = 0; m < nl; ++m) {
            const size_t n = list[m];
            const int t = (ten <= 2) ? (int)(n / k) : (int)n;
            if (vlen) {
                const double *hv = vecs + m * vlen;
                for (int i = 0; i < vlen; ++i) row[i] += vals[m] * hv[i];
            } else {
                for (int c = 0; c < d; ++c) row[c] += vals[m] * elem(x, dt, (size_t)t * d + c);
            }
        }
        free(list);
        free(vecs);
    }
    free(idx);
    free(w);
    free(vals);
    return 0;
}

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
