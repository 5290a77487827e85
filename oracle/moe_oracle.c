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

enum { OR_F32 = 0, OR_BF16 = 1 };

/* Widen element i of an fp32 or bf16 array to double. */
static inline double elem(const void *p, int dt, size_t i) {
    if (dt == OR_F32) return (double)((const float *)p)[i];
    uint32_t bits = ((uint32_t)((const uint16_t *)p)[i]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* sum_c a[off + c] * v[c], c < n, fp64 accumulate.  a is fp32 or bf16, v is fp64. */
static double dot_row(const void *a, int dt, size_t off, const double *v, int n) {
    double acc = 0.0;
    if (dt == OR_F32) {
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

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
