// Fused router: router GEMM (fp32 accumulate), bias-free sigmoid gate,
// group-limited top-k with warp shuffles, weight normalisation.
//
// The layer's routing is the one of "FusionLLM：融合 MLA、GDN 与 MoE 的高效混合
// 架构大模型训练框架", section "混合专家（MoE）" (group-limited routing, bias-free
// sigmoid gating) on the linear router g(x) = W_g x with a fixed k of
// "大模型工程（一）：Transformer 到 MoE", section "MoE 数学：路由、容量与平衡详解".
// Group score = max score inside the group; ties go to the lower index.
//
// Selection compares fp32 logits: sigmoid is monotone, so the kept groups and
// the chosen experts are the ones a comparison of sigmoid scores would pick,
// without the ties that rounding sigmoid(l) to fp32 near 0 or 1 would create.
//
// Gating variants of "大模型工程（一）：Transformer 到 MoE", section "MoE 数学：路由、
// 容量与平衡详解": MOE_GATE_SOFTMAX_TOPK (select on the logits, weights =
// softmax of the k chosen logits) and a selection-only expert bias b[E]
// (aux-loss-free balancing: select on gate score + b, weigh with the unbiased
// scores; gate score = sigmoid(l) for the sigmoid gate, l for softmax).
#include <float.h>
#include <limits.h>

#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {

namespace {

constexpr int kRouteTokens = 32;   // tokens per CTA
constexpr int kRouteKChunk = 32;   // reduction chunk staged in shared memory
constexpr int kRouteThreads = 256;

// Selection key of expert e from its fp32 logit l.
__device__ __forceinline__ float sel_key(float l, int e, int gate, const float* bias) {
    if (bias == nullptr) return l;  // monotone in the gate score for both gates
    const float g = gate == MOE_GATE_SIGMOID ? 1.f / (1.f + expf(-l)) : l;
    return g + bias[e];
}

// Weights of the k chosen experts from their logits (one thread).
__device__ __forceinline__ void gate_weights(const float (&l)[kMaxK], int k, int gate,
                                             float (&w)[kMaxK]) {
    float sum = 0.f;
    if (gate == MOE_GATE_SIGMOID) {
#pragma unroll
        for (int r = 0; r < kMaxK; ++r) {
            if (r >= k) break;
            w[r] = 1.f / (1.f + expf(-l[r]));
            sum += w[r];
        }
    } else {
        float m = l[0];
#pragma unroll
        for (int r = 1; r < kMaxK; ++r)
            if (r < k) m = fmaxf(m, l[r]);
#pragma unroll
        for (int r = 0; r < kMaxK; ++r) {
            if (r >= k) break;
            w[r] = expf(l[r] - m);
            sum += w[r];
        }
    }
#pragma unroll
    for (int r = 0; r < kMaxK; ++r)
        if (r < k) w[r] /= sum;
}

// (v, i) beats (bv, bi): larger value, ties to the lower index; bi == INT_MAX
// marks "nothing yet".
__device__ __forceinline__ bool beats(float v, int i, float bv, int bi) {
    return bi == INT_MAX || v > bv || (v == bv && i < bi);
}

__device__ __forceinline__ void warp_argmax(float& v, int& i) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        float ov = __shfl_xor_sync(0xffffffffu, v, off);
        int oi = __shfl_xor_sync(0xffffffffu, i, off);
        if (oi != INT_MAX && beats(ov, oi, v, i)) {
            v = ov;
            i = oi;
        }
    }
}

// Argmax over each aligned segment of 8 lanes (same tie rule as warp_argmax).
__device__ __forceinline__ void seg8_argmax(float& v, int& i) {
#pragma unroll
    for (int off = 4; off > 0; off >>= 1) {
        float ov = __shfl_xor_sync(0xffffffffu, v, off);
        int oi = __shfl_xor_sync(0xffffffffu, i, off);
        if (oi != INT_MAX && beats(ov, oi, v, i)) {
            v = ov;
            i = oi;
        }
    }
}

// Group-limited top-k of one token from its fp32 logits L[0..E) (shared
// memory), by one warp.  Writes k expert ids (descending, ties to the lower
// index) and the normalised sigmoid weights.
template <int EJ>
__device__ __forceinline__ void warp_topk(const float* L, int lane, int E, int k, int G, int TG,
                                          int gate, const float* __restrict__ bias,
                                          int32_t* __restrict__ idx_out,
                                          float* __restrict__ w_out) {
    const int gsz = E / G;
    // group scores: max key of each group (lane g < G owns group g)
    float gval = -INFINITY;
    if (lane < G)
        for (int e = lane * gsz; e < (lane + 1) * gsz; ++e)
            gval = fmaxf(gval, sel_key(L[e], e, gate, bias));
    uint32_t kept = 0;
    for (int r = 0; r < TG; ++r) {
        float v = -INFINITY;
        int i = INT_MAX;
        if (lane < G && !((kept >> lane) & 1u)) {
            v = gval;
            i = lane;
        }
        warp_argmax(v, i);
        kept |= 1u << i;
    }
    // candidates: experts lane + 32 j inside kept groups
    float cv[EJ];
    bool cand[EJ];
#pragma unroll
    for (int j = 0; j < EJ; ++j) {
        int e = lane + 32 * j;
        cand[j] = e < E && ((kept >> (e / gsz)) & 1u);
        cv[j] = cand[j] ? sel_key(L[e], e, gate, bias) : -INFINITY;
    }
    int sel_e[kMaxK];
    float sel_l[kMaxK];
#pragma unroll
    for (int r = 0; r < kMaxK; ++r) {
        if (r >= k) break;
        float bv = -INFINITY;
        int bi = INT_MAX;
#pragma unroll
        for (int j = 0; j < EJ; ++j) {
            int e = lane + 32 * j;
            if (cand[j] && beats(cv[j], e, bv, bi)) {
                bv = cv[j];
                bi = e;
            }
        }
        warp_argmax(bv, bi);
#pragma unroll
        for (int j = 0; j < EJ; ++j)
            if (lane + 32 * j == bi) cand[j] = false;
        sel_e[r] = bi;
    }
    if (lane == 0) {
#pragma unroll
        for (int r = 0; r < kMaxK; ++r)
            if (r < k) sel_l[r] = L[sel_e[r]];
        float wv[kMaxK];
        gate_weights(sel_l, k, gate, wv);
#pragma unroll
        for (int r = 0; r < kMaxK; ++r) {
            if (r >= k) break;
            idx_out[r] = sel_e[r];
            w_out[r] = wv[r];
        }
    }
}

// CUDA-core router for any E <= 256 (fp32 or bf16 inputs): 32 tokens per CTA.
template <typename TIn, int EJ>
__global__ void __launch_bounds__(kRouteThreads) route_kernel(const TIn* __restrict__ x,
                                                              const TIn* __restrict__ Wr, int T,
                                                              int d, int E, int k, int G, int TG,
                                                              int gate,
                                                              const float* __restrict__ bias,
                                                              int32_t* __restrict__ idx_out,
                                                              float* __restrict__ w_out,
                                                              int* status) {
    extern __shared__ float sm[];
    // phase 1 layout: xs [32][33], ws [E][33]; phase 2 reuses it as logits [32][E+1]
    float* xs = sm;
    float* ws = sm + kRouteTokens * (kRouteKChunk + 1);
    float* logit = sm;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int t0 = blockIdx.x * kRouteTokens;

    pdl_wait();
    if (status != nullptr && blockIdx.x == 0 && tid < 16) status[tid] = 0;

    float acc[4][EJ];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < EJ; ++j) acc[i][j] = 0.f;

    for (int c0 = 0; c0 < d; c0 += kRouteKChunk) {
        for (int i = tid; i < kRouteTokens * kRouteKChunk; i += kRouteThreads) {
            int r = i / kRouteKChunk, c = i % kRouteKChunk;
            int t = t0 + r;
            xs[r * (kRouteKChunk + 1) + c] =
                t < T ? Elem<TIn>::to_f(x[(size_t)t * d + c0 + c]) : 0.f;
        }
        for (int i = tid; i < E * kRouteKChunk; i += kRouteThreads) {
            int r = i / kRouteKChunk, c = i % kRouteKChunk;
            ws[r * (kRouteKChunk + 1) + c] = Elem<TIn>::to_f(Wr[(size_t)r * d + c0 + c]);
        }
        __syncthreads();
#pragma unroll 4
        for (int c = 0; c < kRouteKChunk; ++c) {
            float xv[4], wv[EJ];
#pragma unroll
            for (int i = 0; i < 4; ++i) xv[i] = xs[(warp * 4 + i) * (kRouteKChunk + 1) + c];
#pragma unroll
            for (int j = 0; j < EJ; ++j) {
                int e = lane + 32 * j;
                wv[j] = e < E ? ws[e * (kRouteKChunk + 1) + c] : 0.f;
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < EJ; ++j) acc[i][j] = fmaf(xv[i], wv[j], acc[i][j]);
        }
        __syncthreads();
    }
    // logits to shared memory (NaN treated as -inf so the order stays total)
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < EJ; ++j) {
            int e = lane + 32 * j;
            if (e < E) {
                float v = acc[i][j];
                logit[(warp * 4 + i) * (E + 1) + e] = (v != v) ? -INFINITY : v;
            }
        }
    __syncthreads();
    for (int tt = 0; tt < 4; ++tt) {
        const int tl = warp * 4 + tt;
        const int t = t0 + tl;
        if (t >= T) break;  // warp-uniform
        warp_topk<EJ>(logit + tl * (E + 1), lane, E, k, G, TG, gate, bias, idx_out + (size_t)t * k,
                      w_out + (size_t)t * k);
    }
    pdl_trigger();
}

// ---------------------------------------------------------------------------
// Tensor-core router for bf16, E <= 128, E % 16 == 0: mma.sync m16n8k16
// (bf16 in, fp32 accumulate).  CTA = 8 warps over 32 tokens: warp (wm, wk)
// computes tokens [16 wm, 16 wm + 16) x all E experts over the k-quarter wk of
// every 256-wide chunk of d; the four partial sums are added in fixed order
// (wk = 0..3) through shared memory, so the logits do not depend on timing.
// x and W_router chunks are staged with cp.async (double buffered).
constexpr int kMmaTokens = 32;
constexpr int kMmaKC = 256;             // d per pipeline stage (4 warps x 64)
constexpr int kMmaLd = kMmaKC + 8;      // padded smem row (bf16): conflict-free ldmatrix

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool pred) {
    const uint32_t s = smem_u32(smem);
    const int n = pred ? 16 : 0;  // zero-fill when out of range
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(s), "l"(gmem), "r"(n)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], const void* p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(p)));
}

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4],
                                               uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// NT = E / 8 n-tiles of 8 experts (E = 8 NT, NT even); S cp.async stages
template <int NT, int S>
__global__ void __launch_bounds__(256) route_mma_kernel(const __nv_bfloat16* __restrict__ x,
                                                        const __nv_bfloat16* __restrict__ Wr,
                                                        int T, int d, int E, int k, int G,
                                                        int TG, int gate,
                                                        const float* __restrict__ bias,
                                                        int32_t* __restrict__ idx_out,
                                                        float* __restrict__ w_out,
                                                        int* status) {
    extern __shared__ __align__(16) uint8_t rsm[];
    __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(rsm);  // [S][32][kMmaLd]
    __nv_bfloat16* wsm = xs + S * kMmaTokens * kMmaLd;          // [S][E][kMmaLd]
    float* red = reinterpret_cast<float*>(rsm);                // after the loop: [4][32][E+1]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int wm = warp & 1, wk = warp >> 1;
    const int t0 = blockIdx.x * kMmaTokens;
    pdl_wait();
    if (status != nullptr && blockIdx.x == 0 && tid < 16) status[tid] = 0;

    // each thread copies fixed (row, 16-byte column) pieces of every chunk
    auto load_chunk = [&](int stage, int c0) {
        __nv_bfloat16* xd = xs + stage * kMmaTokens * kMmaLd;
        __nv_bfloat16* wd = wsm + stage * E * kMmaLd;
        // x: 32 rows x 256 cols = 1024 16-byte pieces, 4 per thread
#pragma unroll
        for (int m = 0; m < kMmaTokens * (kMmaKC / 8) / 256; ++m) {
            const int i = tid + 256 * m;
            const int r = i >> 5, c = (i & 31) * 8;
            const int t = t0 + r;
            cp_async16(xd + r * kMmaLd + c, x + (size_t)(t < T ? t : 0) * d + c0 + c, t < T);
        }
        for (int i = tid; i < E * (kMmaKC / 8); i += 256) {
            const int r = i >> 5, c = (i & 31) * 8;
            cp_async16(wd + r * kMmaLd + c, Wr + (size_t)r * d + c0 + c, true);
        }
        cp_async_commit();
    };

    float acc[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[n][q] = 0.f;

    // S-deep cp.async ring: one commit group per chunk (empty groups past the
    // end keep the count uniform), so waiting until S-1 groups are pending
    // means chunk ch has landed
    const int n_chunks = d / kMmaKC;
#pragma unroll
    for (int st = 0; st < S - 1; ++st) {
        if (st < n_chunks)
            load_chunk(st, st * kMmaKC);
        else
            cp_async_commit();
    }
    for (int ch = 0; ch < n_chunks; ++ch) {
        const int nx = ch + S - 1;
        if (nx < n_chunks)
            load_chunk(nx % S, nx * kMmaKC);  // the buffer chunk ch - 1 has been read from
        else
            cp_async_commit();
        cp_async_wait<S - 1>();
        __syncthreads();
        const __nv_bfloat16* xc = xs + (ch % S) * kMmaTokens * kMmaLd;
        const __nv_bfloat16* wc = wsm + (ch % S) * E * kMmaLd;
#pragma unroll
        for (int kk = 0; kk < 64; kk += 16) {
            const int kb = wk * 64 + kk;
            // A fragment: rows 16 wm + (lane & 15), columns kb + 8 (lane >> 4)
            uint32_t a[4];
            ldmatrix_x4(a, xc + (wm * 16 + (lane & 15)) * kMmaLd + kb + 8 * (lane >> 4));
#pragma unroll
            for (int n = 0; n < NT; n += 2) {
                // B fragments of n-tiles n, n+1: expert rows 8n + (lane & 7) + 8 (lane >> 4),
                // k halves by bit 3 of the lane
                uint32_t b[4];
                ldmatrix_x4(b, wc + (8 * n + (lane & 7) + 8 * (lane >> 4)) * kMmaLd + kb +
                                   8 * ((lane >> 3) & 1));
                mma_bf16_16816(acc[n], a, b[0], b[1]);
                mma_bf16_16816(acc[n + 1], a, b[2], b[3]);
            }
        }
        __syncthreads();
    }
    // partial logits of this warp's k-quarter -> red[wk][token][expert]
    const int Ep = E + 1;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        const int r0 = wm * 16 + (lane >> 2), col = 8 * n + 2 * (lane & 3);
        float* base = red + (size_t)wk * kMmaTokens * Ep;
        base[r0 * Ep + col] = acc[n][0];
        base[r0 * Ep + col + 1] = acc[n][1];
        base[(r0 + 8) * Ep + col] = acc[n][2];
        base[(r0 + 8) * Ep + col + 1] = acc[n][3];
    }
    __syncthreads();
    float* logit = red + (size_t)4 * kMmaTokens * Ep;  // [32][E+1]
    for (int i = tid; i < kMmaTokens * E; i += 256) {
        const int r = i / E, e = i % E;
        float v = red[r * Ep + e];
        v += red[(size_t)kMmaTokens * Ep + r * Ep + e];
        v += red[(size_t)2 * kMmaTokens * Ep + r * Ep + e];
        v += red[(size_t)3 * kMmaTokens * Ep + r * Ep + e];
        logit[r * Ep + e] = (v != v) ? -INFINITY : v;
    }
    __syncthreads();
    if (G <= 8 && 8 % G == 0) {
        // 8 lanes per token, all 32 tokens at once: lane `sub` of a token owns
        // experts [sub * NT, sub * NT + NT) (E / 8 = NT of them); a group of
        // E / G experts spans 8 / G consecutive lanes
        const int sub = lane & 7;
        const int tl = warp * 4 + (lane >> 3);
        const int t = t0 + tl;
        const float* L = logit + tl * Ep;
        float v[NT];
#pragma unroll
        for (int i = 0; i < NT; ++i) v[i] = sel_key(L[sub * NT + i], sub * NT + i, gate, bias);
        const int lanes_per_group = 8 / G;
        const int gid = sub / lanes_per_group;
        float gmax = v[0];
#pragma unroll
        for (int i = 1; i < NT; ++i) gmax = fmaxf(gmax, v[i]);
        for (int o = 1; o < lanes_per_group; o <<= 1)
            gmax = fmaxf(gmax, __shfl_xor_sync(0xffffffffu, gmax, o));
        uint32_t kept = 0;
        for (int r = 0; r < TG; ++r) {
            float bv = ((kept >> gid) & 1u) ? -INFINITY : gmax;
            int bi = ((kept >> gid) & 1u) ? INT_MAX : gid;
            seg8_argmax(bv, bi);
            kept |= 1u << bi;
        }
        const bool mine_kept = (kept >> gid) & 1u;
        uint32_t taken = 0;  // bit i: expert sub * NT + i already chosen
        int sel_e[kMaxK];
        float sel_l[kMaxK];
#pragma unroll
        for (int r = 0; r < kMaxK; ++r) {
            if (r >= k) break;
            float bv = -INFINITY;
            int bi = INT_MAX;
            if (mine_kept) {
#pragma unroll
                for (int i = 0; i < NT; ++i)
                    if (!((taken >> i) & 1u) && beats(v[i], sub * NT + i, bv, bi)) {
                        bv = v[i];
                        bi = sub * NT + i;
                    }
            }
            seg8_argmax(bv, bi);
            if (bi / NT == sub) taken |= 1u << (bi - sub * NT);
            sel_e[r] = bi;
        }
        if (sub == 0 && t < T) {
#pragma unroll
            for (int r = 0; r < kMaxK; ++r)
                if (r < k) sel_l[r] = L[sel_e[r]];
            float wv[kMaxK];
            gate_weights(sel_l, k, gate, wv);
#pragma unroll
            for (int r = 0; r < kMaxK; ++r) {
                if (r >= k) break;
                idx_out[(size_t)t * k + r] = sel_e[r];
                w_out[(size_t)t * k + r] = wv[r];
            }
        }
    } else {
        for (int tt = 0; tt < 4; ++tt) {
            const int tl = warp * 4 + tt;
            const int t = t0 + tl;
            if (t >= T) break;  // warp-uniform
            warp_topk<(NT * 8 + 31) / 32>(logit + tl * Ep, lane, E, k, G, TG, gate, bias,
                                          idx_out + (size_t)t * k, w_out + (size_t)t * k);
        }
    }
    pdl_trigger();
}

// ---------------------------------------------------------------------------
// Cluster router for bf16 with d = 256 S (S = 2, 4 or 8 CTAs per cluster):
// the S CTAs of a cluster share 32 tokens and split d, CTA r taking columns
// [256 r, 256 r + 256).  Each CTA loads its x and W_router slices once
// (48 KB at E = 64, d = 2048), forms its partial logits with mma.sync (k
// quarters added in fixed order), and after a cluster barrier CTA r sums the
// S partials of tokens [r 32/S, (r + 1) 32/S) over distributed shared memory
// in rank order and selects their experts.  Every SM streams only a 1/S slice
// of W_router, so small batches are not limited by one SM reading all of it.
__device__ __forceinline__ uint32_t cluster_rank_u32() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ float ld_cluster_f32(const float* local, uint32_t rank) {
    uint32_t a;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_u32(local)), "r"(rank));
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ void cluster_barrier() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
                 ::: "memory");
}

template <int NT, int S>
__global__ void __launch_bounds__(256) route_split_kernel(const __nv_bfloat16* __restrict__ x,
                                                          const __nv_bfloat16* __restrict__ Wr,
                                                          int T, int d, int E, int k, int G,
                                                          int TG, int gate,
                                                          const float* __restrict__ bias,
                                                          int32_t* __restrict__ idx_out,
                                                          float* __restrict__ w_out,
                                                          int* status) {
    extern __shared__ __align__(16) uint8_t rsm[];
    constexpr int kTokPerCta = kMmaTokens / S;
    const int Ep = E + 1;
    __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(rsm);  // [32][kMmaLd]
    __nv_bfloat16* wsm = xs + kMmaTokens * kMmaLd;              // [E][kMmaLd]
    float* red = reinterpret_cast<float*>(rsm);                // after the MMAs: [4][32][E+1]
    const size_t stage_bytes = (size_t)(kMmaTokens + E) * kMmaLd * sizeof(__nv_bfloat16);
    const size_t red_bytes = (size_t)4 * kMmaTokens * Ep * sizeof(float);
    float* part = reinterpret_cast<float*>(rsm + (stage_bytes > red_bytes ? stage_bytes : red_bytes));
    float* lg = part + kMmaTokens * Ep;  // [kTokPerCta][E+1] summed logits
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int wm = warp & 1, wk = warp >> 1;
    const uint32_t rank = cluster_rank_u32();
    const int t0 = (blockIdx.x / S) * kMmaTokens;
    const int c0 = (int)rank * kMmaKC;
    pdl_wait();
    if (status != nullptr && blockIdx.x == 0 && tid < 16) status[tid] = 0;

#pragma unroll
    for (int m = 0; m < kMmaTokens * (kMmaKC / 8) / 256; ++m) {
        const int i = tid + 256 * m;
        const int r = i >> 5, c = (i & 31) * 8;
        const int t = t0 + r;
        cp_async16(xs + r * kMmaLd + c, x + (size_t)(t < T ? t : 0) * d + c0 + c, t < T);
    }
    for (int i = tid; i < E * (kMmaKC / 8); i += 256) {
        const int r = i >> 5, c = (i & 31) * 8;
        cp_async16(wsm + r * kMmaLd + c, Wr + (size_t)r * d + c0 + c, true);
    }
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();

    float acc[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[n][q] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 64; kk += 16) {
        const int kb = wk * 64 + kk;
        uint32_t a[4];
        ldmatrix_x4(a, xs + (wm * 16 + (lane & 15)) * kMmaLd + kb + 8 * (lane >> 4));
#pragma unroll
        for (int n = 0; n < NT; n += 2) {
            uint32_t b[4];
            ldmatrix_x4(b, wsm + (8 * n + (lane & 7) + 8 * (lane >> 4)) * kMmaLd + kb +
                               8 * ((lane >> 3) & 1));
            mma_bf16_16816(acc[n], a, b[0], b[1]);
            mma_bf16_16816(acc[n + 1], a, b[2], b[3]);
        }
    }
    __syncthreads();  // the stage buffers become the k-quarter partials
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        const int r0 = wm * 16 + (lane >> 2), col = 8 * n + 2 * (lane & 3);
        float* base = red + (size_t)wk * kMmaTokens * Ep;
        base[r0 * Ep + col] = acc[n][0];
        base[r0 * Ep + col + 1] = acc[n][1];
        base[(r0 + 8) * Ep + col] = acc[n][2];
        base[(r0 + 8) * Ep + col + 1] = acc[n][3];
    }
    __syncthreads();
    for (int i = tid; i < kMmaTokens * E; i += 256) {
        const int r = i / E, e = i % E;
        float v = red[r * Ep + e];
        v += red[(size_t)kMmaTokens * Ep + r * Ep + e];
        v += red[(size_t)2 * kMmaTokens * Ep + r * Ep + e];
        v += red[(size_t)3 * kMmaTokens * Ep + r * Ep + e];
        part[r * Ep + e] = v;
    }
    cluster_barrier();  // every CTA's partial logits are ready
    for (int i = tid; i < kTokPerCta * E; i += 256) {
        const int r = i / E, e = i % E;
        const float* src = part + ((int)rank * kTokPerCta + r) * Ep + e;
        float v = ld_cluster_f32(src, 0);
#pragma unroll
        for (int q = 1; q < S; ++q) v += ld_cluster_f32(src, (uint32_t)q);
        lg[r * Ep + e] = (v != v) ? -INFINITY : v;
    }
    __syncthreads();
    for (int tt = warp; tt < kTokPerCta; tt += 8) {
        const int t = t0 + (int)rank * kTokPerCta + tt;
        if (t < T)  // warp-uniform
            warp_topk<(NT * 8 + 31) / 32>(lg + tt * Ep, lane, E, k, G, TG, gate, bias,
                                          idx_out + (size_t)t * k, w_out + (size_t)t * k);
    }
    pdl_trigger();
    cluster_barrier();  // no CTA leaves while another may still read its partials
}

size_t route_split_smem(int E, int S) {
    const size_t stage = (size_t)(kMmaTokens + E) * kMmaLd * sizeof(__nv_bfloat16);
    const size_t red = (size_t)4 * kMmaTokens * (E + 1) * sizeof(float);
    return (stage > red ? stage : red) +
           (size_t)(kMmaTokens + kMmaTokens / S) * (E + 1) * sizeof(float);
}

template <int S>
cudaError_t launch_route_split(const void* x, const void* Wr, int T, int d, int E, int k, int G,
                               int TG, int gate, const float* bias, int32_t* idx, float* w,
                               int* status, cudaStream_t s) {
    const size_t smem = route_split_smem(E, S);
    const __nv_bfloat16* xp = static_cast<const __nv_bfloat16*>(x);
    const __nv_bfloat16* wp = static_cast<const __nv_bfloat16*>(Wr);
    const dim3 grid((unsigned)(((T + kMmaTokens - 1) / kMmaTokens) * S));
#define MOE_ROUTE_SPLIT_CASE(NT)                                                              \
    case NT: {                                                                                \
        auto kern = route_split_kernel<NT, S>;                                                \
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                                             (int)smem);                                      \
        if (e != cudaSuccess) return e;                                                       \
        return launch_pdl(kern, grid, dim3(256), smem, s, S, xp, wp, T, d, E, k, G, TG, gate, \
                          bias, idx, w, status);                                              \
    }
    switch (E / 8) {
        MOE_ROUTE_SPLIT_CASE(2)
        MOE_ROUTE_SPLIT_CASE(4)
        MOE_ROUTE_SPLIT_CASE(6)
        MOE_ROUTE_SPLIT_CASE(8)
        MOE_ROUTE_SPLIT_CASE(10)
        MOE_ROUTE_SPLIT_CASE(12)
        MOE_ROUTE_SPLIT_CASE(14)
        MOE_ROUTE_SPLIT_CASE(16)
        default:
            return cudaErrorInvalidValue;
    }
#undef MOE_ROUTE_SPLIT_CASE
}

size_t route_mma_smem(int E, int S) {
    const size_t stage = (size_t)S * (kMmaTokens + E) * kMmaLd * sizeof(__nv_bfloat16);
    const size_t red = (size_t)5 * kMmaTokens * (E + 1) * sizeof(float);
    return stage > red ? stage : red;
}

template <int S>
cudaError_t launch_route_mma_s(const void* x, const void* Wr, int T, int d, int E, int k, int G,
                               int TG, int gate, const float* bias, int32_t* idx, float* w,
                               int* status, cudaStream_t s) {
    const size_t smem = route_mma_smem(E, S);
    const dim3 grid((T + kMmaTokens - 1) / kMmaTokens);
    const __nv_bfloat16* xp = static_cast<const __nv_bfloat16*>(x);
    const __nv_bfloat16* wp = static_cast<const __nv_bfloat16*>(Wr);
#define MOE_ROUTE_MMA_CASE(NT)                                                                \
    case NT: {                                                                                \
        auto kern = route_mma_kernel<NT, S>;                                                  \
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                                             (int)smem);                                      \
        if (e != cudaSuccess) return e;                                                       \
        return launch_pdl(kern, grid, dim3(256), smem, s, 1, xp, wp, T, d, E, k, G, TG, gate, \
                          bias, idx, w, status);                                              \
    }
    switch (E / 8) {
        MOE_ROUTE_MMA_CASE(2)
        MOE_ROUTE_MMA_CASE(4)
        MOE_ROUTE_MMA_CASE(6)
        MOE_ROUTE_MMA_CASE(8)
        MOE_ROUTE_MMA_CASE(10)
        MOE_ROUTE_MMA_CASE(12)
        MOE_ROUTE_MMA_CASE(14)
        MOE_ROUTE_MMA_CASE(16)
        default:
            return cudaErrorInvalidValue;
    }
#undef MOE_ROUTE_MMA_CASE
}

// 4 cp.async stages (one CTA per SM) when the grid fits on the GPU at once
// and E <= 64; otherwise 2 stages, two CTAs per SM
cudaError_t launch_route_mma(const void* x, const void* Wr, int T, int d, int E, int k, int G,
                             int TG, int gate, const float* bias, int32_t* idx, float* w,
                             int* status, cudaStream_t s) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (E <= 64 && (T + kMmaTokens - 1) / kMmaTokens <= sms)
        return launch_route_mma_s<4>(x, Wr, T, d, E, k, G, TG, gate, bias, idx, w, status, s);
    return launch_route_mma_s<2>(x, Wr, T, d, E, k, G, TG, gate, bias, idx, w, status, s);
}

template <typename TIn>
cudaError_t launch_route(const void* x, const void* Wr, int T, int d, int E, int k, int G,
                         int TG, int gate, const float* bias, int32_t* idx, float* w,
                               int* status, cudaStream_t s) {
    const int ej = (E + 31) / 32;
    const size_t p1 = (size_t)(kRouteTokens + E) * (kRouteKChunk + 1);
    const size_t p2 = (size_t)kRouteTokens * (E + 1);
    const size_t smem = sizeof(float) * (p1 > p2 ? p1 : p2);
    const dim3 grid((T + kRouteTokens - 1) / kRouteTokens);
    const TIn* xp = static_cast<const TIn*>(x);
    const TIn* wp = static_cast<const TIn*>(Wr);
#define MOE_ROUTE_CASE(N)                                                                   \
    case N: {                                                                               \
        auto kern = route_kernel<TIn, N>;                                                   \
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                                             (int)smem);                                    \
        if (e != cudaSuccess) return e;                                                     \
        return launch_pdl(kern, grid, dim3(kRouteThreads), smem, s, 1, xp, wp, T, d, E, k, G, \
                          TG, gate, bias, idx, w, status);                                              \
    }
    switch (ej) {
        MOE_ROUTE_CASE(1)
        MOE_ROUTE_CASE(2)
        MOE_ROUTE_CASE(3)
        MOE_ROUTE_CASE(4)
        MOE_ROUTE_CASE(5)
        MOE_ROUTE_CASE(6)
        MOE_ROUTE_CASE(7)
        MOE_ROUTE_CASE(8)
        default:
            return cudaErrorInvalidValue;
    }
#undef MOE_ROUTE_CASE
}

}  // namespace

cudaError_t launch_route_bf16(const void* x, const void* Wr, int T, int d, int E, int k, int G,
                              int TG, int gate, const float* bias, int32_t* idx, float* w,
                               int* status, cudaStream_t s) {
    // tensor-core path for the shapes it tiles exactly; CUDA cores otherwise
    if (E % 16 == 0 && E <= 128 && d % kMmaKC == 0) {
        // small batches: d split over a cluster of S CTAs when d = 256 S (the
        // whole-d kernel's few CTAs would each stream all of W_router); from
        // about 2048 tokens on, the whole-d kernel fills the GPU and is faster
        if (T > 1024)
            return launch_route_mma(x, Wr, T, d, E, k, G, TG, gate, bias, idx, w, status, s);
        if (d == 8 * kMmaKC)
            return launch_route_split<8>(x, Wr, T, d, E, k, G, TG, gate, bias, idx, w, status, s);
        if (d == 4 * kMmaKC)
            return launch_route_split<4>(x, Wr, T, d, E, k, G, TG, gate, bias, idx, w, status, s);
        if (d == 2 * kMmaKC)
            return launch_route_split<2>(x, Wr, T, d, E, k, G, TG, gate, bias, idx, w, status, s);
        return launch_route_mma(x, Wr, T, d, E, k, G, TG, gate, bias, idx, w, status, s);
    }
    return launch_route<__nv_bfloat16>(x, Wr, T, d, E, k, G, TG, gate, bias, idx, w, status, s);
}

cudaError_t launch_route_f32(const void* x, const void* Wr, int T, int d, int E, int k, int G,
                             int TG, int gate, const float* bias, int32_t* idx, float* w,
                               int* status, cudaStream_t s) {
    return launch_route<float>(x, Wr, T, d, E, k, G, TG, gate, bias, idx, w, status, s);
}

}  // namespace moe
