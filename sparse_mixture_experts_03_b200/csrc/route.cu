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
#include <float.h>
#include <limits.h>

#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {

namespace {

constexpr int kRouteTokens = 32;   // tokens per CTA
constexpr int kRouteKChunk = 32;   // reduction chunk staged in shared memory
constexpr int kRouteThreads = 256;

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

template <typename TIn, int EJ>
__global__ void __launch_bounds__(kRouteThreads) route_kernel(const TIn* __restrict__ x,
                                                              const TIn* __restrict__ Wr, int T,
                                                              int d, int E, int k, int G, int TG,
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

    if (status != nullptr && blockIdx.x == 0 && tid < 4) status[tid] = 0;

    float acc[4][EJ];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < EJ; ++j) acc[i][j] = 0.f;

    for (int c0 = 0; c0 < d; c0 += kRouteKChunk) {
        // stage x [32 tokens][32] and W_router [E][32] as fp32
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

    const int gsz = E / G;
    for (int tt = 0; tt < 4; ++tt) {
        const int tl = warp * 4 + tt;
        const int t = t0 + tl;
        if (t >= T) break;  // warp-uniform
        const float* L = logit + tl * (E + 1);
        // group scores: max logit of each group (lane g < G owns group g)
        float gval = -INFINITY;
        if (lane < G)
            for (int e = lane * gsz; e < (lane + 1) * gsz; ++e) gval = fmaxf(gval, L[e]);
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
            cv[j] = cand[j] ? L[e] : -INFINITY;
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
            sel_l[r] = bv;
        }
        if (lane == 0) {
            float s[kMaxK], sum = 0.f;
#pragma unroll
            for (int r = 0; r < kMaxK; ++r) {
                if (r >= k) break;
                s[r] = 1.f / (1.f + expf(-sel_l[r]));
                sum += s[r];
            }
#pragma unroll
            for (int r = 0; r < kMaxK; ++r) {
                if (r >= k) break;
                idx_out[(size_t)t * k + r] = sel_e[r];
                w_out[(size_t)t * k + r] = s[r] / sum;
            }
        }
    }
}

template <typename TIn>
cudaError_t launch_route(const void* x, const void* Wr, int T, int d, int E, int k, int G,
                         int TG, int32_t* idx, float* w, int* status, cudaStream_t s) {
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
        kern<<<grid, kRouteThreads, smem, s>>>(xp, wp, T, d, E, k, G, TG, idx, w, status);  \
        return cudaGetLastError();                                                          \
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
                              int TG, int32_t* idx, float* w, int* status, cudaStream_t s) {
    return launch_route<__nv_bfloat16>(x, Wr, T, d, E, k, G, TG, idx, w, status, s);
}

cudaError_t launch_route_f32(const void* x, const void* Wr, int T, int d, int E, int k, int G,
                             int TG, int32_t* idx, float* w, int* status, cudaStream_t s) {
    return launch_route<float>(x, Wr, T, d, E, k, G, TG, idx, w, status, s);
}

}  // namespace moe
