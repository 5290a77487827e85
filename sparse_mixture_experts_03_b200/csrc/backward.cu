// Memory-bound helper kernels of the layer backward (the GEMMs are the
// CTA-pair kernels of gemm_pair.cu):
//   bwd_gather       x and dy rows into the padded permuted layout (each
//                    token's rows read once); zero padding rows of every
//                    row-indexed GEMM operand
//   router_dlogit    dL/dw from the per-warp partial sums of the SwiGLU
//                    backward epilogue, then dL/dlogit of the chosen experts
//   bwd_combine      dx = shared part + chosen experts' parts + router part,
//                    in a fixed order
//   router_dweight   dW_router[e] = sum of dl * x over expert e's rows: fixed
//                    row slices, then the slices in order
// The gate derivatives follow the chain rule through the gates of
// "FusionLLM：融合 MLA、GDN 与 MoE 的高效混合架构大模型训练框架", section
// "混合专家（MoE）" (sigmoid scores, weights normalised over the chosen
// experts) and of "大模型工程（一）：Transformer 到 MoE", section "MoE 数学：
// 路由、容量与平衡详解" (softmax over the chosen logits).
#include "../../include/moe.h"
#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {

namespace {

// Part 1: one warp per token, its x and dy rows read once (16-byte vectors,
// all of a lane's loads before its stores) and written to the token's k rows.
// Part 2: one warp per row, zeroing padding rows.
__global__ void __launch_bounds__(256)
    bwd_gather_kernel(const uint4* __restrict__ x, const uint4* __restrict__ dy, int T, int vd,
                      int vf, int k, const int32_t* __restrict__ total_rows,
                      const int32_t* __restrict__ row_src, const int32_t* __restrict__ slot_row,
                      uint4* __restrict__ x_perm, uint4* __restrict__ dy_perm,
                      uint4* __restrict__ dgu, uint4* __restrict__ hw) {
    const int lane = threadIdx.x & 31;
    const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int nw = (gridDim.x * blockDim.x) >> 5;
    pdl_wait();
    for (int t = gw; t < T; t += nw) {
        const uint4* xs = x + (size_t)t * vd;
        const uint4* ys = dy + (size_t)t * vd;
        for (int i0 = 0; i0 < vd; i0 += 4 * 32) {
            uint4 a[4], b[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = i0 + u * 32 + lane;
                if (i < vd) {
                    a[u] = __ldcs(xs + i);
                    b[u] = __ldcs(ys + i);
                }
            }
            for (int j = 0; j < k; ++j) {
                const size_t r = (size_t)slot_row[(size_t)t * k + j];
                uint4* xo = x_perm + r * vd;
                uint4* yo = dy_perm + r * vd;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int i = i0 + u * 32 + lane;
                    if (i < vd) {
                        xo[i] = a[u];
                        yo[i] = b[u];
                    }
                }
            }
        }
    }
    // padding rows are K rows of the weight-gradient GEMMs: all zero
    const int total = *total_rows;
    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
    for (int r = gw; r < total; r += nw) {
        if (row_src[r] >= 0) continue;
        uint4* xo = x_perm + (size_t)r * vd;
        uint4* yo = dy_perm + (size_t)r * vd;
        for (int i = lane; i < vd; i += 32) {
            xo[i] = z;
            yo[i] = z;
        }
        uint4* go = dgu + (size_t)r * 2 * vf;
        for (int i = lane; i < 2 * vf; i += 32) go[i] = z;
        uint4* ho = hw + (size_t)r * vf;
        for (int i = lane; i < vf; i += 32) ho[i] = z;
    }
    pdl_trigger();
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// One warp per token.  dw_j: the parts of its slot's row summed in part
// order.  Sigmoid gate (w_j = s_j / S): dl_j = (dw_j - sum_i w_i dw_i) / S *
// s_j (1 - s_j); S and the s_j come from one recomputed logit, that of the
// top choice (w_0 >= 1/k): S = sigmoid(x . Wr[e_0]) / w_0 (fp32 sum of the
// bf16 products), s_j = w_j S.  Softmax over the chosen logits:
// dl_j = w_j (dw_j - sum_i w_i dw_i).
__global__ void __launch_bounds__(256)
    router_dlogit_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ Wr,
                         int T, int d, int k, const int32_t* __restrict__ idx,
                         const float* __restrict__ topk_w, const float* __restrict__ dw_part,
                         int n_parts, const int32_t* __restrict__ slot_row, int gate,
                         float* __restrict__ dl) {
    const int lane = threadIdx.x & 31;
    const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    pdl_wait();
    if (t >= T) {
        pdl_trigger();
        return;
    }
    float dw[kMaxK], w[kMaxK];
    float abar = 0.f;
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
        dw[j] = 0.f;
        w[j] = 0.f;
        if (j < k) {
            // lane l sums parts l, l + 32, ...; then a fixed xor tree (every
            // lane ends with the same sum, in the same order)
            const float* pp = dw_part + (size_t)slot_row[(size_t)t * k + j] * n_parts;
            float acc = 0.f;
            for (int p = lane; p < n_parts; p += 32) acc += pp[p];
            dw[j] = warp_sum(acc);
            w[j] = topk_w[(size_t)t * k + j];
            abar = fmaf(w[j], dw[j], abar);
        }
    }
    float v = 0.f;
    if (gate == MOE_GATE_SIGMOID) {
        const __nv_bfloat16* xr = x + (size_t)t * d;
        const __nv_bfloat16* wr = Wr + (size_t)idx[(size_t)t * k] * d;
        float acc = 0.f;
        for (int c = 2 * lane; c < d; c += 64) {
            const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(xr + c));
            const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(wr + c));
            acc = fmaf(a.x, b.x, acc);
            acc = fmaf(a.y, b.y, acc);
        }
        const float s0 = 1.0f / (1.0f + __expf(-warp_sum(acc)));
        const float S = s0 / w[0];
#pragma unroll
        for (int j = 0; j < kMaxK; ++j)
            if (j == lane) {
                const float sj = w[j] * S;
                v = (dw[j] - abar) / S * sj * (1.0f - sj);
            }
    } else {
#pragma unroll
        for (int j = 0; j < kMaxK; ++j)
            if (j == lane) v = w[j] * (dw[j] - abar);
    }
    if (lane < k) dl[(size_t)t * k + lane] = v;
    pdl_trigger();
}

// 8 columns per thread: dx[t] = base[t] + slot rows (bf16) + dl_j Wr[e_j].
template <int K>
__global__ void __launch_bounds__(256)
    bwd_combine_kernel(const float4* __restrict__ base, const uint4* __restrict__ slots,
                       const float* __restrict__ dl, const int32_t* __restrict__ idx,
                       const uint4* __restrict__ Wr, int T, int d8, float4* __restrict__ dx) {
    const size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
    pdl_wait();
    if (i < (size_t)T * d8) {
        const size_t t = i / d8, c8 = i % d8;
        uint4 raw[K], wraw[K];
        float g[K];
#pragma unroll
        for (int j = 0; j < K; ++j) {
            raw[j] = __ldcs(slots + (t * K + j) * d8 + c8);
            g[j] = dl[t * K + j];
            wraw[j] = __ldg(Wr + (size_t)idx[t * K + j] * d8 + c8);
        }
        float a[8];
        if (base != nullptr) {
            const float4 b0 = __ldcs(base + 2 * i), b1 = __ldcs(base + 2 * i + 1);
            a[0] = b0.x; a[1] = b0.y; a[2] = b0.z; a[3] = b0.w;
            a[4] = b1.x; a[5] = b1.y; a[6] = b1.z; a[7] = b1.w;
        } else {
#pragma unroll
            for (int q = 0; q < 8; ++q) a[q] = 0.f;
        }
#pragma unroll
        for (int j = 0; j < K; ++j) {
            const uint32_t w4[4] = {raw[j].x, raw[j].y, raw[j].z, raw[j].w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                a[2 * h] += __uint_as_float(w4[h] << 16);
                a[2 * h + 1] += __uint_as_float(w4[h] & 0xffff0000u);
            }
        }
#pragma unroll
        for (int j = 0; j < K; ++j) {
            const uint32_t w4[4] = {wraw[j].x, wraw[j].y, wraw[j].z, wraw[j].w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                a[2 * h] = fmaf(g[j], __uint_as_float(w4[h] << 16), a[2 * h]);
                a[2 * h + 1] = fmaf(g[j], __uint_as_float(w4[h] & 0xffff0000u), a[2 * h + 1]);
            }
        }
        __stcs(dx + 2 * i, make_float4(a[0], a[1], a[2], a[3]));
        __stcs(dx + 2 * i + 1, make_float4(a[4], a[5], a[6], a[7]));
    }
    pdl_trigger();
}

// dW_router in two passes with a fixed summation order.  Pass 1: block (e,
// column chunk of 2048, slice z) sums the rows of slice z of expert e's
// segment (the segment cut into kDwSlices nearly equal row ranges), in row
// order, into part[z][e][:]: 8 columns per thread (16-byte loads), 8 rows'
// loads in flight.  The rows' gate gradients go through shared memory 256 at
// a time, so the row loads depend on nothing but the row index (padding rows
// of the segment are zero rows of x_perm and take a zero gradient).  Pass 2
// adds the slices in order z = 0, 1, ...
constexpr int kDwSlices = kDwParts;
constexpr int kDwChunk = 256;

__global__ void __launch_bounds__(256)
    router_dweight_part_kernel(const float* __restrict__ dl, const int32_t* __restrict__ row_src,
                               const int32_t* __restrict__ offsets, const uint4* __restrict__ xp,
                               int E, int d, float* __restrict__ part) {
    __shared__ float s_g[kDwChunk];    // dl of the chunk's rows (0 on padding rows)
    __shared__ int s_ok[kDwChunk];     // the row is a real one
    const int e = blockIdx.x, z = blockIdx.z;
    const int c8 = blockIdx.y * blockDim.x + threadIdx.x;  // group of 8 columns
    const int d8 = d >> 3;
    pdl_wait();
    const int s0 = offsets[e], n = offsets[e + 1] - s0;
    const int r0 = s0 + (int)((long long)z * n / kDwSlices);
    const int r1 = s0 + (int)((long long)(z + 1) * n / kDwSlices);
    float a[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) a[q] = 0.f;
    for (int cb = r0; cb < r1; cb += kDwChunk) {
        const int nr = min(kDwChunk, r1 - cb);
        __syncthreads();  // the previous chunk's gradients are no longer read
        for (int i = threadIdx.x; i < nr; i += blockDim.x) {
            const int src = __ldg(row_src + cb + i);
            s_g[i] = src >= 0 ? __ldg(dl + src) : 0.f;
            s_ok[i] = src >= 0;
        }
        __syncthreads();
        if (c8 < d8) {
            for (int rb = 0; rb < nr; rb += 8) {
                uint4 v[8];
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    if (rb + u < nr) v[u] = __ldg(xp + (size_t)(cb + rb + u) * d8 + c8);
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    if (rb + u >= nr) break;
                    const float g = s_g[rb + u];
                    const uint4 w = s_ok[rb + u] ? v[u] : make_uint4(0u, 0u, 0u, 0u);
                    const uint32_t w4[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        a[2 * h] = fmaf(g, __uint_as_float(w4[h] << 16), a[2 * h]);
                        a[2 * h + 1] = fmaf(g, __uint_as_float(w4[h] & 0xffff0000u), a[2 * h + 1]);
                    }
                }
            }
        }
    }
    if (c8 < d8) {
        float4* o = reinterpret_cast<float4*>(part + ((size_t)z * E + e) * d) + 2 * c8;
        o[0] = make_float4(a[0], a[1], a[2], a[3]);
        o[1] = make_float4(a[4], a[5], a[6], a[7]);
    }
    pdl_trigger();
}

__global__ void __launch_bounds__(256)
    router_dweight_sum_kernel(const float4* __restrict__ part, int n4, float4* __restrict__ dWr) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    pdl_wait();
    if (i < n4) {
        float4 a = part[i];
#pragma unroll
        for (int z = 1; z < kDwSlices; ++z) {
            const float4 b = part[(size_t)z * n4 + i];
            a.x += b.x;
            a.y += b.y;
            a.z += b.z;
            a.w += b.w;
        }
        dWr[i] = a;
    }
    pdl_trigger();
}

}  // namespace

cudaError_t launch_bwd_gather(const void* x, const void* dy, int T, int d, int F, int k,
                              const int32_t* offsets_total, const int32_t* row_src,
                              const int32_t* slot_row, int rows_cap, void* x_perm, void* dy_perm,
                              void* dgu, void* hw, int num_sms, cudaStream_t s) {
    int blocks = (rows_cap + 7) / 8;
    if (blocks > num_sms * 8) blocks = num_sms * 8;
    if (blocks < 1) blocks = 1;
    return launch_pdl(bwd_gather_kernel, dim3(blocks), dim3(256), 0, s, 1,
                      static_cast<const uint4*>(x), static_cast<const uint4*>(dy), T, d / 8, F / 8,
                      k, offsets_total, row_src, slot_row, static_cast<uint4*>(x_perm),
                      static_cast<uint4*>(dy_perm), static_cast<uint4*>(dgu),
                      static_cast<uint4*>(hw));
}

cudaError_t launch_router_dlogit(const void* x, const void* Wr, int T, int d, int k,
                                 const int32_t* idx, const float* topk_w, const float* dw_part,
                                 int n_parts, const int32_t* slot_row, int gate, float* dl,
                                 cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    const unsigned blocks = (unsigned)((T + 7) / 8);
    return launch_pdl(router_dlogit_kernel, dim3(blocks), dim3(256), 0, s, 1,
                      static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(Wr),
                      T, d, k, idx, topk_w, dw_part, n_parts, slot_row, gate, dl);
}

cudaError_t launch_bwd_combine(const float* base, const void* slots, const float* dl,
                               const int32_t* idx, const void* Wr, int T, int d, int k, float* dx,
                               cudaStream_t s) {
    const int d8 = d / 8;
    const size_t n = (size_t)T * d8;
    if (n == 0) return cudaSuccess;
    const unsigned blocks = (unsigned)((n + 255) / 256);
    const float4* b4 = reinterpret_cast<const float4*>(base);
    const uint4* sl = static_cast<const uint4*>(slots);
    const uint4* w = static_cast<const uint4*>(Wr);
    float4* o = reinterpret_cast<float4*>(dx);
    switch (k) {
#define MOE_BWD_COMBINE_K(KK)                                                                \
    case KK:                                                                                 \
        return launch_pdl(bwd_combine_kernel<KK>, dim3(blocks), dim3(256), 0, s, 1, b4, sl, dl, \
                          idx, w, T, d8, o);
        MOE_BWD_COMBINE_K(1) MOE_BWD_COMBINE_K(2) MOE_BWD_COMBINE_K(3) MOE_BWD_COMBINE_K(4)
        MOE_BWD_COMBINE_K(5) MOE_BWD_COMBINE_K(6) MOE_BWD_COMBINE_K(7) MOE_BWD_COMBINE_K(8)
#undef MOE_BWD_COMBINE_K
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_router_dweight(const float* dl, const int32_t* row_src, const int32_t* offsets,
                                  const void* x_perm, int E, int d, float* part, float* dWr,
                                  cudaStream_t s) {
    const unsigned cy = (unsigned)((d / 8 + 255) / 256);
    cudaError_t e = launch_pdl(router_dweight_part_kernel, dim3((unsigned)E, cy, kDwSlices),
                               dim3(256), 0, s, 1, dl, row_src, offsets,
                               static_cast<const uint4*>(x_perm), E, d, part);
    if (e != cudaSuccess) return e;
    const int n4 = E * d / 4;
    return launch_pdl(router_dweight_sum_kernel, dim3((unsigned)((n4 + 255) / 256)), dim3(256), 0,
                      s, 1, reinterpret_cast<const float4*>(part), n4,
                      reinterpret_cast<float4*>(dWr));
}

}  // namespace moe
