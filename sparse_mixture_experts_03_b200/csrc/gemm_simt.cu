// Grouped GEMM for fp32 inputs on CUDA cores (no tensor cores: fp32 operands
// keep their full precision) over expert segments padded to 128 rows, with
// SwiGLU, weighted-scatter and combine epilogues.  Used for fp32 layers,
// which are small; bf16 layers take the CTA-pair tcgen05 kernel.
#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {

namespace {

constexpr int TM = 64, TN = 64, TK = 16;

template <int EPI>
__global__ void __launch_bounds__(256) grouped_gemm_simt_kernel(const float* __restrict__ A,
                                                                const float* __restrict__ B,
                                                                const GemmArgs args, int a_rows) {
    __shared__ float As[TK][TM + 4];
    __shared__ float Bs[2][TK][TN + 4];
    pdl_wait();
    const int n_groups = args.offsets != nullptr ? args.n_groups : 1;
    const int total_rows = args.offsets != nullptr
                               ? args.offsets[n_groups]
                               : (args.static_rows + kRowAlign - 1) / kRowAlign * kRowAlign;
    const int row0 = blockIdx.y * TM;
    if (row0 >= total_rows) return;
    const int nt = blockIdx.x;
    int g = 0;
    if (args.offsets != nullptr) {
        int lo = 0, hi = n_groups - 1;
        while (lo < hi) {
            int mid = (lo + hi + 1) >> 1;
            if (args.offsets[mid] <= row0)
                lo = mid;
            else
                hi = mid - 1;
        }
        g = lo;
    }
    const long long b0 = g * args.b_group_stride + (long long)nt * args.b_tile_step;
    const long long b1 = b0 + args.b_half_off;
    const int K = args.K;
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;

    float acc0[4][4] = {}, acc1[4][4] = {};
    for (int k0 = 0; k0 < K; k0 += TK) {
        for (int i = tid; i < TM * TK; i += 256) {
            int r = i / TK, c = i % TK;
            int ar = row0 + r;
            As[c][r] = ar < a_rows ? A[(size_t)ar * K + k0 + c] : 0.f;
            Bs[0][c][r] = B[(size_t)(b0 + r) * K + k0 + c];
            if (EPI == EPI_SWIGLU) Bs[1][c][r] = B[(size_t)(b1 + r) * K + k0 + c];
        }
        __syncthreads();
#pragma unroll
        for (int c = 0; c < TK; ++c) {
            float av[4], bv[4], uv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                av[i] = As[c][ty * 4 + i];
                bv[i] = Bs[0][c][tx * 4 + i];
                uv[i] = EPI == EPI_SWIGLU ? Bs[1][c][tx * 4 + i] : 0.f;
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    acc0[i][j] = fmaf(av[i], bv[j], acc0[i][j]);
                    if (EPI == EPI_SWIGLU) acc1[i][j] = fmaf(av[i], uv[j], acc1[i][j]);
                }
        }
        __syncthreads();
    }

#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int grow = row0 + ty * 4 + i;
        const int col = nt * args.out_col_step + tx * 4;
        if (EPI == EPI_SWIGLU) {
            if (grow >= args.valid_rows) continue;
            float* o = static_cast<float*>(args.out) + (size_t)grow * args.out_ld + col;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float gt = acc0[i][j];
                o[j] = gt / (1.0f + expf(-gt)) * acc1[i][j];
            }
        } else if (EPI == EPI_SCATTER) {
            const int src = grow < args.valid_rows ? args.row_src[grow] : -1;
            if (src < 0) continue;
            const float wv = args.topk_w[src];
            float* o = static_cast<float*>(args.out) + (size_t)src * args.out_ld + col;
#pragma unroll
            for (int j = 0; j < 4; ++j) o[j] = wv * acc0[i][j];
        } else {
            if (grow >= args.valid_rows) continue;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float a = acc0[i][j];
                for (int s = 0; s < args.k; ++s)
                    a += static_cast<const float*>(
                        args.slots)[((size_t)grow * args.k + s) * args.out_ld + col + j];
                if (args.out_f32)
                    static_cast<float*>(args.out)[(size_t)grow * args.out_ld + col + j] = a;
                else
                    static_cast<__nv_bfloat16*>(args.out)[(size_t)grow * args.out_ld + col + j] =
                        __float2bfloat16_rn(a);
            }
        }
    }
    pdl_trigger();
}

}  // namespace

// grid: N/64 x rows_cap/64 CTAs; blocks past the device-side row total exit.
// a_rows: rows of A that exist (reads beyond are zero).
cudaError_t launch_gemm_simt(int epi, const float* A, const float* B, const GemmArgs& a,
                             int rows_cap, cudaStream_t s) {
    const int n_out = a.n_tiles;  // tiles of 64 output columns
    const dim3 grid(n_out, (rows_cap + TM - 1) / TM);
    const int a_rows = a.offsets != nullptr ? rows_cap : a.static_rows;
    switch (epi) {
        case EPI_SWIGLU:
            return launch_pdl(grouped_gemm_simt_kernel<EPI_SWIGLU>, grid, dim3(256), 0, s, 1, A, B,
                              a, a_rows);
        case EPI_SCATTER:
            return launch_pdl(grouped_gemm_simt_kernel<EPI_SCATTER>, grid, dim3(256), 0, s, 1, A,
                              B, a, a_rows);
        case EPI_COMBINE:
            return launch_pdl(grouped_gemm_simt_kernel<EPI_COMBINE>, grid, dim3(256), 0, s, 1, A,
                              B, a, a_rows);
        default:
            return cudaErrorInvalidValue;
    }
}

}  // namespace moe
