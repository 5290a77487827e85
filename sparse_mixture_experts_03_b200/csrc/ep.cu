// Expert parallelism: the layer split over ranks that each hold E / n_ranks
// of the routed experts ("大模型工程（一）：Transformer 到 MoE", section "混合专家：
// 更多参数，相同 FLOPs": experts spread over GPUs, tokens exchanged all-to-all
// over NVLink; and its Mixtral / Qwen3-MoE / DeepSeek-V3 architecture
// comparison, one expert group per GPU).  The exchange itself is the
// caller's (NCCL all-to-all between these calls); this file has the compute
// on either side of it:
//
//   moe_dispatch          route, permute and copy the rank's own tokens into
//                         expert-contiguous rows (= rank-contiguous, since
//                         rank r owns experts [r E_l, (r+1) E_l)), with each
//                         row's gate weight
//   moe_experts_forward   the received rows (grouped by source rank, then by
//                         local expert) through the local experts: regroup
//                         by expert, gate/up GEMM + SwiGLU, down GEMM whose
//                         epilogue scales each row by its gate weight and
//                         writes it back to its receive position
//   moe_shared_forward    the shared experts on the rank's own tokens (fp32
//                         rows; independent of the exchange, so it can run
//                         while the rows are in flight)
//   moe_combine           y[t] = shared[t] + the k returned rows of token t,
//                         in top-k order (fixed order: bitwise reproducible)
#include <limits.h>

#include <algorithm>

#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr size_t kEpAlign = 1024;
constexpr int kRegroupThreads = 256;
constexpr int kMaxSrcExperts = 2048;  // n_src * E_local of moe_experts_forward

size_t ep_align(size_t v) { return (v + kEpAlign - 1) / kEpAlign * kEpAlign; }

// Exclusive prefix sum of a[0..n) in shared memory by the whole CTA (tmp:
// one int per thread).  Ends with a barrier.
__device__ void block_exclusive_scan(int* a, int n, int* tmp) {
    const int tid = threadIdx.x, nt = blockDim.x;
    const int per = (n + nt - 1) / nt;
    const int b = min(tid * per, n), e = min(b + per, n);
    int sum = 0;
    for (int i = b; i < e; ++i) sum += a[i];
    tmp[tid] = sum;
    __syncthreads();
    if (tid == 0) {
        int run = 0;
        for (int i = 0; i < nt; ++i) {
            const int v = tmp[i];
            tmp[i] = run;
            run += v;
        }
    }
    __syncthreads();
    int run = tmp[tid];
    for (int i = b; i < e; ++i) {
        const int v = a[i];
        a[i] = run;
        run += v;
    }
    __syncthreads();
}

// Rows arrive grouped by source rank, then by local expert (each source's
// dispatch order).  Grouped layout: local expert e owns rows
// [off[e], off[e + 1]), and inside it source 0's rows come first, then
// source 1's, ... (each source's rows in their own order).  row_src[r] = the
// receive position of grouped row r.  Every CTA builds the two (expert,
// source) tables in shared memory; CTA 0 also writes counts / offsets and
// resets the status words (the next launches' tile tickets).
__global__ void __launch_bounds__(kRegroupThreads) ep_regroup_kernel(
    const int32_t* __restrict__ recv_counts, int n_src, int E_l, int R,
    int32_t* __restrict__ counts, int32_t* __restrict__ offsets, int32_t* __restrict__ row_src,
    int* status) {
    __shared__ int s_dst[kMaxSrcExperts + 1];  // (e, src) order: first grouped row
    __shared__ int s_src[kMaxSrcExperts];      // (src, e) order: first receive position
    __shared__ int s_tmp[kRegroupThreads];
    __shared__ int s_tot;
    const int tid = threadIdx.x;
    const int n = n_src * E_l;
    pdl_wait();
    if (status != nullptr && blockIdx.x == 0 && tid < 16) status[tid] = 0;
    for (int i = tid; i < n; i += blockDim.x) {
        const int c = max(recv_counts[i], 0);  // i = src * E_l + e
        s_src[i] = c;
        s_dst[(i % E_l) * n_src + i / E_l] = c;
    }
    if (tid == 0) s_dst[n] = 0;
    __syncthreads();
    block_exclusive_scan(s_src, n, s_tmp);   // receive positions: source-major
    block_exclusive_scan(s_dst, n + 1, s_tmp);  // grouped rows: expert-major; [n] = total
    if (tid == 0) {
        s_tot = s_dst[n];
        if (s_tot > R) set_status(status, MOE_ERR_DEVICE, SITE_PERMUTE, s_tot);
    }
    __syncthreads();
    // counts that do not fit the R rows given: nothing is grouped or computed
    // (zero counts and offsets; the status word says why)
    const bool fits = s_tot <= R;
    const int total = fits ? s_tot : 0;
    if (blockIdx.x == 0) {
        for (int e = tid; e < E_l; e += blockDim.x) {
            counts[e] = fits ? s_dst[(e + 1) * n_src] - s_dst[e * n_src] : 0;
            offsets[e] = fits ? s_dst[e * n_src] : 0;
        }
        if (tid == 0) offsets[E_l] = total;
    }
    for (int r = blockIdx.x * blockDim.x + tid; r < total; r += gridDim.x * blockDim.x) {
        // last (e, src) segment starting at or before r
        int lo = 0, hi = n - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_dst[mid] <= r)
                lo = mid;
            else
                hi = mid - 1;
        }
        const int e = lo / n_src, src = lo % n_src;
        row_src[r] = s_src[src * E_l + e] + (r - s_dst[lo]);
    }
    pdl_trigger();
}

// y[t] = base[t] + rows[slot_row[t*K + 0]] + ... + rows[slot_row[t*K + K-1]]
// in fp32, in that order; rows bf16.  One thread per (token, 8 columns).
template <int K>
__global__ void __launch_bounds__(256) combine_rows_bf16_kernel(
    const uint4* __restrict__ rows, const int32_t* __restrict__ slot_row,
    const float4* __restrict__ base, int T, int d8, int n_rows, void* y, int out_f32,
    int* status) {
    const size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
    pdl_wait();
    if (i >= (size_t)T * d8) return;
    const size_t t = i / d8, c8 = i % d8;
    uint4 raw[K];
#pragma unroll
    for (int j = 0; j < K; ++j) {
        const int r = slot_row[t * K + j];
        if (r >= 0 && r < n_rows) {
            raw[j] = __ldcs(rows + (size_t)r * d8 + c8);
        } else {
            raw[j] = make_uint4(0, 0, 0, 0);
            if (c8 == 0) set_status(status, MOE_ERR_DEVICE, SITE_PERMUTE, r);
        }
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
    if (out_f32) {
        float4* o = static_cast<float4*>(y) + 2 * i;
        __stcs(o, make_float4(a[0], a[1], a[2], a[3]));
        __stcs(o + 1, make_float4(a[4], a[5], a[6], a[7]));
    } else {
        static_cast<uint4*>(y)[i] = make_uint4(pack_bf16x2(a[0], a[1]), pack_bf16x2(a[2], a[3]),
                                               pack_bf16x2(a[4], a[5]), pack_bf16x2(a[6], a[7]));
    }
    pdl_trigger();
}

// Status words 0..15 (status, site, info, tile tickets) to zero.
__global__ void reset_status_kernel(int* status) {
    pdl_wait();
    if (threadIdx.x < 16) status[threadIdx.x] = 0;
    pdl_trigger();
}

// ---- workspace layouts
enum DispatchRegion : int { DP_STATUS, DP_OFFSETS, DP_BLOCK_COUNTS, DP_ROW_SRC, DP_TOTAL };
enum ExpertsRegion : int { EX_STATUS, EX_COUNTS, EX_OFFSETS, EX_ROW_SRC, EX_X, EX_H, EX_TOTAL };
enum SharedRegion : int { SH_STATUS, SH_H, SH_TOTAL };

template <int N>
size_t layout(const size_t (&sizes)[N], size_t (&off)[N + 1]) {
    size_t o = 0;
    for (int i = 0; i < N; ++i) {
        off[i] = o;
        o = ep_align(o + sizes[i]);
    }
    off[N] = o;
    return o;
}

bool dispatch_layout(int T, int E, int k, size_t (&off)[DP_TOTAL + 1]) {
    if (T < 0 || E < 1 || E > kMaxE || k < 1 || k > kMaxK || k > E) return false;
    if ((long long)T * k >= (long long)INT_MAX / 2) return false;
    // block counts: per 256-token block, or per CTA of the one-launch permutation
    const size_t nb = std::max((size_t)(T + kPermBlockTokens - 1) / kPermBlockTokens,
                               (size_t)(T + 31) / 32);
    const size_t sizes[DP_TOTAL] = {sizeof(int) * kStatusWords, sizeof(int) * (E + 1),
                                    sizeof(int) * (nb > 0 ? nb : 1) * E,
                                    sizeof(int) * ((size_t)T * k + 1)};
    layout(sizes, off);
    return true;
}

bool experts_layout(int R, int d, int E_l, int inter, size_t (&off)[EX_TOTAL + 1]) {
    if (R < 0 || d <= 0 || d % 256 != 0 || E_l < 1 || E_l > kMaxE || inter <= 0 ||
        inter % 128 != 0)
        return false;
    if ((long long)R * d >= (1LL << 40)) return false;
    const size_t sizes[EX_TOTAL] = {sizeof(int) * kStatusWords, sizeof(int) * E_l,
                                    sizeof(int) * (E_l + 1),   sizeof(int) * ((size_t)R + 1),
                                    2 * (size_t)R * d,          2 * (size_t)R * inter};
    layout(sizes, off);
    return true;
}

bool shared_layout(int T, int d, int inter, int n_shared, size_t (&off)[SH_TOTAL + 1]) {
    if (T < 0 || d <= 0 || d % 256 != 0 || inter <= 0 || inter % 128 != 0 || n_shared < 1)
        return false;
    const size_t sizes[SH_TOTAL] = {sizeof(int) * kStatusWords,
                                    2 * (size_t)T * n_shared * inter};
    layout(sizes, off);
    return true;
}

template <typename P>
P* region(void* ws, const size_t* off, int i) {
    return reinterpret_cast<P*>(static_cast<char*>(ws) + off[i]);
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

MOE_API size_t moe_dispatch_workspace_bytes(int T, int E, int k) {
    size_t off[DP_TOTAL + 1];
    return dispatch_layout(T, E, k, off) ? off[DP_TOTAL] : 0;
}

MOE_API int moe_dispatch(const void* x, const void* W_router, int T, int d, int E, int k,
                         int n_group, int topk_group, int in_dt, int gate,
                         const float* expert_bias, int32_t* topk_idx, float* topk_w,
                         int32_t* counts, void* x_perm, float* w_perm, int32_t* slot_row,
                         void* workspace, size_t workspace_bytes, void* stream) {
    size_t off[DP_TOTAL + 1];
    if (!dispatch_layout(T, E, k, off) || d <= 0 || d % 256 != 0) return MOE_ERR_INVALID_ARG;
    if (in_dt != MOE_BF16) return MOE_ERR_UNSUPPORTED;
    int st = check_routing(E, k, n_group, topk_group);
    if (st != MOE_OK) return st;
    st = check_gating(gate, expert_bias, nullptr);
    if (st != MOE_OK) return st;
    if (workspace == nullptr || workspace_bytes < off[DP_TOTAL]) return MOE_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (!is_device_ptr(counts) || !aligned(counts, 4)) return MOE_ERR_INVALID_ARG;
    if (T == 0) return ret(cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, s));
    const void* p16[] = {x, W_router, x_perm, workspace};
    for (const void* p : p16)
        if (!is_device_ptr(p) || !aligned(p, 16)) return MOE_ERR_INVALID_ARG;
    const void* p4[] = {topk_idx, topk_w, w_perm, slot_row};
    for (const void* p : p4)
        if (!is_device_ptr(p) || !aligned(p, 4)) return MOE_ERR_INVALID_ARG;
    if (!aligned(workspace, 256)) return MOE_ERR_INVALID_ARG;
    int* status = region<int>(workspace, off, DP_STATUS);
    int32_t* offsets = region<int32_t>(workspace, off, DP_OFFSETS);
    int32_t* row_src = region<int32_t>(workspace, off, DP_ROW_SRC);
    cudaError_t e = launch_route_bf16(x, W_router, T, d, E, k, n_group, topk_group, gate,
                                      expert_bias, topk_idx, topk_w, status, s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    // permutation, rows and their gate weights in one launch (the routing
    // kernel has reset the grid-barrier word of the status region)
    int32_t* block_counts = region<int32_t>(workspace, off, DP_BLOCK_COUNTS);
    if (T <= kSmallPermTokens)
        return ret(launch_permute_gather_small(topk_idx, T, k, E, 1, counts, offsets, row_src,
                                               nullptr, status, x, d, 2, x_perm, num_sms(), s,
                                               slot_row, topk_w, w_perm));
    if (permute_gather_grid_fits(T, E, num_sms()))
        return ret(launch_permute_gather_grid(topk_idx, T, k, E, 1, block_counts, counts, offsets,
                                              row_src, nullptr, status,
                                              status + kGridBarWordPermute, kWaitLimitNs, x, d, 2,
                                              x_perm, num_sms(), s, slot_row, topk_w, w_perm));
    e = launch_permute(topk_idx, T, k, E, block_counts, counts, offsets, row_src, 1, nullptr,
                       status, s, slot_row);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    return ret(launch_gather_rows(x, d, 2, k, offsets + E, row_src, T * k, x_perm, num_sms(), s,
                                  topk_w, w_perm));
}

MOE_API size_t moe_experts_workspace_bytes(int R, int d, int E_local, int inter) {
    size_t off[EX_TOTAL + 1];
    return experts_layout(R, d, E_local, inter, off) ? off[EX_TOTAL] : 0;
}

MOE_API int moe_experts_forward(const void* x_rows, const float* w_rows,
                                const int32_t* recv_counts, int n_src, int R,
                                const void* W_gate_up, const void* W_down, int d, int E_local,
                                int inter, int in_dt, void* y_rows, void* workspace,
                                size_t workspace_bytes, void* stream) {
    size_t off[EX_TOTAL + 1];
    if (!experts_layout(R, d, E_local, inter, off)) return MOE_ERR_INVALID_ARG;
    if (n_src < 1 || (long long)n_src * E_local > kMaxSrcExperts) return MOE_ERR_INVALID_ARG;
    if (in_dt != MOE_BF16) return MOE_ERR_UNSUPPORTED;
    if (workspace == nullptr || workspace_bytes < off[EX_TOTAL]) return MOE_ERR_WORKSPACE;
    if (R == 0) return MOE_OK;
    const void* p16[] = {x_rows, W_gate_up, W_down, y_rows, workspace};
    for (const void* p : p16)
        if (!is_device_ptr(p) || !aligned(p, 16)) return MOE_ERR_INVALID_ARG;
    if (!is_device_ptr(w_rows) || !aligned(w_rows, 4) || !is_device_ptr(recv_counts) ||
        !aligned(recv_counts, 4) || !aligned(workspace, 256))
        return MOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int* status = region<int>(workspace, off, EX_STATUS);
    int32_t* counts = region<int32_t>(workspace, off, EX_COUNTS);
    int32_t* offsets = region<int32_t>(workspace, off, EX_OFFSETS);
    int32_t* row_src = region<int32_t>(workspace, off, EX_ROW_SRC);
    void* xg = region<char>(workspace, off, EX_X);
    void* h = region<char>(workspace, off, EX_H);
    int blocks = (R + kRegroupThreads - 1) / kRegroupThreads;
    if (blocks > 2 * num_sms()) blocks = 2 * num_sms();
    cudaError_t e = launch_pdl(ep_regroup_kernel, dim3(blocks), dim3(kRegroupThreads), 0, s, 1,
                               recv_counts, n_src, E_local, R, counts, offsets, row_src, status);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    // k = 1: row_src holds receive positions, each the source row itself
    e = launch_gather_rows(x_rows, d, 2, 1, offsets + E_local, row_src, R, xg, num_sms(), s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    const int n_pairs = num_sms() / 2;
    PairMaps mp{};
    PairArgs pr{};
    pr.K = d;
    pr.n_ftiles = inter / 128;
    pr.n_groups = E_local;
    pr.counts = counts;
    pr.a_group_stride = 2LL * inter;
    pr.a_tile_step = 128;
    pr.a_cta_step = 64;
    pr.a_mode = 1;
    pr.a_blocks_per_group = 2 * inter / 16;
    pr.out = h;
    pr.out_ld = inter;
    pr.out_col_step = 128;
    pr.status = status;
    pr.sched_counter = status + kSchedWordGateUp;
    pr.wait_limit_ns = kWaitLimitNs;
    if (!make_map_gate_up(&mp.a[0], W_gate_up, (uint64_t)E_local, inter, d) ||
        !make_token_maps(mp.b[0], xg, (uint64_t)R, d))
        return MOE_ERR_CUDA;
    e = launch_pair_gemm(EPI_SWIGLU, EPI_SWIGLU, mp, pr, nullptr, n_pairs, R, s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    PairArgs qr{};
    qr.K = inter;
    qr.n_ftiles = d / 256;
    qr.n_groups = E_local;
    qr.counts = counts;
    qr.a_group_stride = d;
    qr.a_tile_step = 256;
    qr.a_cta_step = 128;
    qr.a_mode = 0;
    qr.out = y_rows;
    qr.out_ld = d;
    qr.out_col_step = 256;
    qr.row_src = row_src;  // grouped row -> receive position
    qr.topk_w = w_rows;    // gate weight of each received row
    qr.k = 1;
    qr.status = status;
    qr.sched_counter = status + kSchedWordDown;
    qr.wait_limit_ns = kWaitLimitNs;
    if (!make_map_rows_atoms(&mp.a[0], W_down, (uint64_t)E_local * d, inter) ||
        !make_token_maps(mp.b[0], h, (uint64_t)R, inter))
        return MOE_ERR_CUDA;
    return ret(launch_pair_gemm(EPI_SCATTER, EPI_SCATTER, mp, qr, nullptr, n_pairs, R, s));
}

MOE_API size_t moe_shared_workspace_bytes(int T, int d, int inter, int n_shared) {
    size_t off[SH_TOTAL + 1];
    return shared_layout(T, d, inter, n_shared, off) ? off[SH_TOTAL] : 0;
}

MOE_API int moe_shared_forward(const void* x, const void* W_shared, int T, int d, int inter,
                               int n_shared, int in_dt, float* y_shared, void* workspace,
                               size_t workspace_bytes, void* stream) {
    size_t off[SH_TOTAL + 1];
    if (!shared_layout(T, d, inter, n_shared, off)) return MOE_ERR_INVALID_ARG;
    if (in_dt != MOE_BF16) return MOE_ERR_UNSUPPORTED;
    if (workspace == nullptr || workspace_bytes < off[SH_TOTAL]) return MOE_ERR_WORKSPACE;
    if (T == 0) return MOE_OK;
    const void* p16[] = {x, W_shared, y_shared, workspace};
    for (const void* p : p16)
        if (!is_device_ptr(p) || !aligned(p, 16)) return MOE_ERR_INVALID_ARG;
    if (!aligned(workspace, 256)) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int* status = region<int>(workspace, off, SH_STATUS);
    void* h = region<char>(workspace, off, SH_H);
    const int SI = n_shared * inter;
    cudaError_t e = launch_pdl(reset_status_kernel, dim3(1), dim3(32), 0, s, 1, status);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    const int n_pairs = num_sms() / 2;
    PairMaps mp{};
    PairArgs ps{};
    ps.K = d;
    ps.n_ftiles = SI / 128;
    ps.counts = nullptr;
    ps.static_rows = T;
    ps.a_tile_step = 128;
    ps.a_cta_step = 64;
    ps.a_mode = 1;
    ps.a_blocks_per_group = 2 * SI / 16;
    ps.out = h;
    ps.out_ld = SI;
    ps.out_col_step = 128;
    ps.status = status;
    ps.sched_counter = status + kSchedWordGateUp;
    ps.wait_limit_ns = kWaitLimitNs;
    if (!make_map_gate_up(&mp.a[0], W_shared, 1, SI, d) ||
        !make_token_maps(mp.b[0], x, (uint64_t)T, d))
        return MOE_ERR_CUDA;
    e = launch_pair_gemm(EPI_SWIGLU, EPI_SWIGLU, mp, ps, nullptr, n_pairs, T, s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    const char* Wsh_dn = static_cast<const char*>(W_shared) + (size_t)2 * SI * d * 2;
    PairArgs qs{};
    qs.K = SI;
    qs.n_ftiles = d / 256;
    qs.counts = nullptr;
    qs.static_rows = T;
    qs.a_tile_step = 256;
    qs.a_cta_step = 128;
    qs.a_mode = 0;
    qs.out = y_shared;
    qs.out_ld = d;
    qs.out_col_step = 256;
    qs.status = status;
    qs.sched_counter = status + kSchedWordDown;
    qs.wait_limit_ns = kWaitLimitNs;
    if (!make_map_rows_atoms(&mp.a[0], Wsh_dn, (uint64_t)d, SI) ||
        !make_token_maps(mp.b[0], h, (uint64_t)T, SI))
        return MOE_ERR_CUDA;
    // one problem: the second epilogue of the pair is unused
    return ret(launch_pair_gemm(EPI_STORE_F32, EPI_SCATTER, mp, qs, nullptr, n_pairs, T, s));
}

MOE_API int moe_combine(const void* rows, int n_rows, const int32_t* slot_row,
                        const float* shared, int T, int d, int k, int out_dt, void* y,
                        void* status_ws, void* stream) {
    if (T < 0 || n_rows < 0 || d <= 0 || d % 8 != 0 || k < 1 || k > kMaxK)
        return MOE_ERR_INVALID_ARG;
    if (out_dt != MOE_F32 && out_dt != MOE_BF16) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!is_device_ptr(rows) || !aligned(rows, 16) || !is_device_ptr(y) || !aligned(y, 16) ||
        !is_device_ptr(slot_row) || !aligned(slot_row, 4))
        return MOE_ERR_INVALID_ARG;
    if (shared != nullptr && (!is_device_ptr(shared) || !aligned(shared, 16)))
        return MOE_ERR_INVALID_ARG;
    if (status_ws != nullptr && (!is_device_ptr(status_ws) || !aligned(status_ws, 256)))
        return MOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int d8 = d / 8;
    const unsigned blocks = (unsigned)(((size_t)T * d8 + 255) / 256);
    const uint4* r4 = static_cast<const uint4*>(rows);
    const float4* b4 = reinterpret_cast<const float4*>(shared);
    const int of = out_dt == MOE_F32 ? 1 : 0;
    int* status = static_cast<int*>(status_ws);
    switch (k) {
#define MOE_COMBINE_ROWS_K(KK)                                                            \
    case KK:                                                                              \
        return ret(launch_pdl(combine_rows_bf16_kernel<KK>, dim3(blocks), dim3(256), 0, s, 1, \
                              r4, slot_row, b4, T, d8, n_rows, y, of, status));
        MOE_COMBINE_ROWS_K(1) MOE_COMBINE_ROWS_K(2) MOE_COMBINE_ROWS_K(3) MOE_COMBINE_ROWS_K(4)
        MOE_COMBINE_ROWS_K(5) MOE_COMBINE_ROWS_K(6) MOE_COMBINE_ROWS_K(7) MOE_COMBINE_ROWS_K(8)
#undef MOE_COMBINE_ROWS_K
        default: return MOE_ERR_INVALID_ARG;
    }
}

}  // extern "C"
