// C ABI of the MoE layer forward: argument checks, workspace layout, TMA
// descriptors and the launch sequence
//   route -> permute (histogram, scan, stable ranks) and gather rows, in one
//   launch
//   -> gate/up grouped GEMM + SwiGLU (routed; shared)
//   -> down grouped GEMM with weighted scatter to token-order slots (routed)
//   -> down GEMM of the shared experts with the fixed-order final sum.
// Everything runs on the caller's stream; nothing here synchronises it except
// moe_get_device_status, and nothing here allocates device memory.
#include <cudaTypedefs.h>

#include <algorithm>
#include <limits.h>
#include <stdlib.h>
#include <string.h>

#include "../../include/moe.h"
#include "moe_internal.h"

namespace {

using namespace moe;

constexpr size_t kRegionAlign = 1024;

struct Layout {
    size_t off[MOE_WS_TOTAL + 1];
    int rows_cap;
    int nb;
};

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

int check_sizes(int T, int d, int E, int k, int inter, int n_shared, int in_dt) {
    if (T < 0 || d <= 0 || E < 1 || E > kMaxE || k < 1 || k > kMaxK || inter <= 0 ||
        n_shared < 0)
        return MOE_ERR_INVALID_ARG;
    if (in_dt != MOE_F32 && in_dt != MOE_BF16) return MOE_ERR_INVALID_ARG;
    if (k > E) return MOE_ERR_INVALID_ARG;
    if ((long long)T * k + 128LL * E >= (long long)INT_MAX) return MOE_ERR_INVALID_ARG;
    if (d % 64 != 0 || inter % 128 != 0) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

bool make_layout(int T, int d, int E, int k, int inter, int n_shared, int in_dt, Layout& L) {
    if (check_sizes(T, d, E, k, inter, n_shared, in_dt) != MOE_OK) return false;
    const size_t esz = in_dt == MOE_BF16 ? 2 : 4;
    const size_t Tk = (size_t)T * k;
    L.rows_cap = (int)(Tk + (size_t)kRowAlign * E);
    L.nb = (T + kPermBlockTokens - 1) / kPermBlockTokens;
    const size_t sizes[MOE_WS_TOTAL] = {
        sizeof(int) * kStatusWords,                     // STATUS
        sizeof(int) * E,                                // COUNTS
        sizeof(int) * (E + 1),                          // OFFSETS
        // BLOCK_COUNTS: per 256-token block, or per CTA (<= ceil(T/32)) of the
        // one-launch permutation
        sizeof(int) * (size_t)std::max(std::max(L.nb, (T + 31) / 32), 1) * E,
        sizeof(int) * Tk,                               // TOPK_IDX
        sizeof(float) * Tk,                             // TOPK_W
        sizeof(int) * (size_t)L.rows_cap,               // ROW_SRC
        esz * (size_t)L.rows_cap * d,                   // X_PERM
        esz * (size_t)L.rows_cap * inter,               // H
        esz * (size_t)T * n_shared * inter,             // H_SHARED
        esz * Tk * d,                                   // SLOTS (in_dt)
        // Y_SHARED: fp32 shared-expert output before the final sum (bf16 layers)
        in_dt == MOE_BF16 ? sizeof(float) * (size_t)T * d * (n_shared > 0 ? 1 : 0) : 0,
    };
    size_t o = 0;
    for (int i = 0; i < MOE_WS_TOTAL; ++i) {
        L.off[i] = o;
        o = align_up(o + sizes[i], kRegionAlign);
    }
    L.off[MOE_WS_TOTAL] = o;
    return true;
}

template <typename T>
T* at(void* ws, const Layout& L, int region) {
    return reinterpret_cast<T*>(static_cast<char*>(ws) + L.off[region]);
}

cudaEvent_t g_stage_events[MOE_N_STAGE_EVENTS];
bool g_stage_events_on = false;

void stage_mark(int i, cudaStream_t s) {
    if (g_stage_events_on && g_stage_events[i] != nullptr) cudaEventRecord(g_stage_events[i], s);
}

cudaEvent_t g_bwd_events[MOE_N_BWD_STAGE_EVENTS];
bool g_bwd_events_on = false;

void bwd_mark(int i, cudaStream_t s) {
    if (g_bwd_events_on && g_bwd_events[i] != nullptr) cudaEventRecord(g_bwd_events[i], s);
}

}  // namespace

extern "C" {

MOE_API int moe_version(void) { return 1; }

MOE_API const char* moe_status_string(int status) {
    switch (status) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_UNSUPPORTED: return "unsupported shape or dtype";
        case MOE_ERR_CUDA: return "CUDA error";
        case MOE_ERR_WORKSPACE: return "workspace missing or too small";
        case MOE_ERR_TIMEOUT: return "device wait timed out";
        case MOE_ERR_DEVICE: return "device bounds check failed";
        default: return "unknown status";
    }
}

MOE_API size_t moe_workspace_bytes(int T, int d, int E, int k, int inter, int n_shared,
                                   int in_dt) {
    Layout L;
    if (!make_layout(T, d, E, k, inter, n_shared, in_dt, L)) return 0;
    return L.off[MOE_WS_TOTAL];
}

MOE_API int moe_workspace_layout(int T, int d, int E, int k, int inter, int n_shared, int in_dt,
                                 size_t* offsets, int n) {
    Layout L;
    if (offsets == nullptr || n < 1 || n > MOE_WS_TOTAL + 1) return MOE_ERR_INVALID_ARG;
    if (!make_layout(T, d, E, k, inter, n_shared, in_dt, L)) return MOE_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i) offsets[i] = L.off[i];
    return MOE_OK;
}

MOE_API int moe_route(const void* x, const void* W_router, int T, int d, int E, int k,
                      int n_group, int topk_group, int in_dt, int32_t* topk_idx, float* topk_w,
                      void* stream) {
    return moe_route_ex(x, W_router, T, d, E, k, n_group, topk_group, in_dt, MOE_GATE_SIGMOID,
                        nullptr, topk_idx, topk_w, stream);
}

MOE_API int moe_route_ex(const void* x, const void* W_router, int T, int d, int E, int k,
                         int n_group, int topk_group, int in_dt, int gate,
                         const float* expert_bias, int32_t* topk_idx, float* topk_w,
                         void* stream) {
    int st = check_sizes(T, d, E, k, 128, 0, in_dt);
    if (st != MOE_OK) return st;
    st = check_routing(E, k, n_group, topk_group);
    if (st != MOE_OK) return st;
    if (T == 0) return MOE_OK;
    st = check_gating(gate, expert_bias, nullptr);
    if (st != MOE_OK) return st;
    if (!is_device_ptr(x) || !is_device_ptr(W_router) || !is_device_ptr(topk_idx) ||
        !is_device_ptr(topk_w))
        return MOE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(W_router, 16) || !aligned(topk_idx, 4) ||
        !aligned(topk_w, 4))
        return MOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (in_dt == MOE_BF16)
        return ret(launch_route_bf16(x, W_router, T, d, E, k, n_group, topk_group, gate,
                                     expert_bias, topk_idx, topk_w, nullptr, s));
    return ret(launch_route_f32(x, W_router, T, d, E, k, n_group, topk_group, gate, expert_bias,
                                topk_idx, topk_w, nullptr, s));
}

MOE_API int moe_forward(const void* x, const void* W_router, const void* W_gate_up,
                        const void* W_down, const void* W_shared, int T, int d, int E, int k,
                        int n_group, int topk_group, int inter, int n_shared, int in_dt,
                        int out_dt, void* y, int32_t* topk_idx_out, float* topk_w_out,
                        void* workspace, size_t workspace_bytes, void* stream) {
    return moe_forward_ex(x, W_router, W_gate_up, W_down, W_shared, T, d, E, k, n_group,
                          topk_group, inter, n_shared, in_dt, out_dt, MOE_GATE_SIGMOID, nullptr,
                          y, topk_idx_out, topk_w_out, nullptr, workspace, workspace_bytes,
                          stream);
}

}  // extern "C"

namespace {
// The forward; with `saved` (bf16 layers) the gate/up epilogue also writes the
// pre-activations the backward reads.
int forward_impl(const void* x, const void* W_router, const void* W_gate_up, const void* W_down,
                 const void* W_shared, int T, int d, int E, int k, int n_group, int topk_group,
                 int inter, int n_shared, int in_dt, int out_dt, int gate,
                 const float* expert_bias, void* y, int32_t* topk_idx_out, float* topk_w_out,
                 int32_t* expert_load, void* saved, void* workspace, size_t workspace_bytes,
                 void* stream) {
    int st = check_sizes(T, d, E, k, inter, n_shared, in_dt);
    if (st != MOE_OK) return st;
    st = check_routing(E, k, n_group, topk_group);
    if (st != MOE_OK) return st;
    if (out_dt != MOE_F32 && out_dt != MOE_BF16) return MOE_ERR_INVALID_ARG;
    if (in_dt == MOE_BF16 && d % 256 != 0) return MOE_ERR_UNSUPPORTED;
    if ((n_shared > 0) != (W_shared != nullptr)) return MOE_ERR_INVALID_ARG;
    Layout L;
    make_layout(T, d, E, k, inter, n_shared, in_dt, L);
    if (workspace == nullptr || workspace_bytes < L.off[MOE_WS_TOTAL]) return MOE_ERR_WORKSPACE;
    st = check_gating(gate, expert_bias, expert_load);
    if (st != MOE_OK) return st;
    if (T == 0) {
        if (expert_load != nullptr)
            return ret(cudaMemsetAsync(expert_load, 0, sizeof(int32_t) * E,
                                       static_cast<cudaStream_t>(stream)));
        return MOE_OK;
    }
    const void* dev_ptrs[] = {x, W_router, W_gate_up, W_down, y, workspace};
    for (const void* p : dev_ptrs)
        if (!is_device_ptr(p) || !aligned(p, 16)) return MOE_ERR_INVALID_ARG;
    if (n_shared > 0 && (!is_device_ptr(W_shared) || !aligned(W_shared, 16)))
        return MOE_ERR_INVALID_ARG;
    if (!aligned(workspace, 256)) return MOE_ERR_INVALID_ARG;
    if ((topk_idx_out != nullptr && (!is_device_ptr(topk_idx_out) || !aligned(topk_idx_out, 4))) ||
        (topk_w_out != nullptr && (!is_device_ptr(topk_w_out) || !aligned(topk_w_out, 4))))
        return MOE_ERR_INVALID_ARG;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int* status = at<int>(workspace, L, MOE_WS_STATUS);
    int32_t* idx = topk_idx_out != nullptr ? topk_idx_out : at<int32_t>(workspace, L, MOE_WS_TOPK_IDX);
    float* w = topk_w_out != nullptr ? topk_w_out : at<float>(workspace, L, MOE_WS_TOPK_W);
    int32_t* counts = at<int32_t>(workspace, L, MOE_WS_COUNTS);
    int32_t* offsets = at<int32_t>(workspace, L, MOE_WS_OFFSETS);
    int32_t* block_counts = at<int32_t>(workspace, L, MOE_WS_BLOCK_COUNTS);
    int32_t* row_src = at<int32_t>(workspace, L, MOE_WS_ROW_SRC);
    void* x_perm = at<char>(workspace, L, MOE_WS_X_PERM);
    void* h = at<char>(workspace, L, MOE_WS_H);
    void* h_sh = at<char>(workspace, L, MOE_WS_H_SHARED);
    void* slots = at<char>(workspace, L, MOE_WS_SLOTS);
    const int SI = n_shared * inter;
    const bool bf16 = in_dt == MOE_BF16;
    const int out_f32 = out_dt == MOE_F32 ? 1 : 0;

    stage_mark(0, s);
    // 1. routing (also resets the status word)
    cudaError_t e = bf16 ? launch_route_bf16(x, W_router, T, d, E, k, n_group, topk_group, gate,
                                             expert_bias, idx, w, status, s)
                         : launch_route_f32(x, W_router, T, d, E, k, n_group, topk_group, gate,
                                            expert_bias, idx, w, status, s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    stage_mark(1, s);
    // 2. permutation: histogram, scan, stable ranks, row gather
    // the CTA-pair GEMMs (bf16) take unpadded expert segments; the CUDA-core
    // kernels (fp32) take segments padded to their 128-row tiles
    if (T <= kSmallPermTokens) {
        e = launch_permute_gather_small(idx, T, k, E, bf16 ? 1 : kRowAlign, counts, offsets,
                                        row_src, expert_load, status, x, d, bf16 ? 2 : 4,
                                        x_perm, num_sms(), s);
    } else if (permute_gather_grid_fits(T, E, num_sms())) {
        e = launch_permute_gather_grid(idx, T, k, E, bf16 ? 1 : kRowAlign, block_counts, counts,
                                       offsets, row_src, expert_load, status,
                                       status + kGridBarWordPermute, kWaitLimitNs, x, d,
                                       bf16 ? 2 : 4, x_perm, num_sms(), s);
    } else {
        e = launch_permute(idx, T, k, E, block_counts, counts, offsets, row_src,
                           bf16 ? 1 : kRowAlign, expert_load, status, s);
        if (e != cudaSuccess) return MOE_ERR_CUDA;
        e = launch_gather_rows(x, d, bf16 ? 2 : 4, k, offsets + E, row_src, L.rows_cap, x_perm,
                               num_sms(), s);
    }
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    stage_mark(2, s);

    const char* Wsh_gu = static_cast<const char*>(W_shared);
    const char* Wsh_dn = Wsh_gu == nullptr ? nullptr
                                           : Wsh_gu + (size_t)2 * SI * d * (bf16 ? 2 : 4);

    if (bf16) {
        // 3. gate/up + SwiGLU: shared experts on all tokens (problem 0: the
        //    longest tiles are handed out first), routed experts (problem 1)
        const int n_pairs = num_sms() / 2;
        PairMaps mp{};
        PairArgs pr{};
        pr.K = d;
        pr.n_ftiles = inter / 128;
        pr.n_groups = E;
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
        const bool train = saved != nullptr;
        if (train) {  // pre-activations in the saved layout, rows in this launch's order
            pr.save = saved;
            pr.gu_rows = T * k;
            pr.feat = inter;
        }
        const int epi_gu = train ? EPI_SWIGLU_SAVE : EPI_SWIGLU;
        // problem 1 (routed) goes in slot 1 when there are shared experts, else slot 0
        const int pr_slot = n_shared > 0 ? 1 : 0;
        if (!make_map_gate_up(&mp.a[pr_slot], W_gate_up, (uint64_t)E, inter, d) ||
            !make_token_maps(mp.b[pr_slot], x_perm, (uint64_t)T * k, d))
            return MOE_ERR_CUDA;
        if (n_shared > 0) {
            PairArgs ps = pr;
            ps.n_ftiles = SI / 128;
            ps.counts = nullptr;
            ps.static_rows = T;
            ps.a_group_stride = 0;
            ps.out = h_sh;
            ps.out_ld = SI;
            ps.a_blocks_per_group = 2 * SI / 16;
            ps.row_src = nullptr;  // shared rows are tokens
            ps.gu_rows = T;
            ps.feat = SI;
            ps.save = train ? static_cast<char*>(saved) + (size_t)T * k * 2 * inter * 2 : nullptr;
            if (!make_map_gate_up(&mp.a[0], Wsh_gu, 1, SI, d) ||
                !make_token_maps(mp.b[0], x, (uint64_t)T, d))
                return MOE_ERR_CUDA;
            e = launch_pair_gemm(epi_gu, epi_gu, mp, ps, &pr, n_pairs, T, s);
        } else {
            e = launch_pair_gemm(epi_gu, epi_gu, mp, pr, nullptr, n_pairs, T, s);
        }
        if (e != cudaSuccess) return MOE_ERR_CUDA;
        stage_mark(3, s);
        // 4. down projections: shared experts into fp32 rows (problem 0),
        //    routed experts weighted into bf16 token-order slots (problem 1)
        PairArgs qr{};
        qr.K = inter;
        qr.n_ftiles = d / 256;
        qr.n_groups = E;
        qr.counts = counts;
        qr.a_group_stride = d;
        qr.a_tile_step = 256;
        qr.a_cta_step = 128;
        qr.a_mode = 0;
        qr.out = slots;
        qr.out_ld = d;
        qr.out_col_step = 256;
        qr.row_src = row_src;
        qr.topk_w = w;
        qr.k = k;
        qr.status = status;
        qr.sched_counter = status + kSchedWordDown;
        qr.wait_limit_ns = kWaitLimitNs;
        const int qr_slot = n_shared > 0 ? 1 : 0;
        if (!make_map_rows_atoms(&mp.a[qr_slot], W_down, (uint64_t)E * d, inter) ||
            !make_token_maps(mp.b[qr_slot], h, (uint64_t)T * k, inter))
            return MOE_ERR_CUDA;
        float* y_sh = nullptr;
        if (n_shared > 0) {
            y_sh = at<float>(workspace, L, MOE_WS_Y_SHARED);
            PairArgs qs = qr;
            qs.K = SI;
            qs.counts = nullptr;
            qs.static_rows = T;
            qs.a_group_stride = 0;
            qs.out = y_sh;
            qs.row_src = nullptr;
            qs.topk_w = nullptr;
            if (!make_map_rows_atoms(&mp.a[0], Wsh_dn, (uint64_t)d, SI) ||
                !make_token_maps(mp.b[0], h_sh, (uint64_t)T, SI))
                return MOE_ERR_CUDA;
            e = launch_pair_gemm(EPI_STORE_F32, EPI_SCATTER, mp, qs, &qr, n_pairs, T, s);
        } else {
            e = launch_pair_gemm(EPI_SCATTER, EPI_SCATTER, mp, qr, nullptr, n_pairs, T, s);
        }
        if (e != cudaSuccess) return MOE_ERR_CUDA;
        stage_mark(4, s);
        // 5. the streaming final sum y = shared + slot_0 + ... + slot_{k-1}
        e = launch_combine_slots(slots, 1, y_sh, T, d, k, y, out_f32, s);
        if (e != cudaSuccess) return MOE_ERR_CUDA;
        stage_mark(5, s);
        return MOE_OK;
    }

    GemmArgs g1{};
    g1.K = d;
    g1.n_groups = E;
    g1.offsets = offsets;
    g1.b_group_stride = 2LL * inter;
    g1.b_half_off = inter;
    g1.valid_rows = INT_MAX;
    g1.out = h;
    g1.out_ld = inter;
    g1.out_f32 = bf16 ? 0 : 1;
    g1.status = status;
    g1.wait_limit_ns = kWaitLimitNs;

    GemmArgs g1s = g1;
    g1s.offsets = nullptr;
    g1s.n_groups = 1;
    g1s.static_rows = T;
    g1s.b_group_stride = 0;
    g1s.b_half_off = SI;
    g1s.valid_rows = T;
    g1s.out = h_sh;
    g1s.out_ld = SI;

    GemmArgs g2{};
    g2.K = inter;
    g2.n_groups = E;
    g2.offsets = offsets;
    g2.b_group_stride = d;
    g2.valid_rows = INT_MAX;
    g2.out = slots;
    g2.out_ld = d;
    g2.row_src = row_src;
    g2.topk_w = w;
    g2.k = k;
    g2.status = status;
    g2.wait_limit_ns = kWaitLimitNs;

    GemmArgs g2s = g2;
    g2s.K = SI;
    g2s.offsets = nullptr;
    g2s.n_groups = 1;
    g2s.static_rows = T;
    g2s.b_group_stride = 0;
    g2s.valid_rows = T;
    g2s.out = y;
    g2s.slots = slots;
    g2s.out_f32 = out_f32;

    // fp32: CUDA-core grouped GEMMs, 64-column output tiles
    const float* Wgu = static_cast<const float*>(W_gate_up);
    const float* Wdn = static_cast<const float*>(W_down);
    g1.n_tiles = inter / 64;
    g1.b_tile_step = 64;
    g1.out_col_step = 64;
    e = launch_gemm_simt(EPI_SWIGLU, static_cast<const float*>(x_perm), Wgu, g1, L.rows_cap, s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    if (n_shared > 0) {
        g1s.n_tiles = SI / 64;
        g1s.b_tile_step = 64;
        g1s.out_col_step = 64;
        e = launch_gemm_simt(EPI_SWIGLU, static_cast<const float*>(x),
                             reinterpret_cast<const float*>(Wsh_gu), g1s,
                             (T + 127) / 128 * 128, s);
        if (e != cudaSuccess) return MOE_ERR_CUDA;
    }
    stage_mark(3, s);
    g2.n_tiles = d / 64;
    g2.b_tile_step = 64;
    g2.b_half_off = 0;
    g2.out_col_step = 64;
    e = launch_gemm_simt(EPI_SCATTER, static_cast<const float*>(h), Wdn, g2, L.rows_cap, s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    stage_mark(4, s);
    if (n_shared > 0) {
        g2s.n_tiles = d / 64;
        g2s.b_tile_step = 64;
        g2s.b_half_off = 0;
        g2s.out_col_step = 64;
        e = launch_gemm_simt(EPI_COMBINE, static_cast<const float*>(h_sh),
                             reinterpret_cast<const float*>(Wsh_dn), g2s,
                             (T + 127) / 128 * 128, s);
    } else {
        e = launch_combine_slots(slots, bf16 ? 1 : 0, nullptr, T, d, k, y, out_f32, s);
    }
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    stage_mark(5, s);
    return MOE_OK;
}
}  // namespace

extern "C" {

MOE_API int moe_forward_ex(const void* x, const void* W_router, const void* W_gate_up,
                           const void* W_down, const void* W_shared, int T, int d, int E, int k,
                           int n_group, int topk_group, int inter, int n_shared, int in_dt,
                           int out_dt, int gate, const float* expert_bias, void* y,
                           int32_t* topk_idx_out, float* topk_w_out, int32_t* expert_load,
                           void* workspace, size_t workspace_bytes, void* stream) {
    return forward_impl(x, W_router, W_gate_up, W_down, W_shared, T, d, E, k, n_group,
                        topk_group, inter, n_shared, in_dt, out_dt, gate, expert_bias, y,
                        topk_idx_out, topk_w_out, expert_load, nullptr, workspace,
                        workspace_bytes, stream);
}

MOE_API size_t moe_saved_bytes(int T, int k, int inter, int n_shared) {
    if (T < 0 || k < 1 || k > kMaxK || inter <= 0 || n_shared < 0) return 0;
    return (size_t)2 * 2 * inter * ((size_t)T * k + (size_t)T * n_shared);
}

MOE_API int moe_forward_train(const void* x, const void* W_router, const void* W_gate_up,
                              const void* W_down, const void* W_shared, int T, int d, int E,
                              int k, int n_group, int topk_group, int inter, int n_shared,
                              int in_dt, int out_dt, int gate, const float* expert_bias,
                              void* y, int32_t* topk_idx_out, float* topk_w_out,
                              int32_t* expert_load, void* saved, size_t saved_bytes,
                              void* workspace, size_t workspace_bytes, void* stream) {
    int st = check_sizes(T, d, E, k, inter, n_shared, in_dt);
    if (st != MOE_OK) return st;
    if (in_dt != MOE_BF16) return MOE_ERR_UNSUPPORTED;
    if (T > 0) {
        if (topk_idx_out == nullptr || topk_w_out == nullptr) return MOE_ERR_INVALID_ARG;
        if (saved == nullptr || !is_device_ptr(saved) || !aligned(saved, 16))
            return MOE_ERR_INVALID_ARG;
        if (saved_bytes < moe_saved_bytes(T, k, inter, n_shared)) return MOE_ERR_INVALID_ARG;
    }
    return forward_impl(x, W_router, W_gate_up, W_down, W_shared, T, d, E, k, n_group,
                        topk_group, inter, n_shared, in_dt, out_dt, gate, expert_bias, y,
                        topk_idx_out, topk_w_out, expert_load, T > 0 ? saved : nullptr,
                        workspace, workspace_bytes, stream);
}

MOE_API int moe_set_stage_events(void* const* events, int n) {
    if (events == nullptr) {
        g_stage_events_on = false;
        return MOE_OK;
    }
    if (n != MOE_N_STAGE_EVENTS) return MOE_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i) g_stage_events[i] = static_cast<cudaEvent_t>(events[i]);
    g_stage_events_on = true;
    return MOE_OK;
}

MOE_API int moe_get_device_status(const void* workspace, int* status, int* where, void* stream) {
    if (workspace == nullptr || status == nullptr) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int buf[2] = {0, 0};
    if (cudaMemcpyAsync(buf, workspace, sizeof(buf), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
    *status = buf[0];
    if (where != nullptr) *where = buf[1];
    return MOE_OK;
}

MOE_API int moe_clear_device_status(void* workspace, void* stream) {
    if (workspace == nullptr) return MOE_ERR_INVALID_ARG;
    return ret(cudaMemsetAsync(workspace, 0, sizeof(int) * kStatusWords,
                               static_cast<cudaStream_t>(stream)));
}

MOE_API int moe_selftest_timeout(void* workspace, int limit_us, void* stream) {
    if (workspace == nullptr || limit_us < 1 || limit_us > 1000000) return MOE_ERR_INVALID_ARG;
    if (!is_device_ptr(workspace)) return MOE_ERR_INVALID_ARG;
    return ret(launch_selftest_timeout(static_cast<int*>(workspace),
                                       (unsigned long long)limit_us * 1000ull,
                                       static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

namespace {

// Workspace of the backward (bf16 layers): regions in this order.
enum BwdRegion : int {
    BW_STATUS, BW_COUNTS, BW_OFFSETS, BW_BLOCK_COUNTS, BW_ROW_SRC, BW_SLOT_ROW, BW_X_PERM,
    BW_DY_PERM, BW_DGU, BW_HW, BW_DW_PART, BW_DL, BW_DX_SLOTS, BW_DGU_SH, BW_HW_SH, BW_DX_SH,
    BW_DWR_PART, BW_TOTAL
};
struct BwdLayout {
    size_t off[BW_TOTAL + 1];
    int rows_cap;
};

bool make_bwd_layout(int T, int d, int E, int k, int inter, int n_shared, BwdLayout& L) {
    if (check_sizes(T, d, E, k, inter, n_shared, MOE_BF16) != MOE_OK) return false;
    if (d % 256 != 0 || inter % 256 != 0) return false;
    const size_t Tk = (size_t)T * k, SI = (size_t)n_shared * inter;
    L.rows_cap = (int)(Tk + (size_t)kRowAlign * E);
    const size_t rc = (size_t)L.rows_cap;
    const int nb = (T + kPermBlockTokens - 1) / kPermBlockTokens;
    const size_t sizes[BW_TOTAL] = {
        sizeof(int) * kStatusWords,             // STATUS (+ tile counters)
        sizeof(int) * E,                        // COUNTS
        sizeof(int) * (E + 1),                  // OFFSETS (segments padded to 128 rows)
        // BLOCK_COUNTS: per 256-token block, or per CTA of the one-launch permutation
        sizeof(int) * (size_t)std::max(std::max(nb, (T + 31) / 32), 1) * E,
        sizeof(int) * rc,                       // ROW_SRC
        sizeof(int) * Tk,                       // SLOT_ROW: slot -> permuted row
        2 * rc * d,                             // X_PERM
        2 * rc * d,                             // DY_PERM
        2 * rc * 2 * inter,                     // DGU: dg | du per permuted row
        2 * rc * inter,                         // HW: w * h per permuted row
        sizeof(float) * rc * (inter / 32),      // DW_PART
        sizeof(float) * Tk,                     // DL
        2 * Tk * d,                             // DX_SLOTS (bf16, slot order)
        2 * (size_t)T * 2 * SI,                 // DGU_SH
        2 * (size_t)T * SI,                     // HW_SH
        n_shared > 0 ? sizeof(float) * (size_t)T * d : 0,  // DX_SH
        sizeof(float) * (size_t)kDwParts * E * d,  // DWR_PART: row-slice sums of dW_router
    };
    size_t o = 0;
    for (int i = 0; i < BW_TOTAL; ++i) {
        L.off[i] = o;
        o = align_up(o + sizes[i], kRegionAlign);
    }
    L.off[BW_TOTAL] = o;
    return true;
}

template <typename T>
T* bat(void* ws, const BwdLayout& L, int region) {
    return reinterpret_cast<T*>(static_cast<char*>(ws) + L.off[region]);
}

}  // namespace

extern "C" {

MOE_API size_t moe_backward_workspace_bytes(int T, int d, int E, int k, int inter,
                                            int n_shared) {
    BwdLayout L;
    if (!make_bwd_layout(T, d, E, k, inter, n_shared, L)) return 0;
    return L.off[BW_TOTAL];
}

MOE_API int moe_backward(const void* x, const void* W_router, const void* W_gate_up,
                         const void* W_down, const void* W_shared, const void* dy,
                         const int32_t* topk_idx, const float* topk_w, const void* saved,
                         int T, int d, int E, int k, int inter, int n_shared, int in_dt,
                         int gate, float* dx, float* dW_router, float* dW_gate_up,
                         float* dW_down, float* dW_shared, void* workspace,
                         size_t workspace_bytes, void* stream) {
    int st = check_sizes(T, d, E, k, inter, n_shared, in_dt);
    if (st != MOE_OK) return st;
    if (in_dt != MOE_BF16 || d % 256 != 0 || inter % 256 != 0) return MOE_ERR_UNSUPPORTED;
    if (gate != MOE_GATE_SIGMOID && gate != MOE_GATE_SOFTMAX_TOPK) return MOE_ERR_INVALID_ARG;
    if ((n_shared > 0) != (W_shared != nullptr) || (n_shared > 0) != (dW_shared != nullptr))
        return MOE_ERR_INVALID_ARG;
    BwdLayout L;
    make_bwd_layout(T, d, E, k, inter, n_shared, L);
    if (workspace == nullptr || workspace_bytes < L.off[BW_TOTAL]) return MOE_ERR_WORKSPACE;
    const void* wptrs[] = {W_router, W_gate_up, W_down, dW_router, dW_gate_up, dW_down, workspace};
    for (const void* p : wptrs)
        if (!is_device_ptr(p) || !aligned(p, 16)) return MOE_ERR_INVALID_ARG;
    if (n_shared > 0 && (!is_device_ptr(W_shared) || !aligned(W_shared, 16) ||
                         !is_device_ptr(dW_shared) || !aligned(dW_shared, 16)))
        return MOE_ERR_INVALID_ARG;
    if (!aligned(workspace, 256)) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int SI = n_shared * inter;
    if (T == 0) {  // no tokens: every weight gradient is zero
        cudaError_t e = cudaMemsetAsync(dW_router, 0, sizeof(float) * (size_t)E * d, s);
        if (e == cudaSuccess)
            e = cudaMemsetAsync(dW_gate_up, 0, sizeof(float) * (size_t)E * 2 * inter * d, s);
        if (e == cudaSuccess)
            e = cudaMemsetAsync(dW_down, 0, sizeof(float) * (size_t)E * d * inter, s);
        if (e == cudaSuccess && n_shared > 0)
            e = cudaMemsetAsync(dW_shared, 0, sizeof(float) * (size_t)3 * SI * d, s);
        return ret(e);
    }
    const void* tptrs[] = {x, dy, topk_idx, topk_w, saved, dx};
    for (const void* p : tptrs)
        if (!is_device_ptr(p) || !aligned(p, 16)) return MOE_ERR_INVALID_ARG;

    int* status = bat<int>(workspace, L, BW_STATUS);
    int32_t* counts = bat<int32_t>(workspace, L, BW_COUNTS);
    int32_t* offsets = bat<int32_t>(workspace, L, BW_OFFSETS);
    int32_t* block_counts = bat<int32_t>(workspace, L, BW_BLOCK_COUNTS);
    int32_t* row_src = bat<int32_t>(workspace, L, BW_ROW_SRC);
    int32_t* slot_row = bat<int32_t>(workspace, L, BW_SLOT_ROW);
    void* x_perm = bat<char>(workspace, L, BW_X_PERM);
    void* dy_perm = bat<char>(workspace, L, BW_DY_PERM);
    void* dgu = bat<char>(workspace, L, BW_DGU);
    void* hw = bat<char>(workspace, L, BW_HW);
    float* dw_part = bat<float>(workspace, L, BW_DW_PART);
    float* dl = bat<float>(workspace, L, BW_DL);
    void* dx_slots = bat<char>(workspace, L, BW_DX_SLOTS);
    void* dgu_sh = bat<char>(workspace, L, BW_DGU_SH);
    void* hw_sh = bat<char>(workspace, L, BW_HW_SH);
    float* dx_sh = n_shared > 0 ? bat<float>(workspace, L, BW_DX_SH) : nullptr;
    const char* Wsh_gu = static_cast<const char*>(W_shared);
    const char* Wsh_dn = Wsh_gu != nullptr ? Wsh_gu + (size_t)2 * SI * d * 2 : nullptr;
    const char* gu_routed = static_cast<const char*>(saved);
    const char* gu_shared = gu_routed + (size_t)T * k * 2 * inter * 2;
    const uint64_t rows_cap = (uint64_t)L.rows_cap;
    const int n_pairs = num_sms() / 2;
    const int rs = n_shared > 0 ? 1 : 0;  // slot of the routed problem in each launch

    // status word and the four launches' tile counters start at zero
    bwd_mark(0, s);
    cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int) * kStatusWords, s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    // 1. the forward's permutation again, with segments padded to 128 rows
    //    (whole k-blocks of the weight-gradient GEMMs), then x / dy rows
    if (T <= kSmallPermTokens)
        e = launch_permute_gather_small(topk_idx, T, k, E, kRowAlign, counts, offsets, row_src,
                                        nullptr, status, nullptr, d, 2, nullptr, num_sms(), s,
                                        slot_row);
    else if (permute_gather_grid_fits(T, E, num_sms()))
        e = launch_permute_gather_grid(topk_idx, T, k, E, kRowAlign, block_counts, counts, offsets,
                                       row_src, nullptr, status, status + kGridBarWordPermute,
                                       kWaitLimitNs, nullptr, d, 2, nullptr, num_sms(), s,
                                       slot_row);
    else
        e = launch_permute(topk_idx, T, k, E, block_counts, counts, offsets, row_src, kRowAlign,
                           nullptr, status, s, slot_row);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    e = launch_bwd_gather(x, dy, T, d, inter, k, offsets + E, row_src, slot_row, L.rows_cap,
                          x_perm, dy_perm, dgu, hw, num_sms(), s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    bwd_mark(1, s);

    PairArgs base{};
    base.n_groups = E;
    base.counts = counts;
    base.seg_align = kRowAlign;
    base.a_tile_step = 256;
    base.a_cta_step = 128;
    base.k = k;
    base.status = status;
    base.wait_limit_ns = kWaitLimitNs;
    auto dense = [&](PairArgs a) {  // the shared experts: one group of T token rows
        a.counts = nullptr;
        a.static_rows = T;
        a.seg_align = 1;
        a.a_group_stride = 0;
        a.row_src = nullptr;
        a.topk_w = nullptr;
        return a;
    };

    // 2. dh = W_down^T dy per chosen expert (weights MN-major), SwiGLU backward
    //    in the epilogue: dg|du, w*h and the parts of dL/dw
    {
        PairMaps mp{};
        PairArgs r = base;
        r.K = d;
        r.n_ftiles = inter / 256;
        r.a_group_stride = d;
        r.row_src = row_src;
        r.topk_w = topk_w;
        r.feat = inter;
        r.gu_rows = T * k;
        r.gu_in = gu_routed;
        r.dgu_out = dgu;
        r.hw_out = hw;
        r.dw_part = dw_part;
        r.sched_counter = status + kSchedWordBwd0;
        if (!make_map_rows_atoms(&mp.a[rs], W_down, (uint64_t)E * d, inter) ||
            !make_token_maps(mp.b[rs], dy_perm, rows_cap, d))
            return MOE_ERR_CUDA;
        if (n_shared > 0) {
            PairArgs sh = dense(r);
            sh.n_ftiles = SI / 256;
            sh.feat = SI;
            sh.gu_rows = T;
            sh.gu_in = gu_shared;
            sh.dgu_out = dgu_sh;
            sh.hw_out = hw_sh;
            sh.dw_part = nullptr;
            if (!make_map_rows_atoms(&mp.a[0], Wsh_dn, (uint64_t)d, SI) ||
                !make_token_maps(mp.b[0], dy, (uint64_t)T, d))
                return MOE_ERR_CUDA;
            e = launch_pair_gemm(EPI_DSWIGLU, EPI_DSWIGLU, mp, sh, &r, n_pairs, T, s, KIND_DGRAD);
        } else {
            e = launch_pair_gemm(EPI_DSWIGLU, EPI_DSWIGLU, mp, r, nullptr, n_pairs, T, s,
                                 KIND_DGRAD);
        }
        if (e != cudaSuccess) return MOE_ERR_CUDA;
        bwd_mark(2, s);
    }
    // 3. dL/dlogit of the chosen experts
    e = launch_router_dlogit(x, W_router, T, d, k, topk_idx, topk_w, dw_part, inter / 32,
                             slot_row, gate, dl, s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    bwd_mark(3, s);
    // 4. dx parts = W_gate_up^T [dg|du] (weights MN-major): chosen experts into
    //    token-order slots, shared experts into fp32 rows
    {
        PairMaps mp{};
        PairArgs r = base;
        r.K = 2 * inter;
        r.n_ftiles = d / 256;
        r.a_group_stride = 2LL * inter;
        r.out = dx_slots;
        r.out_ld = d;
        r.out_col_step = 256;
        r.row_src = row_src;
        r.topk_w = nullptr;  // weight 1: dg|du already carry w
        r.sched_counter = status + kSchedWordBwd0 + 1;
        if (!make_map_rows_atoms(&mp.a[rs], W_gate_up, (uint64_t)E * 2 * inter, d) ||
            !make_token_maps(mp.b[rs], dgu, rows_cap, 2 * inter))
            return MOE_ERR_CUDA;
        if (n_shared > 0) {
            PairArgs sh = dense(r);
            sh.K = 2 * SI;
            sh.out = dx_sh;
            if (!make_map_rows_atoms(&mp.a[0], Wsh_gu, (uint64_t)2 * SI, d) ||
                !make_token_maps(mp.b[0], dgu_sh, (uint64_t)T, 2 * SI))
                return MOE_ERR_CUDA;
            e = launch_pair_gemm(EPI_STORE_F32, EPI_SCATTER, mp, sh, &r, n_pairs, T, s,
                                 KIND_DGRAD);
        } else {
            e = launch_pair_gemm(EPI_SCATTER, EPI_SCATTER, mp, r, nullptr, n_pairs, T, s,
                                 KIND_DGRAD);
        }
        if (e != cudaSuccess) return MOE_ERR_CUDA;
        bwd_mark(4, s);
    }
    // 5. dx = shared part + chosen experts' parts + router part (fixed order)
    e = launch_bwd_combine(dx_sh, dx_slots, dl, topk_idx, W_router, T, d, k, dx, s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    bwd_mark(5, s);
    // 6. dW_down = (w dy)^T h per expert: both operands MN-major, K = the
    //    expert's rows
    {
        PairMaps mp{};
        PairArgs r = base;
        r.n_ftiles = d / 256;
        r.n_ntiles = inter / 256;
        r.m_total = d;
        r.out = dW_down;
        r.out_ld = inter;
        r.sched_counter = status + kSchedWordBwd0 + 2;
        if (!make_map_rows_atoms(&mp.a[rs], dy_perm, rows_cap, d) ||
            !make_map_rows_atoms(&mp.b[rs][kTokenBoxes - 1], hw, rows_cap, inter))
            return MOE_ERR_CUDA;
        if (n_shared > 0) {
            PairArgs sh = dense(r);
            sh.n_ntiles = SI / 256;
            sh.out = const_cast<char*>(reinterpret_cast<const char*>(dW_shared)) +
                     sizeof(float) * (size_t)2 * SI * d;
            sh.out_ld = SI;
            if (!make_map_rows_atoms(&mp.a[0], dy, (uint64_t)T, d) ||
                !make_map_rows_atoms(&mp.b[0][kTokenBoxes - 1], hw_sh, (uint64_t)T, SI))
                return MOE_ERR_CUDA;
            e = launch_pair_gemm(EPI_STORE_ROWS, EPI_STORE_ROWS, mp, sh, &r, n_pairs, 256, s,
                                 KIND_WGRAD);
        } else {
            e = launch_pair_gemm(EPI_STORE_ROWS, EPI_STORE_ROWS, mp, r, nullptr, n_pairs, 256, s,
                                 KIND_WGRAD);
        }
        if (e != cudaSuccess) return MOE_ERR_CUDA;
        bwd_mark(6, s);
    }
    // 7. dW_gate_up = [dg|du]^T x per expert
    {
        PairMaps mp{};
        PairArgs r = base;
        r.n_ftiles = 2 * inter / 256;
        r.n_ntiles = d / 256;
        r.m_total = 2 * inter;
        r.out = dW_gate_up;
        r.out_ld = d;
        r.sched_counter = status + kSchedWordBwd0 + 3;
        if (!make_map_rows_atoms(&mp.a[rs], dgu, rows_cap, 2 * inter) ||
            !make_map_rows_atoms(&mp.b[rs][kTokenBoxes - 1], x_perm, rows_cap, d))
            return MOE_ERR_CUDA;
        if (n_shared > 0) {
            PairArgs sh = dense(r);
            sh.n_ftiles = 2 * SI / 256;
            sh.m_total = 2 * SI;
            sh.out = dW_shared;
            if (!make_map_rows_atoms(&mp.a[0], dgu_sh, (uint64_t)T, 2 * SI) ||
                !make_map_rows_atoms(&mp.b[0][kTokenBoxes - 1], x, (uint64_t)T, d))
                return MOE_ERR_CUDA;
            e = launch_pair_gemm(EPI_STORE_ROWS, EPI_STORE_ROWS, mp, sh, &r, n_pairs, 256, s,
                                 KIND_WGRAD);
        } else {
            e = launch_pair_gemm(EPI_STORE_ROWS, EPI_STORE_ROWS, mp, r, nullptr, n_pairs, 256, s,
                                 KIND_WGRAD);
        }
        if (e != cudaSuccess) return MOE_ERR_CUDA;
        bwd_mark(7, s);
    }
    // 8. dW_router[e] = sum of dl * x over expert e's rows
    e = launch_router_dweight(dl, row_src, offsets, x_perm, E, d,
                              bat<float>(workspace, L, BW_DWR_PART), dW_router, s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    bwd_mark(8, s);
    return MOE_OK;
}

MOE_API int moe_set_backward_stage_events(void* const* events, int n) {
    if (events == nullptr) {
        g_bwd_events_on = false;
        return MOE_OK;
    }
    if (n != MOE_N_BWD_STAGE_EVENTS) return MOE_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i) g_bwd_events[i] = static_cast<cudaEvent_t>(events[i]);
    g_bwd_events_on = true;
    return MOE_OK;
}

}  // extern "C"
