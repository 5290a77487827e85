// Host-side declarations shared by the .cu files of the library (launchers
// and argument structs).  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <utility>

#include "../../include/moe.h"

namespace moe {

// Every kernel of the forward is launched with programmatic dependent launch:
// its CTAs may be scheduled while the previous kernel in the stream is
// finishing (hiding the launch latency between the small stages), and each
// kernel waits (griddepcontrol.wait, which returns once the previous grid has
// completed and its writes are visible) before it reads or writes memory.
// cluster_x > 1 adds a cluster dimension.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, int cluster_x, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    int n = 0;
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
    if (cluster_x > 1) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = (unsigned)cluster_x;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = (unsigned)n;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

constexpr int kMaxE = 256;
constexpr int kMaxGroups = 32;
constexpr int kMaxK = 8;
constexpr int kRowAlign = 128;         // expert segments of the permuted layout are padded to this
constexpr int kPermBlockTokens = 256;  // tokens per block of the permutation kernels
constexpr int kStatusWords = 64;       // int32 words of the status region of the workspace
// status words used as tile ticket counters of the CTA-pair GEMM launches
// (reset to 0, with words 0..15, by the routing kernel at the start of a forward)
constexpr int kSchedWordGateUp = 12;
constexpr int kSchedWordDown = 13;
// arrival counter of the permutation's grid-wide barrier (same reset; the
// backward and the expert-parallel dispatch reset it the same way)
constexpr int kGridBarWordPermute = 14;
// the backward's four CTA-pair launches (the backward clears the whole status
// region first)
constexpr int kSchedWordBwd0 = 20;

// Bound of every device-side wait of the forward and backward kernels.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s per wait

// ---- host helpers (host_util.cu)
// E % n_group == 0, 1 <= topk_group <= n_group, k <= topk_group * E / n_group
int check_routing(int E, int k, int n_group, int topk_group);
// gate is a moe_gate; bias / load, when given, are 4-byte aligned device pointers
int check_gating(int gate, const float* bias, const int32_t* load);
bool aligned(const void* p, size_t a);
// p is device or managed memory (a host pointer is caught before any launch)
bool is_device_ptr(const void* p);
// SM count of the current device (cached)
int num_sms();
inline int ret(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// Epilogue variants of the grouped GEMMs.
enum Epi : int {
    EPI_SWIGLU = 0,     // out = silu(gate) * up (bf16 on the CTA-pair kernel, f32 on CUDA cores)
    EPI_SCATTER = 1,    // slots[row_src[r]] = topk_w[row_src[r]] * acc, rows with row_src < 0
                        // skipped (bf16 slots on the CTA-pair kernel, f32 on CUDA cores)
    EPI_COMBINE = 2,    // y[t] = acc + slots[t*k + 0] + ... + slots[t*k + k-1] (CUDA cores)
    EPI_STORE_F32 = 3,  // out[row] = acc, fp32 (CTA-pair kernel)
    // training (CTA-pair kernel)
    EPI_SWIGLU_SAVE = 4,   // SWIGLU, and the pre-activations gate|up (bf16) to save rows
    EPI_DSWIGLU = 5,       // SwiGLU backward of dh = acc (see PairArgs)
    EPI_STORE_ROWS = 6,    // weight-gradient tile: out[weight row][col] = acc, fp32
};

// Operand layouts and tile shapes of a CTA-pair launch.
enum PairKind : int {
    KIND_FWD = 0,    // A (weights) K-major, B (tokens) K-major; tiles: feature tile x token chunk
    KIND_DGRAD = 1,  // A (weights) MN-major (their transpose is the operand), B K-major
    KIND_WGRAD = 2,  // A and B MN-major (activation rows are K); tiles: M tile x N tile,
                     // K = the group's rows (0 rows: a tile of zeros)
};

// CUDA-core (fp32 layers) grouped GEMM  out[r, n] = sum_c A[r, c] * B[b_row(r, n), c]  over row
// groups.  Rows of group g are [off[g], off[g+1]) of A (a multiple of 128
// rows each); with offsets == nullptr there is one group of static_rows rows.
struct GemmArgs {
    int K;                 // reduction length
    int n_tiles;           // output tiles along N per group
    int n_groups;          // groups (experts); ignored when offsets == nullptr
    const int32_t* offsets;
    int static_rows;
    long long b_group_stride;  // B rows between consecutive groups
    int b_tile_step;           // B rows between consecutive N tiles
    int b_half_off;            // B row offset of the second half of a tile's B rows
    int valid_rows;            // SWIGLU/COMBINE: rows >= valid_rows are not stored
    void* out;
    int out_ld;                // elements per output row
    int out_col_step;          // output columns per N tile
    const int32_t* row_src;    // SCATTER
    const float* topk_w;       // SCATTER
    const void* slots;         // COMBINE: f32 slots
    int k;                     // SCATTER/COMBINE
    int out_f32;               // COMBINE: y dtype (1 f32, 0 bf16); SWIGLU f32 path: 1
    int* status;
    unsigned long long wait_limit_ns;
};

// ---- launchers (return a cudaError_t from the launch)
// gate: MOE_GATE_SIGMOID or MOE_GATE_SOFTMAX_TOPK; bias: device f32[E] selection-only
// expert bias, or nullptr.
cudaError_t launch_route_bf16(const void* x, const void* Wr, int T, int d, int E, int k, int G,
                              int TG, int gate, const float* bias, int32_t* idx, float* w,
                              int* status, cudaStream_t s);
cudaError_t launch_route_f32(const void* x, const void* Wr, int T, int d, int E, int k, int G,
                             int TG, int gate, const float* bias, int32_t* idx, float* w,
                             int* status, cudaStream_t s);

// Segments of the permuted layout are padded to a multiple of `align` rows
// (1: unpadded) with row_src = -1 on padding rows; slot_row (nullable) gets
// the inverse: slot t*k + j -> its row.
cudaError_t launch_permute(const int32_t* idx, int T, int k, int E, int32_t* block_counts,
                           int32_t* counts, int32_t* offsets, int32_t* row_src, int align,
                           int32_t* load_out, int* status, cudaStream_t s,
                           int32_t* slot_row = nullptr);
// x_perm[r] = x[row_src[r] / k] for the rows r < *offsets_total with row_src
// >= 0; with w_dst also w_dst[r] = w_src[row_src[r]].
cudaError_t launch_gather_rows(const void* x, int d, int elem_bytes, int k,
                               const int32_t* offsets_total, const int32_t* row_src,
                               int rows_cap, void* x_perm, int num_sms, cudaStream_t s,
                               const float* w_src = nullptr, float* w_dst = nullptr);
// launch_permute followed by launch_gather_rows in one launch.  T <= 1024:
// several CTAs, each derives the permutation, CTA 0 writes it out.  The k ids
// of a token are distinct.  x == nullptr: no row copies (the permutation
// alone); slot_row (nullable): slot -> row; w_dst (nullable): w_dst[row] =
// w_src[slot].
constexpr int kSmallPermTokens = 1024;
cudaError_t launch_permute_gather_small(const int32_t* idx, int T, int k, int E, int align,
                                       int32_t* counts, int32_t* offsets, int32_t* row_src,
                                       int32_t* load_out, int* status, const void* x, int d,
                                       int elem_bytes, void* x_perm, int num_sms,
                                       cudaStream_t s, int32_t* slot_row = nullptr,
                                       const float* w_src = nullptr, float* w_dst = nullptr);
// T > 1024: the same in one launch of at most num_sms CTAs (token blocks of
// a multiple of 32), which meet at one grid-wide barrier: *grid_bar must be 0
// at launch (a status word the routing kernel, or the backward's status
// reset, zeroes).  block_counts holds min(num_sms, ceil(T/32)) * E int32.
// False from _fits when the per-CTA bitmaps would not fit in shared memory
// (use the separate kernels then).
constexpr size_t kPermGatherGridMaxSmem = 160 * 1024;
bool permute_gather_grid_fits(int T, int E, int num_sms);
cudaError_t launch_permute_gather_grid(const int32_t* idx, int T, int k, int E, int align,
                                      int32_t* block_counts, int32_t* counts, int32_t* offsets,
                                      int32_t* row_src, int32_t* load_out, int* status,
                                      int* grid_bar, unsigned long long wait_limit_ns,
                                      const void* x, int d, int elem_bytes, void* x_perm,
                                      int num_sms, cudaStream_t s, int32_t* slot_row = nullptr,
                                      const float* w_src = nullptr, float* w_dst = nullptr);
// Per-expert counts and unpadded segment offsets of a table of expert ids
// (histogram + scan only); block_counts holds ceil(T/256) * E int32.  Every
// occurrence of an id counts (a row may repeat one); ids outside [0, E) are
// not counted.
cudaError_t launch_expert_counts(const int32_t* idx, int T, int k, int E,
                                 int32_t* block_counts, int32_t* counts, int32_t* offsets,
                                 cudaStream_t s);
// y[t] = base[t] + slots[t*k + 0] + ... + slots[t*k + k-1] in fp32, in that
// order (base: fp32 [T, d] or nullptr for none).
cudaError_t launch_combine_slots(const void* slots, int slots_bf16, const float* base, int T,
                                 int d, int k, void* y, int out_f32, cudaStream_t s);

cudaError_t launch_gemm_simt(int epi, const float* A, const float* B, const GemmArgs& a,
                             int rows_cap, cudaStream_t s);

// Weights x tokens grouped GEMM on CTA pairs (see gemm_pair.cu).  Group g of a
// problem has counts[g] token rows (static_rows when counts == nullptr),
// stored consecutively from row b_row_base in the B tensor; weight rows of
// feature tile ft for the pair's CTA c start at
//   a_row0 = g * a_group_stride + ft * a_tile_step + c * a_cta_step
// (a_mode 0), or are features ft * a_tile_step + c * a_cta_step .. + 63 of
// group g, gate and up interleaved per 16 (a_mode 1).  Output columns of
// feature tile ft start at ft * out_col_step.
struct PairArgs {
    int K;
    int n_ftiles;
    int n_groups;
    const int32_t* counts;
    int static_rows;
    int b_row_base;
    long long a_group_stride;
    int a_tile_step;
    int a_cta_step;
    int a_mode;              // 0: 3-D map {64, rows, K/64}: 128 rows from a_row0
                             // 1: 5-D map {64, 16, 2, G*2F/16, K/64} of a [G][2][F][K]
                             //    gate/up weight: 4 blocks of (16 gate, 16 up) rows
    int a_blocks_per_group;  // a_mode 1: 16-row blocks per group (2F / 16)
    void* out;
    int out_ld;
    int out_col_step;
    const int32_t* row_src;  // SCATTER: permuted row -> t*k + j
    const float* topk_w;     // SCATTER
    const void* slots;       // COMBINE: bf16 [T*k, out_ld]
    int k;
    int out_f32;             // COMBINE
    int* status;
    int* sched_counter;      // problem 0's: tile tickets of the launch, 0 at launch
    unsigned long long wait_limit_ns;
    // ---- training
    int seg_align;           // group segments of B start at multiples of this (0 or 1: packed)
    int n_ntiles;            // KIND_WGRAD: 256-wide tiles along N
    int m_total;             // STORE_ROWS: output rows per group (n_ftiles * 256)
    void* save;              // SWIGLU_SAVE: gate|up pre-activations, bf16, blocks of 16
                             // features: [F/16][gu_rows][16 gate | 16 up], rows in this
                             // launch's order (expert-contiguous, unpadded; or tokens)
    int gu_rows;             // SWIGLU_SAVE / DSWIGLU: rows of the saved layout
    int feat;                // F: SwiGLU features of the problem (inter, or n_shared * inter)
    // DSWIGLU: acc = dh_raw [feature, row] = (W_down^T dy)[row]; w = topk_w[row_src[r]] (1 when
    // row_src == nullptr); reads gate|up of the row's forward position (r minus the padding
    // before its segment) from gu_in (the SWIGLU_SAVE layout), writes
    // dgu_out[r] = (dh * u * silu'(g) | dh * silu(g)) [2F] bf16, hw_out[r] = w * silu(g) * u [F]
    // bf16 and, with dw_part, dw_part[r * (F / 32) + part] = sum over the warp's 32 features of
    // dh_raw * silu(g) * u.
    const void* gu_in;
    void* dgu_out;
    void* hw_out;
    float* dw_part;
};
// Tensor maps of one launch.  Each stage covers 128 of K (two 64-column
// swizzle atoms).  a[p]: weights of problem p, a_mode 0: box {64, 128, 2};
// a_mode 1: box {64, 16, 2, 4, 2}.  b[p][j]: tokens of problem p, 3-D
// {64, rows, K/64}, box {64, 16 (j + 1), 2}: a tile of N tokens loads N/2 rows
// per CTA with the smallest box that covers them.  K must be a multiple of 128.
constexpr int kTokenBoxes = 8;
struct PairMaps {
    CUtensorMap a[2];
    CUtensorMap b[2][kTokenBoxes];
};
// Tensor maps (bf16, 128-byte swizzle).  make_map_rows_atoms: a [rows, K]
// matrix as {64, rows, K/64}, box {64, box_rows, 2} (box_rows rows x 128 of
// K); make_token_maps: the kTokenBoxes maps of one token matrix (boxes of 16,
// 32, ..., 128 rows); make_map_gate_up: a [G][2][F][K] gate/up weight as
// {64, 16, 2, G*2F/16, K/64}, box {64, 16, 2, 4, 2} (4 x (16 gate rows, the
// 16 matching up rows) x 128 of K).  False if the driver rejects the map.
bool make_map_rows_atoms(CUtensorMap* m, const void* base, uint64_t rows, uint64_t K,
                         uint32_t box_rows = 128);
bool make_token_maps(CUtensorMap (&m)[kTokenBoxes], const void* base, uint64_t rows, uint64_t K);
bool make_map_gate_up(CUtensorMap* m, const void* base, uint64_t G, uint64_t F, uint64_t K);
// Epilogue pairs (epi0 for problem 0, epi1 for problem 1): SWIGLU/SWIGLU,
// STORE_F32/SCATTER, SCATTER/SCATTER, SWIGLU_SAVE/SWIGLU_SAVE (KIND_FWD);
// DSWIGLU/DSWIGLU, STORE_F32/SCATTER, SCATTER/SCATTER (KIND_DGRAD);
// STORE_ROWS/STORE_ROWS (KIND_WGRAD).  a1 == nullptr: one problem.
// max_tile_tokens: an upper bound on the tokens of any tile (the batch size,
// capped at 256); up to 128 (and again up to 64) the launch uses a deeper ring
// of smaller stages.
cudaError_t launch_pair_gemm(int epi0, int epi1, const PairMaps& maps, const PairArgs& a0,
                             const PairArgs* a1, int n_pairs, int max_tile_tokens,
                             cudaStream_t s, int kind = KIND_FWD);

// ---- backward helpers (backward.cu)
// Rows of the padded permuted layout (rows [0, offsets_total)): each token's
// x and dy rows are read once and written to its k rows slot_row[t*k + j];
// padding rows (row_src < 0) of x_perm, dy_perm, dgu [2F] and hw [F] are set
// to zero.  bf16.
cudaError_t launch_bwd_gather(const void* x, const void* dy, int T, int d, int F, int k,
                              const int32_t* offsets_total, const int32_t* row_src,
                              const int32_t* slot_row, int rows_cap, void* x_perm, void* dy_perm,
                              void* dgu, void* hw, int num_sms, cudaStream_t s);
// dl[t*k + j] = dL/dlogit of token t's chosen expert j (gate MOE_GATE_*), from
// dw = sum of the dw_part row of its slot, topk_w and the recomputed logits.
cudaError_t launch_router_dlogit(const void* x, const void* Wr, int T, int d, int k,
                                 const int32_t* idx, const float* topk_w, const float* dw_part,
                                 int n_parts, const int32_t* slot_row, int gate, float* dl,
                                 cudaStream_t s);
// dx[t] = base[t] (fp32, nullable) + slots[t*k+0..k-1] (bf16) + sum_j dl[t*k+j] Wr[idx[t*k+j]],
// in that order, fp32.
cudaError_t launch_bwd_combine(const float* base, const void* slots, const float* dl,
                               const int32_t* idx, const void* Wr, int T, int d, int k, float* dx,
                               cudaStream_t s);
// dWr[e] = sum over rows r of expert e's padded segment with row_src[r] >= 0 of
// dl[row_src[r]] * x_perm[r], fp32: kDwParts fixed row slices of the segment
// summed in row order into part [kDwParts, E, d], then the slices in order.
constexpr int kDwParts = 8;
cudaError_t launch_router_dweight(const float* dl, const int32_t* row_src, const int32_t* offsets,
                                  const void* x_perm, int E, int d, float* part, float* dWr,
                                  cudaStream_t s);

cudaError_t launch_selftest_timeout(int* status, unsigned long long limit_ns, cudaStream_t s);

}  // namespace moe
