// Host-side helpers shared by the entry points: pointer and argument checks,
// the SM count, and the TMA tensor maps of the CTA-pair GEMMs.
#include <cudaTypedefs.h>

#include "../../include/moe.h"
#include "moe_internal.h"

namespace moe {

int check_routing(int E, int k, int n_group, int topk_group) {
    if (n_group < 1 || n_group > kMaxGroups || E % n_group != 0) return MOE_ERR_INVALID_ARG;
    if (topk_group < 1 || topk_group > n_group) return MOE_ERR_INVALID_ARG;
    if (k > topk_group * (E / n_group)) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

// gate and optional selection bias / expert-load output: shared checks
int check_gating(int gate, const float* bias, const int32_t* load) {
    if (gate != MOE_GATE_SIGMOID && gate != MOE_GATE_SOFTMAX_TOPK) return MOE_ERR_INVALID_ARG;
    if (bias != nullptr && (!is_device_ptr(bias) || !aligned(bias, 4))) return MOE_ERR_INVALID_ARG;
    if (load != nullptr && (!is_device_ptr(load) || !aligned(load, 4))) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Host-side check that p is memory the device can address (device or managed
// allocation).  Catches host pointers before any kernel could dereference them.
bool is_device_ptr(const void* p) {
    if (p == nullptr) return false;
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged;
}

int num_sms() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (dev < 0 || dev >= 64) return 148;
    if (cached[dev] == 0) {
        int n = 0;
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        cached[dev] = n > 0 ? n : 148;
    }
    return cached[dev];
}

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static bool tried = false;
    if (!tried) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
        tried = true;
    }
    return fn;
}

// bf16 matrix [rows, K] seen as {64, rows, K/64} (inner 64 columns, rows,
// 128-byte k-atoms): one box {64, box_rows, 2} brings box_rows rows x 128 of
// K as two consecutive 128B-swizzled tiles of box_rows x 128 bytes.
bool make_map_rows_atoms(CUtensorMap* m, const void* base, uint64_t rows, uint64_t K,
                         uint32_t box_rows) {
    auto fn = encode_fn();
    if (fn == nullptr || rows == 0 || K % 128 != 0) return false;
    cuuint64_t dims[3] = {64, rows, K / 64};
    cuuint64_t strides[2] = {K * 2, 128};
    cuuint32_t box[3] = {64, box_rows, 2};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// The token maps of one problem: boxes of 16, 32, ..., 128 rows.
bool make_token_maps(CUtensorMap (&m)[kTokenBoxes], const void* base, uint64_t rows, uint64_t K) {
    for (int j = 0; j < kTokenBoxes; ++j)
        if (!make_map_rows_atoms(&m[j], base, rows, K, 16u * (j + 1))) return false;
    return true;
}

// Gate/up weight [G][2][F][K] bf16 (per group: F gate rows, then F up rows)
// seen as {64, 16, 2, G*2F/16, K/64}: 16-row blocks of the whole weight, the
// gate/up axis (F rows apart) and k-atoms.  One box {64, 16, 2, 4, 2} at block
// b of a gate half brings, for 2 k-atoms, 4 x (16 gate rows, the 16 matching
// up rows): 64 features with gate and up interleaved per 16 rows.
bool make_map_gate_up(CUtensorMap* m, const void* base, uint64_t G, uint64_t F, uint64_t K) {
    auto fn = encode_fn();
    if (fn == nullptr || F % 64 != 0 || K % 128 != 0) return false;
    cuuint64_t dims[5] = {64, 16, 2, G * 2 * F / 16, K / 64};
    cuuint64_t strides[4] = {K * 2, F * K * 2, 16 * K * 2, 128};
    cuuint32_t box[5] = {64, 16, 2, 4, 2};
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}


}  // namespace moe
