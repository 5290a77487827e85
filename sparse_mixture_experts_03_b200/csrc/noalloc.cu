// moe_expert_counts_noalloc: per-expert token counts and segment offsets of a
// routing result, with its scratch in a fixed device array instead of a
// caller workspace.
//
// Who needs it: callers that must not allocate device memory (or hand over a
// workspace) on the call path -- for instance a serving step whose device
// memory is planned once up front, where a per-call allocation would either
// synchronise the device or not fit the plan.  The pages have no counterpart
// of this entry point: it is the histogram + exclusive scan of the
// permutation stage on its own, with unpadded segments.  Every occurrence of
// an id counts, so a row that repeats an expert adds it twice.
//
// The scratch is the file-scope array below: nothing is allocated, no
// allocating library is called.  Its device address is taken once per device
// (the first call on a device, with that device current, does this set-up;
// make that first call before any stream capture).  Every call uses the same
// array, so calls that overlap in time -- on two streams, or from two host
// threads -- race on it; callers serialise them.  Nothing in the array has to
// start at zero: each call writes every word it later reads.
#include <mutex>

#include "moe_device.cuh"
#include "moe_internal.h"


namespace moe {
namespace {

// ceil(T / 256) * E int32 words of per-block histograms (256 KiB): for
// example T <= 262144 tokens with E = 64 experts, T <= 65536 with E = 256.
constexpr int kNoAllocScratchWords = 65536;
static __device__ __align__(256) int32_t g_noalloc_scratch[kNoAllocScratchWords];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
int32_t* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device (set-up on the
// first call per device); nullptr on failure.
int32_t* scratch_on_current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (g_scratch_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        g_scratch_ptr[dev] = static_cast<int32_t*>(p);
    }
    return g_scratch_ptr[dev];
}

bool device_ptr(const void* p) {
    cudaPointerAttributes at;
    if (p == nullptr || cudaPointerGetAttributes(&at, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged;
}

}  // namespace
}  // namespace moe

MOE_API int moe_expert_counts_noalloc(const int32_t* topk_idx, int T, int k, int E,
                                      int32_t* counts, int32_t* offsets, void* stream) {
    using namespace moe;
    if (T < 0 || k < 1 || k > kMaxK || E < 1 || E > kMaxE || k > E) return MOE_ERR_INVALID_ARG;
    const long long nb = ((long long)T + kPermBlockTokens - 1) / kPermBlockTokens;
    if (nb * E > kNoAllocScratchWords) return MOE_ERR_WORKSPACE;  // beyond the fixed scratch
    if ((T > 0 && !device_ptr(topk_idx)) || !device_ptr(counts) || !device_ptr(offsets))
        return MOE_ERR_INVALID_ARG;
    int32_t* scratch = scratch_on_current_device();
    if (scratch == nullptr) return MOE_ERR_CUDA;
    const cudaError_t e = launch_expert_counts(topk_idx, T, k, E, scratch, counts, offsets,
                                               static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
