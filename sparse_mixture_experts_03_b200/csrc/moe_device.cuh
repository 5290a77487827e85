// Device-side helpers shared by the MoE kernels: element conversion, the
// device status word, mbarrier / TMA / tcgen05 wrappers (inline PTX for
// sm_100a) and bounded waits.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe.h"
#include "moe_internal.h"

namespace moe {

// Kernel sites recorded in status word [1] when a device check fails.
enum Site : int {
    SITE_NONE = 0,
    SITE_GEMM_PRODUCER = 1,
    SITE_GEMM_MMA = 2,
    SITE_GEMM_EPILOGUE = 3,
    SITE_GEMM_DRAIN = 4,
    SITE_PERMUTE = 5,
    SITE_SELFTEST = 6,
    SITE_GEMM_BOUNDS = 7,
};

// ---------------------------------------------------------------- status
__device__ __forceinline__ void set_status(int* status, int code, int where, int info = 0) {
    if (status == nullptr) return;
    if (atomicCAS(status, 0, code) == 0) {
        status[1] = where;
        status[2] = info;
    }
}

// ---------------------------------------------------------------- launch order
// Wait until the previous kernel of the stream has completed and its memory
// writes are visible (no-op for a kernel launched without programmatic
// dependent launch).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// This CTA's work that later kernels depend on is done: the next kernel may be
// scheduled once every CTA of this grid has signalled or exited.
__device__ __forceinline__ void pdl_trigger() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------- elements
template <typename T> struct Elem;
template <> struct Elem<float> {
    static __device__ __forceinline__ float to_f(float v) { return v; }
};
template <> struct Elem<__nv_bfloat16> {
    static __device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);  // round to nearest even
    return *reinterpret_cast<uint32_t*>(&p);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile(
        "{\n\t.reg .b64 st;\n\t"
        "mbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile(
        "{\n\t.reg .b64 st;\n\t"
        "mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(smem_u32(bar)),
        "r"(bytes)
        : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

// Wait until the phase with parity `parity` of `bar` has completed.  Gives up
// after about `limit_ns` nanoseconds (measured in SM clock cycles at no more
// than 2 GHz, so the real limit is between limit_ns and a few times that), or
// as soon as *abort becomes non-zero (another role of the same CTA gave up).
// On giving up records MOE_ERR_TIMEOUT with `site` (unless another role already
// aborted) and returns false.  The barrier is polled 64 times between checks
// of the clock and of *abort, so a completing phase is seen within one poll.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  volatile int* abort, int* status, int site,
                                                  uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = clock64();
    const uint64_t limit_cycles = limit_ns * 2;
    for (;;) {
#pragma unroll 1
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (abort != nullptr && *abort) return false;
        if ((uint64_t)clock64() - t0 > limit_cycles) {
            if (abort != nullptr) *abort = 1;
            set_status(status, MOE_ERR_TIMEOUT, site);
            return false;
        }
    }
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 32 lanes x 32 consecutive 32-bit columns; thread i of the warp gets lane
// (lane base of taddr) + i.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32"
        " {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15,"
        " %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31},"
        " [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor of a K-major tile written by TMA with
// 128-byte swizzle: rows of 64 bf16 (128 B), 8-row swizzle atoms 1024 B apart.
// Fields (tcgen05 shared memory descriptor): start address >> 4 in bits
// [0,14), leading byte offset (unused for swizzled K-major, 1) in [16,30),
// stride byte offset 1024 >> 4 in [32,46), version 1 in [46,48), layout
// SWIZZLE_128B = 2 in [61,64).
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t smem_addr) {
    return (uint64_t)((smem_addr >> 4) & 0x3FFFu) | ((uint64_t)1u << 16) |
           ((uint64_t)(1024u >> 4) << 32) | ((uint64_t)1u << 46) | ((uint64_t)2u << 61);
}

// Shared-memory matrix descriptor of an MN-major tile written by TMA with
// 128-byte swizzle as [mn block of 64][k row][64 elements]: 64 consecutive
// M (or N) elements per 128-byte row, k rows 128 B apart, 8-row swizzle atoms.
// Leading byte offset = the distance between the 64-element MN blocks
// (mn_block_bytes), stride byte offset = the distance between 8-row k groups
// (1024 B); same version and layout fields as the K-major descriptor.
__device__ __forceinline__ uint64_t sw128_mnmajor_desc(uint32_t smem_addr,
                                                       uint32_t mn_block_bytes) {
    return (uint64_t)((smem_addr >> 4) & 0x3FFFu) |
           ((uint64_t)((mn_block_bytes >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)(1024u >> 4) << 32) | ((uint64_t)1u << 46) | ((uint64_t)2u << 61);
}

// Instruction descriptor for kind::f16: fp32 accumulator, bf16 A and B, M x N.
// Fields: D format [4,6) = 1 (F32), A format [7,10) = 1 (BF16), B format
// [10,13) = 1 (BF16), A major [15] and B major [16] (0 K-major, 1 MN-major),
// N >> 3 in [17,23), M >> 4 in [24,29).
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool a_mn = false,
                                                      bool b_mn = false) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) |
           ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

}  // namespace moe
