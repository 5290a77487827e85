// Grouped GEMM on the 5th-generation tensor cores (tcgen05, sm_100a), fed by
// TMA, accumulating in tensor memory, with the MoE epilogues fused:
//   EPI_SWIGLU   gate/up projection: one tile holds 128 gate rows and the 128
//                matching up rows of B, so the epilogue sees both halves of
//                SwiGLU for the same 128 output columns and writes
//                h = silu(gate) * up as bf16 (SwiGLU: "大模型工程（一）：
//                Transformer 到 MoE", section "变了什么，为什么变", item 3).
//   EPI_SCATTER  down projection of the routed experts: each output row is
//                scaled by its gate weight and written to the token-order
//                slot (t, j) it came from (the weighted combine of the
//                MoEBlock listing, section "混合专家：更多参数，相同 FLOPs").
//   EPI_COMBINE  down projection of the shared experts, with the final sum
//                y = shared + slot_0 + ... + slot_{k-1} in fixed order (the
//                always-on shared experts: "FusionLLM：融合 MLA、GDN 与 MoE 的
//                高效混合架构大模型训练框架", section "模型配置与规模").
//
// The grouped GEMM after routing is named as a fused kernel target on the
// FusionLLM page (section "融合内核"); this is a fresh design for B200:
//   - persistent CTAs (one per SM) walk a tile list built on the device from
//     the per-expert row offsets: tile = (128-row block, N tile); the group
//     (expert) of a row block is found by binary search in the offsets;
//   - warp 0 issues TMA loads (128B swizzle, K-major boxes of 64 x 128) into a
//     4-stage ring; warp 1 issues tcgen05.mma M=128 N=256 K=16 from one
//     thread and commits to mbarriers; warps 2..5 drain the accumulator from
//     TMEM (tcgen05.ld) and run the epilogue;
//   - two 256-column fp32 accumulators (all 512 TMEM columns) let the
//     epilogue of one tile overlap the main loop of the next;
//   - every wait is bounded; a CTA that gives up records MOE_ERR_TIMEOUT in
//     the status word, lets its other roles stop, drains its tensor-core work
//     and frees TMEM before returning.
// No cluster launch and no multicast loads.
#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {

namespace {

constexpr int BM = 128;           // rows per tile (MMA M, TMEM lanes)
constexpr int BK = 64;            // K per stage: one 128-byte swizzle atom of bf16
constexpr int BNB = 256;          // B rows per tile (MMA N)
constexpr int kStages = 4;
constexpr int kABytes = BM * BK * 2;        // 16 KiB
constexpr int kBBytes = BNB * BK * 2;       // 32 KiB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kTmemCols = 512;              // 2 accumulators x 256 fp32 columns
constexpr int kThreads = 192;               // 6 warps
constexpr int kEpiThreads = 128;
constexpr uint32_t kIdesc = idesc_bf16_f32(BM, BNB);
constexpr int kMaxOffsets = kMaxE + 1;

struct __align__(16) SmemTail {
    uint4 stage[kEpiThreads / 32][32 * 8];  // per epilogue warp: 32 rows x 128 B, swizzled
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
    int offsets[2][kMaxOffsets];
};

constexpr size_t kSmemBytes = 1024 /*alignment slack*/ + (size_t)kStages * kStageBytes +
                              sizeof(SmemTail);

__device__ __forceinline__ int find_group(const int* off, int n_groups, int row) {
    int lo = 0, hi = n_groups - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (off[mid] <= row)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

__device__ __forceinline__ float silu_mul(float g, float u) {
    return __fdividef(g, 1.0f + __expf(-g)) * u;
}

// Tile t of the launch belongs to problem 0 when t < tiles0, else to problem 1
// (tile t - tiles0).  Inside a problem: row block t / n_tiles, N tile t % n_tiles.
struct TileRef {
    int p, row0, nt, g;
};

// Epilogue of one tile for the rows of TMEM lane quarter wq (thread `lane`
// holds row wq*32 + lane of the tile).
template <int EPI>
__device__ __forceinline__ void epilogue_tile(uint4* buf, uint32_t taddr, const TileRef& r,
                                              const GemmArgs& args, int lane, int wq, int col0) {
    const int grow = r.row0 + wq * 32 + lane;
    // Epilogue stores go through a per-warp staging buffer: thread `lane`
    // holds row wq*32 + lane after tcgen05.ld; it writes its 128-byte row
    // piece to shared memory (16-byte units XOR-swizzled by row, so both
    // the row-wise writes and the transposed reads are conflict-free),
    // then each store instruction covers 4 rows x 128 contiguous bytes.
    const int rr_lo = lane >> 3, q = lane & 7;
    auto piece = [&](int i) -> uint4 {
        const int rr = i * 4 + rr_lo;
        return buf[rr * 8 + (q ^ (rr & 7))];
    };
    const int row_base = r.row0 + wq * 32;

    if constexpr (EPI == EPI_SWIGLU) {
#pragma unroll 1
        for (int c = 0; c < BNB / 2; c += 64) {
            uint32_t p[32];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t g[32], u[32];
                tmem_ld32(taddr + c + 32 * half, g);
                tmem_ld32(taddr + BNB / 2 + c + 32 * half, u);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    p[16 * half + i] = pack_bf16x2(
                        silu_mul(__uint_as_float(g[2 * i]), __uint_as_float(u[2 * i])),
                        silu_mul(__uint_as_float(g[2 * i + 1]),
                                 __uint_as_float(u[2 * i + 1])));
            }
#pragma unroll
            for (int j = 0; j < 8; ++j)
                buf[lane * 8 + (j ^ (lane & 7))] =
                    make_uint4(p[4 * j], p[4 * j + 1], p[4 * j + 2], p[4 * j + 3]);
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int row = row_base + i * 4 + rr_lo;
                const uint4 v = piece(i);
                if (row < args.valid_rows)
                    *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(args.out) +
                                              (size_t)row * args.out_ld + col0 + c +
                                              8 * q) = v;
            }
            __syncwarp();
        }
    } else if constexpr (EPI == EPI_SCATTER) {
        // slot rows are bf16: w * acc rounded once, 64 columns per staging round
        const int src = grow < args.valid_rows ? args.row_src[grow] : -1;
        const float wv = src >= 0 ? args.topk_w[src] : 0.f;
#pragma unroll 1
        for (int c = 0; c < BNB; c += 64) {
            uint32_t p[32];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t v[32];
                tmem_ld32(taddr + c + 32 * half, v);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    p[16 * half + i] = pack_bf16x2(wv * __uint_as_float(v[2 * i]),
                                                   wv * __uint_as_float(v[2 * i + 1]));
            }
#pragma unroll
            for (int j = 0; j < 8; ++j)
                buf[lane * 8 + (j ^ (lane & 7))] =
                    make_uint4(p[4 * j], p[4 * j + 1], p[4 * j + 2], p[4 * j + 3]);
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int s_rr = __shfl_sync(0xffffffffu, src, i * 4 + rr_lo);
                const uint4 val = piece(i);
                if (s_rr >= 0)
                    *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(args.out) +
                                              (size_t)s_rr * args.out_ld + col0 + c + 8 * q) =
                        val;
            }
            __syncwarp();
        }
    } else {  // EPI_COMBINE
#pragma unroll 1
        for (int c = 0; c < BNB; c += 32) {
            uint32_t v[32];
            tmem_ld32(taddr + c, v);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 8; ++j)
                buf[lane * 8 + (j ^ (lane & 7))] =
                    make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
            __syncwarp();
            float4 a[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint4 u = piece(i);
                a[i] = make_float4(__uint_as_float(u.x), __uint_as_float(u.y),
                                   __uint_as_float(u.z), __uint_as_float(u.w));
            }
            __syncwarp();
            // for 4 rows at a time: all k slot pieces (4 bf16 each) first, then
            // y = shared + slot_0 + ... + slot_{k-1} in that order
#pragma unroll
            for (int h4 = 0; h4 < 8; h4 += 4) {
                uint2 sv[kMaxK][4];
#pragma unroll
                for (int j = 0; j < kMaxK; ++j) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int t = row_base + (h4 + i) * 4 + rr_lo;
                        sv[j][i] = make_uint2(0u, 0u);
                        if (j < args.k && t < args.valid_rows)
                            sv[j][i] = __ldcg(reinterpret_cast<const uint2*>(
                                static_cast<const __nv_bfloat16*>(args.slots) +
                                ((size_t)t * args.k + j) * args.out_ld + col0 + c + 4 * q));
                    }
                }
#pragma unroll
                for (int j = 0; j < kMaxK; ++j) {
                    if (j >= args.k) break;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        float4& ai = a[h4 + i];
                        ai.x += __uint_as_float(sv[j][i].x << 16);
                        ai.y += __uint_as_float(sv[j][i].x & 0xffff0000u);
                        ai.z += __uint_as_float(sv[j][i].y << 16);
                        ai.w += __uint_as_float(sv[j][i].y & 0xffff0000u);
                    }
                }
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int t = row_base + i * 4 + rr_lo;
                if (t >= args.valid_rows) continue;
                const size_t o = (size_t)t * args.out_ld + col0 + c + 4 * q;
                if (args.out_f32) {
                    *reinterpret_cast<float4*>(static_cast<float*>(args.out) + o) = a[i];
                } else {
                    *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(args.out) + o) =
                        make_uint2(pack_bf16x2(a[i].x, a[i].y), pack_bf16x2(a[i].z, a[i].w));
                }
            }
        }
    }
}

template <int EPI0, int EPI1>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA0,
                           const __grid_constant__ CUtensorMap tmB0,
                           const __grid_constant__ CUtensorMap tmA1,
                           const __grid_constant__ CUtensorMap tmB1, const GemmArgs args0,
                           const GemmArgs args1, int n_problems, int* sync_counter) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    SmemTail* tail = reinterpret_cast<SmemTail*>(smem + (size_t)kStages * kStageBytes);
    volatile int* abort_flag = &tail->abort;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&tail->full[s], 1);
            mbar_init(&tail->empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tail->tfull[a], 1);
            mbar_init(&tail->tempty[a], kEpiThreads);
        }
        mbar_init(&tail->drain, 1);
        tail->abort = 0;
        fence_barrier_init();
    }
    for (int p = 0; p < n_problems; ++p) {
        const GemmArgs& a = p == 0 ? args0 : args1;
        if (a.offsets != nullptr) {
            for (int i = tid; i <= a.n_groups; i += kThreads) tail->offsets[p][i] = a.offsets[i];
        } else if (tid == 0) {
            tail->offsets[p][0] = 0;
            tail->offsets[p][1] = (a.static_rows + BM - 1) / BM * BM;
        }
    }
    if (warp == 1) {
        tmem_alloc(&tail->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const uint32_t tmem_base = tail->tmem_base;
    const int ng0 = args0.offsets != nullptr ? args0.n_groups : 1;
    const int ng1 = args1.offsets != nullptr ? args1.n_groups : 1;
    const int tiles0 = (tail->offsets[0][ng0] / BM) * args0.n_tiles;
    const int tiles1 = n_problems > 1 ? (tail->offsets[1][ng1] / BM) * args1.n_tiles : 0;
    const int total_tiles = tiles0 + tiles1;
    const uint64_t limit = args0.wait_limit_ns;
    int* const status = args0.status;

    auto tile_ref = [&](int tile) {
        TileRef r;
        r.p = tile < tiles0 ? 0 : 1;
        const int lt = r.p == 0 ? tile : tile - tiles0;
        const GemmArgs& a = r.p == 0 ? args0 : args1;
        r.row0 = (lt / a.n_tiles) * BM;
        r.nt = lt % a.n_tiles;
        r.g = find_group(tail->offsets[r.p], r.p == 0 ? ng0 : ng1, r.row0);
        return r;
    };

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&tmA0);
            tma_prefetch_desc(&tmB0);
            if (n_problems > 1) {
                tma_prefetch_desc(&tmA1);
                tma_prefetch_desc(&tmB1);
            }
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            uint32_t issued = 0, issued_ph = 0;  // per stage: loaded at least once / parity
            for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
                const TileRef r = tile_ref(tile);
                const GemmArgs& a = r.p == 0 ? args0 : args1;
                const CUtensorMap* mA = r.p == 0 ? &tmA0 : &tmA1;
                const CUtensorMap* mB = r.p == 0 ? &tmB0 : &tmB1;
                const int b0 = (int)(r.g * a.b_group_stride) + r.nt * a.b_tile_step;
                const int b1 = b0 + a.b_half_off;
                const int kb_count = a.K / BK;
                for (int kb = 0; kb < kb_count; ++kb) {
                    if (!mbar_wait_bounded(&tail->empty[s], ph ^ 1u, abort_flag, status,
                                           SITE_GEMM_PRODUCER, limit)) {
                        ok = false;
                        break;
                    }
                    uint8_t* sa = smem + (size_t)s * kStageBytes;
                    uint8_t* sb = sa + kABytes;
                    mbar_arrive_expect_tx(&tail->full[s], kStageBytes);
                    tma_load_2d(sa, mA, &tail->full[s], kb * BK, r.row0);
                    tma_load_2d(sb, mB, &tail->full[s], kb * BK, b0);
                    tma_load_2d(sb + kBBytes / 2, mB, &tail->full[s], kb * BK, b1);
                    issued |= 1u << s;
                    issued_ph = (issued_ph & ~(1u << s)) | (ph << s);
                    if (++s == kStages) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            if (!ok) {
                // let copies already in flight land before the CTA goes away
                for (int i = 0; i < kStages; ++i)
                    if ((issued >> i) & 1u)
                        mbar_wait_bounded(&tail->full[i], (issued_ph >> i) & 1u, nullptr,
                                          nullptr, 0, limit);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            int it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x, ++it) {
                const int acc = it & 1;
                const uint32_t aph = (it >> 1) & 1;
                const int kb_count = (tile < tiles0 ? args0.K : args1.K) / BK;
                if (!mbar_wait_bounded(&tail->tempty[acc], aph ^ 1u, abort_flag, status,
                                       SITE_GEMM_MMA, limit)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BNB);
                for (int kb = 0; kb < kb_count; ++kb) {
                    if (!mbar_wait_bounded(&tail->full[s], ph, abort_flag, status,
                                           SITE_GEMM_MMA, limit)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + (size_t)s * kStageBytes);
                    const uint32_t b_addr = a_addr + kABytes;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        const uint64_t ad = sw128_kmajor_desc(a_addr + kk * 32);
                        const uint64_t bd = sw128_kmajor_desc(b_addr + kk * 32);
                        tc_mma_f16(d_tmem, ad, bd, kIdesc, (kb | kk) != 0 ? 1u : 0u);
                    }
                    tc_commit(&tail->empty[s]);
                    if (++s == kStages) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) break;
                tc_commit(&tail->tfull[acc]);
            }
            // all tensor-core work of this CTA is complete once `drain` fires
            tc_commit(&tail->drain);
            mbar_wait_bounded(&tail->drain, 0u, nullptr, status, SITE_GEMM_DRAIN, limit);
        }
    } else {
        // ------------------------------------------------ epilogue (warps 2..5)
        const int wq = warp & 3;  // TMEM lane quarter this warp may access
        int it = 0;
        for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x, ++it) {
            const int acc = it & 1;
            const uint32_t aph = (it >> 1) & 1;
            const bool got = mbar_wait_bounded(&tail->tfull[acc], aph, abort_flag, status,
                                               SITE_GEMM_EPILOGUE, limit);
            // tcgen05.ld below is warp-collective: leave together or not at all
            if (!__all_sync(0xffffffffu, got)) break;
            tc_fence_after();
            const TileRef r = tile_ref(tile);
            const GemmArgs& args = r.p == 0 ? args0 : args1;
            const uint32_t taddr =
                tmem_base + (uint32_t)(acc * BNB) + ((uint32_t)(wq * 32) << 16);
            const int col0 = r.nt * args.out_col_step;

            if (sync_counter != nullptr && r.p == 1) {
                // the combine reads slot rows written by problem 0's epilogues in
                // other CTAs of this launch (all co-resident): wait until every
                // epilogue warp of every problem-0 tile has published
                bool ok = true;
                if (lane == 0) {
                    const int target = tiles0 * (kEpiThreads / 32);
                    const uint64_t t0 = globaltimer_ns();
                    while (ld_acquire(sync_counter) < target) {
                        if (*abort_flag || globaltimer_ns() - t0 > limit) {
                            ok = false;
                            *abort_flag = 1;
                            set_status(status, MOE_ERR_TIMEOUT, SITE_GEMM_EPILOGUE, 1);
                            break;
                        }
                        __nanosleep(256);
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                __syncwarp();
                if (!ok) break;
            }
            if (r.p == 0)
                epilogue_tile<EPI0>(tail->stage[wq], taddr, r, args0, lane, wq, col0);
            else
                epilogue_tile<EPI1>(tail->stage[wq], taddr, r, args1, lane, wq, col0);
            if (sync_counter != nullptr && r.p == 0) {
                // publish this warp's slot rows to the combine tiles of this launch
                __threadfence();
                __syncwarp();
                if (lane == 0) atomicAdd(sync_counter, 1);
            }
            tc_fence_before();
            mbar_arrive(&tail->tempty[acc]);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

// A kernel that waits on a barrier nothing signals, to exercise the bounded
// wait and the status report without hanging anything.
__global__ void selftest_timeout_kernel(int* status, unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0)
        mbar_wait_bounded(&bar, 0u, &abort_flag, status, SITE_SELFTEST, limit_ns);
}

}  // namespace

size_t gemm_tc_smem_bytes() { return kSmemBytes; }

cudaError_t launch_gemm_tc(int epi, const CUtensorMap& tmA0, const CUtensorMap& tmB0,
                           const GemmArgs& a0, const CUtensorMap* tmA1, const CUtensorMap* tmB1,
                           const GemmArgs* a1, int grid, cudaStream_t s, int* sync_counter) {
    using Kern = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap,
                          const CUtensorMap, const GemmArgs, const GemmArgs, int, int*);
    Kern kern = nullptr;
    switch (epi) {
        case EPI_SWIGLU: kern = grouped_gemm_tc_kernel<EPI_SWIGLU, EPI_SWIGLU>; break;
        case EPI_SCATTER: kern = grouped_gemm_tc_kernel<EPI_SCATTER, EPI_COMBINE>; break;
        case EPI_COMBINE: kern = grouped_gemm_tc_kernel<EPI_COMBINE, EPI_COMBINE>; break;
        default: return cudaErrorInvalidValue;
    }
    if (sync_counter != nullptr && (epi != EPI_SCATTER || a1 == nullptr))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    const int np = a1 != nullptr ? 2 : 1;
    const CUtensorMap& mA1 = np > 1 ? *tmA1 : tmA0;
    const CUtensorMap& mB1 = np > 1 ? *tmB1 : tmB0;
    const GemmArgs& g1 = np > 1 ? *a1 : a0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    // tiles of one launch wait on each other only through sync_counter; the
    // cooperative attribute guarantees every CTA of the grid is resident
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = sync_counter != nullptr ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, tmA0, tmB0, mA1, mB1, a0, g1, np, sync_counter);
}

cudaError_t launch_selftest_timeout(int* status, unsigned long long limit_ns, cudaStream_t s) {
    selftest_timeout_kernel<<<1, 32, 0, s>>>(status, limit_ns);
    return cudaGetLastError();
}

}  // namespace moe
