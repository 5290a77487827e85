// Permutation stage: per-expert histogram, prefix-sum scan, and a coalesced,
// vectorised scatter of token rows into an expert-contiguous layout, so the
// grouped GEMMs see each expert's tokens as one block of rows (the dispatch
// step between routing and the experts: tokens go only to their chosen
// experts, "开源混合架构大模型技术解析", section 四, and 七 item 3 on scheduling
// tokens that route to different experts).
//
// Layout produced: expert e owns rows [offsets[e], offsets[e+1]) of x_perm,
// a segment padded to a multiple of `align` rows (1 for the CTA-pair GEMMs of
// bf16 layers, 128 for the CUDA-core GEMMs of fp32 layers).  Inside a segment
// the real rows come first, in increasing token order (stable), then padding
// rows whose row_src is -1.  row_src[r] = t*k + j for the row holding slot j
// of token t.
//
// Two implementations give the same layout: the forward, the backward and
// the expert-parallel dispatch use one launch that derives the permutation
// from per-expert token bitmaps and copies the rows in the same kernel
// (perm_gather_small_kernel up to 1024 tokens, perm_gather_grid_kernel
// above); the histogram / scan / rank kernels serve the allocation-free
// counts and the sizes whose bitmaps would not fit in shared memory.
#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {

namespace {

constexpr int kWarps = kPermBlockTokens / 32;

// Load the k expert ids of token t (or -1s past T); out-of-range ids are
// recorded as a device error and treated as absent.
__device__ __forceinline__ void load_slots(const int32_t* __restrict__ idx, int t, int T, int k,
                                           int E, int (&my)[kMaxK], int* status) {
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
        int e = -1;
        if (j < k && t < T) {
            e = idx[(size_t)t * k + j];
            if (e < 0 || e >= E) {
                set_status(status, MOE_ERR_DEVICE, SITE_PERMUTE, e);
                e = -1;
            }
        }
        my[j] = e;
    }
}

__device__ __forceinline__ bool holds(const int (&my)[kMaxK], int e) {
    bool h = false;
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) h |= (my[j] == e);
    return h;
}

// Histogram of each block of 256 tokens: block_counts[b][e].  kCountIds
// false: tokens that hold expert e (a routing result names an expert at most
// once per token); true: occurrences of id e in the block's rows, so a row
// that repeats an id counts it as often as it appears.
template <bool kCountIds>
__global__ void __launch_bounds__(kPermBlockTokens) perm_count_kernel(
    const int32_t* __restrict__ idx, int T, int k, int E, int32_t* __restrict__ block_counts,
    int* status) {
    __shared__ int wcnt[kWarps][kMaxE];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int t = blockIdx.x * kPermBlockTokens + tid;
    pdl_wait();
    int my[kMaxK];
    load_slots(idx, t, T, k, E, my, status);
    for (int e = 0; e < E; ++e) {
        int c;
        if constexpr (kCountIds) {
            int m = 0;
#pragma unroll
            for (int j = 0; j < kMaxK; ++j) m += my[j] == e ? 1 : 0;
            c = __reduce_add_sync(0xffffffffu, m);
        } else {
            c = __popc(__ballot_sync(0xffffffffu, holds(my, e)));
        }
        if (lane == 0) wcnt[warp][e] = c;
    }
    __syncthreads();
    for (int e = tid; e < E; e += kPermBlockTokens) {
        int s = 0;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) s += wcnt[w][e];
        block_counts[(size_t)blockIdx.x * E + e] = s;
    }
    pdl_trigger();
}

// One CTA: per expert, exclusive scan of the block histogram over blocks
// (in place), total counts, 128-padded segment offsets, and row_src = -1 on
// the padding rows.  The histogram is staged through shared memory in
// coalesced chunks so the per-expert scans run on-chip.
constexpr int kScanChunkBlocks = 32;

__global__ void __launch_bounds__(1024) perm_scan_kernel(int32_t* __restrict__ block_counts,
                                                         int nb, int E, int align,
                                                         int32_t* __restrict__ counts,
                                                         int32_t* __restrict__ offsets,
                                                         int32_t* __restrict__ row_src,
                                                         int32_t* __restrict__ load_out) {
    __shared__ int s_bc[kScanChunkBlocks * kMaxE];
    __shared__ int s_cnt[kMaxE];
    __shared__ int s_off[kMaxE + 1];
    const int tid = threadIdx.x;
    pdl_wait();
    for (int e = tid; e < E; e += blockDim.x) s_cnt[e] = 0;
    for (int b0 = 0; b0 < nb; b0 += kScanChunkBlocks) {
        const int nbc = min(kScanChunkBlocks, nb - b0);
        __syncthreads();
        for (int i = tid; i < nbc * E; i += blockDim.x) s_bc[i] = block_counts[(size_t)b0 * E + i];
        __syncthreads();
        for (int e = tid; e < E; e += blockDim.x) {
            int run = s_cnt[e];
            for (int b = 0; b < nbc; ++b) {
                int c = s_bc[b * E + e];
                s_bc[b * E + e] = run;
                run += c;
            }
            s_cnt[e] = run;
        }
        __syncthreads();
        for (int i = tid; i < nbc * E; i += blockDim.x) block_counts[(size_t)b0 * E + i] = s_bc[i];
    }
    __syncthreads();
    if (tid < 32) {
        // warp scan of the padded segment sizes
        int carry = 0;
        for (int e0 = 0; e0 < E; e0 += 32) {
            const int e = e0 + tid;
            const int v = e < E ? (s_cnt[e] + align - 1) / align * align : 0;
            int incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                int n = __shfl_up_sync(0xffffffffu, incl, o);
                if (tid >= o) incl += n;
            }
            if (e < E) s_off[e] = carry + incl - v;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (tid == 0) s_off[E] = carry;
    }
    __syncthreads();
    for (int e = tid; e < E; e += blockDim.x) {
        counts[e] = s_cnt[e];
        if (load_out != nullptr) load_out[e] = s_cnt[e];
    }
    for (int e = tid; e <= E; e += blockDim.x) offsets[e] = s_off[e];
    for (int i = tid; i < E * align; i += blockDim.x) {
        int e = i / align, r = i % align;
        int row = s_off[e] + s_cnt[e] + r;
        if (row < s_off[e + 1]) row_src[row] = -1;
    }
    pdl_trigger();
}

// Stable rank of every (token, slot) inside its expert, and row_src of the
// destination row.
__global__ void __launch_bounds__(kPermBlockTokens) perm_rank_kernel(
    const int32_t* __restrict__ idx, int T, int k, int E,
    const int32_t* __restrict__ block_base, const int32_t* __restrict__ offsets,
    int32_t* __restrict__ row_src, int32_t* __restrict__ slot_row, int* status) {
    __shared__ int wbase[kWarps][kMaxE];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int t = blockIdx.x * kPermBlockTokens + tid;
    int my[kMaxK], rank[kMaxK];
    pdl_wait();
    load_slots(idx, t, T, k, E, my, nullptr);
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) rank[j] = 0;
    const unsigned lt = (1u << lane) - 1u;
    for (int e = 0; e < E; ++e) {
        unsigned b = __ballot_sync(0xffffffffu, holds(my, e));
        if (lane == 0) wbase[warp][e] = __popc(b);
#pragma unroll
        for (int j = 0; j < kMaxK; ++j)
            if (my[j] == e) rank[j] = __popc(b & lt);
    }
    __syncthreads();
    for (int e = tid; e < E; e += kPermBlockTokens) {
        int run = offsets[e] + block_base[(size_t)blockIdx.x * E + e];
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            int c = wbase[w][e];
            wbase[w][e] = run;
            run += c;
        }
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
        if (my[j] >= 0) {
            int pos = wbase[warp][my[j]] + rank[j];
            if (pos < offsets[my[j] + 1]) {
                row_src[pos] = t * k + j;
                if (slot_row != nullptr) slot_row[t * k + j] = pos;
            } else
                set_status(status, MOE_ERR_DEVICE, SITE_PERMUTE, pos);
        }
    }
    pdl_trigger();
}

// Largest batch of the one-launch permutation in which every CTA derives
// the whole permutation.
constexpr int kSmallTokens = 1024;
constexpr int kPermGatherThreads = 512;

// Copy token row t of x into row `row` of x_perm: one warp, 16-byte vectors,
// up to 8 per lane in flight.
__device__ __forceinline__ void copy_row_warp(const uint4* __restrict__ x, int vec_per_row, int t,
                                              uint4* __restrict__ x_perm, int row, int lane) {
    const uint4* src = x + (size_t)t * vec_per_row;
    uint4* dst = x_perm + (size_t)row * vec_per_row;
    for (int i0 = 0; i0 < vec_per_row; i0 += 8 * 32) {
        uint4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = i0 + u * 32 + lane;
            if (i < vec_per_row) v[u] = __ldg(src + i);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = i0 + u * 32 + lane;
            if (i < vec_per_row) dst[i] = v[u];
        }
    }
}

// Small batches (T <= 1024) in one launch of several CTAs: every CTA derives
// the whole permutation from the routing result on chip, CTA 0 writes it out
// (counts, offsets, row_src, padding rows, slot_row), and all CTAs copy token
// rows into x_perm (kRows) and gate weights into w_dst (kWeights), one warp
// per (token, slot).  Same layout and order as the kernels above; a routing
// result names an expert at most once per token.
//
// Stable ranks come from a bitmap per expert over the tokens: bit t of
// bits[e] is set when token t chose e, so the rank of token t inside
// segment e is the number of set bits below t -- a per-word prefix count plus
// one masked popcount, independent of E.
template <bool kRows, bool kWeights>
__global__ void __launch_bounds__(kPermGatherThreads) perm_gather_small_kernel(
    const int32_t* __restrict__ idx, int T, int k, int E, int align,
    int32_t* __restrict__ counts, int32_t* __restrict__ offsets, int32_t* __restrict__ row_src,
    int32_t* __restrict__ load_out, int32_t* __restrict__ slot_row, int* status,
    const uint4* __restrict__ x, int vec_per_row, uint4* __restrict__ x_perm,
    const float* __restrict__ w_src, float* __restrict__ w_dst) {
    extern __shared__ __align__(16) uint32_t pg_sm[];
    const int W = (T + 31) >> 5;  // bitmap words per expert
    uint32_t* bits = pg_sm;                                     // [E][W]
    int* pre = reinterpret_cast<int*>(bits + (size_t)E * W);    // [E][W] bits below word w
    int* s_cnt = pre + (size_t)E * W;                           // [E]
    int* s_off = s_cnt + E;                                     // [E + 1]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nwarps = blockDim.x >> 5;
    const int n_slots = T * k;
    const bool writer = blockIdx.x == 0;
    for (int i = tid; i < E * W; i += blockDim.x) bits[i] = 0u;
    pdl_wait();
    __syncthreads();
    for (int s = tid; s < n_slots; s += blockDim.x) {
        const int e = idx[s];
        if (e < 0 || e >= E) {
            if (writer) set_status(status, MOE_ERR_DEVICE, SITE_PERMUTE, e);
            continue;
        }
        const int t = s / k;
        atomicOr(&bits[e * W + (t >> 5)], 1u << (t & 31));
    }
    __syncthreads();
    // per expert (one warp each): exclusive prefix of the word popcounts
    for (int e = warp; e < E; e += nwarps) {
        const int v = lane < W ? __popc(bits[e * W + lane]) : 0;
        int incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += n;
        }
        if (lane < W) pre[e * W + lane] = incl - v;
        if (lane == 31) s_cnt[e] = incl;
    }
    __syncthreads();
    if (warp == 0) {  // segment offsets: exclusive scan of the padded sizes
        int carry = 0;
        for (int e0 = 0; e0 < E; e0 += 32) {
            const int e = e0 + lane;
            const int v = e < E ? (s_cnt[e] + align - 1) / align * align : 0;
            int incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int n = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += n;
            }
            if (e < E) s_off[e] = carry + incl - v;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) s_off[E] = carry;
    }
    __syncthreads();
    // row of slot s (token t, expert e): segment start + stable rank
    auto row_of = [&](int e, int t) {
        const int w = t >> 5;
        return s_off[e] + pre[e * W + w] + __popc(bits[e * W + w] & ((1u << (t & 31)) - 1u));
    };
    if (writer) {
        for (int e = tid; e < E; e += blockDim.x) {
            counts[e] = s_cnt[e];
            if (load_out != nullptr) load_out[e] = s_cnt[e];
        }
        for (int e = tid; e <= E; e += blockDim.x) offsets[e] = s_off[e];
        if (align > 1)
            for (int i = tid; i < E * align; i += blockDim.x) {
                const int e = i / align, r = i % align;
                const int row = s_off[e] + s_cnt[e] + r;
                if (row < s_off[e + 1]) row_src[row] = -1;
            }
        for (int s = tid; s < n_slots; s += blockDim.x) {
            const int e = idx[s];
            if (e < 0 || e >= E) continue;
            const int pos = row_of(e, s / k);
            row_src[pos] = s;
            if (slot_row != nullptr) slot_row[s] = pos;
        }
    }
    // the row copies (kRows) and gate weights (kWeights): one warp per slot
    if constexpr (kRows || kWeights) {
        const int gw = blockIdx.x * nwarps + warp, nw = gridDim.x * nwarps;
        for (int s = gw; s < n_slots; s += nw) {
            const int e = idx[s];
            if (e < 0 || e >= E) continue;
            const int t = s / k;
            const int row = row_of(e, t);
            if constexpr (kWeights) {
                if (lane == 0) w_dst[row] = w_src[s];
            }
            if constexpr (kRows) copy_row_warp(x, vec_per_row, t, x_perm, row, lane);
        }
    }
    pdl_trigger();
}

// Larger batches in one launch: CTA b owns tokens [b TB, (b+1) TB) (TB a
// multiple of 32, one CTA per SM at most, all resident together).
//   1. per-expert bitmaps of its tokens, the per-word prefix counts and its
//      per-expert counts, published in block_counts[b][e];
//   2. a grid-wide barrier (an arrival counter in the status region, reset
//      by the routing kernel; the wait is bounded and reports
//      MOE_ERR_TIMEOUT, after which every CTA that gives up, or sees that
//      another gave up, leaves zero counts and offsets behind);
//   3. every CTA sums the published counts: totals (-> segment offsets) and
//      the counts of the CTAs before it (-> its base inside each segment);
//      CTA 0 writes counts, offsets, padding rows; each CTA writes row_src
//      (and slot_row) of its slots and copies its tokens' rows into x_perm
//      (kRows) and their gate weights into w_dst (kWeights).
// Same layout and stable order as the histogram / scan / rank kernels; the k
// ids of a token are distinct.
template <bool kRows, bool kWeights>
__global__ void __launch_bounds__(kPermGatherThreads) perm_gather_grid_kernel(
    const int32_t* __restrict__ idx, int T, int k, int E, int align, int TB,
    int32_t* __restrict__ block_counts, int32_t* __restrict__ counts,
    int32_t* __restrict__ offsets, int32_t* __restrict__ row_src, int32_t* __restrict__ load_out,
    int32_t* __restrict__ slot_row, int* status, int* grid_bar, unsigned long long wait_limit_ns,
    const uint4* __restrict__ x, int vec_per_row, uint4* __restrict__ x_perm,
    const float* __restrict__ w_src, float* __restrict__ w_dst) {
    extern __shared__ __align__(16) uint32_t pg_sm[];
    const int W = TB >> 5;
    uint32_t* bits = pg_sm;                                   // [E][W]
    int* pre = reinterpret_cast<int*>(bits + (size_t)E * W);  // [E][W]
    int* s_cnt = pre + (size_t)E * W;                         // [E] this CTA's counts
    int* s_tot = s_cnt + E;                                   // [E] all CTAs
    int* s_base = s_tot + E;                                  // [E] CTAs before this one
    int* s_off = s_base + E;                                  // [E + 1]
    __shared__ int s_abort;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nwarps = blockDim.x >> 5;
    const int P = gridDim.x, b = blockIdx.x;
    const int t0 = b * TB, t1 = min(T, t0 + TB);
    const int s0 = t0 * k, s1 = t1 * k;
    const bool writer = b == 0;
    for (int i = tid; i < E * W; i += blockDim.x) bits[i] = 0u;
    for (int e = tid; e < E; e += blockDim.x) {
        s_tot[e] = 0;
        s_base[e] = 0;
    }
    if (tid == 0) s_abort = 0;
    pdl_wait();
    __syncthreads();
    for (int s = s0 + tid; s < s1; s += blockDim.x) {
        const int e = idx[s];
        if (e < 0 || e >= E) {
            set_status(status, MOE_ERR_DEVICE, SITE_PERMUTE, e);
            continue;
        }
        const int t = s / k - t0;
        atomicOr(&bits[e * W + (t >> 5)], 1u << (t & 31));
    }
    __syncthreads();
    for (int e = warp; e < E; e += nwarps) {
        int carry = 0;
        for (int w0 = 0; w0 < W; w0 += 32) {
            const int w = w0 + lane;
            const int v = w < W ? __popc(bits[e * W + w]) : 0;
            int incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int n = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += n;
            }
            if (w < W) pre[e * W + w] = carry + incl - v;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) {
            s_cnt[e] = carry;
            block_counts[(size_t)b * E + e] = carry;
        }
    }
    // grid-wide barrier: every CTA's counts are published
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        atomicAdd(grid_bar, 1);
        const unsigned long long c0 = clock64();
        while (*reinterpret_cast<volatile int*>(grid_bar) < P) {
            if ((unsigned long long)(clock64() - c0) > 2ull * wait_limit_ns) {
                set_status(status, MOE_ERR_TIMEOUT, SITE_PERMUTE, b);
                s_abort = 1;
                break;
            }
            __nanosleep(64);
        }
        __threadfence();
        // a CTA that gave up has recorded MOE_ERR_TIMEOUT before the last
        // arrival could let the others pass: they see it here and give up too
        if (*reinterpret_cast<volatile int*>(status) == MOE_ERR_TIMEOUT) s_abort = 1;
    }
    __syncthreads();
    if (s_abort) {
        // no segment then: the GEMMs see zero routed rows (never a row_src
        // entry this launch did not write)
        for (int e = tid; e <= E; e += blockDim.x) {
            if (e < E) counts[e] = 0;
            offsets[e] = 0;
        }
        return;
    }
    // totals and this CTA's base: column sums of block_counts, split over
    // the threads (parts of the CTA list per expert), combined with integer
    // atomics (order-independent)
    {
        const int parts = max(1, (int)blockDim.x / E);
        const int e = tid % E, part = tid / E;
        if (part < parts) {
            int tot = 0, base = 0;
            for (int q = part; q < P; q += parts) {
                const int c = __ldcg(block_counts + (size_t)q * E + e);
                tot += c;
                if (q < b) base += c;
            }
            atomicAdd(&s_tot[e], tot);
            atomicAdd(&s_base[e], base);
        }
    }
    __syncthreads();
    if (warp == 0) {  // segment offsets: exclusive scan of the padded totals
        int carry = 0;
        for (int e0 = 0; e0 < E; e0 += 32) {
            const int e = e0 + lane;
            const int v = e < E ? (s_tot[e] + align - 1) / align * align : 0;
            int incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int n = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += n;
            }
            if (e < E) s_off[e] = carry + incl - v;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) s_off[E] = carry;
    }
    __syncthreads();
    auto row_of = [&](int e, int t) {  // t relative to t0
        const int w = t >> 5;
        return s_off[e] + s_base[e] + pre[e * W + w] +
               __popc(bits[e * W + w] & ((1u << (t & 31)) - 1u));
    };
    if (writer) {
        for (int e = tid; e < E; e += blockDim.x) {
            counts[e] = s_tot[e];
            if (load_out != nullptr) load_out[e] = s_tot[e];
        }
        for (int e = tid; e <= E; e += blockDim.x) offsets[e] = s_off[e];
        if (align > 1)
            for (int i = tid; i < E * align; i += blockDim.x) {
                const int e = i / align, r = i % align;
                const int row = s_off[e] + s_tot[e] + r;
                if (row < s_off[e + 1]) row_src[row] = -1;
            }
    }
    for (int s = s0 + tid; s < s1; s += blockDim.x) {
        const int e = idx[s];
        if (e < 0 || e >= E) continue;
        const int pos = row_of(e, s / k - t0);
        row_src[pos] = s;
        if (slot_row != nullptr) slot_row[s] = pos;
    }
    if constexpr (kRows || kWeights) {
        for (int s = s0 + warp; s < s1; s += nwarps) {
            const int e = idx[s];
            if (e < 0 || e >= E) continue;
            const int t = s / k;
            const int row = row_of(e, t - t0);
            if constexpr (kWeights) {
                if (lane == 0) w_dst[row] = w_src[s];
            }
            if constexpr (kRows) copy_row_warp(x, vec_per_row, t, x_perm, row, lane);
        }
    }
    pdl_trigger();
}

// x_perm[r] = x[row_src[r] / k] for every real row r < offsets[E]; one warp
// per row, 16-byte vectors, up to 8 vectors per lane loaded before any store
// so each lane keeps 8 loads in flight.  With w_dst, also w_dst[r] =
// w_src[row_src[r]] (the gate weight of the row's slot).
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint4* __restrict__ x,
                                                          int vec_per_row, int k,
                                                          const int32_t* __restrict__ total_rows,
                                                          const int32_t* __restrict__ row_src,
                                                          uint4* __restrict__ x_perm,
                                                          const float* __restrict__ w_src,
                                                          float* __restrict__ w_dst) {
    const int lane = threadIdx.x & 31;
    const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int nw = (gridDim.x * blockDim.x) >> 5;
    pdl_wait();
    const int total = *total_rows;
    for (int r = gw; r < total; r += nw) {
        const int src = row_src[r];
        if (src < 0) continue;
        if (w_dst != nullptr && lane == 0) w_dst[r] = w_src[src];
        const uint4* s = x + (size_t)(src / k) * vec_per_row;
        uint4* dst = x_perm + (size_t)r * vec_per_row;
        for (int i0 = 0; i0 < vec_per_row; i0 += 8 * 32) {
            uint4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int i = i0 + u * 32 + lane;
                if (i < vec_per_row) v[u] = __ldg(s + i);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int i = i0 + u * 32 + lane;
                if (i < vec_per_row) dst[i] = v[u];
            }
        }
    }
    pdl_trigger();
}

// y[t] = base[t] + slots[t*k + 0] + ... + slots[t*k + k-1] in fp32, in that
// order (base = shared-expert output, or none).  8 columns per thread: whole
// slot rows are read with 16-byte loads (bf16) or 2 x 16-byte loads (fp32),
// every slot load of a thread issued before the ordered sum.
template <typename TS>
__global__ void __launch_bounds__(256) combine_slots_kernel(const TS* __restrict__ slots,
                                                            const float* __restrict__ base,
                                                            int T, int d8, int k, void* y,
                                                            int out_f32) {
    const size_t n = (size_t)T * d8;
    pdl_wait();
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
         i += (size_t)gridDim.x * blockDim.x) {
        const size_t t = i / d8, c = (i % d8) * 8;
        const size_t d = (size_t)d8 * 8;
        float a[8];
        if (base != nullptr) {
            const float4 b0 = __ldcs(reinterpret_cast<const float4*>(base + t * d + c));
            const float4 b1 = __ldcs(reinterpret_cast<const float4*>(base + t * d + c) + 1);
            a[0] = b0.x; a[1] = b0.y; a[2] = b0.z; a[3] = b0.w;
            a[4] = b1.x; a[5] = b1.y; a[6] = b1.z; a[7] = b1.w;
        } else {
#pragma unroll
            for (int q = 0; q < 8; ++q) a[q] = 0.f;
        }
        float sv[kMaxK][8];
#pragma unroll
        for (int j = 0; j < kMaxK; ++j) {
            if (j < k) {
                const TS* p = slots + (t * k + j) * d + c;
                if constexpr (sizeof(TS) == 2) {
                    const uint4 u = __ldcs(reinterpret_cast<const uint4*>(p));
                    const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        sv[j][2 * h] = __uint_as_float(w4[h] << 16);
                        sv[j][2 * h + 1] = __uint_as_float(w4[h] & 0xffff0000u);
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < 8; ++q) sv[j][q] = Elem<TS>::to_f(p[q]);
                }
            }
        }
#pragma unroll
        for (int j = 0; j < kMaxK; ++j) {
            if (j >= k) break;
#pragma unroll
            for (int q = 0; q < 8; ++q) a[q] += sv[j][q];
        }
        if (out_f32) {
            float4* o = reinterpret_cast<float4*>(static_cast<float*>(y) + t * d + c);
            o[0] = make_float4(a[0], a[1], a[2], a[3]);
            o[1] = make_float4(a[4], a[5], a[6], a[7]);
        } else {
            *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(y) + t * d + c) =
                make_uint4(pack_bf16x2(a[0], a[1]), pack_bf16x2(a[2], a[3]),
                           pack_bf16x2(a[4], a[5]), pack_bf16x2(a[6], a[7]));
        }
    }
    pdl_trigger();
}

// bf16 slots, k fixed at compile time: one thread per (token, 8 columns), its
// k slot loads (16 B each) and the base loads all issued before the ordered
// sum; nothing is held beyond the raw loads, so a full SM of threads keeps
// enough bytes in flight to stream at HBM speed.
template <int K>
__global__ void __launch_bounds__(256) combine_slots_bf16_kernel(
    const uint4* __restrict__ slots, const float4* __restrict__ base, int T, int d8, void* y,
    int out_f32) {
    const size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
    pdl_wait();
    if (i >= (size_t)T * d8) return;
    const size_t t = i / d8, c8 = i % d8;
    uint4 raw[K];
#pragma unroll
    for (int j = 0; j < K; ++j) raw[j] = __ldcs(slots + (t * K + j) * d8 + c8);
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

}  // namespace

cudaError_t launch_permute(const int32_t* idx, int T, int k, int E, int32_t* block_counts,
                           int32_t* counts, int32_t* offsets, int32_t* row_src, int align,
                           int32_t* load_out, int* status, cudaStream_t s, int32_t* slot_row) {
    const int nb = (T + kPermBlockTokens - 1) / kPermBlockTokens;
    cudaError_t e = launch_pdl(perm_count_kernel<false>, dim3(nb), dim3(kPermBlockTokens), 0, s,
                               1, idx, T, k, E, block_counts, status);
    if (e != cudaSuccess) return e;
    e = launch_pdl(perm_scan_kernel, dim3(1), dim3(1024), 0, s, 1, block_counts, nb, E, align,
                   counts, offsets, row_src, load_out);
    if (e != cudaSuccess) return e;
    return launch_pdl(perm_rank_kernel, dim3(nb), dim3(kPermBlockTokens), 0, s, 1, idx, T, k, E,
                      static_cast<const int32_t*>(block_counts),
                      static_cast<const int32_t*>(offsets), row_src, slot_row, status);
}

cudaError_t launch_permute_gather_small(const int32_t* idx, int T, int k, int E, int align,
                                       int32_t* counts, int32_t* offsets, int32_t* row_src,
                                       int32_t* load_out, int* status, const void* x, int d,
                                       int elem_bytes, void* x_perm, int num_sms,
                                       cudaStream_t s, int32_t* slot_row, const float* w_src,
                                       float* w_dst) {
    if (T > kSmallTokens || T < 1) return cudaErrorInvalidValue;
    const int W = (T + 31) / 32;
    const size_t smem = (size_t)E * W * 8 + (size_t)(2 * E + 1) * 4;
    auto kern = x != nullptr ? (w_dst != nullptr ? perm_gather_small_kernel<true, true>
                                                 : perm_gather_small_kernel<true, false>)
                             : (w_dst != nullptr ? perm_gather_small_kernel<false, true>
                                                 : perm_gather_small_kernel<false, false>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const int warps_per_cta = kPermGatherThreads / 32;
    int blocks = (T * k + warps_per_cta - 1) / warps_per_cta;
    if (blocks > num_sms) blocks = num_sms;
    if (blocks < 1 || (x == nullptr && w_dst == nullptr)) blocks = 1;
    return launch_pdl(kern, dim3((unsigned)blocks), dim3(kPermGatherThreads), smem, s, 1, idx, T,
                      k, E, align, counts, offsets, row_src, load_out, slot_row, status,
                      static_cast<const uint4*>(x), x != nullptr ? d * elem_bytes / 16 : 0,
                      static_cast<uint4*>(x_perm), w_src, w_dst);
}

bool permute_gather_grid_fits(int T, int E, int num_sms) {
    if (T < 1 || num_sms < 1) return false;
    int P = (T + 31) / 32;
    if (P > num_sms) P = num_sms;
    const int TB = ((T + P - 1) / P + 31) / 32 * 32;
    const size_t smem = (size_t)E * (TB / 32) * 8 + (size_t)(4 * E + 1) * 4;
    return smem <= kPermGatherGridMaxSmem;
}

cudaError_t launch_permute_gather_grid(const int32_t* idx, int T, int k, int E, int align,
                                      int32_t* block_counts, int32_t* counts, int32_t* offsets,
                                      int32_t* row_src, int32_t* load_out, int* status,
                                      int* grid_bar, unsigned long long wait_limit_ns,
                                      const void* x, int d, int elem_bytes, void* x_perm,
                                      int num_sms, cudaStream_t s, int32_t* slot_row,
                                      const float* w_src, float* w_dst) {
    if (!permute_gather_grid_fits(T, E, num_sms)) return cudaErrorInvalidValue;
    int P = (T + 31) / 32;
    if (P > num_sms) P = num_sms;
    const int TB = ((T + P - 1) / P + 31) / 32 * 32;
    P = (T + TB - 1) / TB;
    const size_t smem = (size_t)E * (TB / 32) * 8 + (size_t)(4 * E + 1) * 4;
    auto kern = x != nullptr ? (w_dst != nullptr ? perm_gather_grid_kernel<true, true>
                                                 : perm_gather_grid_kernel<true, false>)
                             : (w_dst != nullptr ? perm_gather_grid_kernel<false, true>
                                                 : perm_gather_grid_kernel<false, false>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, dim3((unsigned)P), dim3(kPermGatherThreads), smem,
                      s, 1, idx, T, k, E, align, TB, block_counts, counts, offsets, row_src,
                      load_out, slot_row, status, grid_bar, wait_limit_ns,
                      static_cast<const uint4*>(x), x != nullptr ? d * elem_bytes / 16 : 0,
                      static_cast<uint4*>(x_perm), w_src, w_dst);
}

cudaError_t launch_expert_counts(const int32_t* idx, int T, int k, int E,
                                 int32_t* block_counts, int32_t* counts, int32_t* offsets,
                                 cudaStream_t s) {
    const int nb = (T + kPermBlockTokens - 1) / kPermBlockTokens;
    if (nb > 0)
        perm_count_kernel<true><<<nb, kPermBlockTokens, 0, s>>>(idx, T, k, E, block_counts,
                                                                nullptr);
    // align 1: no padding rows, so the scan writes no row_src entry
    perm_scan_kernel<<<1, 1024, 0, s>>>(block_counts, nb, E, 1, counts, offsets, nullptr, nullptr);
    return cudaGetLastError();
}

cudaError_t launch_gather_rows(const void* x, int d, int elem_bytes, int k,
                               const int32_t* offsets_total, const int32_t* row_src,
                               int rows_cap, void* x_perm, int num_sms, cudaStream_t s,
                               const float* w_src, float* w_dst) {
    const int vec = d * elem_bytes / 16;
    int blocks = num_sms * 8;
    const int need = (rows_cap + 7) / 8;
    if (blocks > need) blocks = need > 0 ? need : 1;
    return launch_pdl(gather_rows_kernel, dim3(blocks), dim3(256), 0, s, 1,
                      static_cast<const uint4*>(x), vec, k, offsets_total, row_src,
                      static_cast<uint4*>(x_perm), w_src, w_dst);
}

cudaError_t launch_combine_slots(const void* slots, int slots_bf16, const float* base, int T,
                                 int d, int k, void* y, int out_f32, cudaStream_t s) {
    const int d8 = d / 8;
    const size_t n = (size_t)T * d8;
    if (slots_bf16) {
        if (n == 0) return cudaSuccess;
        const unsigned blocks16 = (unsigned)((n + 255) / 256);
        const uint4* sl = static_cast<const uint4*>(slots);
        const float4* b4 = reinterpret_cast<const float4*>(base);
        switch (k) {
#define MOE_COMBINE_K(KK)                                                                 \
    case KK:                                                                              \
        return launch_pdl(combine_slots_bf16_kernel<KK>, dim3(blocks16), dim3(256), 0, s, 1, \
                          sl, b4, T, d8, y, out_f32);
            MOE_COMBINE_K(1) MOE_COMBINE_K(2) MOE_COMBINE_K(3) MOE_COMBINE_K(4)
            MOE_COMBINE_K(5) MOE_COMBINE_K(6) MOE_COMBINE_K(7) MOE_COMBINE_K(8)
#undef MOE_COMBINE_K
            default: return cudaErrorInvalidValue;
        }
    }
    int blocks = (int)((n + 255) / 256);
    if (blocks > 148 * 8) blocks = 148 * 8;
    if (blocks < 1) blocks = 1;
    return launch_pdl(combine_slots_kernel<float>, dim3(blocks), dim3(256), 0, s, 1,
                      static_cast<const float*>(slots), base, T, d8, k, y, out_f32);
}

}  // namespace moe
