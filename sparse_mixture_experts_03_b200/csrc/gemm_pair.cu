// Grouped GEMM in "weights x tokens" orientation on CTA pairs (tcgen05
// cta_group::2, sm_100a).
//
// Each expert GEMM out[t, f] = sum_c act[t, c] * W[f, c] is computed as
// D[f, t] = W[f, :] . act[t, :]: the expert's weight rows are the MMA's M
// operand (256 rows per CTA pair, 128 per CTA) and the expert's tokens are
// the N operand (up to 256 per tile, any multiple of 16).  A ragged expert
// therefore costs at most 15 padding columns, not a 128-row tile, and a
// decode-sized batch (a few tokens per expert) becomes a stream of weight
// tiles with a thin N.  The pair splits the weight rows (A) and the token
// rows (B) between its two CTAs; each CTA loads only its own halves with TMA
// into its own shared memory (no multicast).  A pipeline stage covers 128 of
// K: 32 KiB of weights and N/2 token rows per CTA; the ring has 3 stages of
// 64 KiB, or 4 / 5 smaller ones when the batch bounds N by 128 / 64.
//
// Roles (both CTAs, 7 warps each): warps 0 (weights) and 6 (tokens) issue
// one TMA copy each per stage; a stage's full barrier lives in the pair's
// first CTA (the MMA issuer) and receives the transaction bytes of both
// CTAs' copies; warp 1 lane 0 of the first CTA issues tcgen05.mma.cta_group::2
// and frees the stage in both CTAs with one multicast commit; warps 2..5 of
// each CTA read their 32 TMEM lanes (= weight rows) x N columns (= tokens),
// transpose through shared memory and store token-major rows.  Tiles are
// handed out dynamically (a ticket counter, and a ring of decoded tiles that
// every role of the pair reads).
//
// Epilogues:
//   SWIGLU  each warp's 32 weight rows are 16 gate rows and the 16 matching
//           up rows (the gate/up tensor map interleaves them per 16 rows), so
//           h = silu(gate) * up is formed per warp (SwiGLU: "大模型工程（一）：
//           Transformer 到 MoE", section "变了什么，为什么变", item 3) and
//           written as bf16 h[token][feature].
//   SCATTER routed down projection: the row of token column t goes to slot
//           row_src[b_row + t], scaled by its gate weight, stored bf16 (the
//           weighted combine of the MoEBlock listing, section "混合专家：更多
//           参数，相同 FLOPs").
//   STORE_F32 shared down projection, fp32 rows; the final sum
//           y = shared + slot_0 + ... + slot_{k-1} (fixed order) is a separate
//           streaming kernel that reads whole slot rows.
// Every wait is bounded (status word + early exit, never a trap).
#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {

namespace {

constexpr int kAtoms = 2;                        // 128-byte swizzle atoms (64 bf16 of K) per stage
constexpr int kBK = 64 * kAtoms;                 // K per stage
constexpr int kARows = 128;                      // weight rows per CTA (MMA M = 256 per pair)
constexpr int kABytes = kARows * kBK * 2;        // 32 KiB: 2 atoms x 128 weight rows
constexpr int kMaxStages = 6;
constexpr int kAtomBytesA = kARows * 128;        // 16 KiB between the atoms of a tile
constexpr int kNTile = 256;                      // tokens per tile
// The weight producer of the gate/up launch brings the k-block this many
// steps ahead of its current load into L2 (a tile's first touch of a weight
// tile comes from HBM; the ring holds too few bytes to cover that latency)
constexpr int kPrefetchAhead = 2;
constexpr int kTmemCols = 512;                   // 2 accumulators x 256 fp32 columns
constexpr int kThreads = 224;                    // 7 warps: producers 0 and 6, MMA 1, epilogue 2..5
constexpr int kBProducerWarp = 6;
constexpr int kEpiWarps = 4;
constexpr int kMaxGroupsP = kMaxE + 1;
// Tile ids reach every role of a pair through a ring in shared memory, filled
// by CTA 0's weight producer from a global ticket counter (dynamic scheduling:
// a pair takes its next tile when its producer is ready for one).
constexpr int kSchedDepth = 8;
// readers of each ring entry: in CTA 0 the token producer, the MMA issuer and
// the 4 epilogue warps; in CTA 1 both producers and the 4 epilogue warps
constexpr int kSchedReaders = 2 * (2 + kEpiWarps);
// bound of the producers' drain of issued copies when a launch gives up early
constexpr uint64_t kAbortDrainNs = 1000000;  // 1 ms

// One tile of a launch, decoded once by the scheduler and passed through the
// ring as two 16-byte words.
struct __align__(16) Tile {
    int p;       // problem
    int g;       // group (expert)
    int ft;      // feature tile
    int b_row;   // first token row of the tile in the B tensor
    int n_real;  // tokens in the tile (1..256)
    int n;       // MMA N: n_real rounded up to 16
    int end;     // 1: no more tiles for this pair
    int aux;     // KIND_WGRAD: N tile | k-blocks << 16 (b_row is then the first K row)
};

struct __align__(16) PairTail {
    uint4 stage[kEpiWarps * 256];  // per epilogue warp: 32 rows x 128 B staging
    uint64_t full[kMaxStages];
    uint64_t empty[kMaxStages];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint64_t drain;
    uint64_t sched_full[kSchedDepth];   // one arrive from the scheduler per entry
    uint64_t sched_empty[kSchedDepth];  // used in CTA 0: kSchedReaders arrives per entry
    Tile sched_tile[kSchedDepth];
    uint32_t tmem_base;
    int abort;
    int seg_off[2][kMaxGroupsP];   // first token row of each group
    int tile_off[2][kMaxGroupsP];  // first tile of each group
    int cnt[2][kMaxGroupsP];       // token rows of each group
    int useg_off[2][kMaxGroupsP];  // first row of each group with unpadded segments
};

// Load-ring shapes.  A stage holds the weight tile (32 KiB) and up to BMAX
// token rows per CTA (tiles of N <= 2 BMAX tokens); smaller token tiles leave
// room for more stages in flight.
template <int STAGES, int BMAX>
struct Ring {
    static constexpr int kStages = STAGES;
    static constexpr int kBMaxRows = BMAX;
    static constexpr int kBBytes = BMAX * kBK * 2;
    static constexpr int kStageBytes = kABytes + kBBytes;
    static constexpr size_t kSmemBytes = 1024 + (size_t)STAGES * kStageBytes + sizeof(PairTail);
    static_assert(STAGES <= kMaxStages, "stages");
    static_assert(kStageBytes % 1024 == 0, "stages stay 1024-byte aligned (128B swizzle)");
    static_assert(kSmemBytes <= 232448, "shared memory per CTA");
};
using WideRing = Ring<3, 128>;   // tiles of up to 256 tokens: 3 stages of 64 KiB
using MidRing = Ring<4, 64>;     // tiles of up to 128 tokens: 4 stages of 48 KiB
using NarrowRing = Ring<5, 32>;  // tiles of up to 64 tokens: 5 stages of 40 KiB

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// shared::cluster address of the same shared variable in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t map_to_rank(const void* p, uint32_t rank) {
    uint32_t out;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(smem_u32(p)), "r"(rank));
    return out;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
                 ::: "memory");
}
// AND of `ok` over the 4 epilogue warps (also a barrier among them)
__device__ __forceinline__ bool epi_all(bool ok) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred q, o;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.and.pred o, 1, %2, q;\n\t"
        "selp.u32 %0, 1, 0, o;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)ok), "n"(kEpiWarps * 32)
        : "memory");
    return r != 0;
}
// TMA 3-D tile load {64 columns, rows, k-atoms} whose completion is reported
// to an mbarrier of either CTA of the pair (shared::cluster address), no
// multicast.
__device__ __forceinline__ void tma_load_3d_pair(void* smem_dst, const CUtensorMap* map,
                                                 uint32_t bar_cluster, int c0, int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}
// 5-D variant (weights with gate/up interleaving, see PairArgs::a_mode).
__device__ __forceinline__ void tma_load_5d_pair(void* smem_dst, const CUtensorMap* map,
                                                 uint32_t bar_cluster, int c0, int c1, int c2,
                                                 int c3, int c4) {
    asm volatile(
        "cp.async.bulk.tensor.5d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2),
        "r"(c3), "r"(c4)
        : "memory");
}
// L2 prefetch of the box of a tensor map at these coordinates (no shared
// memory written, no completion to wait for).
__device__ __forceinline__ void tma_prefetch_l2_3d(const CUtensorMap* map, int c0, int c1,
                                                   int c2) {
    asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(c0), "r"(c1), "r"(c2)
                 : "memory");
}
__device__ __forceinline__ void tma_prefetch_l2_5d(const CUtensorMap* map, int c0, int c1, int c2,
                                                   int c3, int c4) {
    asm volatile(
        "cp.async.bulk.prefetch.tensor.5d.L2.global.tile [%0, {%1, %2, %3, %4, %5}];" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4)
        : "memory");
}
__device__ __forceinline__ void arrive_expect_tx_local(uint64_t* bar, uint32_t bytes) {
    mbar_arrive_expect_tx(bar, bytes);
}
// The 4 MMAs (K = 16 each) of one 64-deep k-block: descriptors of step kk
// are the base descriptors + AS kk / BS kk (a K-major operand: 2 = 32 bytes
// further along the swizzled rows; an MN-major one: 128 = 16 rows of 128 B
// further); the first accumulates into D only if `accumulate`, the rest
// always do.
template <uint64_t AS = 2, uint64_t BS = 2>
__device__ __forceinline__ void tc_mma4_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "setp.eq.b32 q, %3, %3;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %5, %6, %3, q;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %7, %8, %3, q;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %9, %10, %3, q;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "l"(a_desc + AS), "l"(b_desc + BS),
        "l"(a_desc + 2 * AS), "l"(b_desc + 2 * BS), "l"(a_desc + 3 * AS), "l"(b_desc + 3 * BS)
        : "memory");
}
// arrive (once) on the mbarrier at shared::cluster address `bar` when all
// previously issued tcgen05 operations of this thread have completed
__device__ __forceinline__ void tc_commit_pair(uint32_t bar_cluster) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     bar_cluster)
                 : "memory");
}
// Arrive on the barrier at this shared address in both CTAs of the pair once
// the tcgen05 ops issued so far are complete (one commit, CTA mask 0b11).
__device__ __forceinline__ void tc_commit_both(uint32_t bar_local) {
    asm volatile(
        "{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], m;\n\t}" ::"r"(bar_local)
        : "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster)
                 : "memory");
}
// The same arrive without release semantics (orders no earlier memory access).
__device__ __forceinline__ void mbar_arrive_cluster_relaxed(uint32_t bar_cluster) {
    asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster)
                 : "memory");
}

// Wait for phase `parity` of a local barrier whose arrivals may come from the
// other CTA of the pair (acquire at cluster scope), bounded like
// mbar_wait_bounded.
__device__ __forceinline__ bool mbar_try_wait_cl(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return done != 0;
}
__device__ __forceinline__ bool mbar_wait_cl(uint64_t* bar, uint32_t parity, volatile int* abort,
                                             int* status, int site, uint64_t limit_ns) {
    if (mbar_try_wait_cl(bar, parity)) return true;
    const uint64_t t0 = clock64();
    const uint64_t limit_cycles = limit_ns * 2;
    for (;;) {
#pragma unroll 1
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait_cl(bar, parity)) return true;
        if (abort != nullptr && *abort) return false;
        if ((uint64_t)clock64() - t0 > limit_cycles) {
            if (abort != nullptr) *abort = 1;
            set_status(status, MOE_ERR_TIMEOUT, site);
            return false;
        }
    }
}

__device__ __forceinline__ void st_cluster_v4(uint32_t addr, const int4& v) {
    asm volatile("st.shared::cluster.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x),
                 "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}
__device__ __forceinline__ int4 ld_shared_v4(const void* p) {
    int4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(smem_u32(p))
                 : "memory");
    return v;
}

// Scheduler side of the tile ring (CTA 0's weight producer): entry j of the
// pair's tile sequence goes into both CTAs' rings once all readers are done
// with entry j - kSchedDepth.
__device__ __forceinline__ bool sched_put(PairTail* tail, int j, const Tile& t,
                                          volatile int* abort, int* status, uint64_t limit) {
    const int slot = j % kSchedDepth;
    const uint32_t ph = (uint32_t)(j / kSchedDepth) & 1u;
    if (!mbar_wait_cl(&tail->sched_empty[slot], ph ^ 1u, abort, status, SITE_GEMM_PRODUCER, limit))
        return false;
    const int4* w = reinterpret_cast<const int4*>(&t);
    int4* dst = reinterpret_cast<int4*>(&tail->sched_tile[slot]);
    dst[0] = w[0];
    dst[1] = w[1];
    const uint32_t remote = map_to_rank(&tail->sched_tile[slot], 1);
    st_cluster_v4(remote, w[0]);
    st_cluster_v4(remote + 16, w[1]);
    mbar_arrive(&tail->sched_full[slot]);
    mbar_arrive_cluster(map_to_rank(&tail->sched_full[slot], 1));
    return true;
}
// Reader side: entry j of the tile sequence, then release it to the scheduler.
__device__ __forceinline__ bool sched_get(PairTail* tail, int j, Tile& t, volatile int* abort,
                                          int* status, int site, uint64_t limit) {
    const int slot = j % kSchedDepth;
    const uint32_t ph = (uint32_t)(j / kSchedDepth) & 1u;
    if (!mbar_wait_cl(&tail->sched_full[slot], ph, abort, status, site, limit)) return false;
    int4* w = reinterpret_cast<int4*>(&t);
    w[0] = ld_shared_v4(&tail->sched_tile[slot]);
    w[1] = ld_shared_v4(reinterpret_cast<const int4*>(&tail->sched_tile[slot]) + 1);
    mbar_arrive_cluster(map_to_rank(&tail->sched_empty[slot], 0));
    return true;
}

__device__ __forceinline__ int upper_group(const int* off, int n, int v) {
    // largest g in [0, n) with off[g] <= v
    int lo = 0, hi = n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (off[mid] <= v)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

// tanh by the hardware approximation (relative error about 2^-11, below the
// bf16 rounding of the values it feeds)
__device__ __forceinline__ float tanh_approx(float x) {
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Packed pairs of fp32 values (one 64-bit register pair) for the two-wide
// fp32 arithmetic of sm_100 (fma / mul .rn.f32x2): half the instructions.
__device__ __forceinline__ uint64_t pk2(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ float2 up2(uint64_t v) {
    float2 r;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
    return r;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}

__device__ __forceinline__ float silu_mul(float g, float u) {
    return __fdividef(g, 1.0f + __expf(-g)) * u;
}

// Per-warp staging: 32 rows x 128 B, 16-byte chunk q of row r stored at chunk
// position q ^ (r & 7), so row-wise writes (one row per instruction, lanes
// spread over the row) and transposed reads (one row per lane) are both free
// of bank conflicts.
__device__ __forceinline__ uint8_t* stage_chunk(uint8_t* wb, int row, int chunk) {
    return wb + row * 128 + ((chunk ^ (row & 7)) << 4);
}

// SwiGLU backward epilogue (EPI_DSWIGLU) of one tile for warp quarter wq.
// fp32 transpose (token row i: its 32 features), then lane = token row r:
// dh_raw of features f0 .. f0 + 31 (the warp's TMEM lanes), the saved gate /
// up pre-activations of the row (at its forward position), and per feature
//   h = silu(g) u,  dh = w dh_raw,  dg = dh u silu'(g),  du = dh silu(g),
//   hw = w h,  with silu'(g) = sigmoid(g) (1 + g (1 - sigmoid(g)));
// the sum of dh_raw h over the 32 features is this warp's part of dL/dw.
// The chunk loop stays rolled (its body is large: unrolled it would crowd
// the instruction cache that the producer and MMA warps share), and the
// global reads run ahead of it: the slot of each row two chunks ahead (for its
// gate weight), its gate weight and pre-activations one chunk ahead.
struct DswigluRow {
    int src;
    float w;
    uint4 g[4], u[4];
};

__device__ __forceinline__ int dswiglu_src(const Tile& t, const PairArgs& a, int c0, int lane) {
    const int r = t.b_row + c0 + lane;
    if (c0 + lane >= t.n_real) return -1;
    return a.row_src != nullptr ? a.row_src[r] : r;
}

// rf: the row's index in the forward's row order (the saved layout's rows);
// features f0 .. f0 + 31 are two 16-feature blocks [16 gate | 16 up].
__device__ __forceinline__ void dswiglu_fetch(const PairArgs& a, int src, int rf, int f0,
                                              DswigluRow& row) {
    row.src = src;
    row.w = 1.f;
    if (src < 0) return;
    if (a.row_src != nullptr) row.w = a.topk_w[src];
    const __nv_bfloat16* gu = static_cast<const __nv_bfloat16*>(a.gu_in);
#pragma unroll
    for (int b = 0; b < 2; ++b) {
        const uint4* p = reinterpret_cast<const uint4*>(
            gu + ((size_t)((f0 >> 4) + b) * a.gu_rows + rf) * 32);
        row.g[2 * b] = __ldg(p);
        row.g[2 * b + 1] = __ldg(p + 1);
        row.u[2 * b] = __ldg(p + 2);
        row.u[2 * b + 1] = __ldg(p + 3);
    }
}

__device__ __forceinline__ void dswiglu_epilogue(uint8_t* wb, uint32_t taddr, const Tile& t,
                                                 const PairArgs& a, uint32_t cta, int wq,
                                                 int lane, int row_shift) {
    const int F = a.feat;
    const int f0 = t.ft * 256 + (int)cta * 128 + wq * 32;
    // forward row of this tile's row r: r + row_shift (the forward's segments
    // are unpadded, this launch's are padded to 128 rows)
    const int rf0 = t.b_row + lane + row_shift;
    DswigluRow cur;
    dswiglu_fetch(a, dswiglu_src(t, a, 0, lane), rf0, f0, cur);
    int src_next = dswiglu_src(t, a, 32, lane);
#pragma unroll 1
    for (int cc = 0; cc < kNTile / 32; ++cc) {
        const int c0 = 32 * cc;
        if (c0 >= t.n) break;
        uint32_t v[32];
        tmem_ld32(taddr + (uint32_t)c0, v);
        // the next chunk's reads go out before this chunk's work
        DswigluRow nxt;
        dswiglu_fetch(a, c0 + 32 < t.n ? src_next : -1, rf0 + c0 + 32, f0, nxt);
        src_next = c0 + 64 < t.n ? dswiglu_src(t, a, c0 + 64, lane) : -1;
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            float* rowp = reinterpret_cast<float*>(stage_chunk(wb, i, lane >> 2));
            rowp[lane & 3] = __uint_as_float(v[i]);
        }
        __syncwarp();
        // per lane (= its staged row): dg, du and w h of 32 features.  dg of
        // features 8 qq .. 8 qq + 7 goes back into the lane's own staged row at
        // chunk qq (dh_raw chunks 2 qq, 2 qq + 1 already read), du and w h stay
        // in registers; the rows then leave through the buffer, 4 rows x 128 B
        // (dg | du) and 8 rows x 64 B (w h) per store instruction.
        uint32_t pdu[16], phw[16];
        float part = 0.f;
        if (cur.src >= 0) {
            const uint64_t W2 = pk2(cur.w, cur.w);
            const uint64_t kHalf2 = pk2(0.5f, 0.5f), kOne2 = pk2(1.f, 1.f),
                           kNeg12 = pk2(-1.f, -1.f);
            uint64_t PART = pk2(0.f, 0.f);
            const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(cur.g);
            const __nv_bfloat162* u2 = reinterpret_cast<const __nv_bfloat162*>(cur.u);
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
                uint32_t pdg[4];
#pragma unroll
                for (int hq = 0; hq < 2; ++hq) {
                    const int q = 2 * qq + hq;
                    const float4 c4 = *reinterpret_cast<const float4*>(stage_chunk(wb, lane, q));
                    const uint64_t dr2[2] = {pk2(c4.x, c4.y), pk2(c4.z, c4.w)};
                    float2 odg[2], odu[2], ohw[2];
                    // features 4 q + 2 pp, 4 q + 2 pp + 1 as one pair
#pragma unroll
                    for (int pp = 0; pp < 2; ++pp) {
                        const float2 gg = __bfloat1622float2(g2[2 * q + pp]);
                        const float2 uu = __bfloat1622float2(u2[2 * q + pp]);
                        const uint64_t G = pk2(gg.x, gg.y), U = pk2(uu.x, uu.y);
                        // sigmoid(g) = (1 + tanh(g / 2)) / 2: one hardware tanh each
                        const float2 hg = up2(mul2(G, kHalf2));
                        const uint64_t SG =
                            fma2(pk2(tanh_approx(hg.x), tanh_approx(hg.y)), kHalf2, kHalf2);
                        const uint64_t SILU = mul2(G, SG);
                        const uint64_t H = mul2(SILU, U);
                        PART = fma2(dr2[pp], H, PART);
                        const uint64_t DH = mul2(dr2[pp], W2);
                        // silu'(g) = sigmoid(g) (1 + g (1 - sigmoid(g))) = silu (1 - sg) + sg
                        const uint64_t DS = fma2(SILU, fma2(SG, kNeg12, kOne2), SG);
                        odg[pp] = up2(mul2(mul2(DH, U), DS));
                        odu[pp] = up2(mul2(DH, SILU));
                        ohw[pp] = up2(mul2(H, W2));
                    }
                    pdg[2 * hq] = pack_bf16x2(odg[0].x, odg[0].y);
                    pdg[2 * hq + 1] = pack_bf16x2(odg[1].x, odg[1].y);
                    pdu[4 * qq + 2 * hq] = pack_bf16x2(odu[0].x, odu[0].y);
                    pdu[4 * qq + 2 * hq + 1] = pack_bf16x2(odu[1].x, odu[1].y);
                    phw[4 * qq + 2 * hq] = pack_bf16x2(ohw[0].x, ohw[0].y);
                    phw[4 * qq + 2 * hq + 1] = pack_bf16x2(ohw[1].x, ohw[1].y);
                }
                *reinterpret_cast<uint4*>(stage_chunk(wb, lane, qq)) =
                    make_uint4(pdg[0], pdg[1], pdg[2], pdg[3]);
            }
#pragma unroll
            for (int qq = 0; qq < 4; ++qq)
                *reinterpret_cast<uint4*>(stage_chunk(wb, lane, 4 + qq)) =
                    make_uint4(pdu[4 * qq], pdu[4 * qq + 1], pdu[4 * qq + 2], pdu[4 * qq + 3]);
            const float2 part2 = up2(PART);  // even and odd features' sums
            part = part2.x + part2.y;
            if (a.dw_part != nullptr)
                a.dw_part[(size_t)(t.b_row + c0 + lane) * (F >> 5) + (f0 >> 5)] = part;
        }
        __syncwarp();
        {
            // dg | du: row i = 4 it + lane / 8, 16-byte piece lane % 8
            const int q = lane & 7;
#pragma unroll
            for (int it = 0; it < 8; ++it) {
                const int i = 4 * it + (lane >> 3);
                if (c0 + i < t.n_real) {
                    const uint4 v4 = *reinterpret_cast<const uint4*>(stage_chunk(wb, i, q));
                    __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(a.dgu_out) +
                                         (size_t)(t.b_row + c0 + i) * 2 * F + f0 +
                                         (q < 4 ? q * 8 : F + (q - 4) * 8);
                    *reinterpret_cast<uint4*>(dst) = v4;
                }
            }
        }
        __syncwarp();
        if (cur.src >= 0) {
#pragma unroll
            for (int qq = 0; qq < 4; ++qq)
                *reinterpret_cast<uint4*>(stage_chunk(wb, lane, qq)) =
                    make_uint4(phw[4 * qq], phw[4 * qq + 1], phw[4 * qq + 2], phw[4 * qq + 3]);
        }
        __syncwarp();
        {
            // w h: row i = 8 it + lane / 4, 16-byte piece lane % 4
            const int q = lane & 3;
#pragma unroll
            for (int it = 0; it < 4; ++it) {
                const int i = 8 * it + (lane >> 2);
                if (c0 + i < t.n_real) {
                    const uint4 v4 = *reinterpret_cast<const uint4*>(stage_chunk(wb, i, q));
                    *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.hw_out) +
                                              (size_t)(t.b_row + c0 + i) * F + f0 + q * 8) = v4;
                }
            }
        }
        __syncwarp();
        cur = nxt;
    }
}

// Epilogue of one tile for warp quarter wq of this CTA: TMEM lanes 32 wq ..
// 32 wq + 31 (weight rows) x the tile's N token columns.  Each warp works on
// its own: tcgen05.ld of 32 columns (thread = weight row, registers = tokens),
// transpose through its staging buffer, then thread = token for the stores.
template <int EPI>
__device__ __forceinline__ void pair_epilogue(uint8_t* wb, uint32_t taddr, const Tile& t,
                                              const PairArgs& a, uint32_t cta, int wq, int lane,
                                              int row_shift) {
    if constexpr (EPI == EPI_DSWIGLU) {
        dswiglu_epilogue(wb, taddr, t, a, cta, wq, lane, row_shift);
        return;
    }
    (void)row_shift;
    // SCATTER: slot index and gate weight of every token column of the tile,
    // loaded once per tile (lane l holds columns 32 c + l)
    int srcs[kNTile / 32];
    float wts[kNTile / 32];
    if constexpr (EPI == EPI_SCATTER) {
#pragma unroll
        for (int c = 0; c < kNTile / 32; ++c)
            srcs[c] = 32 * c + lane < t.n_real ? a.row_src[t.b_row + 32 * c + lane] : -1;
#pragma unroll
        for (int c = 0; c < kNTile / 32; ++c)
            wts[c] = srcs[c] >= 0 ? (a.topk_w != nullptr ? a.topk_w[srcs[c]] : 1.f) : 0.f;
    }
#pragma unroll
    for (int cc = 0; cc < kNTile / 32; ++cc) {
        const int c0 = 32 * cc;
        if (c0 >= t.n) break;
        uint32_t v[32];
        tmem_ld32(taddr + (uint32_t)c0, v);  // weight row (lane) x tokens c0 .. c0+31
        tmem_ld_wait();
        const bool tok_ok = c0 + lane < t.n_real;  // after the transpose, lane = token
        if constexpr (EPI == EPI_SWIGLU || EPI == EPI_SWIGLU_SAVE) {
            // The CTA's weight rows are [16 gate, 16 up] per warp quarter: lane
            // i < 16 holds gate feature 16 wq + i, lane i + 16 the matching up
            // row.  fp32 transpose through the staging buffer, then lane = token:
            // h_f = silu(g_f) * u_f for its 16 features, one 32-byte store.
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                float* row = reinterpret_cast<float*>(stage_chunk(wb, i, lane >> 2));
                row[lane & 3] = __uint_as_float(v[i]);
            }
            __syncwarp();
            uint4 h_row[2];   // lane = token: h of its 16 features, bf16
            uint4 sv_row[4];  // SWIGLU_SAVE: its [16 gate | 16 up] pre-activations, bf16
            if (tok_ok) {
                float f[32];
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const float4 c4 = *reinterpret_cast<const float4*>(stage_chunk(wb, lane, q));
                    f[4 * q] = c4.x;
                    f[4 * q + 1] = c4.y;
                    f[4 * q + 2] = c4.z;
                    f[4 * q + 3] = c4.w;
                }
                uint32_t packed[8];
#pragma unroll
                for (int p = 0; p < 8; ++p)
                    packed[p] = pack_bf16x2(silu_mul(f[2 * p], f[16 + 2 * p]),
                                            silu_mul(f[2 * p + 1], f[16 + 2 * p + 1]));
                h_row[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
                h_row[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
                if constexpr (EPI == EPI_SWIGLU_SAVE) {
                    // the pre-activations for the backward: blocks of 16 features,
                    // [block][row][16 gate | 16 up] with this launch's row order, so
                    // the warp's 32 consecutive rows are 2 KiB in one piece
                    // (stored below, through the staged rows)
                    uint32_t pg[8], pu[8];
#pragma unroll
                    for (int p = 0; p < 8; ++p) {
                        pg[p] = pack_bf16x2(f[2 * p], f[2 * p + 1]);
                        pu[p] = pack_bf16x2(f[16 + 2 * p], f[16 + 2 * p + 1]);
                    }
                    sv_row[0] = make_uint4(pg[0], pg[1], pg[2], pg[3]);
                    sv_row[1] = make_uint4(pg[4], pg[5], pg[6], pg[7]);
                    sv_row[2] = make_uint4(pu[0], pu[1], pu[2], pu[3]);
                    sv_row[3] = make_uint4(pu[4], pu[5], pu[6], pu[7]);
                }
            }
            __syncwarp();
            // h rows (32 B each) through the staged rows, 2 lanes per row: each
            // store instruction writes 16 whole 32-byte row pieces (lanes 8 g ..
            // 8 g + 7 take 4 rows 2 apart: disjoint chunk positions)
            if (tok_ok) {
                *reinterpret_cast<uint4*>(stage_chunk(wb, lane, 0)) = h_row[0];
                *reinterpret_cast<uint4*>(stage_chunk(wb, lane, 1)) = h_row[1];
            }
            __syncwarp();
            {
                const int q = lane & 1, g = lane >> 3;
#pragma unroll
                for (int it = 0; it < 2; ++it) {
                    const int i = 16 * it + 2 * ((lane >> 1) & 3) + (g & 1) + 8 * (g >> 1);
                    if (c0 + i < t.n_real)
                        *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) +
                                                  (size_t)(t.b_row + c0 + i) * a.out_ld +
                                                  t.ft * a.out_col_step + cta * 64 + wq * 16 +
                                                  q * 8) =
                            *reinterpret_cast<const uint4*>(stage_chunk(wb, i, q));
                }
            }
            __syncwarp();
            if constexpr (EPI == EPI_SWIGLU_SAVE) {
                // the pre-activations for the backward: blocks of 16 features,
                // [block][row][16 gate | 16 up] with this launch's row order, so
                // the warp's 32 consecutive rows are 2 KiB in one piece; each
                // store instruction writes 512 contiguous bytes (8 rows)
                if (tok_ok) {
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        *reinterpret_cast<uint4*>(stage_chunk(wb, lane, q)) = sv_row[q];
                }
                __syncwarp();
                const int blk = (t.ft * a.out_col_step + (int)cta * 64 + wq * 16) >> 4;
                const int q = lane & 3;
                const int sub = (lane >> 2) & 1, g = lane >> 3;
#pragma unroll
                for (int it = 0; it < 4; ++it) {
                    const int i = 8 * it + g + 4 * sub;
                    if (c0 + i < t.n_real)
                        *reinterpret_cast<uint4*>(
                            static_cast<__nv_bfloat16*>(a.save) +
                            ((size_t)blk * a.gu_rows + t.b_row + c0 + i) * 32 + q * 8) =
                            *reinterpret_cast<const uint4*>(stage_chunk(wb, i, q));
                }
                __syncwarp();
            }
        } else if constexpr (EPI == EPI_SCATTER) {
            // fp32 transpose through the staging buffer (token row i: 32 features x
            // 4 B), then lane = token: its 32 features times its own gate weight,
            // rounded to bf16, one 64-byte store into the token's slot row
            const int src = srcs[cc];
            const float wv = wts[cc];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                float* row = reinterpret_cast<float*>(stage_chunk(wb, i, lane >> 2));
                row[lane & 3] = __uint_as_float(v[i]);
            }
            __syncwarp();
            uint32_t packed[16];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float4 f = *reinterpret_cast<const float4*>(stage_chunk(wb, lane, q));
                packed[2 * q] = pack_bf16x2(wv * f.x, wv * f.y);
                packed[2 * q + 1] = pack_bf16x2(wv * f.z, wv * f.w);
            }
            __syncwarp();
            // the bf16 row (64 B) back into the lane's staged row, then 4 lanes
            // per row: each store instruction writes 8 whole 64-byte row pieces
#pragma unroll
            for (int q = 0; q < 4; ++q)
                *reinterpret_cast<uint4*>(stage_chunk(wb, lane, q)) =
                    make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2],
                               packed[4 * q + 3]);
            __syncwarp();
            {
                // lanes 8 g .. 8 g + 7 take rows r and r + 4 (disjoint chunk
                // positions of the swizzle: no bank conflict)
                const int q = lane & 3;
                const int sub = (lane >> 2) & 1, g = lane >> 3;
#pragma unroll
                for (int it = 0; it < 4; ++it) {
                    const int i = 8 * it + g + 4 * sub;
                    const int si = __shfl_sync(0xffffffffu, src, i);
                    if (si >= 0) {
                        const uint4 v4 = *reinterpret_cast<const uint4*>(stage_chunk(wb, i, q));
                        *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) +
                                                  (size_t)si * a.out_ld + t.ft * a.out_col_step +
                                                  cta * 128 + wq * 32 + q * 8) = v4;
                    }
                }
            }
            __syncwarp();
        } else if constexpr (EPI == EPI_STORE_ROWS) {
            // weight-gradient tile: lane = output row (TMEM lane), 32 columns per
            // chunk.  Rows go through the staging buffer so that each store
            // instruction writes 4 whole 128-byte row segments.  A tile of an
            // empty group (no k-blocks) stores zeros.
            const bool zero = (t.aux >> 16) == 0;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                float4 c4 = make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                        __uint_as_float(v[4 * q + 2]),
                                        __uint_as_float(v[4 * q + 3]));
                if (zero) c4 = make_float4(0.f, 0.f, 0.f, 0.f);
                *reinterpret_cast<float4*>(stage_chunk(wb, lane, q)) = c4;
            }
            __syncwarp();
            float* ob = static_cast<float*>(a.out) +
                        ((size_t)t.g * a.m_total + t.ft * 256 + cta * 128 + wq * 32) * a.out_ld +
                        (size_t)(t.aux & 0xFFFF) * 256 + c0;
#pragma unroll
            for (int it = 0; it < 8; ++it) {
                const int row = it * 4 + (lane >> 3), q = lane & 7;
                *reinterpret_cast<float4*>(ob + (size_t)row * a.out_ld + q * 4) =
                    *reinterpret_cast<const float4*>(stage_chunk(wb, row, q));
            }
            __syncwarp();
        } else {  // EPI_STORE_F32: out[b_row + token][col] = acc, fp32
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                // token row i: 32 features x 4 B = 128 B in chunks 0..7
                float* row = reinterpret_cast<float*>(stage_chunk(wb, i, lane >> 2));
                row[lane & 3] = __uint_as_float(v[i]);
            }
            __syncwarp();
            {
                // 8 lanes per token row: each store instruction writes 4 whole
                // 128-byte row pieces
                const int q = lane & 7;
#pragma unroll
                for (int it = 0; it < 8; ++it) {
                    const int i = 4 * it + (lane >> 3);
                    if (c0 + i < t.n_real)
                        *reinterpret_cast<float4*>(static_cast<float*>(a.out) +
                                                   (size_t)(t.b_row + c0 + i) * a.out_ld +
                                                   t.ft * a.out_col_step + cta * 128 + wq * 32 +
                                                   q * 4) =
                            *reinterpret_cast<const float4*>(stage_chunk(wb, i, q));
                }
            }
            __syncwarp();
        }
    }
}

template <int EPI0, int EPI1, class RING, int KIND>
__global__ void __launch_bounds__(kThreads, 1)
    pair_gemm_kernel(const __grid_constant__ PairMaps maps, const PairArgs args0,
                     const PairArgs args1, int n_problems) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    constexpr int kStages = RING::kStages;
    constexpr int kStageBytes = RING::kStageBytes;
    PairTail* tail = reinterpret_cast<PairTail*>(smem + (size_t)kStages * kStageBytes);
    volatile int* abort_flag = &tail->abort;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t cta = cluster_ctarank();  // 0: MMA issuer of the pair
    const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
    int* const status = args0.status;
    const uint64_t limit = args0.wait_limit_ns;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&tail->full[s], 2);   // used in CTA 0: its two producers' expect_tx
            mbar_init(&tail->empty[s], 1);  // one commit from the MMA issuer
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tail->tfull[a], 1);
            mbar_init(&tail->tempty[a], 2 * kEpiWarps);  // used in CTA 0: both CTAs' warps
        }
        mbar_init(&tail->drain, 1);
        for (int i = 0; i < kSchedDepth; ++i) {
            mbar_init(&tail->sched_full[i], 1);
            mbar_init(&tail->sched_empty[i], kSchedReaders);
        }
        tail->abort = 0;
        fence_barrier_init();
    }
    if (KIND == KIND_FWD && warp == 0 && lane == 0) {
        // The weights are inputs no earlier kernel writes: while the previous
        // kernels (routing, permutation) finish, bring this CTA's half of the
        // weight tile of the pair's first tile into L2.  The first tile is
        // the pair's index; a problem with expert counts (not yet known here)
        // is taken to have one token chunk per expert, as at small batches
        // (a wrong guess only prefetches a tile another pair will load).
        int lt = pair, p = 0;
        const int ng0_s = args0.counts != nullptr ? args0.n_groups : 1;
        if (args0.counts == nullptr && n_problems > 1) {
            const int tiles0_s = ((args0.static_rows + kNTile - 1) / kNTile) * args0.n_ftiles;
            if (lt >= tiles0_s) {
                lt -= tiles0_s;
                p = 1;
            }
        }
        const PairArgs& a = p == 0 ? args0 : args1;
        const int ng = p == 0 ? ng0_s : (args1.counts != nullptr ? args1.n_groups : 1);
        int g, ft;
        if (a.counts == nullptr) {
            g = 0;
            ft = lt % a.n_ftiles;
        } else {
            g = lt / a.n_ftiles;
            ft = lt % a.n_ftiles;
        }
        if (g < ng && a.n_ftiles > 0) {
            const CUtensorMap* m = &maps.a[p];
            const int kb_n = a.K / kBK;
            const int a_row0 = (int)(g * a.a_group_stride) + ft * a.a_tile_step +
                               (int)cta * a.a_cta_step;
            const int blk = g * a.a_blocks_per_group +
                            ((ft * a.a_tile_step + (int)cta * a.a_cta_step) >> 4);
            for (int kb = 0; kb < kb_n; ++kb) {
                if (a.a_mode == 0)
                    tma_prefetch_l2_3d(m, 0, a_row0, kb * kAtoms);
                else
                    tma_prefetch_l2_5d(m, 0, 0, 0, blk, kb * kAtoms);
            }
        }
    }
    // everything below reads or writes memory of earlier kernels (counts,
    // token rows, outputs): wait until the previous kernel has completed
    pdl_wait();
    // group offsets of both problems: rows and tiles (exclusive prefix sums)
    if (warp == 0) {
        for (int p = 0; p < n_problems; ++p) {
            const PairArgs& a = p == 0 ? args0 : args1;
            const int ng = a.counts != nullptr ? a.n_groups : 1;
            const int al = a.seg_align > 1 ? a.seg_align : 1;
            int carry_r = 0, carry_t = 0, carry_u = 0;
            for (int g0 = 0; g0 < ng; g0 += 32) {
                const int g = g0 + lane;
                const int c = g < ng ? (a.counts != nullptr ? a.counts[g] : a.static_rows) : 0;
                // rows the group occupies in B (segments padded to `al` rows)
                const int cr = (c + al - 1) / al * al;
                const int tl = KIND == KIND_WGRAD ? (g < ng ? a.n_ftiles * a.n_ntiles : 0)
                                                  : ((c + kNTile - 1) / kNTile) * a.n_ftiles;
                int ir = cr, it = tl, iu = c;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int nr = __shfl_up_sync(0xffffffffu, ir, o);
                    const int nt = __shfl_up_sync(0xffffffffu, it, o);
                    const int nu = __shfl_up_sync(0xffffffffu, iu, o);
                    if (lane >= o) {
                        ir += nr;
                        it += nt;
                        iu += nu;
                    }
                }
                if (g < ng) {
                    tail->seg_off[p][g] = carry_r + ir - cr;
                    tail->tile_off[p][g] = carry_t + it - tl;
                    tail->cnt[p][g] = c;
                    tail->useg_off[p][g] = carry_u + iu - c;
                }
                carry_r += __shfl_sync(0xffffffffu, ir, 31);
                carry_t += __shfl_sync(0xffffffffu, it, 31);
                carry_u += __shfl_sync(0xffffffffu, iu, 31);
            }
            if (lane == 0) {
                tail->seg_off[p][ng] = carry_r;
                tail->tile_off[p][ng] = carry_t;
            }
        }
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&tail->tmem_base)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();  // barrier init of both CTAs visible before any cross-CTA signal
    tc_fence_after();

    const uint32_t tmem_base = tail->tmem_base;
    const int ng0 = args0.counts != nullptr ? args0.n_groups : 1;
    const int ng1 = args1.counts != nullptr ? args1.n_groups : 1;
    const int tiles0 = tail->tile_off[0][ng0];
    const int tiles1 = n_problems > 1 ? tail->tile_off[1][ng1] : 0;
    const int total_tiles = tiles0 + tiles1;

    // tile -> (problem, expert, feature tile, token chunk); inside an expert the
    // feature tile is the slow index so the token chunks of one weight tile are
    // neighbours in the tile order (weights fetched from HBM once, re-read in L2)
    auto decode = [&](int tile) {
        Tile t;
        t.p = tile < tiles0 ? 0 : 1;
        const PairArgs& a = t.p == 0 ? args0 : args1;
        const int lt = t.p == 0 ? tile : tile - tiles0;
        const int ng = t.p == 0 ? ng0 : ng1;
        t.g = upper_group(tail->tile_off[t.p], ng, lt);
        const int cnt = tail->cnt[t.p][t.g];
        const int local = lt - tail->tile_off[t.p][t.g];
        t.end = 0;
        if (KIND == KIND_WGRAD) {
            // M tile slow, N tile fast; K runs over the group's rows (padded
            // to whole k-blocks with zero rows, or past the end of a dense
            // problem's rows, which the tensor map fills with zeros)
            t.ft = local / a.n_ntiles;
            t.b_row = a.b_row_base + tail->seg_off[t.p][t.g];
            t.n_real = kNTile;
            t.n = kNTile;
            t.aux = (local % a.n_ntiles) | (((cnt + kBK - 1) / kBK) << 16);
            return t;
        }
        const int nch = (cnt + kNTile - 1) / kNTile;
        // routed experts: feature tile slow, token chunk fast (a weight tile's
        // chunks are neighbours); dense problems: token chunk slow, feature tile
        // fast (pairs running together cover whole token rows)
        const bool dense = a.counts == nullptr;
        t.ft = dense ? local % a.n_ftiles : local / nch;
        const int ch = dense ? local / a.n_ftiles : local % nch;
        // the expert's tokens split into nch nearly equal chunks (sizes differ by
        // at most one row), so tiles of one expert take the same time
        const int r0 = (int)((long long)ch * cnt / nch);
        const int r1 = (int)((long long)(ch + 1) * cnt / nch);
        t.b_row = a.b_row_base + tail->seg_off[t.p][t.g] + r0;
        t.n_real = r1 - r0;
        t.n = (t.n_real + 15) & ~15;
        t.aux = 0;
        return t;
    };

    if (warp == 0 || warp == kBProducerWarp) {
        // ------------------------------------------------ TMA producers (both CTAs)
        // Warp 0 loads the weight tile, warp kBProducerWarp the token tile, one
        // 32 KiB copy each per stage.  CTA 0's weight producer is also the
        // pair's scheduler: it draws the pair's tiles from the ticket counter
        // (the first one is the pair's index) and publishes them; every other
        // role reads the ring.
        const bool is_a = warp == 0;
        const bool is_sched = is_a && cta == 0;
        if (lane == 0) {
            for (int p = 0; p < n_problems; ++p) {
                if (is_a) {
                    tma_prefetch_desc(&maps.a[p]);
                } else {
                    for (int j = 0; j < kTokenBoxes; ++j) tma_prefetch_desc(&maps.b[p][j]);
                }
            }
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            int next = pair;
            // stages this lane has issued a copy into, and the parity of the
            // full-barrier phase of that copy (for the drain on abort)
            uint32_t issued = 0, issued_ph = 0;
            for (int j = 0; ok; ++j) {
                Tile t;
                if (is_sched) {
                    if (next < total_tiles) {
                        t = decode(next);
                        if (t.n > 2 * RING::kBMaxRows) {
                            // a token tile larger than this ring's stages: the
                            // launch chose the wrong ring; stop every role cleanly
                            set_status(status, MOE_ERR_DEVICE, SITE_GEMM_BOUNDS, t.n);
                            t = Tile{};
                            t.end = 1;
                            next = total_tiles;
                        }
                        // the ticket's latency is hidden behind this tile's loads
                        next = n_pairs + atomicAdd(args0.sched_counter, 1);
                    } else {
                        t = Tile{};
                        t.end = 1;
                    }
                    if (!sched_put(tail, j, t, abort_flag, status, limit)) break;
                } else if (!sched_get(tail, j, t, abort_flag, status, SITE_GEMM_PRODUCER, limit)) {
                    break;
                }
                if (t.end) break;
                const PairArgs& a = t.p == 0 ? args0 : args1;
                // token rows per CTA: N/2, loaded with the box of 16 rb rows (an
                // MN-major token operand: 128 K rows x 2 blocks of 64 columns)
                const int rb = KIND == KIND_WGRAD ? 8 : ((t.n >> 1) + 15) >> 4;
                const CUtensorMap* m = is_a ? &maps.a[t.p] : &maps.b[t.p][rb - 1];
                const uint32_t op_bytes = is_a ? (uint32_t)kABytes : (uint32_t)rb * 4096u;
                const int a_row0 = (int)(t.g * a.a_group_stride) + t.ft * a.a_tile_step +
                                   (int)cta * a.a_cta_step;
                const int b_row0 = t.b_row + (int)cta * (t.n >> 1);
                // MN-major weights (KIND_DGRAD): rows = K of group g, 64-column
                // blocks = this CTA's 128 M rows; MN-major activations
                // (KIND_WGRAD): rows = K from the group's first row
                const int a_mn_row = KIND == KIND_WGRAD ? t.b_row : (int)(t.g * a.a_group_stride);
                const int a_mn_blk = (t.ft * a.a_tile_step + (int)cta * a.a_cta_step) >> 6;
                const int b_mn_blk = ((t.aux & 0xFFFF) * kNTile + (int)cta * (kNTile / 2)) >> 6;
                const int kb_count = KIND == KIND_WGRAD ? (t.aux >> 16) : a.K / kBK;
                for (int kb = 0; kb < kb_count; ++kb) {
                    if (!mbar_wait_bounded(&tail->empty[s], ph ^ 1u, abort_flag, status,
                                           SITE_GEMM_PRODUCER, limit)) {
                        ok = false;
                        break;
                    }
                    uint8_t* sa = smem + (size_t)s * kStageBytes;
                    // both CTAs' copies of this operand complete on CTA 0's barrier
                    if (cta == 0) arrive_expect_tx_local(&tail->full[s], 2u * op_bytes);
                    const uint32_t fb = map_to_rank(&tail->full[s], 0);
                    const int atom = kb * kAtoms;
                    if (!is_a) {
                        if (KIND == KIND_WGRAD)  // 128 K rows x this CTA's 128 N columns
                            tma_load_3d_pair(sa + kABytes, m, fb, 0, t.b_row + kb * kBK, b_mn_blk);
                        else  // 16 rb token rows x 2 k-atoms (rows past the tile's N/2 unused)
                            tma_load_3d_pair(sa + kABytes, m, fb, 0, b_row0, atom);
                    } else if (KIND != KIND_FWD) {
                        // 128 K rows x this CTA's 128 M columns
                        tma_load_3d_pair(sa, m, fb, 0, a_mn_row + kb * kBK, a_mn_blk);
                    } else if (a.a_mode == 0) {
                        // 128 consecutive weight rows x 2 k-atoms
                        tma_load_3d_pair(sa, m, fb, 0, a_row0, atom);
                    } else {
                        // 4 blocks x (16 gate rows, 16 up rows) of features
                        // ft * a_tile_step + cta * a_cta_step ... + 63 of group g, x 2 k-atoms
                        const int blk = t.g * a.a_blocks_per_group +
                                        ((t.ft * a.a_tile_step + (int)cta * a.a_cta_step) >> 4);
                        tma_load_5d_pair(sa, m, fb, 0, 0, 0, blk, atom);
                        // the same rows kPrefetchAhead k-blocks further on towards L2
                        if (kb + kPrefetchAhead < kb_count)
                            tma_prefetch_l2_5d(m, 0, 0, 0, blk, atom + kPrefetchAhead * kAtoms);
                    }
                    issued |= 1u << s;
                    issued_ph = (issued_ph & ~(1u << s)) | (ph << s);
                    if (++s == kStages) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            if (!ok) {
                // Leaving early (a wait ran out or another role gave up): no
                // copy this lane issued may still be writing this CTA's shared
                // memory when the CTA exits.  In the pair's first CTA every
                // issued stage's full barrier is waited for (it also counts
                // the other CTA's bytes of that stage); a stage the other CTA
                // never filled does not complete and ends the bounded wait.
                // The second CTA cannot wait on those barriers, so it holds
                // for a fixed settle time, far above a copy's latency.
                if (cta == 0) {
                    for (int st = 0; st < kStages; ++st)
                        if (issued & (1u << st))
                            mbar_wait_bounded(&tail->full[st], (issued_ph >> st) & 1u, nullptr,
                                              status, SITE_GEMM_DRAIN, kAbortDrainNs);
                } else if (issued != 0) {
                    const uint64_t t0 = clock64();
                    while ((uint64_t)clock64() - t0 < 2 * kAbortDrainNs) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (CTA 0 of the pair)
        if (lane == 0 && cta == 0) {
            int s = 0;
            uint32_t ph = 0;
            int it = 0;
            bool ok = true;
            // everything the k-block loop needs is precomputed: the loop body is
            // one barrier poll, one block of 4 MMAs and two commits (a single
            // thread issues them, so its instruction count per MMA bounds the rate)
            const uint32_t empty_loc0 = smem_u32(&tail->empty[0]);
            // operand layouts: K-major (k16 steps of 32 B inside 128-byte rows,
            // 64-deep atoms 16 KiB apart for A) or MN-major (k16 steps of 16
            // rows x 128 B; 64-column blocks 16 KiB apart)
            constexpr bool kAMn = KIND != KIND_FWD;
            constexpr bool kBMn = KIND == KIND_WGRAD;
            const uint64_t adesc0 = kAMn ? sw128_mnmajor_desc(smem_u32(smem), 16384u)
                                         : sw128_kmajor_desc(smem_u32(smem));
            const uint64_t bdesc0 = kBMn ? sw128_mnmajor_desc(smem_u32(smem) + kABytes, 16384u)
                                         : sw128_kmajor_desc(smem_u32(smem) + kABytes);
            constexpr uint64_t kAStep = kAMn ? 128 : 2;
            constexpr uint64_t kBStep = kBMn ? 128 : 2;
            constexpr uint64_t kAHalf = kAMn ? 4 * 128 : (kAtomBytesA >> 4);
            constexpr uint64_t kStageDesc = kStageBytes >> 4;  // descriptor step per stage
            for (;; ++it) {
                Tile t;
                if (!sched_get(tail, it, t, abort_flag, status, SITE_GEMM_MMA, limit)) {
                    ok = false;
                    break;
                }
                if (t.end) break;
                const PairArgs& a = t.p == 0 ? args0 : args1;
                const int acc = it & 1;
                const uint32_t aph = (it >> 1) & 1;
                if (!mbar_wait_bounded(&tail->tempty[acc], aph ^ 1u, abort_flag, status,
                                       SITE_GEMM_MMA, limit)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * kNTile);
                const uint32_t idesc = idesc_bf16_f32(2 * kARows, t.n, kAMn, kBMn);
                // the token tile's second k-atom starts 16 rb rows x 128 B after its
                // first (K-major); MN-major: 4 k16 steps further
                const uint64_t b_atom_desc =
                    kBMn ? 4 * 128 : (uint64_t)(((t.n >> 1) + 15) >> 4) * (2048 >> 4);
                const int kb_count = KIND == KIND_WGRAD ? (t.aux >> 16) : a.K / kBK;
                uint32_t accum = 0;
                for (int kb = 0; kb < kb_count; ++kb) {
                    if (!mbar_try_wait(&tail->full[s], ph) &&
                        !mbar_wait_bounded(&tail->full[s], ph, abort_flag, status, SITE_GEMM_MMA,
                                           limit)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = adesc0 + (uint64_t)s * kStageDesc;
                    const uint64_t bd = bdesc0 + (uint64_t)s * kStageDesc;
#pragma unroll
                    for (int at = 0; at < kAtoms; ++at) {
                        tc_mma4_pair<kAStep, kBStep>(d_tmem, ad + (uint64_t)at * kAHalf,
                                                     bd + (uint64_t)at * b_atom_desc, idesc,
                                                     accum);
                        accum = 1;
                    }
                    // stage s free in both CTAs once these MMAs have read it
                    tc_commit_both(empty_loc0 + (uint32_t)(s * 8));
                    if (++s == kStages) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) break;
                tc_commit_both(smem_u32(&tail->tfull[acc]));
            }
            if (!ok) *abort_flag = 1;
            // all tensor-core work of the pair is complete once `drain` fires
            tc_commit_pair(smem_u32(&tail->drain));
            mbar_wait_bounded(&tail->drain, 0u, nullptr, status, SITE_GEMM_DRAIN, limit);
        }
    } else {
        // ------------------------------------------------ epilogue (warps 2..5, both CTAs)
        const int wq = warp & 3;  // TMEM lane quarter this warp may access
        uint8_t* wstage = reinterpret_cast<uint8_t*>(tail->stage) + wq * 4096;
        // Entry `it` of the tile ring, broadcast to the warp.  The epilogue reads
        // one entry ahead: entry it + 1 is taken once tile it's accumulator is
        // ready and before tile it's stores, so the release that frees the
        // ring entry does not wait for those stores to drain.
        auto get_tile = [&](int it, Tile& t) {
            bool ok = true;
            if (lane == 0) ok = sched_get(tail, it, t, abort_flag, status, SITE_GEMM_EPILOGUE, limit);
            int* w = reinterpret_cast<int*>(&t);
#pragma unroll
            for (int q = 0; q < 8; ++q) w[q] = __shfl_sync(0xffffffffu, w[q], 0);
            return __shfl_sync(0xffffffffu, (int)ok, 0) != 0;
        };
        Tile t_next{};
        bool ok_next = get_tile(0, t_next);
        for (int it = 0;; ++it) {
            const Tile t = t_next;
            const bool sched_ok = ok_next;
            // the 4 warps read the same sequence: they vote before leaving so
            // that none is left waiting on a named barrier
            if (!epi_all(sched_ok)) {
                *abort_flag = 1;
                break;
            }
            if (t.end) break;
            const int acc = it & 1;
            const uint32_t aph = (it >> 1) & 1;
            const bool got = mbar_wait_bounded(&tail->tfull[acc], aph, abort_flag, status,
                                               SITE_GEMM_EPILOGUE, limit);
            // the epilogue warps synchronise on named barriers: leave together
            if (!epi_all(got)) {
                *abort_flag = 1;
                break;
            }
            tc_fence_after();
            // the next ring entry (always published: the last tile is followed
            // by an end entry)
            ok_next = get_tile(it + 1, t_next);
            const uint32_t taddr =
                tmem_base + (uint32_t)(acc * kNTile) + ((uint32_t)(wq * 32) << 16);
            // lane quarter wq = weight rows 32 wq .. 32 wq + 31 of this CTA
            const int row_shift = tail->useg_off[t.p][t.g] - tail->seg_off[t.p][t.g];
            if (t.p == 0)
                pair_epilogue<EPI0>(wstage, taddr, t, args0, cta, wq, lane, row_shift);
            else
                pair_epilogue<EPI1>(wstage, taddr, t, args1, cta, wq, lane, row_shift);
            // The accumulator is free: tcgen05.wait::ld has completed this warp's
            // TMEM reads, and the tcgen05 fence pair orders them before the MMA
            // thread's reuse.  The arrive is relaxed: the tile's global stores
            // need no ordering against the MMAs, and a release here would wait
            // for all of them to drain.
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster_relaxed(map_to_rank(&tail->tempty[acc], 0));
        }
    }

    pdl_trigger();
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();  // no CTA leaves while its pair may still signal or read it
    tc_fence_after();
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"(kTmemCols)
                     : "memory");
}

// A bounded wait on a barrier that nothing signals: it must end with
// MOE_ERR_TIMEOUT in the status word (site SITE_SELFTEST), not hang.
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

cudaError_t launch_selftest_timeout(int* status, unsigned long long limit_ns, cudaStream_t s) {
    selftest_timeout_kernel<<<1, 32, 0, s>>>(status, limit_ns);
    return cudaGetLastError();
}

namespace {
template <class RING, int KIND>
cudaError_t launch_pair_ring(int epi0, int epi1, const PairMaps& maps, const PairArgs& a0,
                             const PairArgs* a1, int n_pairs, cudaStream_t s) {
    using Kern = void (*)(const PairMaps, const PairArgs, const PairArgs, int);
    Kern kern = nullptr;
    if constexpr (KIND == KIND_FWD) {
        if (epi0 == EPI_SWIGLU && epi1 == EPI_SWIGLU)
            kern = pair_gemm_kernel<EPI_SWIGLU, EPI_SWIGLU, RING, KIND>;
        else if (epi0 == EPI_SWIGLU_SAVE && epi1 == EPI_SWIGLU_SAVE)
            kern = pair_gemm_kernel<EPI_SWIGLU_SAVE, EPI_SWIGLU_SAVE, RING, KIND>;
        else if (epi0 == EPI_STORE_F32 && epi1 == EPI_SCATTER)
            kern = pair_gemm_kernel<EPI_STORE_F32, EPI_SCATTER, RING, KIND>;
        else if (epi0 == EPI_SCATTER && epi1 == EPI_SCATTER)
            kern = pair_gemm_kernel<EPI_SCATTER, EPI_SCATTER, RING, KIND>;
    } else if constexpr (KIND == KIND_DGRAD) {
        if (epi0 == EPI_DSWIGLU && epi1 == EPI_DSWIGLU)
            kern = pair_gemm_kernel<EPI_DSWIGLU, EPI_DSWIGLU, RING, KIND>;
        else if (epi0 == EPI_STORE_F32 && epi1 == EPI_SCATTER)
            kern = pair_gemm_kernel<EPI_STORE_F32, EPI_SCATTER, RING, KIND>;
        else if (epi0 == EPI_SCATTER && epi1 == EPI_SCATTER)
            kern = pair_gemm_kernel<EPI_SCATTER, EPI_SCATTER, RING, KIND>;
    } else {
        if (epi0 == EPI_STORE_ROWS && epi1 == EPI_STORE_ROWS)
            kern = pair_gemm_kernel<EPI_STORE_ROWS, EPI_STORE_ROWS, RING, KIND>;
    }
    if (kern == nullptr) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)RING::kSmemBytes);
    if (e != cudaSuccess) return e;
    const int np = a1 != nullptr ? 2 : 1;
    return launch_pdl(kern, dim3(2 * n_pairs), dim3(kThreads), RING::kSmemBytes, s, 2, maps, a0,
                      np > 1 ? *a1 : a0, np);
}

template <int KIND>
cudaError_t launch_pair_kind(int epi0, int epi1, const PairMaps& maps, const PairArgs& a0,
                             const PairArgs* a1, int n_pairs, int max_tile_tokens,
                             cudaStream_t s) {
    if (max_tile_tokens <= 2 * NarrowRing::kBMaxRows)
        return launch_pair_ring<NarrowRing, KIND>(epi0, epi1, maps, a0, a1, n_pairs, s);
    if (max_tile_tokens <= 2 * MidRing::kBMaxRows)
        return launch_pair_ring<MidRing, KIND>(epi0, epi1, maps, a0, a1, n_pairs, s);
    return launch_pair_ring<WideRing, KIND>(epi0, epi1, maps, a0, a1, n_pairs, s);
}
}  // namespace

cudaError_t launch_pair_gemm(int epi0, int epi1, const PairMaps& maps, const PairArgs& a0,
                             const PairArgs* a1, int n_pairs, int max_tile_tokens,
                             cudaStream_t s, int kind) {
    if (a0.sched_counter == nullptr) return cudaErrorInvalidValue;
    switch (kind) {
        case KIND_FWD:
            return launch_pair_kind<KIND_FWD>(epi0, epi1, maps, a0, a1, n_pairs, max_tile_tokens,
                                              s);
        case KIND_DGRAD:
            return launch_pair_kind<KIND_DGRAD>(epi0, epi1, maps, a0, a1, n_pairs,
                                                max_tile_tokens, s);
        case KIND_WGRAD:  // tiles are always 256 columns wide
            return launch_pair_ring<WideRing, KIND_WGRAD>(epi0, epi1, maps, a0, a1, n_pairs, s);
        default:
            return cudaErrorInvalidValue;
    }
}

}  // namespace moe
