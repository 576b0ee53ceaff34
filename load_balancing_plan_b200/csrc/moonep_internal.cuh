// moonep_internal.cuh -- shared pieces of the MoonEP sm_100a library:
// workspace layout arithmetic (host and device), header word indices, kernel
// parameter blocks, and inline-PTX wrappers for mbarriers and TMA bulk copies.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "moonep.h"

namespace moonep {

// ---------------------------------------------------------------------------
// workspace header words
// ---------------------------------------------------------------------------
enum : int {
    HDR_STATUS = 0,
    HDR_FALLBACK = 1,
    HDR_NREP = 2,
    HDR_MIGRATED = 3,
    HDR_NRANGES = 4,
    HDR_CFG = 5,  // 8 words: R L S K H B C C_max
    HDR_NRX = 13,
    HDR_FLAGS = 14,  // plan flags (MOONEP_PLAN_*)
    HDR_NSLOT = 15,  // pieces with a prefetch slot
    HDR_BAR_COUNT = 16,
    HDR_BAR_GEN = 17,
    HDR_TABLES_ONLY = 18,  // kTablesOnlyMark: a copy of the header and tables without the dispatch scratch
    HDR_EP = 19,           // 0: the workspace of a single-GPU plan; rank + 1: of expert-parallel rank `rank`
    HDR_TOTAL_SPILL = 20,
    HDR_PEND = 21,
    HDR_COUNT_DONE = 22,   // counting CTAs finished (moonep_ep_count_exchange)
};

// Token ranges of the dispatch grid.  The plan counts copies per (expert,
// range) so each dispatch CTA can number its copies without looking at other
// ranges.  Ranges are short (about kRangeTokens tokens) and far more numerous
// than the CTAs the GPU holds at once (kMinRanges: two per SM of a B200; the
// dispatch CTAs' shared memory lets three be resident at H = 7168, and waves
// of 444 measured no faster), so
// the resident CTAs always work on neighbouring token ranges and their row
// stores land close together in every expert's segment (DRAM pages stay
// open): on the mid workload dispatch takes 666 us with 4-token ranges, 689
// with 16-token ranges and 734 with one 110-token range per resident CTA.  Q
// is a whole number of such waves, so the last wave is full, and at most
// kBaseWords / N so that the per-(expert, range) table stays small.
#ifndef MOONEP_MIN_RANGES
#define MOONEP_MIN_RANGES 296
#endif
constexpr int64_t kMinRanges = MOONEP_MIN_RANGES;
#ifndef MOONEP_RANGE_TOKENS
#define MOONEP_RANGE_TOKENS 4
#endif
constexpr int64_t kRangeTokens = MOONEP_RANGE_TOKENS;
#ifndef MOONEP_BASE_WORDS_LOG2
#define MOONEP_BASE_WORDS_LOG2 22
#endif
constexpr int64_t kBaseWords = int64_t(1) << MOONEP_BASE_WORDS_LOG2;
// The plan counts ranges in blocks of consecutive ranges (one CTA counts a
// block); kBlocks blocks at most, one per SM of a B200 but the one whose CTA
// plans, so that each counting CTA loads all the ids it counts in one batch
// and keeps its block's histogram over the grid barrier.
#ifndef MOONEP_BLOCKS
#define MOONEP_BLOCKS 147
#endif
constexpr int64_t kBlocks = MOONEP_BLOCKS;

// combine and combine_backward: deal units to the CTAs round-robin
// (1) instead of one contiguous share each (0)
#ifndef MOONEP_INTERLEAVE
#define MOONEP_INTERLEAVE 0
#endif
#ifndef MOONEP_RANGE_WAVES
#define MOONEP_RANGE_WAVES 1
#endif
__host__ __device__ inline int64_t num_ranges(int64_t T, int64_t N) {
    if (!MOONEP_RANGE_WAVES) {
        int64_t q = T / kRangeTokens;
        const int64_t cap = kBaseWords / (N > 0 ? N : 1);
        if (q > cap) q = cap;
        if (q < kMinRanges) q = kMinRanges;
        return q < T ? q : (T > 0 ? T : 0);
    }
    const int64_t wave_tokens = kRangeTokens * kMinRanges;
    int64_t w = (T + wave_tokens / 2) / wave_tokens;  // waves, rounded to the nearest
    const int64_t wcap = kBaseWords / ((N > 0 ? N : 1) * kMinRanges);
    if (w > wcap) w = wcap;
    if (w < 1) w = 1;
    const int64_t q = w * kMinRanges;
    return q < T ? q : (T > 0 ? T : 0);
}

__host__ __device__ inline int64_t num_blocks(int64_t Q) { return Q < kBlocks ? Q : kBlocks; }

// block b of NB holds ranges [b*Q/NB, (b+1)*Q/NB); range q is in block
// floor(((q+1)*NB - 1) / Q) (the last b with b*Q/NB <= q)
__host__ __device__ inline int64_t block_first_range(int64_t b, int64_t Q, int64_t NB) { return b * Q / NB; }
__host__ __device__ inline int64_t block_of_range(int64_t q, int64_t Q, int64_t NB) { return ((q + 1) * NB - 1) / Q; }

// token range q of Q: [q*T/Q, (q+1)*T/Q)
__host__ __device__ inline int64_t range_begin(int64_t q, int64_t T, int64_t Q) { return q * T / Q; }

// pieces: a receiver's range of the spill stream touches consecutive chunks,
// so pieces <= spilled chunks + receivers - 1 < N + R (slots no longer bound
// them once pieces may read their weights remotely)
__host__ __device__ inline int64_t max_pieces(int R, int L, int B) {
    (void)B;
    return (int64_t)R * L + R;
}

// Fills the layout for a plan whose dispatch numbers the copies of T tokens:
// all R*S of them on one GPU (compute_layout), or one rank's S under expert
// parallelism, where each rank dispatches its own tokens.
__host__ __device__ inline void compute_layout_tokens(const moonep_cfg_t &c, int64_t T, moonep_ws_layout_t &l) {
    const int64_t N = (int64_t)c.R * c.L, R = c.R;
    const int64_t RB = (int64_t)c.R * c.B > 0 ? (int64_t)c.R * c.B : 1;
    const int64_t P = max_pieces(c.R, c.L, c.B);
    const int64_t NR = 2 * N + P;
    const int64_t SEG = R * (2 * (int64_t)c.L + c.B);
    int64_t o = MOONEP_WS_HEADER_WORDS;
    l.n_ranges = num_ranges(T, N);
    l.n_blocks = num_blocks(l.n_ranges);
    l.max_pieces = P;
    l.cnt = o; o += N;
    l.keep = o; o += N;
    l.spill = o; o += N;
    l.home_off = o; o += N;
    l.fb_cnt = o; o += N;
    l.fb_off = o; o += N;
    l.load = o; o += R;
    l.deficit = o; o += R;
    l.fill = o; o += R;
    l.slots_used = o; o += R;
    l.slot_expert = o; o += RB;
    l.slot_cnt = o; o += RB;
    l.slot_off = o; o += RB;
    l.slot_first_j = o; o += RB;
    l.rep_ptr = o; o += N + 1;
    l.rep_expert = o; o += P;
    l.rep_recv = o; o += P;
    l.rep_slot = o; o += P;
    l.rep_first_j = o; o += P;
    l.rep_cnt = o; o += P;
    l.rep_off = o; o += P;
    l.recv_ptr = o; o += R + 1;
    l.slot_piece = o; o += RB;
    l.rx_expert = o; o += N;
    l.route_ptr = o; o += N + 1;
    l.route_end = o; o += NR;
    l.route_base = o; o += NR;
    l.seg_off = o; o += SEG;
    l.seg_len = o; o += SEG;
    l.alloc = o; o += N * R;
    o = (o + 3) & ~(int64_t)3;
    l.tables_end = o;
    l.base = o;
    o += N * (l.n_ranges > 0 ? l.n_ranges : 1);
    l.blk = o;
    o += N * (l.n_blocks > 0 ? l.n_blocks : 1);
    o = (o + 3) & ~(int64_t)3;
    l.words = o;
}

__host__ __device__ inline void compute_layout(const moonep_cfg_t &c, moonep_ws_layout_t &l) {
    compute_layout_tokens(c, (int64_t)c.R * c.S, l);
}

// ---------------------------------------------------------------------------
// kernel parameter blocks
// ---------------------------------------------------------------------------
// plan kernel modes: the whole plan of one GPU's R*S tokens (kPlanFull);
// under expert parallelism, first the counts of one rank's S tokens
// (kPlanCount: histogram into counts_out, per-range scratch into ws), then,
// once every rank's counts are gathered, the plan from them
// (kPlanFromCounts: identical tables on every rank, and this rank's copy
// numbers offset by the copies of the lower ranks)
enum : int32_t { kPlanFull = 0, kPlanCount = 1, kPlanFromCounts = 2 };

struct PlanParams {
    moonep_cfg_t cfg;
    int32_t flags;
    int32_t N;
    int64_t T, Q;
    const int32_t *ids;
    int32_t *ws;
    moonep_ws_layout_t lay;
    int64_t wait_limit;
    int32_t mode;              // kPlan*
    int32_t rank;              // expert-parallel rank (kPlanCount, kPlanFromCounts)
    int32_t *counts_out;       // kPlanCount: [N + 1] (counts, then status bits)
    const int32_t *counts_all; // kPlanFromCounts: [R][N + 1], every rank's counts_out
    int32_t *const *counts_peers; // kPlanCount: device table [R] of every rank's counts_all, or NULL
    uint64_t mK, mT;           // floor((2^64 - 1) / d) + 1 for d = K and d = T (set at launch)
};

struct DispatchParams {
    moonep_cfg_t cfg;
    int32_t N;
    int32_t npc;          // pieces per row
    int64_t T, Q;
    uint32_t row_bytes;   // H * 2
    uint32_t piece_bytes; // stage size; every piece but the last is this size
    const uint8_t *x;
    const int32_t *ids;
    uint8_t *recv;
    int32_t *dest;
    int32_t *ws;
    moonep_ws_layout_t lay;
    int64_t wait_limit;
    uint8_t *const *recv_peers;  // expert parallelism: every rank's receive buffer [C_max][H] (device array of R)
    int32_t ep_tag;              // 0, or rank + 1 under expert parallelism
};

struct CombineParams {
    moonep_cfg_t cfg;
    int64_t T;
    int64_t units;        // T * units_per_token
    int32_t upt;          // units (row chunks) per token
    int32_t hv;           // 16-byte vectors per row (H / 8)
    int64_t rows_total;   // R * C_max
    uint32_t chunk_bytes; // bytes of each of the K rows per unit (last chunk may be shorter)
    int32_t stages;       // shared-memory stages
    const uint4 *y;
    const int32_t *dest;
    const float *w;
    uint4 *out;
    int32_t *ws;
    int64_t wait_limit;
    const uint8_t *const *y_peers;  // expert parallelism: every rank's expert outputs [C_max][H]
    int32_t ep_tag;
};

struct BackwardParams {
    moonep_cfg_t cfg;
    int64_t T;
    int32_t hv;           // 16-byte vectors per row (H / 8)
    int32_t upt;          // row chunks per token
    uint32_t chunk_bytes; // bytes per row chunk (the last may be shorter)
    int32_t stages;       // shared-memory stages
    int64_t rows_total;   // R * C_max
    int64_t wait_limit;
    const uint4 *grad_out;
    const uint4 *y;       // may be NULL when grad_w is NULL
    const int32_t *dest;
    const float *w;
    uint4 *grad_y;
    float *grad_w;        // may be NULL
    int32_t *ws;
    // expert parallelism (NULL otherwise): row dest[t][k] = q * C_max + j is
    // row j of rank q's buffer, reached through these device tables [R]
    const uint8_t *const *y_peers;
    uint8_t *const *grad_y_peers;
    int32_t ep_tag;       // rank + 1, or 0
};

struct CopyParams {
    moonep_cfg_t cfg;
    int64_t wait_limit;
    int64_t vecs;         // 16-byte vectors per expert
    const uint4 *src;
    uint4 *dst;
    int32_t *ws;
    moonep_ws_layout_t lay;
    // expert parallelism (ep_tag = rank + 1): prefetch reads the home ranks'
    // weights [L][elems] through peers and writes this rank's slots [B][elems]
    // (dst); reduce_grad adds the receivers' replica slots [B][elems] (read
    // and cleared through peers) into this rank's gradients [L][elems] (src)
    uint8_t *const *peers;
    int32_t ep_tag;
};

struct CopyOutParams {
    moonep_cfg_t cfg;
    int64_t Q;            // token ranges of the plan (workspace check)
    int64_t wait_limit;
    int64_t row_vecs;     // 16-byte vectors per row
    const uint4 *src;     // receive buffer [R, C_max, H]
    uint4 *dst;           // the caller's copy, same shape
    int32_t *ws;
    moonep_ws_layout_t lay;
};
constexpr int kCopyOutThreads = 256;

// ---------------------------------------------------------------------------
// device helpers
// ---------------------------------------------------------------------------
#ifdef __CUDACC__
__device__ __forceinline__ int ld_cg(const int32_t *p) { return __ldcg(p); }

// Whether the workspace status holds an error bit, read once by thread 0 and
// shared with the whole CTA: another CTA may set a bit at any moment, and the
// threads of one CTA must take the same early exit.
__device__ __forceinline__ bool block_status_failed(const int32_t *ws) {
    __shared__ int s_failed;
    if (threadIdx.x == 0) s_failed = (__ldcg(ws + HDR_STATUS) & MOONEP_ST_ERROR_MASK) != 0;
    __syncthreads();
    return s_failed != 0;
}

// Whether the workspace holds a plan for this configuration, token ranges
// and kind (ep_tag: 0 for a single-GPU plan, rank + 1 for an expert-parallel
// rank's).
__device__ __forceinline__ bool cfg_matches(const int32_t *ws, const moonep_cfg_t &c, int64_t Q, int32_t ep_tag = 0) {
    const int32_t *h = ws + HDR_CFG;
    return __ldcg(h + 0) == c.R && __ldcg(h + 1) == c.L && __ldcg(h + 2) == c.S &&
           __ldcg(h + 3) == c.K && __ldcg(h + 4) == c.H && __ldcg(h + 5) == c.B &&
           __ldcg(h + 6) == c.C && __ldcg(h + 7) == c.C_max && __ldcg(ws + HDR_NRANGES) == (int32_t)Q &&
           __ldcg(ws + HDR_EP) == ep_tag;
}

// A workspace whose header word HDR_TABLES_ONLY holds this value is a copy of
// the plan header and tables alone (moonep_plan_noalloc's output): it lacks
// the dispatch scratch (base, blk) that lies past tables_end.  The value is a
// repeated byte so a single-word memset writes it.
constexpr int32_t kTablesOnlyMark = 0x5A5A5A5A;

__device__ __forceinline__ bool tables_only(const int32_t *ws) {
    return __ldcg(ws + HDR_TABLES_ONLY) == kTablesOnlyMark;
}

__device__ __forceinline__ unsigned lanemask_lt() {
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// bounded mbarrier wait; returns false if it gave up after `limit` polls
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity, int64_t limit) {
    int64_t n = 0;
    while (!mbar_try_wait(bar, parity))
        if (++n > limit) return false;
    return true;
}

// barrier over the `count` threads of named barrier `id` (id 0 is __syncthreads)
__device__ __forceinline__ void named_barrier(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// TMA bulk copy global -> shared, completion counted on an mbarrier
__device__ __forceinline__ void bulk_g2s(void *dst_smem, const void *src, uint32_t bytes, uint64_t *bar,
                                         uint64_t pol) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
            smem_u32(dst_smem)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(pol)
        : "memory");
}

// TMA bulk copy shared -> global, tracked by bulk async-groups (no cache hint)
__device__ __forceinline__ void bulk_s2g_plain(void *dst, const void *src_smem, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(smem_u32(src_smem)),
                 "r"(bytes)
                 : "memory");
}

// TMA bulk copy global -> shared without a cache hint
__device__ __forceinline__ void bulk_g2s_plain(void *dst_smem, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst_smem)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

// TMA bulk copy shared -> global, tracked by bulk async-groups
__device__ __forceinline__ void bulk_s2g(void *dst, const void *src_smem, uint32_t bytes, uint64_t pol) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group.L2::cache_hint [%0], [%1], %2, %3;" ::"l"(dst),
                 "r"(smem_u32(src_smem)), "r"(bytes), "l"(pol)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

template <int N>
__device__ __forceinline__ void bulk_wait_all() {
    asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ int warp_incl_scan(int v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int t = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += t;
    }
    return v;
}
#endif

}  // namespace moonep

namespace moonep {
// Raises a kernel's dynamic shared-memory limit on the current device only
// when a launch needs more than was set before, so steady-state launches make
// no attribute call (`cache` holds one entry per device).
//
// MOONEP_CARVEOUT (percent of the unified L1/shared storage given to shared
// memory, -1 = the driver's choice) is requested for every kernel alike, so
// consecutive kernels of a step never make the SM change its split.
#ifndef MOONEP_CARVEOUT
#define MOONEP_CARVEOUT -1
#endif
inline cudaError_t set_smem_limit(const void *func, size_t smem, std::atomic<size_t> *cache) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    const size_t want = smem > 0 ? smem : 1;
    if (cache[dev].load(std::memory_order_relaxed) >= want) return cudaSuccess;
    if (MOONEP_CARVEOUT >= 0) {
        e = cudaFuncSetAttribute(func, cudaFuncAttributePreferredSharedMemoryCarveout, MOONEP_CARVEOUT);
        if (e != cudaSuccess) return e;
    }
    e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess) cache[dev].store(want, std::memory_order_relaxed);
    return e;
}
}  // namespace moonep

// launchers (defined in the kernel files, called by the C ABI layer)
namespace moonep {
cudaError_t launch_plan(const PlanParams &p, int grid, size_t smem, cudaStream_t s);
size_t plan_smem_bytes(int N);
const void *plan_kernel_ptr();
cudaError_t launch_dispatch(const DispatchParams &p, size_t smem, cudaStream_t s);
cudaError_t dispatch_smem_config(int N, uint32_t row_bytes, int ctas_per_sm, uint32_t *piece_bytes,
                                 int *npc, size_t *smem, bool ep = false);
cudaError_t launch_combine(const CombineParams &p, int grid, size_t smem, cudaStream_t s);
cudaError_t combine_config(int K, int hv, uint32_t *chunk, int *upt, int *stages, size_t *smem, bool ep = false);
const void *combine_kernel_ptr();
cudaError_t launch_prefetch(const CopyParams &p, int grid, cudaStream_t s);
cudaError_t launch_reduce_grad(const CopyParams &p, int sms, cudaStream_t s);
int set_error(int code, const char *msg);
cudaError_t launch_copy_out(const CopyOutParams &p, int sms, cudaStream_t s);
cudaError_t launch_combine_backward(const BackwardParams &p, int grid, size_t smem, cudaStream_t s);
cudaError_t combine_backward_config(int K, int hv, bool with_grad_w, uint32_t *chunk, int *upt, int *stages,
                                    size_t *smem);
}  // namespace moonep
