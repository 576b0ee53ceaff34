// weights.cu -- moonep_prefetch and moonep_reduce_grad, the two
// bandwidth-bound kernels around the replicated experts (twodots.gr "MoonEP
// balances AI experts in MoE models", memory-contract paragraphs: weights of
// the duplicated experts are preloaded into the prefetch slots [E, E+B);
// their gradients go to a separate fp32 reduce buffer, and reduce_grad adds
// each rank's own experts' replica slots to the local parameter gradient and
// clears the used slots; "The Busiest Rank Sets Your Step Time", flowchart:
// weight prefetch, reduce_grad).
//
// Both walk lists the plan leaves in the workspace (the replica pieces, and
// the experts that have at least one).  prefetch moves 32 KB chunks with TMA
// bulk copies (one warp per SM, a pipeline of shared-memory stages), reading
// each chunk of a replicated expert once and storing it to every slot of
// that expert.
// reduce_grad deals units of a few KB of one expert's gradient to warps; each
// warp keeps two units' loads in flight (the next unit's home and replica
// vectors are loaded before the current unit is added and stored).  Under
// expert parallelism (kEp) both reach the other ranks' buffers through a
// table of peer pointers: prefetch reads the home rank's weights,
// reduce_grad reads and clears the receivers' replica gradients.
#include "moonep_internal.cuh"

namespace moonep {

namespace {

constexpr int kThreads = 256;
constexpr int kChunkVecs = 2048;   // 32 KB of fp32 per chunk

#ifndef MOONEP_PREFETCH_CHUNK
#define MOONEP_PREFETCH_CHUNK 32768  // bytes per bulk copy
#endif
#ifndef MOONEP_PREFETCH_STAGES
#define MOONEP_PREFETCH_STAGES 6
#endif
#ifndef MOONEP_PREFETCH_STORE_HINT
#define MOONEP_PREFETCH_STORE_HINT 1  // 1: evict-first L2 hint on the slot stores too
#endif
#ifndef MOONEP_PREFETCH_LOOKAHEAD
#define MOONEP_PREFETCH_LOOKAHEAD 4
#endif
#ifndef MOONEP_PREFETCH_ONCE
#define MOONEP_PREFETCH_ONCE 1  // 1: one read per replicated expert, stored to all its slots
#endif
#ifndef MOONEP_PREFETCH_ONCE_LOOKAHEAD
#define MOONEP_PREFETCH_ONCE_LOOKAHEAD 1  // loads ahead in the read-once pipeline (its store groups are larger)
#endif
constexpr int kPfOnceAhead = MOONEP_PREFETCH_ONCE_LOOKAHEAD;
static_assert(MOONEP_PREFETCH_STAGES - MOONEP_PREFETCH_ONCE_LOOKAHEAD - 1 >= 0, "stage reuse needs an older store group");
#ifndef MOONEP_PREFETCH_INTERLEAVE
#define MOONEP_PREFETCH_INTERLEAVE 0  // 1: units dealt to the CTAs round-robin instead of contiguous shares
#endif
constexpr uint32_t kPfChunk = MOONEP_PREFETCH_CHUNK;
constexpr int kPfStages = MOONEP_PREFETCH_STAGES;
constexpr int kPfAhead = MOONEP_PREFETCH_LOOKAHEAD;
static_assert(kPfStages - kPfAhead - 1 >= 0, "stage reuse needs an older store group");

// Prefetch: one warp per CTA, one CTA per SM; lane 0 runs a TMA pipeline over
// the units (piece, 32 KB chunk) of this CTA: bulk load global -> shared
// (mbarrier), bulk store shared -> global (bulk groups), kPfAhead loads in
// flight, a stage reused once its store has read it.  Every wait is bounded.
// The pieces are those with a slot: all of them on one GPU, this rank's
// (kEp; they are contiguous in the plan's slot-piece list, which is
// receiver-major) under expert parallelism, where the source is the home
// rank's weights [L][elems] through the peer table and the destination the
// rank's own slots [B][elems].
template <bool kEp>
__global__ void __launch_bounds__(32, 1) prefetch_kernel(const __grid_constant__ CopyParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    int32_t *ws = p.ws;
    if (block_status_failed(ws)) return;
    if (!cfg_matches(ws, p.cfg, p.lay.n_ranges, p.ep_tag)) {
        if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(ws + HDR_STATUS, MOONEP_ST_CFG);
        return;
    }
    if (threadIdx.x != 0) return;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + (size_t)kPfStages * kPfChunk);
    for (int s = 0; s < kPfStages; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
    fence_proxy_async_smem();

    const int B = p.cfg.B, L = p.cfg.L;
    // slotted pieces handled: [sp0, sp0 + P) of the slot-piece list
    int64_t sp0 = 0, P = 0;
    if (kEp) {
        const int rank = p.ep_tag - 1;
        for (int r = 0; r < rank; ++r) sp0 += __ldg(ws + p.lay.slots_used + r);
        P = __ldg(ws + p.lay.slots_used + rank);
    } else {
        P = __ldcg(ws + HDR_NSLOT);  // pieces with a slot (all, under the headroom rule)
    }
    const int64_t bytes_per = p.vecs * 16;
    const int64_t cps = (bytes_per + kPfChunk - 1) / kPfChunk;
    const int64_t units = P * cps;
    // the CTA's units: u0 + it * ustep for it < n
    const int64_t ustep = MOONEP_PREFETCH_INTERLEAVE ? gridDim.x : 1;
    const int64_t u0 = MOONEP_PREFETCH_INTERLEAVE ? blockIdx.x : (int64_t)blockIdx.x * units / gridDim.x;
    const int64_t n = MOONEP_PREFETCH_INTERLEAVE
                          ? (blockIdx.x < units ? (units - 1 - blockIdx.x) / gridDim.x + 1 : 0)
                          : (int64_t)(blockIdx.x + 1) * units / gridDim.x - u0;
    const uint8_t *src_base = reinterpret_cast<const uint8_t *>(p.src);
    uint8_t *dst_base = reinterpret_cast<uint8_t *>(p.dst);
    const uint64_t pol = policy_evict_first();
    bool fail = false;
    int64_t issued = 0, stored = 0;
    for (int64_t it = 0; it < n + kPfAhead; ++it) {
        if (it < n) {
            const int64_t u = u0 + it * ustep;
            const int64_t sp = u / cps, c = u - sp * cps;
            const int gp = __ldg(ws + p.lay.slot_piece + sp0 + sp);
            const int e = __ldg(ws + p.lay.rep_expert + gp);
            const uint8_t *src = kEp ? p.peers[e / L] + (int64_t)(e % L) * bytes_per : src_base + (int64_t)e * bytes_per;
            const uint32_t bytes = (uint32_t)min((int64_t)kPfChunk, bytes_per - c * kPfChunk);
            const int s = (int)(it % kPfStages);
            if (it >= kPfStages) bulk_wait_read<kPfStages - kPfAhead - 1>();
            mbar_arrive_expect_tx(&bars[s], bytes);
            bulk_g2s(smem + (size_t)s * kPfChunk, src + c * kPfChunk, bytes, &bars[s], pol);
            issued = it + 1;
        }
        const int64_t j = it - kPfAhead;
        if (j >= 0 && j < n) {
            const int s = (int)(j % kPfStages);
            int64_t w = 0;
            while (!mbar_try_wait(&bars[s], (uint32_t)((j / kPfStages) & 1)))
                if (++w > p.wait_limit) {
                    fail = true;
                    break;
                }
            if (fail) break;
            const int64_t u = u0 + j * ustep;
            const int64_t sp = u / cps, c = u - sp * cps;
            const int gp = __ldg(ws + p.lay.slot_piece + sp0 + sp);
            const int64_t slot = kEp ? (int64_t)__ldg(ws + p.lay.rep_slot + gp)
                                     : (int64_t)__ldg(ws + p.lay.rep_recv + gp) * B + __ldg(ws + p.lay.rep_slot + gp);
            const uint32_t bytes = (uint32_t)min((int64_t)kPfChunk, bytes_per - c * kPfChunk);
            if (MOONEP_PREFETCH_STORE_HINT)
                bulk_s2g(dst_base + slot * bytes_per + c * kPfChunk, smem + (size_t)s * kPfChunk, bytes, pol);
            else
                bulk_s2g_plain(dst_base + slot * bytes_per + c * kPfChunk, smem + (size_t)s * kPfChunk, bytes);
            bulk_commit();
            stored = j + 1;
        }
    }
    bulk_wait_all<0>();
    if (fail) {
        // let the loads still in flight land before the CTA exits
        const int64_t drain = p.wait_limit > (int64_t(1) << 20) ? p.wait_limit : (int64_t(1) << 20);
        for (int64_t u = stored; u < issued; ++u) {
            int64_t w = 0;
            while (!mbar_try_wait(&bars[u % kPfStages], (uint32_t)((u / kPfStages) & 1)))
                if (++w > drain) break;
        }
        atomicOr(ws + HDR_STATUS, MOONEP_ST_TIMEOUT);
    }
}

// Prefetch on one GPU, reading each replicated expert once: a unit is one
// 32 KB chunk of one replicated expert's weights, loaded into a stage once
// and stored from there to the slot of every piece of that expert (an expert
// replicated on n receivers costs one read and n writes, not n of each).
// Units are dealt to the CTAs round-robin, so every CTA gets a like mix of
// experts with few and many replicas.  Pieces without a slot (remote
// weights) take no copy; an expert with none is not read.  One load ahead
// (not four): a unit's store group is n times larger than its load, and with
// one load ahead four store groups may still be reading their stages when a
// stage is reused (training workload, kernel alone: 531 us with 1 ahead, 555
// with 2, 558 with 4; mid: 111, 113-115, 115).
__global__ void __launch_bounds__(32, 1) prefetch_once_kernel(const __grid_constant__ CopyParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    int32_t *ws = p.ws;
    if (block_status_failed(ws)) return;
    if (!cfg_matches(ws, p.cfg, p.lay.n_ranges, p.ep_tag)) {
        if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(ws + HDR_STATUS, MOONEP_ST_CFG);
        return;
    }
    if (threadIdx.x != 0) return;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + (size_t)kPfStages * kPfChunk);
    for (int s = 0; s < kPfStages; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
    fence_proxy_async_smem();

    const int B = p.cfg.B;
    const int64_t nrx = __ldcg(ws + HDR_NRX);
    const int64_t bytes_per = p.vecs * 16;
    const int64_t cps = (bytes_per + kPfChunk - 1) / kPfChunk;
    const int64_t units = nrx * cps;
    const int64_t u0 = blockIdx.x, ustep = gridDim.x;
    const int64_t n = blockIdx.x < units ? (units - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    const uint8_t *src_base = reinterpret_cast<const uint8_t *>(p.src);
    uint8_t *dst_base = reinterpret_cast<uint8_t *>(p.dst);
    const uint64_t pol = policy_evict_first();
    bool fail = false;
    int64_t issued = 0, stored = 0;
    for (int64_t it = 0; it < n + kPfOnceAhead; ++it) {
        if (it < n) {
            const int64_t u = u0 + it * ustep;
            const int64_t x = u / cps, c = u - x * cps;
            const int e = __ldg(ws + p.lay.rx_expert + x);
            const int pb = __ldg(ws + p.lay.rep_ptr + e), pe = __ldg(ws + p.lay.rep_ptr + e + 1);
            bool any = false;
            for (int q = pb; q < pe && !any; ++q) any = __ldg(ws + p.lay.rep_slot + q) >= 0;
            const uint32_t bytes = (uint32_t)min((int64_t)kPfChunk, bytes_per - c * kPfChunk);
            const int s = (int)(it % kPfStages);
            if (it >= kPfStages) bulk_wait_read<kPfStages - kPfOnceAhead - 1>();
            mbar_arrive_expect_tx(&bars[s], any ? bytes : 0u);
            if (any) bulk_g2s(smem + (size_t)s * kPfChunk, src_base + (int64_t)e * bytes_per + c * kPfChunk, bytes,
                              &bars[s], pol);
            issued = it + 1;
        }
        const int64_t j = it - kPfOnceAhead;
        if (j >= 0 && j < n) {
            const int s = (int)(j % kPfStages);
            int64_t w = 0;
            while (!mbar_try_wait(&bars[s], (uint32_t)((j / kPfStages) & 1)))
                if (++w > p.wait_limit) {
                    fail = true;
                    break;
                }
            if (fail) break;
            const int64_t u = u0 + j * ustep;
            const int64_t x = u / cps, c = u - x * cps;
            const int e = __ldg(ws + p.lay.rx_expert + x);
            const int pb = __ldg(ws + p.lay.rep_ptr + e), pe = __ldg(ws + p.lay.rep_ptr + e + 1);
            const uint32_t bytes = (uint32_t)min((int64_t)kPfChunk, bytes_per - c * kPfChunk);
            for (int q = pb; q < pe; ++q) {
                const int sl = __ldg(ws + p.lay.rep_slot + q);
                if (sl < 0) continue;
                const int64_t slot = (int64_t)__ldg(ws + p.lay.rep_recv + q) * B + sl;
                if (MOONEP_PREFETCH_STORE_HINT)
                    bulk_s2g(dst_base + slot * bytes_per + c * kPfChunk, smem + (size_t)s * kPfChunk, bytes, pol);
                else
                    bulk_s2g_plain(dst_base + slot * bytes_per + c * kPfChunk, smem + (size_t)s * kPfChunk, bytes);
            }
            bulk_commit();
            stored = j + 1;
        }
    }
    bulk_wait_all<0>();
    if (fail) {
        const int64_t drain = p.wait_limit > (int64_t(1) << 20) ? p.wait_limit : (int64_t(1) << 20);
        for (int64_t u = stored; u < issued; ++u) {
            int64_t w = 0;
            while (!mbar_try_wait(&bars[u % kPfStages], (uint32_t)((u / kPfStages) & 1)))
                if (++w > drain) break;
        }
        atomicOr(ws + HDR_STATUS, MOONEP_ST_TIMEOUT);
    }
}

__device__ __forceinline__ void add4(float4 &a, const float4 &b) {
    a.x = __fadd_rn(a.x, b.x);
    a.y = __fadd_rn(a.y, b.y);
    a.z = __fadd_rn(a.z, b.z);
    a.w = __fadd_rn(a.w, b.w);
}

// reduce_grad, CTA form (MOONEP_REDUCE_GRAD_CTA=1; one GPU only; kept to
// reproduce the comparison with the warp form): the same sums, a persistent
// grid striding over the units (replicated expert, 32 KB chunk), thread 0
// of each CTA collecting the unit's replica slots between two barriers.
__global__ void __launch_bounds__(kThreads) reduce_grad_kernel(const __grid_constant__ CopyParams p) {
    int32_t *ws = p.ws;
    if (block_status_failed(ws)) return;
    if (!cfg_matches(ws, p.cfg, p.lay.n_ranges)) {
        if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(ws + HDR_STATUS, MOONEP_ST_CFG);
        return;
    }
    __shared__ int64_t s_slot[64];   // replica slots of the unit's expert (<= R <= 64)
    const int64_t nrx = __ldcg(ws + HDR_NRX);
    const int64_t cps = (p.vecs + kChunkVecs - 1) / kChunkVecs;
    const int64_t units = nrx * cps;
    const int B = p.cfg.B;
    float4 *g_home = reinterpret_cast<float4 *>(const_cast<uint4 *>(p.src));
    float4 *g_rep = reinterpret_cast<float4 *>(p.dst);
    constexpr int kRepBatch = 4;
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int64_t u = blockIdx.x; u < units; u += gridDim.x) {
        const int64_t x = u / cps, c = u - x * cps;
        const int e = __ldg(ws + p.lay.rx_expert + x);
        const int pb = __ldg(ws + p.lay.rep_ptr + e), pe = __ldg(ws + p.lay.rep_ptr + e + 1);
        __shared__ int s_np;
        __syncthreads();  // s_slot and s_np of the previous unit are no longer read
        if (threadIdx.x == 0) {
            // the expert's pieces in receiver order; pieces without a slot
            // (remote weights) carry no replica gradient
            int n = 0;
            for (int q = pb; q < pe; ++q) {
                const int sl = __ldg(ws + p.lay.rep_slot + q);
                if (sl >= 0) s_slot[n++] = ((int64_t)__ldg(ws + p.lay.rep_recv + q) * B + sl) * p.vecs;
            }
            s_np = n;
        }
        __syncthreads();
        const int np = s_np;
        const int64_t n = min((int64_t)kChunkVecs, p.vecs - c * kChunkVecs);
        const int64_t off = c * kChunkVecs;
        float4 *home = g_home + (int64_t)e * p.vecs + off;
        for (int64_t i = threadIdx.x; i < n; i += 2 * kThreads) {
            const int64_t i2 = i + kThreads;
            const bool two = i2 < n;
            float4 a0 = __ldcs(home + i);
            float4 a1 = two ? __ldcs(home + i2) : z;
            for (int q0 = 0; q0 < np; q0 += kRepBatch) {
                float4 r0[kRepBatch], r1[kRepBatch];
#pragma unroll
                for (int qq = 0; qq < kRepBatch; ++qq) {
                    if (q0 + qq < np) {
                        const float4 *rp = g_rep + s_slot[q0 + qq] + off;
                        r0[qq] = __ldcs(rp + i);
                        r1[qq] = two ? __ldcs(rp + i2) : z;
                    }
                }
#pragma unroll
                for (int qq = 0; qq < kRepBatch; ++qq)
                    if (q0 + qq < np) {
                        add4(a0, r0[qq]);
                        add4(a1, r1[qq]);
                    }
            }
            __stcs(home + i, a0);
            if (two) __stcs(home + i2, a1);
            for (int q = 0; q < np; ++q) {
                float4 *rp = g_rep + s_slot[q] + off;
                __stcs(rp + i, z);
                if (two) __stcs(rp + i2, z);
            }
        }
    }
}


// reduce_grad: g_home[e] = (((g_home[e] + rep_1) + rep_2) + ...) in ascending
// receiver order (the plan's piece order within an expert), then rep_i = 0.
// Each CTA first copies the plan's lists (replicated experts, their piece
// ranges, and every piece's slot) into shared memory once.  Then every warp
// strides over units of 32 x kRgVecs 16-byte vectors of one replicated
// expert, unit u going to warp u mod (warps in the grid), so the warps in
// flight at any moment work on neighbouring stretches of the same
// gradients.  A warp loads its next unit (home vectors and the first
// kRgBatch replicas) before it adds and stores the current one, so two
// units' loads are in flight per warp; no barrier separates units.  On the
// mid workload (3 replicated experts, 8 replicas, 1.29 GB) this runs 207 us
// against 230 us for the CTA form; the form without the look-ahead unit
// (8 vectors per lane, 2 replicas per batch) ran 210 us.
//
// kEp: expert parallelism.  Only the rank's own experts (a contiguous
// stretch of the ascending replicated-expert list), their home gradients
// [L][elems] local, each replica read and cleared through the peer table.
#ifndef MOONEP_RG_VECS
#define MOONEP_RG_VECS 6
#endif
#ifndef MOONEP_RG_BATCH
#define MOONEP_RG_BATCH 1
#endif
#ifndef MOONEP_RG_THREADS
#define MOONEP_RG_THREADS 256
#endif
#ifndef MOONEP_RG_MINB
#define MOONEP_RG_MINB 1  // CTAs per SM the register budget is set for
#endif
constexpr int kRgVecs = MOONEP_RG_VECS;
constexpr int kRgBatch = MOONEP_RG_BATCH;
constexpr int kRgThreads = MOONEP_RG_THREADS;
constexpr int kRgUnit = 32 * kRgVecs;

template <bool kEp>
__global__ void __launch_bounds__(kRgThreads, MOONEP_RG_MINB) reduce_grad_pipe_kernel(const __grid_constant__ CopyParams p) {
    extern __shared__ __align__(16) int rg_sm[];
    int32_t *ws = p.ws;
    if (block_status_failed(ws)) return;
    if (!cfg_matches(ws, p.cfg, p.lay.n_ranges, p.ep_tag)) {
        if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(ws + HDR_STATUS, MOONEP_ST_CFG);
        return;
    }
    const int N = p.cfg.R * p.cfg.L, B = p.cfg.B, L = p.cfg.L;
    const int nrx_all = __ldcg(ws + HDR_NRX);
    const int P = __ldcg(ws + HDR_NREP);
    // [N] expert, [N] first piece, [N] end piece, [max_pieces] slot, then
    // (kEp) the peer table, 8-byte aligned
    int *s_e = rg_sm, *s_pb = rg_sm + N, *s_pe = rg_sm + 2 * N, *s_slot = rg_sm + 3 * N;
    float4 **s_peer = reinterpret_cast<float4 **>(rg_sm + ((3 * N + p.lay.max_pieces + 1) & ~1));
    // the replicated experts handled: all, or (kEp) the rank's own, which
    // form the stretch [x0, x0 + nrx) of the ascending list
    int x0 = 0, nrx = nrx_all;
    if (kEp) {
        const int lo = (p.ep_tag - 1) * L, hi = lo + L;
        int below = 0, mine = 0;
        for (int b0 = 0; b0 < nrx_all; b0 += kRgThreads) {
            const int x = b0 + threadIdx.x;
            const int e = x < nrx_all ? __ldcg(ws + p.lay.rx_expert + x) : N;
            below += __syncthreads_count(e < lo);
            mine += __syncthreads_count(e >= lo && e < hi);
        }
        x0 = below;
        nrx = mine;
        for (int r = threadIdx.x; r < p.cfg.R; r += kRgThreads) s_peer[r] = reinterpret_cast<float4 *>(p.peers[r]);
    }
    for (int x = threadIdx.x; x < nrx; x += kRgThreads) {
        const int e = __ldcg(ws + p.lay.rx_expert + x0 + x);
        s_e[x] = kEp ? e - (p.ep_tag - 1) * L : e;  // row of the home gradient array
        s_pb[x] = __ldcg(ws + p.lay.rep_ptr + e);
        s_pe[x] = __ldcg(ws + p.lay.rep_ptr + e + 1);
    }
    // slot of every piece as receiver * B + slot; -1: no slot (remote
    // weights: such a piece has no replica gradient)
    for (int q = threadIdx.x; q < P; q += kRgThreads) {
        const int sl = __ldcg(ws + p.lay.rep_slot + q);
        s_slot[q] = sl >= 0 ? __ldcg(ws + p.lay.rep_recv + q) * B + sl : -1;
    }
    __syncthreads();

    const int lane = threadIdx.x & 31;
    constexpr int kWarpsPerCta = kRgThreads / 32;
    const int64_t gw = (int64_t)blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
    const int64_t tw = (int64_t)gridDim.x * kWarpsPerCta;
    const int64_t vecs = p.vecs;
    const int64_t upe = (vecs + kRgUnit - 1) / kRgUnit;
    const int64_t units = (int64_t)nrx * upe;
    float4 *g_home = reinterpret_cast<float4 *>(const_cast<uint4 *>(p.src));
    float4 *g_rep = reinterpret_cast<float4 *>(p.dst);
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    auto replica = [&](int sl) -> float4 * {
        return kEp ? s_peer[sl / B] + (int64_t)(sl % B) * vecs : g_rep + (int64_t)sl * vecs;
    };

    struct Unit {
        int64_t off;
        int e, pb, pe;
    };
    auto meta = [&](int64_t u) {
        Unit m;
        const int x = (int)(u / upe);
        m.off = (u - (int64_t)x * upe) * kRgUnit + lane;
        m.e = s_e[x];
        m.pb = s_pb[x];
        m.pe = s_pe[x];
        return m;
    };
    auto load_batch = [&](const Unit &m, int q0, float4 (&r)[kRgBatch][kRgVecs], int (&sl)[kRgBatch]) {
#pragma unroll
        for (int qq = 0; qq < kRgBatch; ++qq) {
            sl[qq] = q0 + qq < m.pe ? s_slot[q0 + qq] : -1;
            const float4 *rp = replica(sl[qq] < 0 ? 0 : sl[qq]);
#pragma unroll
            for (int v = 0; v < kRgVecs; ++v) {
                const int64_t i = m.off + 32 * v;
                r[qq][v] = (sl[qq] >= 0 && i < vecs) ? __ldcs(rp + i) : z;
            }
        }
    };
    auto add_batch = [&](float4 (&h)[kRgVecs], float4 (&r)[kRgBatch][kRgVecs], int (&sl)[kRgBatch]) {
#pragma unroll
        for (int qq = 0; qq < kRgBatch; ++qq)
            if (sl[qq] >= 0) {
#pragma unroll
                for (int v = 0; v < kRgVecs; ++v) add4(h[v], r[qq][v]);
            }
    };
    auto load = [&](const Unit &m, float4 (&h)[kRgVecs], float4 (&r)[kRgBatch][kRgVecs], int (&sl)[kRgBatch]) {
        const float4 *home = g_home + (int64_t)m.e * vecs;
#pragma unroll
        for (int v = 0; v < kRgVecs; ++v) {
            const int64_t i = m.off + 32 * v;
            h[v] = i < vecs ? __ldcs(home + i) : z;
        }
        load_batch(m, m.pb, r, sl);
    };
    auto finish = [&](const Unit &m, float4 (&h)[kRgVecs], float4 (&r)[kRgBatch][kRgVecs], int (&sl)[kRgBatch]) {
        add_batch(h, r, sl);
        // replicas beyond the first batch: loaded and added here
        for (int q0 = m.pb + kRgBatch; q0 < m.pe; q0 += kRgBatch) {
            load_batch(m, q0, r, sl);
            add_batch(h, r, sl);
        }
        float4 *home = g_home + (int64_t)m.e * vecs;
#pragma unroll
        for (int v = 0; v < kRgVecs; ++v) {
            const int64_t i = m.off + 32 * v;
            if (i < vecs) __stcs(home + i, h[v]);
        }
        for (int q = m.pb; q < m.pe; ++q) {
            const int sq = s_slot[q];
            if (sq < 0) continue;
            float4 *rp = replica(sq);
#pragma unroll
            for (int v = 0; v < kRgVecs; ++v) {
                const int64_t i = m.off + 32 * v;
                if (i < vecs) __stcs(rp + i, z);
            }
        }
    };

    float4 ha[kRgVecs], ra[kRgBatch][kRgVecs], hb[kRgVecs], rb[kRgBatch][kRgVecs];
    int sla[kRgBatch], slb[kRgBatch];
    if (gw >= units) return;
    Unit ma = meta(gw);
    load(ma, ha, ra, sla);
    for (int64_t u = gw; u < units; u += 2 * tw) {
        const bool has_b = u + tw < units;
        Unit mb;
        if (has_b) {
            mb = meta(u + tw);
            load(mb, hb, rb, slb);
        }
        finish(ma, ha, ra, sla);
        if (!has_b) break;
        if (u + 2 * tw < units) {
            ma = meta(u + 2 * tw);
            load(ma, ha, ra, sla);
        }
        finish(mb, hb, rb, slb);
    }
}

}  // namespace

#ifndef MOONEP_PREFETCH_CTAS_PER_SM
#define MOONEP_PREFETCH_CTAS_PER_SM 1
#endif
cudaError_t launch_prefetch(const CopyParams &p, int grid, cudaStream_t s) {
    grid *= MOONEP_PREFETCH_CTAS_PER_SM;
    const size_t smem = (size_t)kPfStages * kPfChunk + kPfStages * 8;
    if (p.peers) {
        static std::atomic<size_t> smem_set_ep[64];
        cudaError_t err = set_smem_limit((const void *)prefetch_kernel<true>, smem, smem_set_ep);
        if (err != cudaSuccess) return err;
        prefetch_kernel<true><<<grid, 32, smem, s>>>(p);
        return cudaGetLastError();
    }
    if (MOONEP_PREFETCH_ONCE) {
        static std::atomic<size_t> smem_set1[64];
        cudaError_t err = set_smem_limit((const void *)prefetch_once_kernel, smem, smem_set1);
        if (err != cudaSuccess) return err;
        prefetch_once_kernel<<<grid, 32, smem, s>>>(p);
        return cudaGetLastError();
    }
    static std::atomic<size_t> smem_set[64];
    cudaError_t err = set_smem_limit((const void *)prefetch_kernel<false>, smem, smem_set);
    if (err != cudaSuccess) return err;
    prefetch_kernel<false><<<grid, 32, smem, s>>>(p);
    return cudaGetLastError();
}

#ifndef MOONEP_REDUCE_GRAD_CTA
#define MOONEP_REDUCE_GRAD_CTA 0
#endif
#ifndef MOONEP_RG_CTAS_PER_SM
#define MOONEP_RG_CTAS_PER_SM 0  // 0: as many as fit (occupancy)
#endif

template <bool kEp>
static cudaError_t launch_reduce_grad_pipe(const CopyParams &p, int sms, cudaStream_t s) {
    const int N = p.cfg.R * p.cfg.L;
    const size_t smem = (size_t)(((3 * N + p.lay.max_pieces + 1) & ~1) + 2 * 64) * sizeof(int);
    const void *fn = (const void *)reduce_grad_pipe_kernel<kEp>;
    static std::atomic<size_t> smem_set[64];
    static std::atomic<int> per_sm_cache[64];
    cudaError_t err = set_smem_limit(fn, smem, smem_set);
    if (err != cudaSuccess) return err;
    int per_sm = MOONEP_RG_CTAS_PER_SM;
    if (per_sm <= 0) {
        // CTAs per SM for this shared-memory size, cached per device (the
        // size follows N; recomputed when it changes)
        int dev = 0;
        err = cudaGetDevice(&dev);
        if (err != cudaSuccess) return err;
        const int key = (int)(smem & 0x7fffffff);
        static std::atomic<int> smem_key[64];
        if (dev >= 0 && dev < 64 && smem_key[dev].load() == key && per_sm_cache[dev].load() > 0) {
            per_sm = per_sm_cache[dev].load();
        } else {
            err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kRgThreads, smem);
            if (err != cudaSuccess) return err;
            if (per_sm < 1) per_sm = 1;
            if (dev >= 0 && dev < 64) {
                per_sm_cache[dev].store(per_sm);
                smem_key[dev].store(key);
            }
        }
    }
    reduce_grad_pipe_kernel<kEp><<<sms * per_sm, kRgThreads, smem, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_reduce_grad(const CopyParams &p, int sms, cudaStream_t s) {
    if (p.peers) return launch_reduce_grad_pipe<true>(p, sms, s);
    if (MOONEP_REDUCE_GRAD_CTA) {
        static std::atomic<size_t> smem_set[64];
        cudaError_t err = set_smem_limit((const void *)reduce_grad_kernel, 0, smem_set);
        if (err != cudaSuccess) return err;
        reduce_grad_kernel<<<sms * 8, kThreads, 0, s>>>(p);
        return cudaGetLastError();
    }
    return launch_reduce_grad_pipe<false>(p, sms, s);
}

}  // namespace moonep
