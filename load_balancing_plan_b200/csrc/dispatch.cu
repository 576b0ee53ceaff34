// dispatch.cu -- moonep_dispatch: sender-side destination rows fused with the
// row scatter of the hidden states ("The Busiest Rank Sets Your Step Time:
// Running MoonEP's Planning Code Ourselves", section "What the technique is":
// the sending side computes the receiver's final per-expert position and
// writes there, so no receive-buffer-to-compute-buffer copy exists;
// agentlenshq "MoonshotAI/MoonEP", "How it works": fused permute).
//
// One CTA per token range (the ranges the plan counted: about 4 tokens each;
// the grid is a whole number of waves of two CTAs per SM, and at H = 7168 a
// CTA's 66 KB of shared memory lets three be resident; at any moment the
// stores of all CTAs go to neighbouring rows of each expert's segment).  Warp 0
// numbers the range's copies in ascending g: for each group of 32 ids it
// finds equal experts with __match_any_sync, ranks lanes within a group by
// popcount, and adds a per-expert running counter kept in shared memory
// (initialised from the plan's base + blk prefixes), which gives the copy index
// j of every (token, k); j maps to a flat row through the expert's route
// entries.  Lane 0 then moves the data with TMA bulk copies: each row piece
// of x is loaded once into a shared-memory stage (mbarrier completion) and
// stored K times straight to its destination rows (bulk async-groups), with
// kLookahead loads in flight ahead of the stores.  Numbering runs just ahead
// of the copies, so its cost hides under them.  No multicast.
//
// MOONEP_DISPATCH_LOADER=1 builds a variant in which a loader warp fills the
// stages with 16-byte loads and the TMA unit only stores.  With one long
// token range per resident CTA it was 4% faster (the x loads no longer queued
// behind the stores); with the short ranges the plan makes, the plain
// TMA pipeline is about 1% ahead, so it is the default.
#include "moonep_internal.cuh"

namespace moonep {

namespace {

#ifndef MOONEP_DISPATCH_STAGES
#define MOONEP_DISPATCH_STAGES 8     // shared-memory stages
#endif
#ifndef MOONEP_DISPATCH_LOOKAHEAD
#define MOONEP_DISPATCH_LOOKAHEAD 6  // loads issued ahead of the stores
#endif
#ifndef MOONEP_DISPATCH_LOADER
#define MOONEP_DISPATCH_LOADER 0     // 1: a loader warp fetches x with plain loads, TMA only stores; 0: TMA loads too
#endif
#ifndef MOONEP_DISPATCH_HINTS
#define MOONEP_DISPATCH_HINTS 3      // bit 0: evict-first on the x loads, bit 1: on the row stores
#endif
constexpr int kStages = MOONEP_DISPATCH_STAGES;
constexpr int kLookahead = MOONEP_DISPATCH_LOOKAHEAD;
constexpr int kRing = 2048;     // destination ring entries (ids)
constexpr uint32_t kMaxPiece = 32768;
static_assert(kStages - kLookahead - 1 >= 0, "stage reuse needs an older store group");

struct Smem {
    uint8_t *stages;
    uint64_t *bars;
    int32_t *ring;
    int32_t *ctr;
};

__device__ __forceinline__ Smem carve(uint8_t *base, uint32_t piece_bytes) {
    Smem s;
    s.stages = base;
    s.bars = reinterpret_cast<uint64_t *>(base + (size_t)kStages * piece_bytes);
    s.ring = reinterpret_cast<int32_t *>(s.bars + kStages);
    s.ctr = s.ring + kRing;
    return s;
}

// number the next 32 copies of the range (warp-wide)
__device__ __forceinline__ bool rank_group(const DispatchParams &p, const Smem &sm, int64_t g0, int64_t l0,
                                           int64_t nids) {
    const int lane = threadIdx.x & 31;
    const int32_t *ws = p.ws;
    const int64_t l = l0 + lane;
    const bool valid = l < nids;
    int e = valid ? __ldg(p.ids + g0 + l) : -1;
    bool bad = false;
    if (valid && (unsigned)e >= (unsigned)p.N) {
        e = -1;
        bad = true;
    }
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rin = __popc(peers & lanemask_lt());
    const int b = e >= 0 ? sm.ctr[e] : 0;
    __syncwarp();
    if (e >= 0 && rin == 0) sm.ctr[e] = b + __popc(peers);
    __syncwarp();
    int d = -1;
    if (e >= 0) {
        const int j = b + rin;
        const int pb = __ldg(ws + p.lay.route_ptr + e), pe = __ldg(ws + p.lay.route_ptr + e + 1);
        for (int x = pb; x < pe; ++x)
            if (j < __ldg(ws + p.lay.route_end + x)) {
                d = __ldg(ws + p.lay.route_base + x) + j;
                break;
            }
        if (d < 0 || (int64_t)d >= (int64_t)p.cfg.R * p.cfg.C_max) {
            d = -1;
            bad = true;
        }
    }
    if (valid) {
        sm.ring[l % kRing] = d;
        p.dest[g0 + l] = d;
    }
    __syncwarp();
    return __any_sync(0xffffffffu, bad);
}

// Copy numbers of range q start after the earlier ranges of its block and
// the earlier blocks (base + blk).  Only the counters of the experts the
// range routes to are read: each thread loads those of the ids it covers,
// kInitBatch ids at a time with all their loads in flight (equal ids store
// equal values), so the cost follows the range's ids, not the expert count.
constexpr int kInitBatch = 4;
__device__ __forceinline__ void init_counters(const DispatchParams &p, int32_t *ctr, int64_t q, int64_t g0,
                                              int64_t nids, int tid, int nthreads) {
    const int32_t *ws = p.ws;
    const int64_t NB = p.lay.n_blocks;
    const int32_t *base = ws + p.lay.base + q * p.N;                    // base[q][e] = base[e]
    const int32_t *blk = ws + p.lay.blk + block_of_range(q, p.Q, NB);   // blk[e][b] = blk[e * NB]
    for (int64_t l0 = 0; l0 < nids; l0 += (int64_t)kInitBatch * nthreads) {
        int e[kInitBatch], v[kInitBatch];
#pragma unroll
        for (int u = 0; u < kInitBatch; ++u) {
            const int64_t l = l0 + tid + (int64_t)u * nthreads;
            e[u] = l < nids ? __ldg(p.ids + g0 + l) : -1;
        }
#pragma unroll
        for (int u = 0; u < kInitBatch; ++u)
            if ((unsigned)e[u] < (unsigned)p.N)
                v[u] = __ldg(base + e[u]) + __ldg(blk + (int64_t)e[u] * NB);
#pragma unroll
        for (int u = 0; u < kInitBatch; ++u)
            if ((unsigned)e[u] < (unsigned)p.N) ctr[e[u]] = v[u];
    }
}

// kEp: expert parallelism.  The CTA's tokens are one rank's (T = S), their
// copy numbers start after the lower ranks' copies (the plan's blk prefix
// carries them), and a row goes to the receive buffer of its destination
// rank through a table of peer pointers (kept in shared memory after the
// counters) instead of one buffer [R][C_max][H].
template <bool kEp>
__global__ void __launch_bounds__(32, 1) dispatch_kernel(const __grid_constant__ DispatchParams p) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    const int lane = threadIdx.x;
    int32_t *ws = p.ws;
    const int64_t q = blockIdx.x;
    if (block_status_failed(ws)) return;
    // a tables-only copy has no base/blk scratch: refuse it before reading them
    if (!cfg_matches(ws, p.cfg, p.Q, p.ep_tag) || tables_only(ws)) {
        if (lane == 0) atomicOr(ws + HDR_STATUS, MOONEP_ST_CFG);
        return;
    }
    const Smem sm = carve(smem_raw, p.piece_bytes);
    const int K = p.cfg.K, npc = p.npc;
    const int64_t t0 = range_begin(q, p.T, p.Q), t1 = range_begin(q + 1, p.T, p.Q);
    const int64_t ntok = t1 - t0;
    const int64_t g0 = t0 * K, nids = ntok * K;
    uint8_t **s_peer = reinterpret_cast<uint8_t **>(sm.ctr + ((p.N + 1) & ~1));
    if (kEp)
        for (int r = lane; r < p.cfg.R; r += 32) s_peer[r] = p.recv_peers[r];
    const int64_t Cm = p.cfg.C_max;
    init_counters(p, sm.ctr, q, g0, nids, lane, 32);
    if (lane == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(&sm.bars[s], 1);
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    __syncwarp();

    const int64_t nunits = ntok * npc;
    const uint32_t last_piece = p.row_bytes - (uint32_t)(npc - 1) * p.piece_bytes;
    const uint64_t pol = policy_evict_first();

    int64_t nranked = 0;
    bool bad = false;
    bool fail = false;
    int64_t issued = 0, stored = 0;
    for (int64_t it = 0; it < nunits + kLookahead; ++it) {
        if (it < nunits) {
            const int64_t i = it / npc;
            while (nranked < (i + 1) * K) {
                bad |= rank_group(p, sm, g0, nranked, nids);
                nranked = min(nranked + 32, nids);
            }
            if (lane == 0) {
                const int s = (int)(it % kStages);
                const int pc = (int)(it - i * npc);
                const uint32_t bytes = pc == npc - 1 ? last_piece : p.piece_bytes;
                if (it >= kStages) bulk_wait_read<kStages - kLookahead - 1>();
                mbar_arrive_expect_tx(&sm.bars[s], bytes);
                uint8_t *dsm = sm.stages + (size_t)s * p.piece_bytes;
                const uint8_t *src = p.x + (t0 + i) * (int64_t)p.row_bytes + (int64_t)pc * p.piece_bytes;
                if (MOONEP_DISPATCH_HINTS & 1)
                    bulk_g2s(dsm, src, bytes, &sm.bars[s], pol);
                else
                    bulk_g2s_plain(dsm, src, bytes, &sm.bars[s]);
            }
            issued = it + 1;
        }
        const int64_t j = it - kLookahead;
        if (j >= 0 && j < nunits) {
            if (lane == 0) {
                const int s = (int)(j % kStages);
                const uint32_t par = (uint32_t)((j / kStages) & 1);
                int64_t n = 0;
                while (!mbar_try_wait(&sm.bars[s], par))
                    if (++n > p.wait_limit) {
                        fail = true;
                        break;
                    }
                if (!fail) {
                    const int64_t i = j / npc;
                    const int pc = (int)(j - i * npc);
                    const uint32_t bytes = pc == npc - 1 ? last_piece : p.piece_bytes;
                    const uint8_t *src = sm.stages + (size_t)s * p.piece_bytes;
                    for (int k = 0; k < K; ++k) {
                        const int d = sm.ring[(i * K + k) % kRing];
                        if (d >= 0) {
                            uint8_t *row = kEp ? s_peer[d / Cm] + (int64_t)(d % Cm) * p.row_bytes
                                               : p.recv + (int64_t)d * p.row_bytes;
                            uint8_t *dst = row + (int64_t)pc * p.piece_bytes;
                            if (MOONEP_DISPATCH_HINTS & 2)
                                bulk_s2g(dst, src, bytes, pol);
                            else
                                bulk_s2g_plain(dst, src, bytes);
                        }
                    }
                    bulk_commit();
                }
            }
            fail = __shfl_sync(0xffffffffu, (int)fail, 0) != 0;
            if (fail) break;
            stored = j + 1;
        }
    }
    if (lane == 0) {
        bulk_wait_all<0>();
        if (fail) {
            // let the loads still in flight land before the CTA exits (with a
            // limit of its own, at least 2^20 polls, whatever wait_limit is)
            const int64_t drain = p.wait_limit > (int64_t(1) << 20) ? p.wait_limit : (int64_t(1) << 20);
            for (int64_t u = stored; u < issued; ++u) {
                int64_t n = 0;
                while (!mbar_try_wait(&sm.bars[u % kStages], (uint32_t)((u / kStages) & 1)))
                    if (++n > drain) break;
            }
            atomicOr(ws + HDR_STATUS, MOONEP_ST_TIMEOUT);
        }
        if (bad) atomicOr(ws + HDR_STATUS, MOONEP_ST_DEST);
    }
}

// The same dispatch with the x rows fetched by kLoaderWarps loader warps
// with ordinary 16-byte loads (registers, then shared memory, a proxy fence
// and an mbarrier arrive), so the SM's TMA unit carries only the row stores.
// Warp 0 numbers the copies and issues the K bulk stores of each unit; once
// the store group of unit j - kRelease has read its stage, it hands that stage
// back on the stage's "empty" mbarrier.  Shared memory: stages, kStages "full"
// then kStages "empty" barriers, ring, counters.
#ifndef MOONEP_DISPATCH_LOADER_WARPS
#define MOONEP_DISPATCH_LOADER_WARPS 1
#endif
constexpr int kLoaderWarps = MOONEP_DISPATCH_LOADER_WARPS;
constexpr int kVec = 16;       // 16-byte vectors per lane per pass (8 KB per warp)
#ifndef MOONEP_DISPATCH_RELEASE
#define MOONEP_DISPATCH_RELEASE 2
#endif
constexpr int kRelease = MOONEP_DISPATCH_RELEASE;  // store groups left reading their stages
static_assert(kRelease >= 1 && kRelease < kStages, "a stage is handed back before its next load needs it");

__global__ void __launch_bounds__(32 * (1 + kLoaderWarps), 1)
    dispatch_loader_kernel(const __grid_constant__ DispatchParams p) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int32_t *ws = p.ws;
    const int64_t q = blockIdx.x;
    if (block_status_failed(ws)) return;
    if (!cfg_matches(ws, p.cfg, p.Q) || tables_only(ws)) {
        if (threadIdx.x == 0) atomicOr(ws + HDR_STATUS, MOONEP_ST_CFG);
        return;
    }
    Smem sm;
    sm.stages = smem_raw;
    sm.bars = reinterpret_cast<uint64_t *>(smem_raw + (size_t)kStages * p.piece_bytes);
    uint64_t *empty = sm.bars + kStages;
    sm.ring = reinterpret_cast<int32_t *>(empty + kStages);
    sm.ctr = sm.ring + kRing;
    const int K = p.cfg.K, npc = p.npc;
    {
        const int64_t t0 = range_begin(q, p.T, p.Q), t1 = range_begin(q + 1, p.T, p.Q);
        init_counters(p, sm.ctr, q, t0 * K, (t1 - t0) * K, threadIdx.x, blockDim.x);
    }
    if (threadIdx.x == 0) {
        for (int st = 0; st < kStages; ++st) {
            mbar_init(&sm.bars[st], 1);
            mbar_init(&empty[st], 1);
        }
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    __syncthreads();

    const int64_t t0 = range_begin(q, p.T, p.Q), t1 = range_begin(q + 1, p.T, p.Q);
    const int64_t ntok = t1 - t0;
    const int64_t g0 = t0 * K, nids = ntok * K;
    const int64_t nunits = ntok * npc;
    const uint32_t last_piece = p.row_bytes - (uint32_t)(npc - 1) * p.piece_bytes;

    if (warp > 0) {
        // ------------------------------------------------------ loaders
        for (int64_t u = warp - 1; u < nunits; u += kLoaderWarps) {
            const int st = (int)(u % kStages);
            int ok = 1;
            if (lane == 0 && u >= kStages)
                ok = mbar_wait_bounded(&empty[st], (uint32_t)(((u / kStages) - 1) & 1), p.wait_limit);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) {
                if (lane == 0) atomicOr(ws + HDR_STATUS, MOONEP_ST_TIMEOUT);
                break;
            }
            const int64_t i = u / npc;
            const int pc = (int)(u - i * npc);
            const uint32_t bytes = pc == npc - 1 ? last_piece : p.piece_bytes;
            const uint4 *src = reinterpret_cast<const uint4 *>(p.x + (t0 + i) * (int64_t)p.row_bytes +
                                                               (int64_t)pc * p.piece_bytes);
            uint4 *dst = reinterpret_cast<uint4 *>(sm.stages + (size_t)st * p.piece_bytes);
            const int nv = (int)(bytes >> 4);
            for (int v0 = 0; v0 < nv; v0 += 32 * kVec) {
                uint4 v[kVec];
#pragma unroll
                for (int k = 0; k < kVec; ++k)
                    if (v0 + lane + 32 * k < nv) v[k] = __ldcs(src + v0 + lane + 32 * k);
#pragma unroll
                for (int k = 0; k < kVec; ++k)
                    if (v0 + lane + 32 * k < nv) dst[v0 + lane + 32 * k] = v[k];
            }
            fence_proxy_async_smem();  // these generic-proxy writes before the bulk stores read them
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.bars[st]);
        }
        return;
    }
    // ---------------------------------------------------------- warp 0
    int64_t nranked = 0;
    bool bad = false, fail = false;
    for (int64_t j = 0; j < nunits; ++j) {
        const int64_t i = j / npc;
        while (nranked < (i + 1) * K) {
            bad |= rank_group(p, sm, g0, nranked, nids);
            nranked = min(nranked + 32, nids);
        }
        if (lane == 0) {
            const int st = (int)(j % kStages);
            if (!mbar_wait_bounded(&sm.bars[st], (uint32_t)((j / kStages) & 1), p.wait_limit)) {
                fail = true;
            } else {
                const int pc = (int)(j - i * npc);
                const uint32_t bytes = pc == npc - 1 ? last_piece : p.piece_bytes;
                const uint8_t *src = sm.stages + (size_t)st * p.piece_bytes;
                for (int k = 0; k < K; ++k) {
                    const int d = sm.ring[(i * K + k) % kRing];
                    if (d < 0) continue;
                    uint8_t *dst = p.recv + (int64_t)d * p.row_bytes + (int64_t)pc * p.piece_bytes;
                    if (MOONEP_DISPATCH_HINTS & 2)
                        bulk_s2g(dst, src, bytes, policy_evict_first());
                    else
                        bulk_s2g_plain(dst, src, bytes);
                }
                bulk_commit();
                bulk_wait_read<kRelease>();
                if (j >= kRelease) mbar_arrive(&empty[(j - kRelease) % kStages]);
            }
        }
        fail = __shfl_sync(0xffffffffu, (int)fail, 0) != 0;
        if (fail) break;
    }
    if (lane == 0) {
        bulk_wait_all<0>();
        if (fail) atomicOr(ws + HDR_STATUS, MOONEP_ST_TIMEOUT);
        if (bad) atomicOr(ws + HDR_STATUS, MOONEP_ST_DEST);
    }
}

}  // namespace

#ifndef MOONEP_DISPATCH_FILL_SMEM
#define MOONEP_DISPATCH_FILL_SMEM 0  // 1: at most ctas_per_sm resident CTAs (two: 25% slower than three)
#endif
// Shared memory: kStages pieces + barriers + ring + N counters (+ the peer
// table under expert parallelism), sized so that `ctas_per_sm` CTAs fit one
// SM (227 KB usable per SM on sm_100).
cudaError_t dispatch_smem_config(int N, uint32_t row_bytes, int ctas_per_sm, uint32_t *piece_bytes, int *npc,
                                 size_t *smem, bool ep) {
    const size_t budget = (size_t)(228 * 1024) / (size_t)ctas_per_sm - 1024;  // 1 KB reserved per CTA
    const size_t fixed = (size_t)kStages * 8 + (size_t)kRing * 4 + (size_t)N * 4 + 128 + (ep ? 8 + 64 * 8 : 0);
    if (budget <= fixed) return cudaErrorInvalidValue;
    size_t maxp = (budget - fixed) / kStages;
    if (maxp > kMaxPiece) maxp = kMaxPiece;
    maxp &= ~(size_t)127;
    if (maxp < 128) return cudaErrorInvalidValue;
    int n = (int)((row_bytes + maxp - 1) / maxp);
    uint32_t pb = (uint32_t)(((row_bytes + n - 1) / n + 127) & ~127u);  // 128-byte aligned stages
    while ((size_t)pb > maxp) {
        ++n;
        pb = (uint32_t)(((row_bytes + n - 1) / n + 127) & ~127u);
    }
    n = (int)((row_bytes + pb - 1) / pb);
    *piece_bytes = pb;
    *npc = n;
    *smem = (size_t)kStages * pb + fixed;
#if MOONEP_DISPATCH_FILL_SMEM
    // take the whole per-CTA budget, so that no more than ctas_per_sm CTAs
    // are resident on an SM
    if (*smem < budget) *smem = budget;
#endif
    return cudaSuccess;
}

cudaError_t launch_dispatch(const DispatchParams &p, size_t smem, cudaStream_t s) {
    if (p.recv_peers) {
        static std::atomic<size_t> smem_set_ep[64];
        cudaError_t err = set_smem_limit((const void *)dispatch_kernel<true>, smem, smem_set_ep);
        if (err != cudaSuccess) return err;
        dispatch_kernel<true><<<(unsigned)p.Q, 32, smem, s>>>(p);
        return cudaGetLastError();
    }
    if (MOONEP_DISPATCH_LOADER) {
        static std::atomic<size_t> smem_set2[64];
        const size_t smem2 = smem + (size_t)kStages * 8;  // the "empty" barriers
        cudaError_t err = set_smem_limit((const void *)dispatch_loader_kernel, smem2, smem_set2);
        if (err != cudaSuccess) return err;
        dispatch_loader_kernel<<<(unsigned)p.Q, 32 * (1 + kLoaderWarps), smem2, s>>>(p);
        return cudaGetLastError();
    }
    static std::atomic<size_t> smem_set[64];
    cudaError_t err = set_smem_limit((const void *)dispatch_kernel<false>, smem, smem_set);
    if (err != cudaSuccess) return err;
    dispatch_kernel<false><<<(unsigned)p.Q, 32, smem, s>>>(p);
    return cudaGetLastError();
}

}  // namespace moonep
