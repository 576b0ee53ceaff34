// weights.cu -- moonep_prefetch and moonep_reduce_grad, the two
// bandwidth-bound kernels around the replicated experts (twodots.gr "MoonEP
// balances AI experts in MoE models", memory-contract paragraphs: weights of
// the duplicated experts are preloaded into the prefetch slots [E, E+B);
// their gradients go to a separate fp32 reduce buffer, and reduce_grad adds
// each rank's own experts' replica slots to the local parameter gradient and
// clears the used slots; "The Busiest Rank Sets Your Step Time", flowchart:
// weight prefetch, reduce_grad).
//
// Both walk a list the plan leaves in the workspace (the replica pieces, and
// the experts that have at least one) and split every expert into 32 KB
// chunks.  prefetch moves each chunk with TMA bulk copies (one warp per SM,
// a pipeline of shared-memory stages); reduce_grad hands chunks to a
// persistent grid whose threads keep two 16-byte vectors of the home gradient
// and up to four replicas each in flight before adding them in order.
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
constexpr uint32_t kPfChunk = MOONEP_PREFETCH_CHUNK;
constexpr int kPfStages = MOONEP_PREFETCH_STAGES;
constexpr int kPfAhead = MOONEP_PREFETCH_LOOKAHEAD;
static_assert(kPfStages - kPfAhead - 1 >= 0, "stage reuse needs an older store group");

// Prefetch: one warp per CTA, one CTA per SM; lane 0 runs a TMA pipeline over
// the units (piece, 32 KB chunk) of this CTA: bulk load global -> shared
// (mbarrier), bulk store shared -> global (bulk groups), kPfAhead loads in
// flight, a stage reused once its store has read it.  Every wait is bounded.
__global__ void __launch_bounds__(32, 1) prefetch_kernel(const __grid_constant__ CopyParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    int32_t *ws = p.ws;
    if (block_status_failed(ws)) return;
    if (!cfg_matches(ws, p.cfg, p.lay.n_ranges)) {
        if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(ws + HDR_STATUS, MOONEP_ST_CFG);
        return;
    }
    if (threadIdx.x != 0) return;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + (size_t)kPfStages * kPfChunk);
    for (int s = 0; s < kPfStages; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
    fence_proxy_async_smem();

    const int64_t P = __ldcg(ws + HDR_NSLOT);  // pieces with a slot (all, under the headroom rule)
    const int64_t bytes_per = p.vecs * 16;
    const int64_t cps = (bytes_per + kPfChunk - 1) / kPfChunk;
    const int64_t units = P * cps;
    const int64_t u0 = (int64_t)blockIdx.x * units / gridDim.x;
    const int64_t u1 = (int64_t)(blockIdx.x + 1) * units / gridDim.x;
    const int64_t n = u1 - u0;
    const int B = p.cfg.B;
    const uint8_t *src_base = reinterpret_cast<const uint8_t *>(p.src);
    uint8_t *dst_base = reinterpret_cast<uint8_t *>(p.dst);
    const uint64_t pol = policy_evict_first();
    bool fail = false;
    int64_t issued = 0, stored = 0;
    for (int64_t it = 0; it < n + kPfAhead; ++it) {
        if (it < n) {
            const int64_t u = u0 + it;
            const int64_t sp = u / cps, c = u - sp * cps;
            const int gp = __ldg(ws + p.lay.slot_piece + sp);
            const int e = __ldg(ws + p.lay.rep_expert + gp);
            const uint32_t bytes = (uint32_t)min((int64_t)kPfChunk, bytes_per - c * kPfChunk);
            const int s = (int)(it % kPfStages);
            if (it >= kPfStages) bulk_wait_read<kPfStages - kPfAhead - 1>();
            mbar_arrive_expect_tx(&bars[s], bytes);
            bulk_g2s(smem + (size_t)s * kPfChunk, src_base + (int64_t)e * bytes_per + c * kPfChunk, bytes, &bars[s],
                     pol);
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
            const int64_t u = u0 + j;
            const int64_t sp = u / cps, c = u - sp * cps;
            const int gp = __ldg(ws + p.lay.slot_piece + sp);
            const int64_t slot = (int64_t)__ldg(ws + p.lay.rep_recv + gp) * B + __ldg(ws + p.lay.rep_slot + gp);
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

__device__ __forceinline__ void add4(float4 &a, const float4 &b) {
    a.x = __fadd_rn(a.x, b.x);
    a.y = __fadd_rn(a.y, b.y);
    a.z = __fadd_rn(a.z, b.z);
    a.w = __fadd_rn(a.w, b.w);
}

// g_home[e] = (((g_home[e] + rep_1) + rep_2) + ...) in ascending receiver
// order (the plan's piece order within an expert), then rep_i = 0.  A
// persistent grid strides over the units (replicated expert, 32 KB chunk);
// consecutive units of a CTA are a grid apart, so every CTA sees every
// expert and the experts' different replica counts even out.
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

}  // namespace

cudaError_t launch_prefetch(const CopyParams &p, int grid, cudaStream_t s) {
    const size_t smem = (size_t)kPfStages * kPfChunk + kPfStages * 8;
    static std::atomic<size_t> smem_set[64];
    cudaError_t err = set_smem_limit((const void *)prefetch_kernel, smem, smem_set);
    if (err != cudaSuccess) return err;
    prefetch_kernel<<<grid, 32, smem, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_reduce_grad(const CopyParams &p, int sms, cudaStream_t s) {
    static std::atomic<size_t> smem_set[64];
    cudaError_t err = set_smem_limit((const void *)reduce_grad_kernel, 0, smem_set);
    if (err != cudaSuccess) return err;
    reduce_grad_kernel<<<sms * 8, kThreads, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace moonep
