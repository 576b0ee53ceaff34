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
// the experts that have at least one), split every expert into 16 KB chunks
// and hand chunks to a persistent grid.  Vectors are 16 bytes wide; loads
// are issued before stores so each thread keeps several in flight.
#include "moonep_internal.cuh"

namespace moonep {

namespace {

constexpr int kThreads = 256;
constexpr int kChunkVecs = 1024;   // 16 KB per chunk
constexpr int kPerThread = kChunkVecs / kThreads;

__global__ void __launch_bounds__(kThreads) prefetch_kernel(const __grid_constant__ CopyParams p) {
    int32_t *ws = p.ws;
    if (__ldcg(ws + HDR_STATUS) & MOONEP_ST_ERROR_MASK) return;
    if (!cfg_matches(ws, p.cfg, p.lay.n_ranges)) {
        if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(ws + HDR_STATUS, MOONEP_ST_CFG);
        return;
    }
    const int64_t P = __ldcg(ws + HDR_NREP);
    const int64_t cps = (p.vecs + kChunkVecs - 1) / kChunkVecs;
    const int64_t units = P * cps;
    const int B = p.cfg.B;
    for (int64_t u = blockIdx.x; u < units; u += gridDim.x) {
        const int64_t gp = u / cps, c = u - gp * cps;
        const int e = __ldg(ws + p.lay.rep_expert + gp);
        const int64_t slot = (int64_t)__ldg(ws + p.lay.rep_recv + gp) * B + __ldg(ws + p.lay.rep_slot + gp);
        const uint4 *src = p.src + (int64_t)e * p.vecs + c * kChunkVecs;
        uint4 *dst = p.dst + slot * p.vecs + c * kChunkVecs;
        const int64_t n = min((int64_t)kChunkVecs, p.vecs - c * kChunkVecs);
        uint4 v[kPerThread];
#pragma unroll
        for (int i = 0; i < kPerThread; ++i) {
            const int64_t x = threadIdx.x + (int64_t)i * kThreads;
            if (x < n) v[i] = __ldcs(src + x);
        }
#pragma unroll
        for (int i = 0; i < kPerThread; ++i) {
            const int64_t x = threadIdx.x + (int64_t)i * kThreads;
            if (x < n) __stcs(dst + x, v[i]);
        }
    }
}

__device__ __forceinline__ void add4(float4 &a, const float4 &b) {
    a.x = __fadd_rn(a.x, b.x);
    a.y = __fadd_rn(a.y, b.y);
    a.z = __fadd_rn(a.z, b.z);
    a.w = __fadd_rn(a.w, b.w);
}

// g_home[e] = (((g_home[e] + rep_1) + rep_2) + ...) in ascending receiver
// order (the plan's piece order within an expert), then rep_i = 0.
__global__ void __launch_bounds__(kThreads) reduce_grad_kernel(const __grid_constant__ CopyParams p) {
    int32_t *ws = p.ws;
    if (__ldcg(ws + HDR_STATUS) & MOONEP_ST_ERROR_MASK) return;
    if (!cfg_matches(ws, p.cfg, p.lay.n_ranges)) {
        if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(ws + HDR_STATUS, MOONEP_ST_CFG);
        return;
    }
    const int64_t nrx = __ldcg(ws + HDR_NRX);
    const int64_t cps = (p.vecs + kChunkVecs - 1) / kChunkVecs;
    const int64_t units = nrx * cps;
    const int B = p.cfg.B;
    float4 *g_home = reinterpret_cast<float4 *>(const_cast<uint4 *>(p.src));
    float4 *g_rep = reinterpret_cast<float4 *>(p.dst);
    constexpr int kRepBatch = 4;
    for (int64_t u = blockIdx.x; u < units; u += gridDim.x) {
        const int64_t x = u / cps, c = u - x * cps;
        const int e = __ldg(ws + p.lay.rx_expert + x);
        const int pb = __ldg(ws + p.lay.rep_ptr + e), pe = __ldg(ws + p.lay.rep_ptr + e + 1);
        const int64_t n = min((int64_t)kChunkVecs, p.vecs - c * kChunkVecs);
        float4 *home = g_home + (int64_t)e * p.vecs + c * kChunkVecs;
        for (int64_t i = threadIdx.x; i < n; i += kThreads) {
            float4 acc = __ldcs(home + i);
            for (int q0 = pb; q0 < pe; q0 += kRepBatch) {
                float4 r[kRepBatch];
#pragma unroll
                for (int qq = 0; qq < kRepBatch; ++qq) {
                    const int q = q0 + qq;
                    if (q < pe) {
                        const int64_t slot =
                            (int64_t)__ldg(ws + p.lay.rep_recv + q) * B + __ldg(ws + p.lay.rep_slot + q);
                        r[qq] = __ldcs(g_rep + slot * p.vecs + c * kChunkVecs + i);
                    }
                }
#pragma unroll
                for (int qq = 0; qq < kRepBatch; ++qq)
                    if (q0 + qq < pe) add4(acc, r[qq]);
            }
            __stcs(home + i, acc);
            const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int q = pb; q < pe; ++q) {
                const int64_t slot = (int64_t)__ldg(ws + p.lay.rep_recv + q) * B + __ldg(ws + p.lay.rep_slot + q);
                __stcs(g_rep + slot * p.vecs + c * kChunkVecs + i, z);
            }
        }
    }
}

}  // namespace

cudaError_t launch_prefetch(const CopyParams &p, int grid, cudaStream_t s) {
    prefetch_kernel<<<grid, kThreads, 0, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_reduce_grad(const CopyParams &p, int grid, cudaStream_t s) {
    reduce_grad_kernel<<<grid, kThreads, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace moonep
