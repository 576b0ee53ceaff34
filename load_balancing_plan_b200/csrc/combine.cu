// combine.cu -- moonep_combine: gather of the expert outputs back into token
// order fused with the top-K weighted sum ("The Busiest Rank Sets Your Step
// Time: Running MoonEP's Planning Code Ourselves", flowchart: combine
// gathers results back into token order; agentlenshq "MoonshotAI/MoonEP",
// "How it works": fused unpermute).
//
// out[t] = bf16_rne(acc), acc = 0.0f, acc = fmaf(w[t][k], float(y[dest[t][k]]),
// acc) for k = 0..K-1 in that order.  HBM-bound: K row reads and one row
// write per token.  A unit of work is one token x 256 hidden values (one
// 16-byte vector per lane of a warp); each warp takes a contiguous run of
// units, so it reloads a token's K destinations and weights only when the
// token changes, and keeps min(K, 8) independent 16-byte loads per lane in
// flight.  Rows are read and written with streaming cache hints.
#include <cuda_bf16.h>

#include "moonep_internal.cuh"

namespace moonep {

namespace {

constexpr int kThreads = 256;
constexpr int kVecPerLane = 1;          // 16-byte vectors per lane per unit
constexpr int kUnitVecs = 32 * kVecPerLane;
constexpr int kKBatch = 8;              // rows loaded before their fmas

__device__ __forceinline__ void fma8(float *acc, float w, const uint4 &v) {
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(h[i]);
        acc[2 * i] = __fmaf_rn(w, f.x, acc[2 * i]);
        acc[2 * i + 1] = __fmaf_rn(w, f.y, acc[2 * i + 1]);
    }
}

__device__ __forceinline__ uint4 pack8(const float *acc) {
    uint4 v;
    __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
    return v;
}

__global__ void __launch_bounds__(kThreads, 2) combine_kernel(const __grid_constant__ CombineParams p) {
    if (__ldcg(p.ws + HDR_STATUS) & MOONEP_ST_ERROR_MASK) return;
    const int lane = threadIdx.x & 31;
    if (!cfg_matches(p.ws, p.cfg, num_ranges(p.T))) {
        if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(p.ws + HDR_STATUS, MOONEP_ST_CFG);
        return;
    }
    const int64_t gw = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t nw = ((int64_t)gridDim.x * kThreads) >> 5;
    const int64_t u0 = gw * p.units / nw, u1 = (gw + 1) * p.units / nw;
    const int K = p.cfg.K;
    const int hv = p.hv;

    int64_t cur = -1;
    int dk = 0, dk2 = 0;      // dest of k = lane, lane + 32
    float wk = 0.f, wk2 = 0.f;
    bool tok_ok = true;
    bool bad = false;
    for (int64_t u = u0; u < u1; ++u) {
        const int64_t t = u / p.upt;
        const int sg = (int)(u - t * p.upt);
        if (t != cur) {
            cur = t;
            dk = lane < K ? __ldg(p.dest + t * K + lane) : 0;
            wk = lane < K ? __ldg(p.w + t * K + lane) : 0.f;
            dk2 = lane + 32 < K ? __ldg(p.dest + t * K + lane + 32) : 0;
            wk2 = lane + 32 < K ? __ldg(p.w + t * K + lane + 32) : 0.f;
            const bool okl = (dk >= 0 && (int64_t)dk < p.rows_total) && (dk2 >= 0 && (int64_t)dk2 < p.rows_total);
            tok_ok = __all_sync(0xffffffffu, okl);
            bad |= !tok_ok;
        }
        if (!tok_ok) continue;
        float acc[kVecPerLane][8];
#pragma unroll
        for (int v = 0; v < kVecPerLane; ++v)
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[v][i] = 0.f;
        const int vb = sg * kUnitVecs + lane;
        for (int k0 = 0; k0 < K; k0 += kKBatch) {
            uint4 ld[kKBatch][kVecPerLane];
            float wb[kKBatch];
#pragma unroll
            for (int kk = 0; kk < kKBatch; ++kk) {
                const int k = k0 + kk;
                const int d = __shfl_sync(0xffffffffu, k < 32 ? dk : dk2, k & 31);
                wb[kk] = __shfl_sync(0xffffffffu, k < 32 ? wk : wk2, k & 31);
#pragma unroll
                for (int v = 0; v < kVecPerLane; ++v) {
                    const int vi = vb + v * 32;
                    if (k < K && vi < hv)
                        ld[kk][v] = __ldcs(p.y + (int64_t)d * hv + vi);
                    else
                        ld[kk][v] = make_uint4(0, 0, 0, 0);
                }
            }
#pragma unroll
            for (int kk = 0; kk < kKBatch; ++kk) {
                if (k0 + kk < K) {
#pragma unroll
                    for (int v = 0; v < kVecPerLane; ++v) fma8(acc[v], wb[kk], ld[kk][v]);
                }
            }
        }
#pragma unroll
        for (int v = 0; v < kVecPerLane; ++v) {
            const int vi = vb + v * 32;
            if (vi < hv) __stcs(p.out + t * hv + vi, pack8(acc[v]));
        }
    }
    if (bad && lane == 0) atomicOr(p.ws + HDR_STATUS, MOONEP_ST_DEST);
}

}  // namespace

const void *combine_kernel_ptr() { return (const void *)combine_kernel; }

cudaError_t launch_combine(const CombineParams &p, int grid, cudaStream_t s) {
    combine_kernel<<<grid, kThreads, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace moonep
