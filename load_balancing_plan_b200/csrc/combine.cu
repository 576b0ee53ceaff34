// combine.cu -- moonep_combine: gather of the expert outputs back into token
// order fused with the top-K weighted sum ("The Busiest Rank Sets Your Step
// Time: Running MoonEP's Planning Code Ourselves", flowchart: combine
// gathers results back into token order; agentlenshq "MoonshotAI/MoonEP",
// "How it works": fused unpermute).
//
// out[t] = bf16_rne(acc), acc = 0.0f, acc = fmaf(w[t][k], float(y[dest[t][k]]),
// acc) for k = 0..K-1 in that order.  The same kernel with no weights is the
// dispatch backward: grad_x[t] = bf16_rne(fp32 sum over k of grad_recv[dest]).
//
// HBM-bound: K row reads and one row write per token.  One persistent CTA
// per SM runs a TMA pipeline.  A unit of work is one chunk of one token's
// row (chunk_bytes of each of its K source rows).  Warp 0 produces: for each
// unit it waits for a free shared-memory stage, posts the byte count on the
// stage's "full" mbarrier, and its lanes issue the K bulk copies
// global -> shared (lane k copies row k); it also parks the token's K
// weights next to the stage.  Warps 1..8 consume: they wait on "full", read
// the K chunks from shared memory (16 bytes per thread per row, conflict
// free), accumulate in fp32 in k order, store the bf16 result with a
// streaming hint and release the stage on its "empty" mbarrier.  Up to
// `stages` units are in flight per SM, so the gather is never short of
// outstanding bytes.  Every wait is bounded.  No multicast.
#include <cuda_bf16.h>

#include "moonep_internal.cuh"

namespace moonep {

namespace {

#ifndef MOONEP_COMBINE_CONSUMERS
#define MOONEP_COMBINE_CONSUMERS 8   // consumer warps per CTA
#endif
#ifndef MOONEP_COMBINE_CHUNK
#define MOONEP_COMBINE_CHUNK 8192    // bytes of each source row per unit (upper bound)
#endif
#ifndef MOONEP_COMBINE_SMEM_KB
#define MOONEP_COMBINE_SMEM_KB 220   // shared memory for the stages
#endif

constexpr int kConsumerWarps = MOONEP_COMBINE_CONSUMERS;
constexpr int kThreads = 32 * (1 + kConsumerWarps);
constexpr int kMaxStages = 8;
constexpr int kMaxK = 64;

struct StageInfo {
    int64_t t;       // token
    int32_t c;       // chunk of the row
    uint32_t bytes;  // bytes of this chunk
    int32_t valid;   // all K destinations in range
    int32_t pad;
};

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

// kEp: expert parallelism.  The tokens are one rank's (T = S) and a source
// row lives in the expert-output buffer of its rank, reached through a table
// of peer pointers kept in shared memory after the weights.
template <bool kEp>
__global__ void __launch_bounds__(kThreads, 1) combine_kernel(const __grid_constant__ CombineParams p) {
    extern __shared__ __align__(1024) uint8_t smem[];
    int32_t *ws = p.ws;
    if (block_status_failed(ws)) return;
    if (!cfg_matches(ws, p.cfg, num_ranges(p.T, (int64_t)p.cfg.R * p.cfg.L), p.ep_tag)) {
        if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(ws + HDR_STATUS, MOONEP_ST_CFG);
        return;
    }
    const int K = p.cfg.K;
    const int NS = p.stages;
    const uint32_t CH = p.chunk_bytes;
    const size_t stage_bytes = (size_t)K * CH;
    uint8_t *stages = smem;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + (size_t)NS * stage_bytes);
    uint64_t *empty = full + kMaxStages;
    StageInfo *info = reinterpret_cast<StageInfo *>(empty + kMaxStages);
    float *sw = reinterpret_cast<float *>(info + kMaxStages);  // [kMaxStages][kMaxK]
    const uint8_t **s_peer = reinterpret_cast<const uint8_t **>(sw + kMaxStages * kMaxK);  // [R] (kEp)

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (kEp)
        for (int r = threadIdx.x; r < p.cfg.R; r += kThreads) s_peer[r] = p.y_peers[r];
    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    __syncthreads();

    // the CTA's units: a contiguous share, or (MOONEP_INTERLEAVE) every
    // gridDim.x-th unit, so that the CTAs work on neighbouring tokens
    const int64_t u0 = MOONEP_INTERLEAVE ? blockIdx.x : (int64_t)blockIdx.x * p.units / gridDim.x;
    const int64_t ustep = MOONEP_INTERLEAVE ? gridDim.x : 1;
    const int64_t nun = MOONEP_INTERLEAVE ? (blockIdx.x < p.units ? (p.units - 1 - blockIdx.x) / gridDim.x + 1 : 0)
                                          : (int64_t)(blockIdx.x + 1) * p.units / gridDim.x - u0;
    const int64_t row_bytes = (int64_t)p.hv * 16;
    const uint32_t last = (uint32_t)(row_bytes - (int64_t)(p.upt - 1) * CH);
    const uint64_t pol = policy_evict_first();
    const uint8_t *y = reinterpret_cast<const uint8_t *>(p.y);

    if (warp == 0) {
        // ------------------------------------------------------- producer
        int64_t cur = -1;
        int dk = 0, dk2 = 0;
        float wk = 0.f, wk2 = 0.f;
        int valid = 1;
        bool bad = false, fail = false;
        int64_t i = 0;
        for (int64_t u = u0; i < nun; u += ustep, ++i) {
            const int s = (int)(i % NS);
            if (i >= NS) {
                int ok = 1;
                if (lane == 0) ok = mbar_wait_bounded(&empty[s], (uint32_t)(((i / NS) - 1) & 1), p.wait_limit);
                if (!__shfl_sync(0xffffffffu, ok, 0)) {
                    fail = true;
                    break;
                }
            }
            const int64_t t = u / p.upt;
            const int c = (int)(u - t * p.upt);
            if (t != cur) {
                cur = t;
                // no weights (dispatch backward): every weight is 1, and
                // fmaf(1, v, acc) is exactly the fp32 sum acc + v
                dk = lane < K ? __ldg(p.dest + t * K + lane) : 0;
                wk = lane < K ? (p.w ? __ldg(p.w + t * K + lane) : 1.f) : 0.f;
                dk2 = lane + 32 < K ? __ldg(p.dest + t * K + lane + 32) : 0;
                wk2 = lane + 32 < K ? (p.w ? __ldg(p.w + t * K + lane + 32) : 1.f) : 0.f;
                const bool okl = dk >= 0 && (int64_t)dk < p.rows_total && dk2 >= 0 && (int64_t)dk2 < p.rows_total;
                valid = __all_sync(0xffffffffu, okl) ? 1 : 0;
                bad |= !valid;
            }
            const uint32_t bytes = c == p.upt - 1 ? last : CH;
            if (lane < K) sw[s * kMaxK + lane] = wk;
            if (lane + 32 < K) sw[s * kMaxK + lane + 32] = wk2;
            __syncwarp();  // every lane's weights before lane 0's release
            if (lane == 0) {
                info[s].t = t;
                info[s].c = c;
                info[s].bytes = bytes;
                info[s].valid = valid;
                mbar_arrive_expect_tx(&full[s], valid ? (uint32_t)K * bytes : 0u);
            }
            __syncwarp();
            if (valid) {
                uint8_t *st = stages + (size_t)s * stage_bytes;
                const int64_t Cm = p.cfg.C_max;
                if (lane < K) {
                    const uint8_t *row = kEp ? s_peer[dk / Cm] + (int64_t)(dk % Cm) * row_bytes
                                             : y + (int64_t)dk * row_bytes;
                    bulk_g2s(st + (size_t)lane * CH, row + (int64_t)c * CH, bytes, &full[s], pol);
                }
                if (lane + 32 < K) {
                    const uint8_t *row = kEp ? s_peer[dk2 / Cm] + (int64_t)(dk2 % Cm) * row_bytes
                                             : y + (int64_t)dk2 * row_bytes;
                    bulk_g2s(st + (size_t)(lane + 32) * CH, row + (int64_t)c * CH, bytes, &full[s], pol);
                }
            }
        }
        // every copy issued must land before the CTA exits
        if (lane == 0) {
            const int64_t drain = p.wait_limit > (int64_t(1) << 20) ? p.wait_limit : (int64_t(1) << 20);
            for (int64_t j = (i > NS ? i - NS : 0); j < i; ++j)
                mbar_wait_bounded(&full[j % NS], (uint32_t)((j / NS) & 1), drain);
            if (fail) atomicOr(ws + HDR_STATUS, MOONEP_ST_TIMEOUT);
            if (bad) atomicOr(ws + HDR_STATUS, MOONEP_ST_DEST);
        }
    } else {
        // ------------------------------------------------------- consumers
        const int ct = threadIdx.x - 32;
        int64_t i = 0;
        for (int64_t u = u0; i < nun; u += ustep, ++i) {
            const int s = (int)(i % NS);
            if (!mbar_wait_bounded(&full[s], (uint32_t)((i / NS) & 1), p.wait_limit)) {
                if (ct == 0) atomicOr(ws + HDR_STATUS, MOONEP_ST_TIMEOUT);
                break;
            }
            const StageInfo inf = info[s];
            if (inf.valid) {
                const uint8_t *st = stages + (size_t)s * stage_bytes;
                const float *wv = sw + s * kMaxK;
                const int nv = (int)(inf.bytes >> 4);
                uint4 *dst = p.out + inf.t * p.hv + (int64_t)inf.c * (CH >> 4);
                for (int v = ct; v < nv; v += 32 * kConsumerWarps) {
                    float acc[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) acc[q] = 0.f;
                    for (int k = 0; k < K; ++k) {
                        const uint4 val = *reinterpret_cast<const uint4 *>(st + (size_t)k * CH + (size_t)v * 16);
                        fma8(acc, wv[k], val);
                    }
                    __stcs(dst + v, pack8(acc));
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }
    }
}

}  // namespace

const void *combine_kernel_ptr() { return (const void *)combine_kernel<false>; }

// chunk: the row split into equal pieces (multiples of 16 bytes) of at most
// MOONEP_COMBINE_CHUNK bytes, fewer when K is large (K*chunk <= 8 chunks);
// stages fill MOONEP_COMBINE_SMEM_KB of shared memory (at most kMaxStages).
// Large bulk copies matter: 8 KB copies move about 1.5x the bytes per second
// of 4 KB ones on B200.
cudaError_t combine_config(int K, int hv, uint32_t *chunk, int *upt, int *stages, size_t *smem, bool ep) {
    if (K < 1 || K > kMaxK || hv < 1) return cudaErrorInvalidValue;
    uint32_t cap = MOONEP_COMBINE_CHUNK;
    while ((uint32_t)K * cap > 8u * MOONEP_COMBINE_CHUNK && cap > 512) cap >>= 1;
    const uint32_t row = (uint32_t)hv * 16;
    const int n = (int)((row + cap - 1) / cap);
    const uint32_t ch = (((row + n - 1) / n) + 15) & ~15u;
    const size_t stage = (size_t)K * ch;
    const size_t fixed = 2 * kMaxStages * 8 + kMaxStages * sizeof(StageInfo) + kMaxStages * kMaxK * 4 + 128 +
                         (ep ? 64 * 8 : 0);
    int ns = (int)((MOONEP_COMBINE_SMEM_KB * 1024 - fixed) / stage);
    if (ns > kMaxStages) ns = kMaxStages;
    if (ns < 2) return cudaErrorInvalidValue;
    *chunk = ch;
    *upt = (int)((row + ch - 1) / ch);
    *stages = ns;
    *smem = (size_t)ns * stage + fixed;
    return cudaSuccess;
}

cudaError_t launch_combine(const CombineParams &p, int grid, size_t smem, cudaStream_t s) {
    if (p.y_peers) {
        static std::atomic<size_t> smem_set_ep[64];
        cudaError_t err = set_smem_limit((const void *)combine_kernel<true>, smem, smem_set_ep);
        if (err != cudaSuccess) return err;
        combine_kernel<true><<<grid, kThreads, smem, s>>>(p);
        return cudaGetLastError();
    }
    static std::atomic<size_t> smem_set[64];
    cudaError_t err = set_smem_limit((const void *)combine_kernel<false>, smem, smem_set);
    if (err != cudaSuccess) return err;
    combine_kernel<false><<<grid, kThreads, smem, s>>>(p);
    return cudaGetLastError();
}

}  // namespace moonep
