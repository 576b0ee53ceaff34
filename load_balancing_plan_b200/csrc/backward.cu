// backward.cu -- moonep_combine_backward: the backward of the combine step
// for training ("The Busiest Rank Sets Your Step Time: Running MoonEP's
// Planning Code Ourselves", flowchart: in training the backward pass follows
// the layer's data path; combine is linear in the expert outputs and in the
// router weights, so its backward is a weighted dispatch of the output
// gradient plus one inner product per (token, k)):
//
//   grad_y[dest[t][k]] = bf16_rne(fp32(w[t][k] * grad_out[t]))
//   grad_w[t][k]       = sum_h grad_out[t][h] * y[dest[t][k]][h]   (fp32)
//
// HBM-bound: one read of grad_out per token, K row writes and, for grad_w,
// K row reads.  One persistent CTA per SM owns a contiguous run of whole
// tokens.  Warp 0 produces: per unit (one chunk of one token's row) it bulk
// copies the grad_out chunk and, for grad_w, the K matching chunks of y into
// a shared-memory stage (TMA, "full" mbarrier).  Warps 1..8 consume: each
// thread takes 16-byte vectors of the chunk, stores the K scaled vectors to
// the dispatched rows and adds the products into its own per-k partial sums
// in shared memory.  After a token's last chunk the consumers reduce the
// partial sums (warp butterflies, then the 8 warps in order), so grad_w does
// not depend on timing.  Every wait is bounded; no multicast.
//
// Expert parallelism (kEp): the tokens are one rank's (T = S) and a row
// q * C_max + j of dest is row j of rank q's buffer.  The producer turns each
// destination into two device addresses once per token (y through y_peers,
// grad_y through grad_y_peers) and hands the grad_y address to the consumers
// in shared memory, so the stores reach the peers' buffers directly.
#include <cuda_bf16.h>

#include "moonep_internal.cuh"

namespace moonep {

namespace {

#ifndef MOONEP_CB_WARPS
#define MOONEP_CB_WARPS 8
#endif
constexpr int kConsumerWarps = MOONEP_CB_WARPS;
constexpr int kConsumers = 32 * kConsumerWarps;
constexpr int kThreads = 32 + kConsumers;
constexpr int kMaxStages = 8;
constexpr int kMaxK = 64;

struct StageInfo {
    int64_t t;       // token
    int32_t c;       // chunk of the row
    uint32_t bytes;  // bytes of this chunk
    int32_t valid;   // all K destinations in range
    int32_t pad;
};

template <bool kEp>
__global__ void __launch_bounds__(kThreads, 1) combine_backward_kernel(const __grid_constant__ BackwardParams p) {
    extern __shared__ __align__(1024) uint8_t smem[];
    int32_t *ws = p.ws;
    if (block_status_failed(ws)) return;
    if (!cfg_matches(ws, p.cfg, num_ranges(p.T, (int64_t)p.cfg.R * p.cfg.L), p.ep_tag)) {
        if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(ws + HDR_STATUS, MOONEP_ST_CFG);
        return;
    }
    const int K = p.cfg.K;
    const bool want_w = p.grad_w != nullptr;
    const int NS = p.stages;
    const uint32_t CH = p.chunk_bytes;
    const int rows_per_stage = 1 + (want_w ? K : 0);
    const size_t stage_bytes = (size_t)rows_per_stage * CH;
    uint8_t *stages = smem;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + (size_t)NS * stage_bytes);
    uint64_t *empty = full + kMaxStages;
    StageInfo *info = reinterpret_cast<StageInfo *>(empty + kMaxStages);
    float *sw = reinterpret_cast<float *>(info + kMaxStages);        // [kMaxStages][kMaxK] weights
    int32_t *sd = reinterpret_cast<int32_t *>(sw + kMaxStages * kMaxK);  // [kMaxStages][kMaxK] dests
    uint4 **sgy = reinterpret_cast<uint4 **>(sd + kMaxStages * kMaxK);   // [kMaxStages][kMaxK] grad_y rows (kEp)
    float *s_red = reinterpret_cast<float *>(sgy + kMaxStages * kMaxK);   // [kMaxK][kConsumerWarps]
    float *s_part = s_red + kMaxK * kConsumerWarps;                       // [K][kConsumers]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    if (want_w)
        for (int i = threadIdx.x; i < K * kConsumers; i += kThreads) s_part[i] = 0.f;
    __syncthreads();

    // the CTA's tokens (whole tokens, so grad_w needs no cross-CTA sum): a
    // contiguous share, or (MOONEP_INTERLEAVE) every gridDim.x-th token, so
    // that the CTAs work on neighbouring tokens; unit i of the CTA is chunk
    // i % upt of its (i / upt)-th token
    const int64_t tb = MOONEP_INTERLEAVE ? blockIdx.x : (int64_t)blockIdx.x * p.T / gridDim.x;
    const int64_t tstep = MOONEP_INTERLEAVE ? gridDim.x : 1;
    const int64_t ntk = MOONEP_INTERLEAVE ? (blockIdx.x < p.T ? (p.T - 1 - blockIdx.x) / gridDim.x + 1 : 0)
                                          : (int64_t)(blockIdx.x + 1) * p.T / gridDim.x - tb;
    const int64_t nun = ntk * p.upt;
    auto unit_of = [&](int64_t i) { return (tb + (i / p.upt) * tstep) * p.upt + i % p.upt; };
    const int64_t row_bytes = (int64_t)p.hv * 16;
    const uint32_t last = (uint32_t)(row_bytes - (int64_t)(p.upt - 1) * CH);
    const uint64_t pol = policy_evict_first();
    const uint8_t *gsrc = reinterpret_cast<const uint8_t *>(p.grad_out);
    const uint8_t *ysrc = reinterpret_cast<const uint8_t *>(p.y);

    if (warp == 0) {
        // ------------------------------------------------------- producer
        int64_t cur = -1;
        int dk = 0, dk2 = 0;
        float wk = 0.f, wk2 = 0.f;
        const uint8_t *yk = nullptr, *yk2 = nullptr;  // the K rows of y (kEp: on their ranks)
        uint4 *gk = nullptr, *gk2 = nullptr;          // the K rows of grad_y (kEp)
        int valid = 1;
        bool bad = false, fail = false;
        int64_t i = 0;
        for (int64_t u = unit_of(0); i < nun; ++i, u = unit_of(i)) {
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
                dk = lane < K ? __ldg(p.dest + t * K + lane) : 0;
                wk = lane < K ? __ldg(p.w + t * K + lane) : 0.f;
                dk2 = lane + 32 < K ? __ldg(p.dest + t * K + lane + 32) : 0;
                wk2 = lane + 32 < K ? __ldg(p.w + t * K + lane + 32) : 0.f;
                const bool okl = dk >= 0 && (int64_t)dk < p.rows_total && dk2 >= 0 && (int64_t)dk2 < p.rows_total;
                valid = __all_sync(0xffffffffu, okl) ? 1 : 0;
                bad |= !valid;
                if (valid) {
                    if (kEp) {
                        const uint32_t Cm = (uint32_t)p.cfg.C_max;
                        const uint32_t q = (uint32_t)dk / Cm, q2 = (uint32_t)dk2 / Cm;
                        const int64_t j = (int64_t)((uint32_t)dk - q * Cm), j2 = (int64_t)((uint32_t)dk2 - q2 * Cm);
                        if (lane < K) {
                            gk = reinterpret_cast<uint4 *>(__ldg(reinterpret_cast<const uint64_t *>(p.grad_y_peers) + q)) +
                                 j * p.hv;
                            if (want_w) yk = reinterpret_cast<const uint8_t *>(
                                                 __ldg(reinterpret_cast<const uint64_t *>(p.y_peers) + q)) + j * row_bytes;
                        }
                        if (lane + 32 < K) {
                            gk2 = reinterpret_cast<uint4 *>(__ldg(reinterpret_cast<const uint64_t *>(p.grad_y_peers) + q2)) +
                                  j2 * p.hv;
                            if (want_w) yk2 = reinterpret_cast<const uint8_t *>(
                                                  __ldg(reinterpret_cast<const uint64_t *>(p.y_peers) + q2)) + j2 * row_bytes;
                        }
                    } else if (want_w) {
                        yk = ysrc + (int64_t)dk * row_bytes;
                        yk2 = ysrc + (int64_t)dk2 * row_bytes;
                    }
                }
            }
            const uint32_t bytes = c == p.upt - 1 ? last : CH;
            if (lane < K) {
                sw[s * kMaxK + lane] = wk;
                sd[s * kMaxK + lane] = dk;
                if (kEp) sgy[s * kMaxK + lane] = gk;
            }
            if (lane + 32 < K) {
                sw[s * kMaxK + lane + 32] = wk2;
                sd[s * kMaxK + lane + 32] = dk2;
                if (kEp) sgy[s * kMaxK + lane + 32] = gk2;
            }
            __syncwarp();  // every lane's weights and rows before lane 0's release
            if (lane == 0) {
                info[s].t = t;
                info[s].c = c;
                info[s].bytes = bytes;
                info[s].valid = valid;
                mbar_arrive_expect_tx(&full[s], valid ? (uint32_t)rows_per_stage * bytes : 0u);
            }
            __syncwarp();
            if (valid) {
                uint8_t *st = stages + (size_t)s * stage_bytes;
                if (lane == 0) bulk_g2s(st, gsrc + t * row_bytes + (int64_t)c * CH, bytes, &full[s], pol);
                if (want_w) {
                    if (lane < K) bulk_g2s(st + (size_t)(1 + lane) * CH, yk + (int64_t)c * CH, bytes, &full[s], pol);
                    if (lane + 32 < K)
                        bulk_g2s(st + (size_t)(33 + lane) * CH, yk2 + (int64_t)c * CH, bytes, &full[s], pol);
                }
            }
        }
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
        const int cw = ct >> 5;
        int64_t i = 0;
        bool ok = true;
        for (int64_t u = unit_of(0); i < nun; ++i, u = unit_of(i)) {
            const int s = (int)(i % NS);
            if (ok && !mbar_wait_bounded(&full[s], (uint32_t)((i / NS) & 1), p.wait_limit)) {
                if (ct == 0) atomicOr(ws + HDR_STATUS, MOONEP_ST_TIMEOUT);
                ok = false;  // keep joining the token-end barriers, touch nothing
            }
            const StageInfo inf = info[s];
            if (ok && inf.valid) {
                const uint8_t *st = stages + (size_t)s * stage_bytes;
                const float *wv = sw + s * kMaxK;
                const int32_t *dv = sd + s * kMaxK;
                uint4 *const *gv_rows = sgy + s * kMaxK;
                const int nv = (int)(inf.bytes >> 4);
                const int64_t col = (int64_t)inf.c * (CH >> 4);
                for (int v = ct; v < nv; v += kConsumers) {
                    const uint4 gv = *reinterpret_cast<const uint4 *>(st + (size_t)v * 16);
                    const __nv_bfloat162 *gh = reinterpret_cast<const __nv_bfloat162 *>(&gv);
                    float gf[8];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float2 f = __bfloat1622float2(gh[q]);
                        gf[2 * q] = f.x;
                        gf[2 * q + 1] = f.y;
                    }
                    for (int k = 0; k < K; ++k) {
                        const float w = wv[k];
                        uint4 o;
                        __nv_bfloat162 *oh = reinterpret_cast<__nv_bfloat162 *>(&o);
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            oh[q] = __floats2bfloat162_rn(__fmul_rn(w, gf[2 * q]), __fmul_rn(w, gf[2 * q + 1]));
                        uint4 *dst = kEp ? gv_rows[k] : p.grad_y + (int64_t)dv[k] * p.hv;
                        __stcs(dst + col + v, o);
                        if (want_w) {
                            const uint4 yv = *reinterpret_cast<const uint4 *>(st + (size_t)(1 + k) * CH + (size_t)v * 16);
                            const __nv_bfloat162 *yh = reinterpret_cast<const __nv_bfloat162 *>(&yv);
                            float a = s_part[k * kConsumers + ct];
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                const float2 f = __bfloat1622float2(yh[q]);
                                a = __fmaf_rn(gf[2 * q], f.x, a);
                                a = __fmaf_rn(gf[2 * q + 1], f.y, a);
                            }
                            s_part[k * kConsumers + ct] = a;
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            // the decision depends on u only, so all consumers join the same barriers
            const int64_t tu = u / p.upt;
            if (want_w && u - tu * p.upt == p.upt - 1) {
                // the token's last chunk: reduce the partial sums in a fixed order
                named_barrier(1, kConsumers);
                for (int k = 0; k < K; ++k) {
                    float a = s_part[k * kConsumers + ct];
                    s_part[k * kConsumers + ct] = 0.f;
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) a = __fadd_rn(a, __shfl_xor_sync(0xffffffffu, a, o));
                    if (lane == 0) s_red[k * kConsumerWarps + cw] = a;
                }
                named_barrier(1, kConsumers);
                if (ok && inf.valid && ct < K) {
                    float a = 0.f;
                    for (int q = 0; q < kConsumerWarps; ++q) a = __fadd_rn(a, s_red[ct * kConsumerWarps + q]);
                    p.grad_w[tu * K + ct] = a;
                }
            }
        }
    }
}

}  // namespace

// chunk: the row split into the fewest equal pieces (multiples of 16 bytes,
// at most 32 KB) such that three stages of (1 + K) pieces fit in shared
// memory beside the fixed tables; large bulk copies move the most bytes.
// Both forms of the kernel use the same layout (the grad_y row pointers are
// reserved in the single-GPU form too), so they split rows alike and sum
// grad_w in the same order.
cudaError_t combine_backward_config(int K, int hv, bool with_grad_w, uint32_t *chunk, int *upt, int *stages,
                                    size_t *smem) {
    if (K < 1 || K > kMaxK || hv < 1) return cudaErrorInvalidValue;
    const size_t rows = 1 + (with_grad_w ? (size_t)K : 0);
    const size_t fixed = 2 * kMaxStages * 8 + kMaxStages * sizeof(StageInfo) + 2 * kMaxStages * kMaxK * 4 +
                         (size_t)kMaxStages * kMaxK * 8 + kMaxK * kConsumerWarps * 4 +
                         (with_grad_w ? (size_t)K * kConsumers * 4 : 0) + 128;
    const size_t budget = 220 * 1024;
    if (fixed + rows * 16 * 3 > budget) return cudaErrorInvalidValue;
    const uint32_t row = (uint32_t)hv * 16;
    uint32_t ch = row;
    for (int n = 1;; ++n) {
        ch = (((row + n - 1) / n) + 15) & ~15u;
        if (ch <= 32768 && rows * ch * 3 <= budget - fixed) break;
        if (ch <= 16) return cudaErrorInvalidValue;
    }
    const size_t stage = rows * ch;
    int ns = (int)((budget - fixed) / stage);
    if (ns > kMaxStages) ns = kMaxStages;
    if (ns < 2) return cudaErrorInvalidValue;
    *chunk = ch;
    *upt = (int)((row + ch - 1) / ch);
    *stages = ns;
    *smem = (size_t)ns * stage + fixed;
    return cudaSuccess;
}

cudaError_t launch_combine_backward(const BackwardParams &p, int grid, size_t smem, cudaStream_t s) {
    if (p.grad_y_peers) {
        static std::atomic<size_t> smem_set_ep[64];
        cudaError_t err = set_smem_limit((const void *)combine_backward_kernel<true>, smem, smem_set_ep);
        if (err != cudaSuccess) return err;
        combine_backward_kernel<true><<<grid, kThreads, smem, s>>>(p);
        return cudaGetLastError();
    }
    static std::atomic<size_t> smem_set[64];
    cudaError_t err = set_smem_limit((const void *)combine_backward_kernel<false>, smem, smem_set);
    if (err != cudaSuccess) return err;
    combine_backward_kernel<false><<<grid, kThreads, smem, s>>>(p);
    return cudaGetLastError();
}

}  // namespace moonep
