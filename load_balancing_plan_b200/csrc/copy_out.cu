// copy_out.cu -- moonep_copy_out: the zero_copy = false path.  The
// application normally works on views of the receive buffer, which the next
// dispatch or combine overwrites; a caller that keeps the dispatched rows
// longer (autograd saving them for the backward pass, for one) takes its own
// copy (twodots.gr "MoonEP balances AI experts in MoE models": the paragraph
// on zero-copy communication and static shapes, and the one on the lifetime
// of zero-copy views).
//
// Only the rows the plan uses are copied, to the same rows of the caller's
// buffer, so the plan's segment tables describe the copy as well.  On rank r
// those rows are two contiguous runs: [0, fill[r]) -- the local segments,
// then the slotted pieces, then any remote pieces -- and, from row C, the
// fallback segments of r's own experts.  The default kernel moves them with
// TMA bulk copies through shared memory (below); MOONEP_COPY_OUT_TMA=0 builds
// the first form, in which CTA (x, r, part) copies its share of run `part` of
// rank r with 16-byte streaming loads and stores, four in flight per thread
// (it tops out at about 5.9 TB/s, held back by the LSU queue).
#include "moonep_internal.cuh"

namespace moonep {

namespace {

constexpr int kUnroll = 4;

__global__ void __launch_bounds__(kCopyOutThreads, 6) copy_out_kernel(const __grid_constant__ CopyOutParams p) {
    int32_t *ws = p.ws;
    if (block_status_failed(ws)) return;
    if (!cfg_matches(ws, p.cfg, p.Q)) {
        if (threadIdx.x == 0) atomicOr(ws + HDR_STATUS, MOONEP_ST_CFG);
        return;
    }
    const int r = blockIdx.y, part = blockIdx.z;
    const int L = p.cfg.L, B = p.cfg.B, SEG = 2 * L + B;
    __shared__ int s_n;
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        int n = 0;
        if (part == 0) {
            n = lane == 0 ? __ldg(ws + p.lay.fill + r) : 0;
        } else {
            for (int loc = lane; loc < L; loc += 32) n += __ldg(ws + p.lay.seg_len + r * SEG + L + B + loc);
        }
        for (int o = 16; o > 0; o >>= 1) n += __shfl_xor_sync(0xffffffffu, n, o);
        if (lane == 0) s_n = n;
    }
    __syncthreads();
    const int64_t n = s_n;
    const int64_t row0 = part == 0 ? 0 : p.cfg.C;
    if (n <= 0) return;
    if (row0 + n > p.cfg.C_max) {
        if (threadIdx.x == 0) atomicOr(ws + HDR_STATUS, MOONEP_ST_DEST);
        return;
    }
    const int64_t base = ((int64_t)r * p.cfg.C_max + row0) * p.row_vecs;
    const int64_t nv = n * p.row_vecs;
    const uint4 *src = p.src + base;
    uint4 *dst = p.dst + base;
    // blocks of kUnroll * kCopyOutThreads vectors: thread t moves vectors
    // t, t + 256, t + 512, t + 768 of each block (coalesced per warp)
    constexpr int kChunk = kUnroll * kCopyOutThreads;
    for (int64_t c0 = (int64_t)blockIdx.x * kChunk; c0 < nv; c0 += (int64_t)gridDim.x * kChunk) {
        const uint4 *s = src + c0 + threadIdx.x;
        uint4 *d = dst + c0 + threadIdx.x;
        const int64_t rem = nv - c0 - threadIdx.x;
        if (rem > (kUnroll - 1) * kCopyOutThreads) {
            uint4 t[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) t[u] = __ldcs(s + u * kCopyOutThreads);
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) __stcs(d + u * kCopyOutThreads, t[u]);
        } else {
#pragma unroll
            for (int u = 0; u < kUnroll; ++u)
                if (u * kCopyOutThreads < rem) __stcs(d + u * kCopyOutThreads, __ldcs(s + u * kCopyOutThreads));
        }
    }
}

// The same copy through shared memory with TMA bulk copies
// (MOONEP_COPY_OUT_TMA, the default): one warp per SM, lane 0 runs a pipeline
// of kCoStages 32 KB stages over the CTA's contiguous share of the 32 KB
// chunks of all 2R runs (bulk load global -> shared on an mbarrier, bulk
// store shared -> global, kCoAhead loads in flight, evict-first hints on
// both sides).  The runs' byte extents are worked out by the warp first
// (fill[r] rows from row 0; the fallback segments' total from row C).
#ifndef MOONEP_COPY_OUT_TMA
#define MOONEP_COPY_OUT_TMA 1
#endif
constexpr uint32_t kCoChunk = 32768;
constexpr int kCoStages = 6;
constexpr int kCoAhead = 4;
constexpr int kCoMaxRuns = 128;  // 2 runs per rank, R <= 64
static_assert(kCoStages - kCoAhead - 1 >= 0, "stage reuse needs an older store group");

__global__ void __launch_bounds__(32, 1) copy_out_tma_kernel(const __grid_constant__ CopyOutParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ int64_t s_start[kCoMaxRuns];   // byte offset of the run in recv / out
    __shared__ int64_t s_bytes[kCoMaxRuns];
    __shared__ int64_t s_first[kCoMaxRuns + 1];  // first chunk of each run (prefix)
    int32_t *ws = p.ws;
    if (block_status_failed(ws)) return;
    if (!cfg_matches(ws, p.cfg, p.Q)) {
        if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(ws + HDR_STATUS, MOONEP_ST_CFG);
        return;
    }
    const int lane = threadIdx.x;
    const int R = p.cfg.R, L = p.cfg.L, B = p.cfg.B, SEG = 2 * L + B;
    const int64_t row_bytes = p.row_vecs * 16;
    const int nruns = 2 * R;
    // runs: 2r = rows [0, fill[r]) of rank r, 2r+1 = its fallback rows from C
    bool bad = false;
    for (int r = 0; r < R; ++r) {
        int nfb = 0;
        for (int loc = lane; loc < L; loc += 32) nfb += __ldg(ws + p.lay.seg_len + r * SEG + L + B + loc);
        for (int o = 16; o > 0; o >>= 1) nfb += __shfl_xor_sync(0xffffffffu, nfb, o);
        if (lane == 0) {
            const int nfill = __ldg(ws + p.lay.fill + r);
            const int64_t base = (int64_t)r * p.cfg.C_max;
            if (nfill < 0 || nfill > p.cfg.C_max || nfb < 0 || (int64_t)p.cfg.C + nfb > p.cfg.C_max) bad = true;
            s_start[2 * r] = base * row_bytes;
            s_bytes[2 * r] = bad ? 0 : (int64_t)nfill * row_bytes;
            s_start[2 * r + 1] = (base + p.cfg.C) * row_bytes;
            s_bytes[2 * r + 1] = bad ? 0 : (int64_t)nfb * row_bytes;
        }
    }
    __syncwarp();
    if (lane == 0) {
        int64_t c = 0;
        for (int q = 0; q < nruns; ++q) {
            s_first[q] = c;
            c += (s_bytes[q] + kCoChunk - 1) / kCoChunk;
        }
        s_first[nruns] = c;
        if (bad && blockIdx.x == 0) atomicOr(ws + HDR_STATUS, MOONEP_ST_DEST);
    }
    __syncwarp();
    if (lane != 0) return;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + (size_t)kCoStages * kCoChunk);
    for (int st = 0; st < kCoStages; ++st) mbar_init(&bars[st], 1);
    fence_mbar_init();
    fence_proxy_async_smem();

    const int64_t units = s_first[nruns];
    const int64_t u0 = (int64_t)blockIdx.x * units / gridDim.x;
    const int64_t n = (int64_t)(blockIdx.x + 1) * units / gridDim.x - u0;
    const uint8_t *src = reinterpret_cast<const uint8_t *>(p.src);
    uint8_t *dst = reinterpret_cast<uint8_t *>(p.dst);
    const uint64_t pol = policy_evict_first();
    // unit -> (byte offset, bytes); runs ascend in s_first and the CTA's units
    // too, so the loads and the stores each keep a run cursor
    auto locate = [&](int64_t u, int &run, int64_t &off, uint32_t &bytes) {
        while (run + 1 < nruns && s_first[run + 1] <= u) ++run;
        const int64_t k = u - s_first[run];
        off = s_start[run] + k * kCoChunk;
        bytes = (uint32_t)min((int64_t)kCoChunk, s_bytes[run] - k * kCoChunk);
    };
    int run_l = 0, run_s = 0;
    bool fail = false;
    int64_t issued = 0, stored = 0;
    for (int64_t it = 0; it < n + kCoAhead; ++it) {
        if (it < n) {
            const int st = (int)(it % kCoStages);
            int64_t off;
            uint32_t bytes;
            locate(u0 + it, run_l, off, bytes);
            if (it >= kCoStages) bulk_wait_read<kCoStages - kCoAhead - 1>();
            mbar_arrive_expect_tx(&bars[st], bytes);
            bulk_g2s(smem + (size_t)st * kCoChunk, src + off, bytes, &bars[st], pol);
            issued = it + 1;
        }
        const int64_t j = it - kCoAhead;
        if (j >= 0 && j < n) {
            const int st = (int)(j % kCoStages);
            if (!mbar_wait_bounded(&bars[st], (uint32_t)((j / kCoStages) & 1), p.wait_limit)) {
                fail = true;
                break;
            }
            int64_t off;
            uint32_t bytes;
            locate(u0 + j, run_s, off, bytes);
            bulk_s2g(dst + off, smem + (size_t)st * kCoChunk, bytes, pol);
            bulk_commit();
            stored = j + 1;
        }
    }
    bulk_wait_all<0>();
    if (fail) {
        // let the loads still in flight land before the CTA exits
        const int64_t drain = p.wait_limit > (int64_t(1) << 20) ? p.wait_limit : (int64_t(1) << 20);
        for (int64_t u = stored; u < issued; ++u)
            mbar_wait_bounded(&bars[u % kCoStages], (uint32_t)((u / kCoStages) & 1), drain);
        atomicOr(ws + HDR_STATUS, MOONEP_ST_TIMEOUT);
    }
}

}  // namespace

cudaError_t launch_copy_out(const CopyOutParams &p, int sms, cudaStream_t s) {
    if (MOONEP_COPY_OUT_TMA) {
        const size_t smem = (size_t)kCoStages * kCoChunk + kCoStages * 8;
        static std::atomic<size_t> smem_set[64];
        cudaError_t err = set_smem_limit((const void *)copy_out_tma_kernel, smem, smem_set);
        if (err != cudaSuccess) return err;
        copy_out_tma_kernel<<<sms, 32, smem, s>>>(p);
        return cudaGetLastError();
    }
    // the CTAs one wave holds (6 of 256 threads per SM), shared by the R fill runs
    const int per_rank = (int)((6 * (int64_t)sms + p.cfg.R - 1) / p.cfg.R);
    const dim3 grid((unsigned)(per_rank > 0 ? per_rank : 1), (unsigned)p.cfg.R, 2);
    copy_out_kernel<<<grid, kCopyOutThreads, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace moonep
