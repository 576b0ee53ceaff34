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
// fallback segments of r's own experts.  CTA (x, r, part) copies its share of
// run `part` of rank r with 16-byte streaming loads and stores, four in flight
// per thread; the runs are HBM-bound copies, so plain coalesced vector
// accesses with enough bytes in flight reach the copy bandwidth.
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

}  // namespace

cudaError_t launch_copy_out(const CopyOutParams &p, int blocks_per_rank, cudaStream_t s) {
    const dim3 grid((unsigned)blocks_per_rank, (unsigned)p.cfg.R, 2);
    copy_out_kernel<<<grid, kCopyOutThreads, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace moonep
