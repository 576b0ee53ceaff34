// plan.cu -- moonep_plan: the online redundant-expert planning kernel.
//
// "The Busiest Rank Sets Your Step Time: Running MoonEP's Planning Code
// Ourselves", section "What the technique is" (flowchart: router output
// topk_experts / tokens_per_expert -> planning kernel deciding online which
// experts to duplicate and where), and twodots.gr "MoonEP balances AI
// experts in MoE models" (the GPU planner; the planner emits cu_seqlens).
//
// One persistent cooperative kernel, 512 threads per CTA, one CTA per SM:
//   phase A  every CTA counts the top-K ids of its token ranges into a
//            shared-memory histogram, writes the per-(expert, range) counts
//            and adds them to the global tokens_per_expert (cnt);
//   barrier  one bounded grid barrier (gives up after wait_limit polls and
//            records MOONEP_ST_TIMEOUT; all CTAs are co-resident by the
//            cooperative launch, so it normally completes at once);
//   phase B  CTA 0 runs the planner on cnt (keep/spill split, spill stream,
//            receiver walk, pieces, slots, fallback, route/segment/alloc
//            tables) while CTAs 1.. turn the per-range counts into
//            exclusive prefixes (one warp per expert column).
//
// The spill planner.  Spilled rows form one stream, expert by expert in
// ascending order (chunk m of expert e spans stream positions [A_e, A_e +
// spill_e)).  Receivers (ranks with deficit > 0) are visited in ascending
// order; receiver r starts where the previous one stopped, at position p_r,
// and takes rows until it has either filled its deficit or used its B slots
// (one slot per chunk it touches).  That is exactly "each chunk goes to the
// lowest-index rank that still has room and a free slot", computed as a walk
// over at most R receivers instead of over the chunks.  Rows past the last
// receiver's stop fall back to their home rank's headroom.
#include "moonep_internal.cuh"

namespace moonep {

namespace {

constexpr int kPlanThreads = 512;
constexpr int kWarps = kPlanThreads / 32;
constexpr int kMaxR = 64;

// Exclusive scan of n ints (in and out may alias) by the whole CTA; returns
// the total.  Each thread owns a contiguous run of ceil(n / 512) entries.
__device__ int block_excl_scan(const int *in, int *out, int n, int *s_tmp) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int per = (n + kPlanThreads - 1) / kPlanThreads;
    const int lo = min(tid * per, n), hi = min(lo + per, n);
    int sum = 0;
    for (int i = lo; i < hi; ++i) sum += in[i];
    int incl = warp_incl_scan(sum);
    if (lane == 31) s_tmp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int v = lane < kWarps ? s_tmp[lane] : 0;
        int iv = warp_incl_scan(v);
        if (lane < kWarps) s_tmp[lane] = iv - v;
        if (lane == kWarps - 1) s_tmp[32] = iv;
    }
    __syncthreads();
    int run = s_tmp[warp] + incl - sum;
    for (int i = lo; i < hi; ++i) {
        int v = in[i];
        out[i] = run;
        run += v;
    }
    int total = s_tmp[32];
    __syncthreads();
    return total;
}

// first m >= i with ce[m] > v (ce strictly increasing over [0, M)); warp-wide
__device__ int advance_chunk(const int *ce, int M, int i, int v) {
    const int lane = threadIdx.x & 31;
    while (true) {
        int idx = i + lane;
        bool le = idx < M && ce[idx] <= v;
        unsigned bal = __ballot_sync(0xffffffffu, le);
        if (bal == 0xffffffffu) {
            i += 32;
            continue;
        }
        return i + __ffs(~bal) - 1;
    }
}

// Bounded grid barrier over gridDim.x CTAs (counters zeroed by the caller's
// memset before the launch).  Returns false if this CTA gave up waiting.
__device__ bool grid_barrier(int32_t *ws, int64_t limit) {
    __shared__ int s_ok;
    __syncthreads();
    if (threadIdx.x == 0) {
        volatile int32_t *gen = ws + HDR_BAR_GEN;
        int g = *gen;
        __threadfence();
        int arrived = atomicAdd(ws + HDR_BAR_COUNT, 1);
        bool ok = true;
        if (arrived == (int)gridDim.x - 1) {
            atomicExch(ws + HDR_BAR_COUNT, 0);
            __threadfence();
            atomicAdd(ws + HDR_BAR_GEN, 1);
        } else {
            int64_t n = 0;
            while (*gen == g) {
                if (++n > limit) {
                    ok = false;
                    break;
                }
                __nanosleep(64);
            }
        }
        __threadfence();
        s_ok = ok;
    }
    __syncthreads();
    return s_ok != 0;
}

// Exclusive prefix of one expert's per-range counts, in place (one warp).
__device__ void scan_column(int32_t *col, int64_t Q) {
    const int lane = threadIdx.x & 31;
    int carry = 0;
    for (int64_t q0 = 0; q0 < Q; q0 += 32 * 16) {
        int v[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            int64_t q = q0 + u * 32 + lane;
            v[u] = q < Q ? __ldcg(col + q) : 0;
        }
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            int incl = warp_incl_scan(v[u]);
            int64_t q = q0 + u * 32 + lane;
            if (q < Q) col[q] = carry + incl - v[u];
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
    }
}

// The planner (one CTA).  Shared memory: six arrays of N ints + small ones.
__device__ void plan_tables(const PlanParams &p, int *sm) {
    const moonep_cfg_t &c = p.cfg;
    const int N = p.N, R = c.R, L = c.L, B = c.B, C = c.C, Cm = c.C_max;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const moonep_ws_layout_t &lay = p.lay;
    int32_t *ws = p.ws;

    int *s_cnt = sm;        // copies per expert
    int *s_x = sm + N;      // scans
    int *s_sp = sm + 2 * N; // spill per expert
    int *s_ce = sm + 3 * N; // chunk end positions in the spill stream
    int *s_ch = sm + 4 * N; // chunk -> expert
    int *s_y = sm + 5 * N;  // scratch
    __shared__ int s_def[kMaxR], s_rp[kMaxR], s_rt[kMaxR], s_ri0[kMaxR], s_rnp[kMaxR], s_rpb[kMaxR];
    __shared__ int s_tmp[33];
    __shared__ int s_misc[4];  // 0 p_end, 1 n_rx, 2 pieces, 3 capacity error

    for (int e = tid; e < N; e += kPlanThreads) s_cnt[e] = __ldcg(ws + lay.cnt + e);
    if (tid < 4) s_misc[tid] = 0;
    __syncthreads();

    // keep/spill: each home rank keeps rows in local-expert order up to C
    const int total = block_excl_scan(s_cnt, s_x, N, s_tmp);
    for (int e = tid; e < N; e += kPlanThreads) {
        const int h = e / L;
        const int hx = s_x[e] - s_x[h * L];
        const int ce = s_cnt[e];
        const int k = min(ce, max(0, C - hx));
        ws[lay.keep + e] = k;
        ws[lay.home_off + e] = min(hx, C);
        ws[lay.spill + e] = ce - k;
        s_sp[e] = ce - k;
    }
    for (int h = tid; h < R; h += kPlanThreads) {
        const int lo = s_x[h * L];
        const int hi = h + 1 < R ? s_x[(h + 1) * L] : total;
        const int ld = hi - lo;
        const int d = C - min(ld, C);
        ws[lay.load + h] = ld;
        ws[lay.deficit + h] = d;
        s_def[h] = d;
    }
    __syncthreads();

    // the spill stream and its chunks
    const int total_spill = block_excl_scan(s_sp, s_x, N, s_tmp);  // s_x = A_e
    for (int e = tid; e < N; e += kPlanThreads) s_y[e] = s_sp[e] > 0 ? 1 : 0;
    __syncthreads();
    const int M = block_excl_scan(s_y, s_y, N, s_tmp);  // s_y = chunk index
    for (int e = tid; e < N; e += kPlanThreads)
        if (s_sp[e] > 0) {
            s_ce[s_y[e]] = s_x[e] + s_sp[e];
            s_ch[s_y[e]] = e;
        }
    __syncthreads();

    // receiver walk: receiver r takes the stream from p_r until its deficit
    // is filled or it has touched B chunks
    if (warp == 0) {
        int pos = 0, i0 = 0;
        for (int r = 0; r < R; ++r) {
            const int d = s_def[r];
            int take = 0, np = 0, ir = i0;
            const int pr = pos;
            if (d > 0 && pos < total_spill && B > 0) {
                i0 = advance_chunk(s_ce, M, i0, pos);
                const int i1 = min(i0 + B - 1, M - 1);
                take = min(d, s_ce[i1] - pos);
                const int il = advance_chunk(s_ce, M, i0, pos + take - 1);
                np = il - i0 + 1;
                ir = i0;
                pos += take;
            }
            if (lane == 0) {
                s_rp[r] = pr;
                s_rt[r] = take;
                s_ri0[r] = ir;
                s_rnp[r] = np;
            }
        }
        // pieces per receiver -> exclusive prefix (R <= 64: two per lane)
        const int a = lane < R ? s_rnp[lane] : 0;
        const int b = lane + 32 < R ? s_rnp[lane + 32] : 0;
        const int ia = warp_incl_scan(a);
        const int tot_a = __shfl_sync(0xffffffffu, ia, 31);
        const int ib = warp_incl_scan(b);
        if (lane < R) s_rpb[lane] = ia - a;
        if (lane + 32 < R) s_rpb[lane + 32] = tot_a + ib - b;
        const int P = tot_a + __shfl_sync(0xffffffffu, ib, 31);
        // replicated experts are the chunks that start before the walk's end
        const int nrx = pos > 0 ? advance_chunk(s_ce, M, 0, pos - 1) + 1 : 0;
        if (lane == 0) {
            s_misc[0] = pos;
            s_misc[1] = nrx;
            s_misc[2] = P;
        }
    }
    __syncthreads();
    const int p_end = s_misc[0], nrx = s_misc[1], P = s_misc[2];

    for (int r = tid; r < R; r += kPlanThreads) {
        ws[lay.fill + r] = C - s_def[r] + s_rt[r];
        ws[lay.slots_used + r] = s_rnp[r];
    }
    for (int e = tid; e < N; e += kPlanThreads) s_y[e] = 0;  // pieces per expert
    __syncthreads();

    // pieces and slots
    for (int idx = tid; idx < R * B; idx += kPlanThreads) {
        const int r = idx / B, b = idx - r * B;
        if (b < s_rnp[r]) {
            const int i = s_ri0[r] + b;
            const int e = s_ch[i];
            const int ce = s_ce[i], cs = ce - s_sp[e];
            const int lo = max(s_rp[r], cs), hi = min(s_rp[r] + s_rt[r], ce);
            const int n = hi - lo;
            const int fj = (s_cnt[e] - s_sp[e]) + (lo - cs);
            const int soff = (C - s_def[r]) + (lo - s_rp[r]);
            const int gp = s_rpb[r] + b;
            ws[lay.rep_expert + gp] = e;
            ws[lay.rep_recv + gp] = r;
            ws[lay.rep_slot + gp] = b;
            ws[lay.rep_first_j + gp] = fj;
            ws[lay.rep_cnt + gp] = n;
            ws[lay.slot_expert + idx] = e;
            ws[lay.slot_cnt + idx] = n;
            ws[lay.slot_off + idx] = soff;
            ws[lay.slot_first_j + idx] = fj;
            // route entry of this piece: after e's home entry and e's earlier pieces
            ws[lay.route_end + 2 * e + 1 + gp] = fj + n;
            ws[lay.route_base + 2 * e + 1 + gp] = r * Cm + soff - fj;
            atomicAdd(&s_y[e], 1);
        } else {
            ws[lay.slot_expert + idx] = -1;
            ws[lay.slot_cnt + idx] = 0;
            ws[lay.slot_off + idx] = C - s_def[r] + s_rt[r];
            ws[lay.slot_first_j + idx] = 0;
        }
    }
    for (int x = tid; x < nrx; x += kPlanThreads) ws[lay.rx_expert + x] = s_ch[x];
    __syncthreads();
    block_excl_scan(s_y, s_y, N, s_tmp);  // s_y = rep_ptr

    // fallback rows: the stream beyond the walk's end, per chunk
    for (int e = tid; e < N; e += kPlanThreads) {
        int fb = 0;
        if (s_sp[e] > 0) {
            const int cs = s_x[e], ce = cs + s_sp[e];
            fb = max(0, ce - max(cs, p_end));
        }
        s_x[e] = fb;
        ws[lay.fb_cnt + e] = fb;
    }
    __syncthreads();
    block_excl_scan(s_x, s_ce, N, s_tmp);  // s_ce = exclusive prefix of fb_cnt
    // (s_x still holds fb_cnt)
    for (int e = tid; e < N; e += kPlanThreads) {
        const int h = e / L;
        const int fbo = C + (s_ce[e] - s_ce[h * L]);
        const int fb = s_x[e];
        const int keep = s_cnt[e] - s_sp[e];
        const int rp = s_y[e];
        const int rn = (e + 1 < N ? s_y[e + 1] : P) - rp;
        ws[lay.fb_off + e] = fbo;
        ws[lay.rep_ptr + e] = rp;
        ws[lay.route_ptr + e] = 2 * e + rp;
        ws[lay.route_end + 2 * e + rp] = keep;
        ws[lay.route_base + 2 * e + rp] = h * Cm + ws[lay.home_off + e];
        ws[lay.route_end + 2 * e + rp + rn + 1] = s_cnt[e];
        ws[lay.route_base + 2 * e + rp + rn + 1] = h * Cm + fbo - (s_cnt[e] - fb);
        if ((e % L) == L - 1 && fbo + fb > Cm) s_misc[3] = 1;
    }
    if (tid == 0) {
        ws[lay.rep_ptr + N] = P;
        ws[lay.route_ptr + N] = 2 * N + P;
    }
    // segment tables [R][2L+B]: local, slot, fallback
    const int SEG = 2 * L + B;
    for (int idx = tid; idx < R * SEG; idx += kPlanThreads) {
        const int r = idx / SEG, s = idx - r * SEG;
        int off, len;
        if (s < L) {
            const int e = r * L + s;
            off = ws[lay.home_off + e];
            len = s_cnt[e] - s_sp[e];
        } else if (s < L + B) {
            off = ws[lay.slot_off + r * B + (s - L)];
            len = ws[lay.slot_cnt + r * B + (s - L)];
        } else {
            const int e = r * L + (s - L - B);
            off = C + (s_ce[e] - s_ce[r * L]);
            len = s_x[e];
        }
        ws[lay.seg_off + idx] = off;
        ws[lay.seg_len + idx] = len;
    }
    // allocation table: zero, then home (keep + fallback) and pieces
    for (int64_t i = tid; i < (int64_t)N * R; i += kPlanThreads) ws[lay.alloc + i] = 0;
    __syncthreads();
    for (int e = tid; e < N; e += kPlanThreads)
        ws[lay.alloc + (int64_t)e * R + e / L] = s_cnt[e] - s_sp[e] + s_x[e];
    for (int gp = tid; gp < P; gp += kPlanThreads)
        ws[lay.alloc + (int64_t)ws[lay.rep_expert + gp] * R + ws[lay.rep_recv + gp]] = ws[lay.rep_cnt + gp];
    __syncthreads();
    if (tid == 0) {
        const int fallback = total_spill - p_end;
        int st = 0;
        if (s_misc[3]) st |= MOONEP_ST_CAPACITY;
        if (fallback > 0) st |= MOONEP_ST_FALLBACK;
        ws[HDR_FALLBACK] = fallback;
        ws[HDR_NREP] = P;
        ws[HDR_MIGRATED] = total_spill - fallback;
        ws[HDR_NRX] = nrx;
        ws[HDR_TOTAL_SPILL] = total_spill;
        ws[HDR_PEND] = p_end;
        __threadfence();
        if (st) atomicOr(ws + HDR_STATUS, st);
    }
}

__global__ void __launch_bounds__(kPlanThreads, 1) plan_kernel(const __grid_constant__ PlanParams p) {
    extern __shared__ __align__(16) int sm[];
    const int N = p.N, K = p.cfg.K;
    const int tid = threadIdx.x;
    int32_t *ws = p.ws;
    const moonep_ws_layout_t &lay = p.lay;

    // phase A: per-range histograms
    bool bad = false;
    for (int64_t q = blockIdx.x; q < p.Q; q += gridDim.x) {
        for (int e = tid; e < N; e += kPlanThreads) sm[e] = 0;
        __syncthreads();
        const int64_t i0 = range_begin(q, p.T, p.Q) * K, i1 = range_begin(q + 1, p.T, p.Q) * K;
        for (int64_t i = i0 + tid; i < i1; i += kPlanThreads) {
            const int e = __ldg(p.ids + i);
            if ((unsigned)e < (unsigned)N)
                atomicAdd(&sm[e], 1);
            else
                bad = true;
        }
        __syncthreads();
        for (int e = tid; e < N; e += kPlanThreads) {
            const int v = sm[e];
            ws[lay.base + (int64_t)e * p.Q + q] = v;
            if (v) atomicAdd(ws + lay.cnt + e, v);
        }
        __syncthreads();
    }
    if (bad) atomicOr(ws + HDR_STATUS, MOONEP_ST_EXPERT_ID);
    if (blockIdx.x == 0 && tid < 8) ws[HDR_CFG + tid] = (&p.cfg.R)[tid];
    if (blockIdx.x == 0 && tid == 0) ws[HDR_NRANGES] = (int32_t)p.Q;
    __threadfence();

    if (!grid_barrier(ws, p.wait_limit)) {
        if (tid == 0) atomicOr(ws + HDR_STATUS, MOONEP_ST_TIMEOUT);
        return;
    }
    const int st = __ldcg(ws + HDR_STATUS);
    if (st & MOONEP_ST_ERROR_MASK) return;

    // phase B: column prefixes on CTAs 1.. (or all on CTA 0 if alone)
    const int warp = tid >> 5;
    if (gridDim.x == 1) {
        for (int e = warp; e < N; e += kWarps) scan_column(ws + lay.base + (int64_t)e * p.Q, p.Q);
        __syncthreads();
        plan_tables(p, sm);
    } else if (blockIdx.x == 0) {
        plan_tables(p, sm);
    } else {
        const int gw = (blockIdx.x - 1) * kWarps + warp;
        const int nw = (gridDim.x - 1) * kWarps;
        for (int e = gw; e < N; e += nw) scan_column(ws + lay.base + (int64_t)e * p.Q, p.Q);
    }
}

}  // namespace

size_t plan_smem_bytes(int N) { return (size_t)6 * (N > 0 ? N : 1) * sizeof(int); }

const void *plan_kernel_ptr() { return (const void *)plan_kernel; }

cudaError_t launch_plan(const PlanParams &p, int grid, size_t smem, cudaStream_t s) {
    void *args[] = {(void *)&p};
    return cudaLaunchCooperativeKernel((const void *)plan_kernel, dim3(grid), dim3(kPlanThreads), args, smem, s);
}

}  // namespace moonep
