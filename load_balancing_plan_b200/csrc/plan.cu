// plan.cu -- moonep_plan: the online redundant-expert planning kernel.
//
// "The Busiest Rank Sets Your Step Time: Running MoonEP's Planning Code
// Ourselves", section "What the technique is" (flowchart: router output
// topk_experts / tokens_per_expert -> planning kernel deciding online which
// experts to duplicate and where), and twodots.gr "MoonEP balances AI
// experts in MoE models" (the GPU planner; the planner emits cu_seqlens).
//
// One persistent cooperative kernel, 512 threads per CTA, one CTA per SM:
//   phase A  every CTA walks blocks of consecutive token ranges, counting
//            the top-K ids into a running shared-memory histogram; it
//            stores the running count before each range (base: copies of e
//            in the block's earlier ranges) and the block total (blk), and
//            adds the totals to the global tokens_per_expert (cnt);
//   barrier  one bounded grid barrier (gives up after wait_limit polls and
//            records MOONEP_ST_TIMEOUT; all CTAs are co-resident by the
//            cooperative launch, so it normally completes at once);
//   phase B  CTA 0 runs the planner on cnt (keep/spill split, spill stream,
//            receiver walk, pieces, slots, fallback, route/segment/alloc
//            tables) while CTAs 1.. turn the block totals into exclusive
//            prefixes (one warp per expert column).
//
// The spill planner.  Spilled rows form one stream, expert by expert in
// ascending order (chunk m of expert e spans stream positions [A_e, A_e +
// spill_e)).  Receivers (ranks with deficit > 0) are visited in ascending
// order; receiver r starts where the previous one stopped, at position p_r,
// and takes rows until it has either filled its deficit or used its B slots
// (one slot per chunk it touches).  That is exactly "each chunk goes to the
// lowest-index rank that still has room and a free slot", computed as a walk
// over at most R receivers instead of over the chunks.  Rows past the last
// receiver's stop fall back to their home rank's headroom.  Plan flags: with
// MOONEP_PLAN_REMOTE_WEIGHTS the B limit is dropped (pieces past a receiver's
// B-th read their weights remotely); with MOONEP_PLAN_ONE_GROUP a receiver
// also stops where the stream leaves its first chunk's home group.
#include "moonep_internal.cuh"

namespace moonep {

namespace {

constexpr int kPlanThreads = 512;

// MOONEP_PLAN_TRACE: development builds stamp %globaltimer (ns) at the phase
// boundaries of CTA 0 into header words 32..55 of the workspace (12 stamps),
// and the grid's start and counting-end spread into words 56..61.
#ifdef MOONEP_PLAN_TRACE
__device__ __forceinline__ void trace(int32_t *ws, int slot) {
    if (threadIdx.x == 0) {
        uint64_t t;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
        reinterpret_cast<unsigned long long *>(ws + 32)[slot] = t;
    }
}
#define TRACE(ws, slot) trace(ws, slot)
// every CTA: words 56..57 the latest end of a counting phase, 58..59 the
// complement of the earliest start, 60..61 the latest start
__device__ __forceinline__ void trace_grid(int32_t *ws, bool start) {
    if (threadIdx.x == 0) {
        unsigned long long t;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
        unsigned long long *w = reinterpret_cast<unsigned long long *>(ws + 56);
        if (start) {
            atomicMax(w + 1, ~t);
            atomicMax(w + 2, t);
        } else {
            atomicMax(w, t);
        }
    }
}
#define TRACE_GRID(ws, start) trace_grid(ws, start)
#else
#define TRACE(ws, slot) ((void)0)
#define TRACE_GRID(ws, start) ((void)0)
#endif
constexpr int kWarps = kPlanThreads / 32;
constexpr int kMaxR = 64;
#ifndef MOONEP_ID_BATCH
#define MOONEP_ID_BATCH 8  // ids per thread loaded together in the counting phase (16: the plan
                           // ran 9 us slower in the step on training, its code no longer cold-friendly)
#endif
constexpr int kIdBatch = MOONEP_ID_BATCH;
// Above this many experts the whole CTA plans.  Alone and warm, one warp
// plans a few hundred experts faster (no block barriers), but right after
// GBs of streaming traffic, as in a real step, the CTA-wide planner wins at
// every size measured: 36 -> 28 us at 64 experts, 57 -> 40 us at 256, 42 ->
// 30 us at 384.
#ifndef MOONEP_WARP_PLANNER_MAX_N
#define MOONEP_WARP_PLANNER_MAX_N 32
#endif
constexpr int kWarpPlannerMaxN = MOONEP_WARP_PLANNER_MAX_N;
// The receiver walk: first all receivers at once, checked, then one after
// another only if a chunk limit stops some receiver (1); always one after
// another (0).  On 16 receivers the sequential walk took 5-7 us of the plan.
#ifndef MOONEP_PLAN_SPEC_WALK
#define MOONEP_PLAN_SPEC_WALK 1
#endif
// Counting: the block's totals per expert from its histogram's columns after
// the counting (1) or by a second shared-memory atomic per id (0); the
// token and range of an id by multiply-high with a reciprocal made at launch
// (1) or by 32-bit division (0).  floor(n / d) = hi64(n * m) with
// m = floor((2^64 - 1) / d) + 1 holds for every n, d < 2^32, d >= 2: m
// exceeds 2^64 / d by at most 1, so n * m / 2^64 exceeds n / d by less than
// 2^-32 < 1 / d, which cannot carry n / d past the next integer.
#ifndef MOONEP_PLAN_TOT_SUM
#define MOONEP_PLAN_TOT_SUM 0  // 1 measured no faster alone, and slower with the multiply-high division
#endif
#ifndef MOONEP_PLAN_FASTDIV
#define MOONEP_PLAN_FASTDIV 1
#endif

// The planner and its scans run once per plan, cold: after a step's GBs of
// streaming no line of their code is in any cache, and each line fetched costs
// a round trip to L2 or HBM.  Their loops are therefore not unrolled
// (`#pragma unroll 1`): at 512 threads and up to a few thousand experts they
// run one or a few iterations per thread, so unrolled copies only lengthen
// the code.  Inside the training step this took the plan from 32.5 to 26 us.
//
// Exclusive scan of n ints (in and out may alias) by one warp; returns the
// total.  Lane l owns the contiguous run [l*per, (l+1)*per), per = ceil(n/32).
__device__ int warp_excl_scan(const int *in, int *out, int n) {
    const int lane = threadIdx.x & 31;
    const int per = (n + 31) >> 5;
    const int lo = min(lane * per, n), hi = min(lo + per, n);
    int sum = 0;
    #pragma unroll 1
    for (int i = lo; i < hi; ++i) sum += in[i];
    const int incl = warp_incl_scan(sum);
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    int run = incl - sum;
    #pragma unroll 1
    for (int i = lo; i < hi; ++i) {
        const int v = in[i];
        out[i] = run;
        run += v;
    }
    __syncwarp();
    return total;
}

// The same by the whole CTA (kPlanThreads threads, contiguous runs of
// ceil(n / kPlanThreads)); s_tmp holds 33 ints.
__device__ int block_excl_scan(const int *in, int *out, int n, int *s_tmp) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int per = (n + kPlanThreads - 1) / kPlanThreads;
    const int lo = min(tid * per, n), hi = min(lo + per, n);
    int sum = 0;
    #pragma unroll 1
    for (int i = lo; i < hi; ++i) sum += in[i];
    const int incl = warp_incl_scan(sum);
    if (lane == 31) s_tmp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int v = lane < kWarps ? s_tmp[lane] : 0;
        const int iv = warp_incl_scan(v);
        if (lane < kWarps) s_tmp[lane] = iv - v;
        if (lane == kWarps - 1) s_tmp[32] = iv;
    }
    __syncthreads();
    int run = s_tmp[warp] + incl - sum;
    #pragma unroll 1
    for (int i = lo; i < hi; ++i) {
        const int v = in[i];
        out[i] = run;
        run += v;
    }
    const int total = s_tmp[32];
    __syncthreads();
    return total;
}

// Two exclusive scans at once (a and b of n ints each; a's input and output
// may alias, as may b's, but not one with the other): the same runs per
// thread and the same barriers as one scan.  Returns both totals.
__device__ int2 warp_excl_scan2(const int *ia, int *oa, const int *ib, int *ob, int n) {
    const int lane = threadIdx.x & 31;
    const int per = (n + 31) >> 5;
    const int lo = min(lane * per, n), hi = min(lo + per, n);
    int sa = 0, sb = 0;
#pragma unroll 1
    for (int i = lo; i < hi; ++i) {
        sa += ia[i];
        sb += ib[i];
    }
    const int xa = warp_incl_scan(sa), xb = warp_incl_scan(sb);
    const int2 tot = make_int2(__shfl_sync(0xffffffffu, xa, 31), __shfl_sync(0xffffffffu, xb, 31));
    int ra = xa - sa, rb = xb - sb;
#pragma unroll 1
    for (int i = lo; i < hi; ++i) {
        const int a = ia[i], b = ib[i];
        oa[i] = ra;
        ob[i] = rb;
        ra += a;
        rb += b;
    }
    __syncwarp();
    return tot;
}

// s_tmp holds 66 ints
__device__ int2 block_excl_scan2(const int *ia, int *oa, const int *ib, int *ob, int n, int *s_tmp) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int per = (n + kPlanThreads - 1) / kPlanThreads;
    const int lo = min(tid * per, n), hi = min(lo + per, n);
    int sa = 0, sb = 0;
#pragma unroll 1
    for (int i = lo; i < hi; ++i) {
        sa += ia[i];
        sb += ib[i];
    }
    const int xa = warp_incl_scan(sa), xb = warp_incl_scan(sb);
    if (lane == 31) {
        s_tmp[warp] = xa;
        s_tmp[33 + warp] = xb;
    }
    __syncthreads();
    if (warp == 0) {
        const int va = lane < kWarps ? s_tmp[lane] : 0, vb = lane < kWarps ? s_tmp[33 + lane] : 0;
        const int ja = warp_incl_scan(va), jb = warp_incl_scan(vb);
        if (lane < kWarps) {
            s_tmp[lane] = ja - va;
            s_tmp[33 + lane] = jb - vb;
        }
        if (lane == kWarps - 1) {
            s_tmp[32] = ja;
            s_tmp[65] = jb;
        }
    }
    __syncthreads();
    int ra = s_tmp[warp] + xa - sa, rb = s_tmp[33 + warp] + xb - sb;
#pragma unroll 1
    for (int i = lo; i < hi; ++i) {
        const int a = ia[i], b = ib[i];
        oa[i] = ra;
        ob[i] = rb;
        ra += a;
        rb += b;
    }
    const int2 tot = make_int2(s_tmp[32], s_tmp[65]);
    __syncthreads();
    return tot;
}

// first m in [0, M) with a[m] > v, or M (a strictly increasing); one thread
__device__ __forceinline__ int first_above(const int *a, int M, int v) {
    int lo = 0, hi = M;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (a[mid] > v)
            hi = mid;
        else
            lo = mid + 1;
    }
    return lo;
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
// MOONEP_BARRIER_ONCE (the default) builds the form for a kernel that passes
// one barrier per launch: thread 0 of each CTA releases the CTA's writes
// (the CTA barrier orders them before its fence) and adds one to the
// counter, then waits until the counter reaches the grid size; no
// generation word and no reset, so the last CTA to arrive is not delayed by
// two more atomics.  0 builds the reusable form with a generation word.
#ifndef MOONEP_BARRIER_ONCE
#define MOONEP_BARRIER_ONCE 1
#endif
__device__ bool grid_barrier(int32_t *ws, int64_t limit) {
    __shared__ int s_ok;
    __syncthreads();
    if (MOONEP_BARRIER_ONCE && threadIdx.x == 0) {
        volatile int32_t *count = ws + HDR_BAR_COUNT;
        __threadfence();
        atomicAdd(ws + HDR_BAR_COUNT, 1);
        bool ok = true;
        int64_t n = 0;
        while (*count < (int)gridDim.x) {
            if (++n > limit) {
                ok = false;
                break;
            }
            __nanosleep(32);
        }
        __threadfence();
        s_ok = ok;
    } else if (!MOONEP_BARRIER_ONCE && threadIdx.x == 0) {
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

// Exclusive prefix of one expert's per-block counts, in place (one warp),
// starting from carry0.  The column has Q <= kBlocks entries (one per block
// of token ranges): lane l owns the run [l*per, (l+1)*per), per =
// ceil(Q / 32) <= kScanPer, so one warp scan covers the column.
constexpr int kScanPer = (int)((kBlocks + 31) / 32);
__device__ void scan_column(int32_t *col, int64_t Q, int carry0 = 0) {
    const int lane = threadIdx.x & 31;
    const int per = (int)((Q + 31) >> 5);
    const int lo = min(lane * per, (int)Q), hi = min(lo + per, (int)Q);
    int v[kScanPer];
    int sum = 0;
#pragma unroll
    for (int u = 0; u < kScanPer; ++u) {
        v[u] = lo + u < hi ? __ldcg(col + lo + u) : 0;
        sum += v[u];
    }
    const int incl = warp_incl_scan(sum);
    int run = carry0 + incl - sum;
#pragma unroll
    for (int u = 0; u < kScanPer; ++u) {
        if (lo + u < hi) col[lo + u] = run;
        run += v[u];
    }
}

// The planner, run by NT threads of CTA 0: one warp (NT = 32, no block-wide
// barriers; up to kWarpPlannerMaxN experts) or the whole CTA (NT =
// kPlanThreads, above that).  Every intermediate lives in
// shared memory (seven arrays of N ints and a few of R); global memory is
// only written.  The receiver walk is sequential and always runs on warp 0.
template <int NT>
__device__ void plan_tables(const PlanParams &p, int *sm) {
    const moonep_cfg_t &c = p.cfg;
    const int N = p.N, R = c.R, L = c.L, B = c.B, C = c.C, Cm = c.C_max;
    const int SEG = 2 * L + B;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int NW = NT / 32;
    const moonep_ws_layout_t &lay = p.lay;
    int32_t *ws = p.ws;

    int *s_cnt = sm;          // copies per expert
    int *s_x = sm + N;        // scans: cnt prefix, then spill-stream starts, then fb_cnt
    int *s_sp = sm + 2 * N;   // spill per expert
    int *s_ce = sm + 3 * N;   // chunk end positions in the spill stream, then fb prefix
    int *s_ch = sm + 4 * N;   // chunk -> expert
    int *s_y = sm + 5 * N;    // chunk index, then pieces per expert -> rep_ptr
    int *s_hoff = sm + 6 * N; // row of the expert's local segment
    __shared__ int s_def[kMaxR], s_rp[kMaxR], s_rt[kMaxR], s_ri0[kMaxR], s_rnp[kMaxR], s_rpb[kMaxR], s_spb[kMaxR];
    __shared__ int s_tmp[66];
    __shared__ int s_misc[6];  // 0 p_end, 1 P, 2 NSLOT, 3 nrx, 4 capacity error
    const bool remote = (p.flags & MOONEP_PLAN_REMOTE_WEIGHTS) != 0;
    const bool one_group = (p.flags & MOONEP_PLAN_ONE_GROUP) != 0;
    auto sync = [] {
        if (NT == 32)
            __syncwarp();
        else
            __syncthreads();
    };
    auto scan = [&](const int *in, int *out, int n) {
        return NT == 32 ? warp_excl_scan(in, out, n) : block_excl_scan(in, out, n, s_tmp);
    };
    auto scan2 = [&](const int *ia, int *oa, const int *ib, int *ob, int n) {
        return NT == 32 ? warp_excl_scan2(ia, oa, ib, ob, n) : block_excl_scan2(ia, oa, ib, ob, n, s_tmp);
    };

    TRACE(ws, 3);
    if (tid == 0) s_misc[4] = 0;
    // keep/spill: each home rank keeps rows in local-expert order up to C
    const int total = scan(s_cnt, s_x, N);
    #pragma unroll 1
    for (int e = tid; e < N; e += NT) {
        const int h = e / L;
        const int hx = s_x[e] - s_x[h * L];
        const int ce = s_cnt[e];
        const int k = min(ce, max(0, C - hx));
        const int ho = min(hx, C);
        s_hoff[e] = ho;
        s_sp[e] = ce - k;
        s_y[e] = ce - k > 0 ? 1 : 0;
        ws[lay.keep + e] = k;
        ws[lay.home_off + e] = ho;
        ws[lay.spill + e] = ce - k;
        ws[lay.seg_off + h * SEG + (e - h * L)] = ho;
        ws[lay.seg_len + h * SEG + (e - h * L)] = k;
    }
    #pragma unroll 1
    for (int h = tid; h < R; h += NT) {
        const int lo = s_x[h * L];
        const int hi = h + 1 < R ? s_x[(h + 1) * L] : total;
        const int ld = hi - lo;
        const int d = C - min(ld, C);
        ws[lay.load + h] = ld;
        ws[lay.deficit + h] = d;
        s_def[h] = d;
    }
    sync();

    // the spill stream and its chunks
    // s_x = A_e (the spill stream's starts), s_y = chunk index
    const int2 t2 = scan2(s_sp, s_x, s_y, s_y, N);
    const int total_spill = t2.x, M = t2.y;
    #pragma unroll 1
    for (int e = tid; e < N; e += NT)
        if (s_sp[e] > 0) {
            s_ce[s_y[e]] = s_x[e] + s_sp[e];
            s_ch[s_y[e]] = e;
        }
    sync();
    TRACE(ws, 4);

    if (warp == 0) {
        // receiver walk: receiver r takes the stream from p_r until its
        // deficit is filled or (headroom rule) it has touched B chunks or
        // (one-group rule) the stream leaves its first chunk's home group
        int pos = 0;
        bool walked = false;
#if MOONEP_PLAN_SPEC_WALK
        {
            // All receivers at once, two per lane: if no chunk limit stops a
            // receiver, receiver r starts at min(D_r, total) (D_r: the
            // deficits of the receivers before it that take part) and takes
            // min(d_r, total - start).  Each lane then checks its receivers'
            // limits at those starts; if every take fits, these starts and
            // takes are exactly the walk's (each receiver's take is the
            // walk's take at the walk's start, by induction over r), else
            // the walk below runs one receiver after another.
            int a[2], st[2], tk[2], ci[2], np[2];
            bool ok = true;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int r = lane + 32 * h;
                a[h] = (r < R && (remote || B > 0)) ? max(s_def[r], 0) : 0;
            }
            const int ia = warp_incl_scan(a[0]);
            const int ta = __shfl_sync(0xffffffffu, ia, 31);
            const int ib = warp_incl_scan(a[1]);
            const int da[2] = {ia - a[0], ta + ib - a[1]};
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                st[h] = min(da[h], total_spill);
                tk[h] = min(a[h], total_spill - st[h]);
                ci[h] = 0;
                np[h] = 0;
                if (tk[h] > 0) {
                    const int i0 = first_above(s_ce, M, st[h]);
                    int i1 = remote ? M - 1 : min(i0 + B - 1, M - 1);
                    if (one_group) i1 = min(i1, first_above(s_ch, M, (s_ch[i0] / L + 1) * L - 1) - 1);
                    if (s_ce[i1] - st[h] < tk[h]) ok = false;
                    ci[h] = i0;
                    np[h] = first_above(s_ce, M, st[h] + tk[h] - 1) - i0 + 1;
                }
            }
            walked = __all_sync(0xffffffffu, ok);
            if (walked) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int r = lane + 32 * h;
                    if (r < R) {
                        s_rp[r] = st[h];
                        s_rt[r] = tk[h];
                        s_ri0[r] = ci[h];
                        s_rnp[r] = np[h];
                    }
                }
                pos = min(ta + __shfl_sync(0xffffffffu, ib, 31), total_spill);
            }
        }
#endif
        int i0 = 0;
        #pragma unroll 1
        for (int r = 0; r < R && !walked; ++r) {
            const int d = s_def[r];
            int take = 0, np = 0, ir = i0;
            const int pr = pos;
            if (d > 0 && pos < total_spill && (remote || B > 0)) {
                i0 = advance_chunk(s_ce, M, i0, pos);
                int i1 = remote ? M - 1 : min(i0 + B - 1, M - 1);
                if (one_group) {
                    // stop at the last chunk of the first chunk's home group
                    // (chunk experts ascend, so it is one before the first
                    // chunk of an expert of a later group)
                    const int h = s_ch[i0] / L;
                    i1 = min(i1, advance_chunk(s_ch, M, i0, (h + 1) * L - 1) - 1);
                }
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
        __syncwarp();
        // pieces per receiver -> exclusive prefix (R <= 64: two per lane), and
        // the same for the pieces that get a slot (the first B of each receiver)
        const int na = lane < R ? s_rnp[lane] : 0;
        const int nb = lane + 32 < R ? s_rnp[lane + 32] : 0;
        const int ia = warp_incl_scan(na);
        const int tot_a = __shfl_sync(0xffffffffu, ia, 31);
        const int ib = warp_incl_scan(nb);
        if (lane < R) s_rpb[lane] = ia - na;
        if (lane + 32 < R) s_rpb[lane + 32] = tot_a + ib - nb;
        const int sa = min(na, B), sb = min(nb, B);
        const int isa = warp_incl_scan(sa);
        const int tot_sa = __shfl_sync(0xffffffffu, isa, 31);
        const int isb = warp_incl_scan(sb);
        if (lane < R) s_spb[lane] = isa - sa;
        if (lane + 32 < R) s_spb[lane + 32] = tot_sa + isb - sb;
        // every lane takes part in these shuffles (a full-mask shuffle must
        // not sit under a lane-dependent branch)
        const int P_all = tot_a + __shfl_sync(0xffffffffu, ib, 31);
        const int nslot_all = tot_sa + __shfl_sync(0xffffffffu, isb, 31);
        // replicated experts are the chunks that start before the walk's end
        const int nrx = pos > 0 ? advance_chunk(s_ce, M, 0, pos - 1) + 1 : 0;
        if (lane == 0) {
            s_misc[0] = pos;
            s_misc[1] = P_all;
            s_misc[2] = nslot_all;
            s_misc[3] = nrx;
        }
    }
    #pragma unroll 1
    for (int e = tid; e < N; e += NT) s_y[e] = 0;  // pieces per expert
    sync();
    const int p_end = s_misc[0], P = s_misc[1], NSLOT = s_misc[2], nrx = s_misc[3];
    #pragma unroll 1
    for (int r = tid; r < R; r += NT) {
        ws[lay.fill + r] = C - s_def[r] + s_rt[r];
        ws[lay.slots_used + r] = min(s_rnp[r], B);
        ws[lay.recv_ptr + r] = s_rpb[r];
    }
    if (tid == 0) ws[lay.recv_ptr + R] = P;
    TRACE(ws, 5);

    // pieces (a warp per receiver), their slots and slot segments, route
    // entries and alloc entries
    #pragma unroll 1
    for (int r = warp; r < R; r += NW) {
        const int npr = s_rnp[r];
        #pragma unroll 1
        for (int b = lane; b < npr; b += 32) {
            const int i = s_ri0[r] + b;
            const int e = s_ch[i];
            const int ce = s_ce[i], cs = ce - s_sp[e];
            const int lo = max(s_rp[r], cs), hi = min(s_rp[r] + s_rt[r], ce);
            const int n = hi - lo;
            const int fj = (s_cnt[e] - s_sp[e]) + (lo - cs);
            const int off = (C - s_def[r]) + (lo - s_rp[r]);
            const int gp = s_rpb[r] + b;
            const int slot = b < B ? b : -1;
            ws[lay.rep_expert + gp] = e;
            ws[lay.rep_recv + gp] = r;
            ws[lay.rep_slot + gp] = slot;
            ws[lay.rep_first_j + gp] = fj;
            ws[lay.rep_cnt + gp] = n;
            ws[lay.rep_off + gp] = off;
            if (slot >= 0) {
                const int idx = r * B + slot;
                const int sg = r * SEG + L + slot;
                ws[lay.slot_expert + idx] = e;
                ws[lay.slot_cnt + idx] = n;
                ws[lay.slot_off + idx] = off;
                ws[lay.slot_first_j + idx] = fj;
                ws[lay.seg_off + sg] = off;
                ws[lay.seg_len + sg] = n;
                ws[lay.slot_piece + s_spb[r] + slot] = gp;
            }
            // route entry of this piece: after e's home entry and e's earlier pieces
            ws[lay.route_end + 2 * e + 1 + gp] = fj + n;
            ws[lay.route_base + 2 * e + 1 + gp] = r * Cm + off - fj;
            ws[lay.alloc + (int64_t)e * R + r] = n;
            atomicAdd(&s_y[e], 1);
        }
    }
    // slots no piece took
    #pragma unroll 1
    for (int idx = tid; idx < R * B; idx += NT) {
        const int r = idx / B, b = idx - r * B;
        if (b < s_rnp[r]) continue;
        const int sg = r * SEG + L + b;
        const int fill = C - s_def[r] + s_rt[r];
        ws[lay.slot_expert + idx] = -1;
        ws[lay.slot_cnt + idx] = 0;
        ws[lay.slot_off + idx] = fill;
        ws[lay.slot_first_j + idx] = 0;
        ws[lay.seg_off + sg] = fill;
        ws[lay.seg_len + sg] = 0;
    }
    #pragma unroll 1
    for (int x = tid; x < nrx; x += NT) ws[lay.rx_expert + x] = s_ch[x];
    // fallback rows: the stream beyond the walk's end, per chunk (s_x: A_e -> fb_cnt)
    #pragma unroll 1
    for (int e = tid; e < N; e += NT) {
        int fb = 0;
        if (s_sp[e] > 0) {
            const int cs = s_x[e], ce = cs + s_sp[e];
            fb = max(0, ce - max(cs, p_end));
        }
        s_x[e] = fb;
        ws[lay.fb_cnt + e] = fb;
    }
    sync();
    TRACE(ws, 6);
    scan2(s_y, s_y, s_x, s_ce, N);  // s_y = rep_ptr, s_ce = exclusive prefix of fb_cnt
    int cap_err = 0;
    #pragma unroll 1
    for (int e = tid; e < N; e += NT) {
        const int h = e / L;
        const int fbo = C + (s_ce[e] - s_ce[h * L]);
        const int fb = s_x[e];
        const int keep = s_cnt[e] - s_sp[e];
        const int rp = s_y[e];
        const int rn = (e + 1 < N ? s_y[e + 1] : P) - rp;
        const int sg = h * SEG + L + B + (e - h * L);
        ws[lay.fb_off + e] = fbo;
        ws[lay.rep_ptr + e] = rp;
        ws[lay.route_ptr + e] = 2 * e + rp;
        ws[lay.route_end + 2 * e + rp] = keep;
        ws[lay.route_base + 2 * e + rp] = h * Cm + s_hoff[e];
        ws[lay.route_end + 2 * e + rp + rn + 1] = s_cnt[e];
        ws[lay.route_base + 2 * e + rp + rn + 1] = h * Cm + fbo - (s_cnt[e] - fb);
        ws[lay.seg_off + sg] = fbo;
        ws[lay.seg_len + sg] = fb;
        ws[lay.alloc + (int64_t)e * R + h] = keep + fb;
        if ((e % L) == L - 1 && fbo + fb > Cm) cap_err = 1;
    }
    if (cap_err) s_misc[4] = 1;
    sync();
    if (tid == 0) {
        ws[lay.rep_ptr + N] = P;
        ws[lay.route_ptr + N] = 2 * N + P;
        const int fallback = total_spill - p_end;
        int st = 0;
        if (s_misc[4]) st |= MOONEP_ST_CAPACITY;
        if (fallback > 0) st |= MOONEP_ST_FALLBACK;
        ws[HDR_FALLBACK] = fallback;
        ws[HDR_NREP] = P;
        ws[HDR_MIGRATED] = total_spill - fallback;
        ws[HDR_NRX] = nrx;
        ws[HDR_FLAGS] = p.flags;
        ws[HDR_NSLOT] = NSLOT;
        ws[HDR_TOTAL_SPILL] = total_spill;
        ws[HDR_PEND] = p_end;
        TRACE(ws, 7);
        __threadfence();
        if (st) atomicOr(ws + HDR_STATUS, st);
    }
}

// Expert parallelism, the counts' exchange fused into the counting launch:
// the last counting CTA to finish copies the rank's finished counts [N + 1]
// into row `rank` of every rank's counts_all, through the peer table (plain
// stores, no multicast).  Each CTA releases its atomics and counts itself
// done; the one that sees every other CTA done acquires and copies, so no CTA
// waits for another.  After every rank's launch has completed (the caller's
// barrier), each counts_all holds all R rows, as an all-gather would leave it.
// (Not inlined: it runs only under expert parallelism, and the single-GPU
// plan's code stays as it was.)
__device__ __noinline__ void push_counts(const PlanParams &p) {
    __shared__ int s_last;
    const int N = p.N;
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const int done = atomicAdd(p.ws + HDR_COUNT_DONE, 1);
        s_last = done == (int)gridDim.x - 1;
        if (s_last) __threadfence();
    }
    __syncthreads();
    if (!s_last) return;
    const int64_t row = (int64_t)p.rank * (N + 1);
    for (int i = threadIdx.x; i <= N; i += blockDim.x) {
        const int v = __ldcg(p.counts_out + i);
        for (int q = 0; q < p.cfg.R; ++q) {
            int32_t *dst = reinterpret_cast<int32_t *>(__ldg(reinterpret_cast<const uint64_t *>(p.counts_peers) + q));
            dst[row + i] = v;
        }
    }
}

// Expert parallelism: the plan from every rank's counts ([R][N + 1]: the
// copies of each expert among the rank's tokens, then the rank's status
// bits).  CTA 0 sums the columns into tokens_per_expert (cnt) and plans
// exactly as the single-GPU plan does, so every rank derives the same
// tables; the other CTAs turn this rank's per-block counts into copy
// numbers, starting each expert at the copies the lower ranks hold (copies
// are numbered in ascending g = (r*S + s)*K + k across ranks).  A kernel of
// its own: the single-GPU plan kernel's code stays as small as before (its
// in-step time is bound by instruction fetches of run-once code).
__global__ void __launch_bounds__(kPlanThreads, 1) plan_from_counts_kernel(const __grid_constant__ PlanParams p) {
    extern __shared__ __align__(16) int sm[];
    const int N = p.N, R = p.cfg.R;
    const int tid = threadIdx.x, warp = tid >> 5;
    int32_t *ws = p.ws;
    const moonep_ws_layout_t &lay = p.lay;
    const int64_t NB = lay.n_blocks;
    const int64_t row = (int64_t)N + 1;
    if (block_status_failed(ws)) return;  // this rank's count found a bad id
    if (gridDim.x == 1 || blockIdx.x > 0) {
        const int gw = gridDim.x == 1 ? warp : (blockIdx.x - 1) * kWarps + warp;
        const int nw = gridDim.x == 1 ? kWarps : (gridDim.x - 1) * kWarps;
        for (int e = gw; e < N; e += nw) {
            int carry = 0;
            for (int r = 0; r < p.rank; ++r) carry += __ldg(p.counts_all + r * row + e);
            scan_column(ws + lay.blk + (int64_t)e * NB, NB, carry);
        }
        if (blockIdx.x > 0) return;
    }
    __shared__ int s_st;
    if (tid == 0) s_st = 0;
    __syncthreads();
    for (int r = tid; r < R; r += kPlanThreads) {
        const int st = __ldg(p.counts_all + r * row + N);
        if (st) atomicOr(&s_st, st);
    }
    for (int e = tid; e < N; e += kPlanThreads) {
        int c = 0;
        for (int r = 0; r < R; ++r) c += __ldg(p.counts_all + r * row + e);
        sm[e] = c;
        ws[lay.cnt + e] = c;
    }
    for (int64_t i = tid; i < (int64_t)N * R; i += kPlanThreads) ws[lay.alloc + i] = 0;
    __syncthreads();
    if (s_st & MOONEP_ST_ERROR_MASK) {
        // a bad id on some rank: no rank plans, so no rank dispatches
        if (tid == 0) atomicOr(ws + HDR_STATUS, s_st & MOONEP_ST_ERROR_MASK);
        return;
    }
    if (tid < 8) ws[HDR_CFG + tid] = (&p.cfg.R)[tid];
    if (tid == 0) {
        ws[HDR_NRANGES] = (int32_t)p.Q;
        ws[HDR_EP] = p.rank + 1;
    }
    __syncthreads();
    if (N > kWarpPlannerMaxN)
        plan_tables<kPlanThreads>(p, sm);
    else if (warp == 0)
        plan_tables<32>(p, sm);
}

__global__ void __launch_bounds__(kPlanThreads, 1) plan_kernel(const __grid_constant__ PlanParams p) {
    extern __shared__ __align__(16) int sm[];
    const int N = p.N, K = p.cfg.K;
    const int tid = threadIdx.x;
    int32_t *ws = p.ws;
    const moonep_ws_layout_t &lay = p.lay;

    if (blockIdx.x == 0) TRACE(ws, 0);
    TRACE_GRID(ws, true);
    // phase A: each counting CTA takes blocks of consecutive token ranges and
    // counts the block's ids into a shared-memory histogram per (range,
    // expert) and into the block's totals per expert -- all of a block's ids
    // are loaded in one batch of up to kIdBatch per thread, so a block costs
    // about one memory latency however many ranges it holds.  The totals go
    // to blk[e][b] and into the global tokens_per_expert (cnt).  Then one
    // thread per expert walks the block's ranges in order: base[q][e] =
    // copies of e in the block's earlier ranges (stored only where range q
    // has a copy of e: a range of a few tokens routes to few experts, and
    // dispatch reads no other entry).
    //
    // For the plan proper on more than one CTA, CTA 0 counts no block (it
    // plans after the barrier) and CTA k >= 1 counts block k - 1.  With one
    // block per counting CTA the histogram stays in shared memory over the
    // barrier and the range walk runs after it, beside the planner: only
    // dispatch reads base, and the barrier's fence would otherwise wait for
    // those thousands of scattered stores (3-4 us on the training workload).
    bool bad = false;
    const int64_t NB = lay.n_blocks;
    // copies per expert: into the plan's cnt, or (counting one rank's tokens
    // under expert parallelism) into the rank's counts_out
    int32_t *cnt_acc = p.mode == kPlanCount ? p.counts_out : ws + lay.cnt;
    // the range of token t is ((t + 1) * Q - 1) / T; in 32 bits when that
    // cannot overflow (every configuration up to 2^32 / Q tokens)
    const bool div32 = (uint64_t)(p.T + 1) * (uint64_t)p.Q < (uint64_t(1) << 32);
    const bool planner_apart = p.mode == kPlanFull && gridDim.x > 1;
    const int64_t b_step = planner_apart ? gridDim.x - 1 : gridDim.x;
    const int64_t b_first = planner_apart ? (blockIdx.x == 0 ? NB : (int64_t)blockIdx.x - 1) : blockIdx.x;
    const bool defer_walk = planner_apart && NB <= b_step;
    int64_t walk_qa = 0;
    int walk_nr = 0;
    bool walk_pending = false;
    auto walk = [&](int64_t qa, int nr) {
        for (int e = tid; e < N; e += kPlanThreads) {
            int run = 0;
            int32_t *dst = ws + lay.base + qa * N + e;
            const int *src = sm + e;
#pragma unroll 8
            for (int r = 0; r < nr; ++r, dst += N, src += N) {
                // dispatch reads base[q][e] only where range q routes to e
                const int c = *src;
                if (c) *dst = run;
                run += c;
            }
        }
    };
    for (int64_t b = b_first; b < NB; b += b_step) {
        const int64_t qa = block_first_range(b, p.Q, NB), qb = block_first_range(b + 1, p.Q, NB);
        const int nr = (int)(qb - qa);
        int *tot = sm + nr * N;  // the block's copies per expert
        {
            const int nz = nr * N + N;
            int4 *sm4 = reinterpret_cast<int4 *>(sm);
            for (int i = tid; i < nz / 4; i += kPlanThreads) sm4[i] = make_int4(0, 0, 0, 0);
            for (int i = (nz & ~3) + tid; i < nz; i += kPlanThreads) sm[i] = 0;
        }
        __syncthreads();
        if (blockIdx.x == 1) TRACE(ws, 9);
        const int64_t i0 = range_begin(qa, p.T, p.Q) * K, i1 = range_begin(qb, p.T, p.Q) * K;
        for (int64_t b0 = i0; b0 < i1; b0 += (int64_t)kIdBatch * kPlanThreads) {
            int v[kIdBatch];
#pragma unroll
            for (int u = 0; u < kIdBatch; ++u) {
                const int64_t i = b0 + tid + (int64_t)u * kPlanThreads;
                v[u] = i < i1 ? __ldg(p.ids + i) : -1;
            }
#pragma unroll
            for (int u = 0; u < kIdBatch; ++u) {
                const int64_t i = b0 + tid + (int64_t)u * kPlanThreads;
                if (i < i1) {
                    if ((unsigned)v[u] < (unsigned)N) {
                        // the range of token i / K: the last q with q*T/Q <= t
                        int64_t t, q;
                        if (MOONEP_PLAN_FASTDIV) {
                            const uint32_t iu = (uint32_t)i;  // i < T*K < 2^31
                            t = K == 1 ? (int64_t)iu : (int64_t)__umul64hi((uint64_t)iu, p.mK);
                            const uint32_t nq = (uint32_t)(t + 1) * (uint32_t)p.Q - 1u;
                            q = div32 ? (p.T == 1 ? (int64_t)nq : (int64_t)__umul64hi((uint64_t)nq, p.mT))
                                      : ((t + 1) * p.Q - 1) / p.T;
                        } else {
                            t = (int64_t)((uint32_t)i / (uint32_t)K);  // i < T*K < 2^31
                            q = div32 ? (int64_t)(((uint32_t)(t + 1) * (uint32_t)p.Q - 1u) / (uint32_t)p.T)
                                      : ((t + 1) * p.Q - 1) / p.T;
                        }
                        atomicAdd(&sm[(q - qa) * N + v[u]], 1);
                        if (!MOONEP_PLAN_TOT_SUM) atomicAdd(&tot[v[u]], 1);
                    } else {
                        bad = true;
                    }
                }
            }
        }
        __syncthreads();
        if (blockIdx.x == 1) TRACE(ws, 10);
        for (int e = tid; e < N; e += kPlanThreads) {
            int c = 0;
            if (MOONEP_PLAN_TOT_SUM) {
#pragma unroll 8
                for (int r = 0; r < nr; ++r) c += sm[r * N + e];
            } else {
                c = tot[e];
            }
            ws[lay.blk + (int64_t)e * NB + b] = c;
            if (c) atomicAdd(cnt_acc + e, c);
        }
        if (defer_walk) {
            walk_qa = qa;
            walk_nr = nr;
            walk_pending = true;
        } else {
            walk(qa, nr);
            __syncthreads();
        }
        if (blockIdx.x == 1) TRACE(ws, 11);
    }
    TRACE_GRID(ws, false);
    if (bad) atomicOr(ws + HDR_STATUS, MOONEP_ST_EXPERT_ID);
    if (p.mode == kPlanCount) {
        // the status travels with the counts, so every rank learns of it
        if (bad) atomicOr(p.counts_out + N, MOONEP_ST_EXPERT_ID);
        if (p.counts_peers) push_counts(p);
        return;
    }
    // the allocation table is only written after the barrier: clear it now,
    // spread over the whole grid
    for (int64_t i = (int64_t)blockIdx.x * kPlanThreads + tid; i < (int64_t)N * p.cfg.R;
         i += (int64_t)gridDim.x * kPlanThreads)
        ws[lay.alloc + i] = 0;
    if (blockIdx.x == 0) TRACE(ws, 1);
    if (blockIdx.x == 0 && tid < 8) ws[HDR_CFG + tid] = (&p.cfg.R)[tid];
    if (blockIdx.x == 0 && tid == 0) ws[HDR_NRANGES] = (int32_t)p.Q;
    if (!MOONEP_BARRIER_ONCE) __threadfence();

    if (!grid_barrier(ws, p.wait_limit)) {
        if (tid == 0) atomicOr(ws + HDR_STATUS, MOONEP_ST_TIMEOUT);
        return;
    }
    if (blockIdx.x == 0) TRACE(ws, 2);
    if (block_status_failed(ws)) return;

    // phase B: exclusive prefixes of the block totals per expert on CTAs 1..
    // (or all on CTA 0 if alone); CTA 0 loads cnt with all its threads, then
    // plans (one warp, or all warps for more than kWarpPlannerMaxN experts)
    const int warp = tid >> 5;
    if (gridDim.x == 1)
        for (int e = warp; e < N; e += kWarps) scan_column(ws + lay.blk + (int64_t)e * NB, NB);
    if (blockIdx.x == 0) {
        for (int e = tid; e < N; e += kPlanThreads) sm[e] = __ldcg(ws + lay.cnt + e);
        __syncthreads();
        if (N > kWarpPlannerMaxN)
            plan_tables<kPlanThreads>(p, sm);
        else if (warp == 0)
            plan_tables<32>(p, sm);
    } else {
        // the block's range walk, from the histogram kept in shared memory
        if (walk_pending) walk(walk_qa, walk_nr);
        const int gw = (blockIdx.x - 1) * kWarps + warp;
        const int nw = (gridDim.x - 1) * kWarps;
        for (int e = gw; e < N; e += nw) scan_column(ws + lay.blk + (int64_t)e * NB, NB);
        __syncthreads();
        if (blockIdx.x == 1) TRACE(ws, 8);
    }
}

}  // namespace

// Dynamic shared memory of the plan: 7 arrays of N ints for the planner, or
// phase A's (range, expert) histogram of a block and its totals,
// (ceil(Q / NB) + 1) * N ints, whichever is larger.  With Q <=
// max(kMinRanges, kBaseWords / N) and NB = min(Q, kBlocks),
// ceil(Q / NB) * N <= kBaseWords / kBlocks + N.
size_t plan_smem_bytes(int N) {
    const int64_t n = N > 0 ? N : 1;
    const int64_t a = 7 * n, b = kBaseWords / kBlocks + 2 * n + 4;
    return (size_t)(a > b ? a : b) * sizeof(int);
}

const void *plan_kernel_ptr() { return (const void *)plan_kernel; }

static uint64_t reciprocal64(int64_t d) { return d >= 2 ? ~uint64_t(0) / (uint64_t)d + 1 : 0; }

cudaError_t launch_plan(const PlanParams &p_in, int grid, size_t smem, cudaStream_t s) {
    PlanParams p = p_in;
    p.mK = reciprocal64(p.cfg.K);
    p.mT = reciprocal64(p.T);
    if (p.mode == kPlanFromCounts) {
        static std::atomic<size_t> smem_set[64];
        cudaError_t err = set_smem_limit((const void *)plan_from_counts_kernel, smem, smem_set);
        if (err != cudaSuccess) return err;
        plan_from_counts_kernel<<<grid, kPlanThreads, smem, s>>>(p);
        return cudaGetLastError();
    }
    if (p.mode == kPlanCount) {
        // no grid barrier when only counting: an ordinary launch
        plan_kernel<<<grid, kPlanThreads, smem, s>>>(p);
        return cudaGetLastError();
    }
    void *args[] = {(void *)&p};
    return cudaLaunchCooperativeKernel((const void *)plan_kernel, dim3(grid), dim3(kPlanThreads), args, smem, s);
}

}  // namespace moonep
