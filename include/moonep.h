/*
 * moonep.h -- C ABI of the MoonEP hot path on NVIDIA B200 (sm_100a).
 *
 * MoonEP ("Moonshot AI Open-Sources MoonEP: A Perfectly Balanced Expert
 * Parallelism Library for MoE Training", TL;DR) gives every expert-parallel
 * rank exactly C = S*K rows per MoE layer, whatever the router skew, by
 * planning a few redundant copies of hot experts online on the GPU and
 * routing the overflow to them.  This library implements the data path of
 * one layer for R expert-parallel ranks simulated as partitions of one
 * symmetric buffer in a single GPU's memory:
 *
 *   moonep_plan         histogram of the router's top-K ids, keep/spill split,
 *                       redundant-expert (spill) planner, all tables; one
 *                       persistent kernel, no host synchronisation
 *   moonep_dispatch     sender-side destination rows fused with the row
 *                       scatter of the hidden states (zero-copy permute)
 *   moonep_combine      gather of the expert outputs fused with the top-K
 *                       weighted fp32 sum (unpermute)
 *   moonep_prefetch     copy of the replicated experts' weights into the
 *                       receivers' prefetch slots
 *   moonep_reduce_grad  replica gradients added to the home experts'
 *                       gradients, used slots cleared
 *   moonep_combine_backward, moonep_dispatch_backward
 *                       the adjoints of combine and dispatch, for training
 *
 * Notation.  R ranks; L experts per rank; N = R*L experts; expert e lives on
 * home rank home(e) = e / L at local index e % L (the contiguous blocking of
 * the weight tensor in "The Busiest Rank Sets Your Step Time: Running
 * MoonEP's Planning Code Ourselves", section "Installation and integration");
 * S tokens per rank, T = R*S tokens; K experts per token; H hidden size; B
 * prefetch slots per rank; C = S*K rows per rank; C_max >= C rows allocated
 * per rank (rows [C, C_max) are the headroom for fallback rows).  A routed
 * copy has global index g = (r*S + s)*K + k for token s of rank r.
 *
 * Spill rule (the pages give no planning algorithm; this is the library's
 * rule).  Each home rank keeps its rows in local-expert order up to C.  The
 * overflow ("spilled chunks"), taken expert by expert in ascending expert
 * order, goes to the lowest-index ranks that still have room below C and a
 * free prefetch slot; each (expert, receiver) piece takes one slot.  Rows no
 * receiver can take stay on the home rank in the headroom, from row C on.
 * The copies of expert e are numbered j = 0, 1, ... in ascending g; copy j
 * goes home while j < keep[e], then through e's replica pieces in ascending
 * receiver order, then to the fallback rows.
 *
 * Row layout of rank r in the receive buffer recv[R][C_max][H] (the
 * "cu_seqlens" the group GEMM consumes, twodots.gr "MoonEP balances AI
 * experts in MoE models", memory-contract paragraphs): local segments of
 * experts r*L .. r*L+L-1 packed from row 0, then slots b = 0..B-1 packed
 * after them, then padding up to C (only if receivers ran out of slots),
 * then fallback segments of r's own experts from row C.  When no row falls
 * back every rank holds exactly C rows and rows [0, C) are all used.
 *
 * Ownership.  The caller allocates every device buffer, including the plan
 * workspace; the library never allocates or frees device memory.  Device
 * pointers must be 16-byte aligned (4-byte for int32/fp32 arrays); H must be
 * a multiple of 8 so each bf16 row is a whole number of 16-byte vectors.
 * Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 * default stream) except moonep_plan_read, which synchronises it.  The
 * receive buffer's rows are views valid until the next dispatch or combine
 * into the same buffer (twodots.gr, zero-copy views); rows outside the
 * plan's segments are never written.
 *
 * Errors.  Every call returns MOONEP_OK or a synchronous host error
 * (MOONEP_ERR_ARG: bad configuration, null or misaligned pointer, size out
 * of range; MOONEP_ERR_CUDA: a CUDA call failed; MOONEP_ERR_DEVICE: the
 * device is not sm_100).  moonep_last_error() describes the last one on the
 * calling thread.  Data-dependent errors are recorded on the device in the
 * workspace status word without host synchronisation (MOONEP_ST_* bits); a
 * call that finds an error bit set in the workspace writes nothing.
 * moonep_plan_read returns the status to the host.
 *
 * Limits: 1 <= R <= 64; N <= 4096; 1 <= K <= 64; 8 <= H <= 1048576;
 * 0 <= B <= 1024 and R*B <= 65536; T*K and R*C_max below 2^31.
 */
#ifndef MOONEP_H
#define MOONEP_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOONEP_API __attribute__((visibility("default")))
#else
#define MOONEP_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
    int32_t R, L, S, K, H, B, C, C_max; /* C must equal S*K; C_max >= C */
} moonep_cfg_t;

typedef struct {
    int32_t status;        /* MOONEP_ST_* bits                               */
    int32_t fallback_rows; /* rows kept on their home rank beyond C          */
    int32_t n_replicas;    /* replica pieces = used prefetch slots            */
    int32_t migrated_rows; /* rows placed on a rank other than their home    */
} moonep_plan_info_t;

/* host return codes */
#define MOONEP_OK 0
#define MOONEP_ERR_ARG 1
#define MOONEP_ERR_CUDA 2
#define MOONEP_ERR_DEVICE 3

/* device status bits (workspace word 0) */
#define MOONEP_ST_EXPERT_ID 0x1   /* a top-K id outside [0, N)                          */
#define MOONEP_ST_CAPACITY 0x2    /* fallback rows do not fit in [C, C_max)             */
#define MOONEP_ST_TIMEOUT 0x4     /* a bounded device wait gave up                      */
#define MOONEP_ST_DEST 0x8        /* combine met a destination outside [0, R*C_max)     */
#define MOONEP_ST_CFG 0x10        /* workspace planned for another configuration        */
#define MOONEP_ST_ERROR_MASK 0xFF
#define MOONEP_ST_FALLBACK 0x100  /* informational: fallback_rows > 0                   */

/* Workspace layout: offsets in int32 words from the workspace base.  The
 * header occupies words [0, MOONEP_WS_HEADER_WORDS):
 *   0 status, 1 fallback_rows, 2 n_replicas, 3 migrated_rows, 4 n_ranges,
 *   5..12 the cfg it was planned for, 13 replicated-expert count,
 *   14 plan flags, 15 pieces with a slot, 18 0x5A5A5A5A in a tables-only
 *   copy made by moonep_plan_noalloc (0 in a full workspace).
 * Tables ([N] unless noted): cnt = copies per expert (tokens_per_expert);
 * keep, spill, home_off (row of e's local segment), fb_cnt, fb_off (row of
 * e's fallback segment); [R]: load (copies homed on r), deficit (C - load,
 * floored at 0), fill (rows used below C), slots_used; [R*B]: slot_expert
 * (-1 = empty), slot_cnt, slot_off, slot_first_j (first copy index j held);
 * rep_ptr [N+1] (CSR over pieces, pieces in ascending (expert, receiver)
 * order) and per piece rep_expert, rep_recv, rep_slot (-1 = no slot:
 * remote weights), rep_first_j, rep_cnt, rep_off (first row on the
 * receiver); recv_ptr [R+1] (the pieces of receiver r are [recv_ptr[r],
 * recv_ptr[r+1]): piece order is receiver-major as well); slot_piece (the
 * pieces that have a slot, in piece order); rx_expert (experts with >= 1
 * piece, ascending); route_ptr [N+1],
 * route_end, route_base (copy j of e goes to flat row route_base[p] + j for
 * the first entry p of e with j < route_end[p]); seg_off, seg_len
 * [R][2L+B] (L local, B slot, L fallback segments per rank); alloc [N][R]
 * (rows of expert e on rank r, fallback included: the allocation table);
 * base [n_ranges][N] (copies of e in the earlier token ranges of the range's
 * block; written only where the range has a copy of e) and blk [N][n_blocks]
 * (copies of e in earlier blocks; a block is n_ranges / n_blocks consecutive
 * ranges): dispatch scratch, copy numbers start at base + blk.  Tables
 * from `cnt` up to, not including, `base` are contiguous. */
#define MOONEP_WS_HEADER_WORDS 64
typedef struct {
    int64_t words;      /* total size in int32 words                  */
    int64_t n_ranges;   /* token ranges of the dispatch grid           */
    int64_t max_pieces; /* capacity of the per-piece arrays            */
    int64_t cnt, keep, spill, home_off, fb_cnt, fb_off;
    int64_t load, deficit, fill, slots_used;
    int64_t slot_expert, slot_cnt, slot_off, slot_first_j;
    int64_t rep_ptr, rep_expert, rep_recv, rep_slot, rep_first_j, rep_cnt;
    int64_t rx_expert;
    int64_t route_ptr, route_end, route_base;
    int64_t seg_off, seg_len;
    int64_t alloc;
    int64_t tables_end; /* = base                                      */
    int64_t base;
    int64_t rep_off, recv_ptr, slot_piece; /* (between rep_cnt and rx_expert in memory) */
    int64_t n_blocks;   /* blocks of consecutive token ranges          */
    int64_t blk;
} moonep_ws_layout_t;

/* Per-rank buffer sizes in bytes, as a real deployment would allocate them
 * ("The Busiest Rank Sets Your Step Time", memory-cost table): dispatch =
 * C_max*H*2 (bf16 rows), prefetch = B*elems*2 (bf16 weights), reduce =
 * B*elems*4 (fp32 gradients), for elems weight elements per expert. */
typedef struct {
    int64_t dispatch_bytes, prefetch_bytes, reduce_bytes;
} moonep_rank_bytes_t;

/* Validates cfg and fills the workspace layout.  MOONEP_OK or ERR_ARG. */
MOONEP_API int moonep_ws_layout(const moonep_cfg_t *cfg, moonep_ws_layout_t *out);

/* Workspace size in bytes for cfg (0 if cfg is invalid). */
MOONEP_API size_t moonep_plan_workspace_bytes(const moonep_cfg_t *cfg);

/* Per-rank buffer sizes for cfg and `elems_per_expert` weight elements. */
MOONEP_API int moonep_rank_bytes(const moonep_cfg_t *cfg, int64_t elems_per_expert, moonep_rank_bytes_t *out);

/* Plan ("The Busiest Rank Sets Your Step Time", section "What the technique
 * is", flowchart: router output -> planning kernel).  topk_idx: device int32
 * [R][S][K] expert ids.  ws: device workspace of moonep_plan_workspace_bytes
 * bytes, 16-byte aligned, owned by the caller; fully rewritten.  One memset
 * of the header and one persistent cooperative kernel; no host sync. */
MOONEP_API int moonep_plan(const moonep_cfg_t *cfg, const int32_t *topk_idx, void *ws, void *stream);

/* Plan flags for moonep_plan_ex. */
#define MOONEP_PLAN_REMOTE_WEIGHTS 0x1
#define MOONEP_PLAN_ONE_GROUP 0x2

/* moonep_plan with flags.  MOONEP_PLAN_REMOTE_WEIGHTS selects the pages'
 * inference fallback instead of the headroom rule: when a receiver would need
 * more replicas than its B prefetch slots, the group GEMM reads the expert's
 * weights from its home rank (twodots.gr "MoonEP balances AI experts in MoE
 * models", memory-contract paragraphs; "The Busiest Rank Sets Your Step
 * Time", "Installation and integration"), so receivers take spilled rows while
 * they have room whatever their slots.  Their first B pieces get slots; later
 * pieces have rep_slot = -1 and follow the slotted ones on the receiver (rows
 * rep_off[p] .. rep_off[p] + rep_cnt[p]).  No row falls back: every rank
 * holds exactly C rows and C_max = C suffices.  prefetch copies slotted pieces
 * only, reduce_grad reduces slotted pieces only (remote pieces carry no
 * gradient slot: the mode is for inference).
 * MOONEP_PLAN_ONE_GROUP keeps the headroom rule and adds the pages' planner
 * variant in which a rank duplicates experts of at most one remote home group
 * ("The Busiest Rank Sets Your Step Time", "Installation and integration",
 * the paragraph on B after the weight-tensor figure): a receiver stops at the
 * end of the home group its first piece comes from, so it never holds pieces
 * of more than L = E/R experts and B = L slots always suffice.  The price is
 * balance: rows that no receiver may take fall back to their home rank's
 * headroom (rows from C), so C_max must leave room for them.  The two flags
 * exclude each other (MOONEP_ERR_ARG).  flags = 0 is moonep_plan. */
MOONEP_API int moonep_plan_ex(const moonep_cfg_t *cfg, int32_t flags, const int32_t *topk_idx, void *ws,
                              void *stream);

/* Dispatch (same flowchart: dispatch sends tokens straight to their final
 * slot on the remote rank).  x: device bf16 [R*S][H] hidden states;
 * topk_idx: the ids given to moonep_plan; recv: device bf16 [R][C_max][H];
 * dest: device int32 [R][S][K], written with the flat row rank*C_max + row of
 * every copy.  recv[dest[g]] = x[token(g)] bitwise. */
MOONEP_API int moonep_dispatch(const moonep_cfg_t *cfg, void *ws, const void *x, const int32_t *topk_idx,
                    void *recv, int32_t *dest, void *stream);

/* Copy-out, the zero_copy = false path (twodots.gr "MoonEP balances AI
 * experts in MoE models": the application works on views of the
 * communication buffer, which the next dispatch or combine overwrites, so a
 * caller that keeps the rows longer -- autograd saving them for the backward
 * pass, for one -- needs zero_copy = false, i.e. a copy of its own).
 * recv: device bf16 [R][C_max][H] after moonep_dispatch with this plan; out:
 * device bf16 [R][C_max][H] owned by the caller, not overlapping recv
 * (MOONEP_ERR_ARG).  Copies every row the plan uses -- on rank r the rows
 * [0, fill[r]) and the fallback segments of r's experts from row C -- to the
 * same row of out, bitwise; other rows of out are not written, so the plan's
 * segment tables index out as they index recv.  Both pointers 16-byte
 * aligned.  Status bits as for dispatch (a failed plan: nothing written). */
MOONEP_API int moonep_copy_out(const moonep_cfg_t *cfg, void *ws, const void *recv, void *out, void *stream);

/* Generation of the zero-copy views tied to a workspace: the number of
 * moonep_dispatch and moonep_combine calls launched with `ws` so far in this
 * process (host-side count; no GPU work, never fails; 0 for an unknown ws).
 * A view taken at generation g is stale once the generation moves past g. */
MOONEP_API int64_t moonep_view_generation(const void *ws);

/* Combine (same flowchart: combine gathers results back into token order).
 * y: device bf16 [R][C_max][H] expert outputs in the dispatched layout;
 * dest: from moonep_dispatch; topk_w: device fp32 [R][S][K] router weights;
 * out: device bf16 [R*S][H].  out[t] = bf16_rne(acc), acc = 0.0f then
 * acc = fmaf(w[t][k], float(y[dest[t][k]]), acc) for k = 0..K-1. */
MOONEP_API int moonep_combine(const moonep_cfg_t *cfg, void *ws, const void *y, const int32_t *dest,
                   const float *topk_w, void *out, void *stream);

/* Combine backward, for training ("The Busiest Rank Sets Your Step Time",
 * flowchart: the backward pass of the layer follows its forward path; combine
 * is linear in the expert outputs and in the router weights).  grad_out:
 * device bf16 [R*S][H], the gradient of `out`; y, dest, topk_w: as given to
 * moonep_combine; grad_y: device bf16 [R][C_max][H], written at every
 * dispatched row: grad_y[dest[t][k]] = bf16_rne(fp32(w[t][k] *
 * grad_out[t])); grad_w: device fp32 [R][S][K] or NULL: grad_w[t][k] = sum
 * over h of grad_out[t][h] * y[dest[t][k]][h], accumulated in fp32 (the
 * order is fixed, so results repeat exactly; it is not the plain left-to-right
 * order).  y may be NULL when grad_w is NULL.  Rows outside the plan's
 * segments are not written. */
MOONEP_API int moonep_combine_backward(const moonep_cfg_t *cfg, void *ws, const void *grad_out, const void *y,
                                       const int32_t *dest, const float *topk_w, void *grad_y, float *grad_w,
                                       void *stream);

/* Dispatch backward, for training: the adjoint of the row scatter.
 * grad_recv: device bf16 [R][C_max][H], the gradient of the dispatched rows;
 * grad_x: device bf16 [R*S][H]: grad_x[t] = bf16_rne(acc), acc = 0.0f then
 * acc = acc + float(grad_recv[dest[t][k]]) for k = 0..K-1 (fp32). */
MOONEP_API int moonep_dispatch_backward(const moonep_cfg_t *cfg, void *ws, const void *grad_recv,
                                        const int32_t *dest, void *grad_x, void *stream);

/* Prefetch (twodots.gr: weights of the duplicated experts are loaded into
 * the prefetch slots [E, E+B) before the experts run).  w_home: device bf16
 * [N][elems_per_expert]; w_slot: device bf16 [R][B][elems_per_expert];
 * w_slot[r][b] = w_home[slot_expert[r][b]] for used slots only.
 * elems_per_expert must be a positive multiple of 8. */
MOONEP_API int moonep_prefetch(const moonep_cfg_t *cfg, void *ws, const void *w_home, void *w_slot,
                    int64_t elems_per_expert, void *stream);

/* Replica gradient reduction (twodots.gr: reduce_grad adds the replica
 * slots of a rank's own experts to the local parameter gradient and clears
 * the used slots).  g_home: device fp32 [N][elems]; g_rep: device fp32
 * [R][B][elems].  For each replicated expert, in ascending receiver order,
 * g_home[e] = g_home[e] + g_rep[r][b] (fp32 adds); then g_rep[r][b] = 0.
 * Unused slots are not touched: zero g_rep once after allocating it.
 * elems_per_expert must be a positive multiple of 4. */
MOONEP_API int moonep_reduce_grad(const moonep_cfg_t *cfg, void *ws, float *g_home, float *g_rep,
                       int64_t elems_per_expert, void *stream);

/* Reads the plan header (and, if host_tables is not NULL, the tables from
 * `cnt` up to `base`, i.e. layout.tables_end - layout.cnt words, into
 * host_tables) after synchronising `stream`. */
MOONEP_API int moonep_plan_read(const moonep_cfg_t *cfg, const void *ws, moonep_plan_info_t *info,
                     int32_t *host_tables, void *stream);

/* The pages have no counterpart to this entry point.  moonep_plan for
 * callers that cannot allocate device memory themselves (a plug-in handed
 * tensors but no allocator, or a process whose device memory belongs to a
 * pooled allocator that must not see extra cudaMalloc calls): the workspace
 * lives in a static 2 MiB device array inside the library (held by every
 * GPU that loads it until exit) and the plan header and tables, words
 * [0, layout.tables_end) of the workspace layout, are copied into
 * tables_out (device, at least layout.tables_end int32 words, 16-byte
 * aligned, caller-owned).  Same kernel and results as moonep_plan; allocates
 * nothing.  The copy is tables only: it lacks the dispatch scratch that
 * follows the tables in a full workspace, and its header word 18 says so.
 * moonep_plan_read, moonep_prefetch, moonep_reduce_grad, moonep_copy_out,
 * moonep_combine and the backward pair read only the header and tables and
 * accept it as `ws`; moonep_dispatch refuses it (MOONEP_ST_CFG set in its
 * status word, nothing else written) and needs a full moonep_plan workspace.
 * Configurations whose workspace (moonep_plan_workspace_bytes) exceeds
 * 2 MiB are refused with MOONEP_ERR_ARG before any GPU work.  The first call
 * on a device looks up the array's device address and keeps it for the
 * life of the CUDA context (after cudaDeviceReset the library must not be
 * called on that device again in the process); make that first call before
 * any stream capture.  Every call shares the array, so calls that overlap
 * on the GPU race: serialise them. */
MOONEP_API int moonep_plan_noalloc(const moonep_cfg_t *cfg, const int32_t *topk_idx, int32_t *tables_out,
                                   void *stream);

/* ------------------------------------------------------------------------
 * Expert parallelism: one rank per GPU ("The Busiest Rank Sets Your Step
 * Time", section "Installation and integration": eight ranks over NVLink,
 * the weight tensor mapped from each home rank; twodots.gr "MoonEP balances
 * AI experts in MoE models", memory-contract paragraphs: dispatch writes
 * into the other ranks' receive buffers, prefetch reads weights from the
 * home rank, reduce_grad reads the replica gradients from the receivers).
 *
 * Rank r holds its own S tokens (topk_idx, topk_w and x of [S][K], [S][K]
 * and [S][H]; rows s of rank r are global tokens r*S + s), its receive
 * buffer recv_r [C_max][H], its experts' weights [L][elems] and gradients
 * [L][elems], and its slots [B][elems] (bf16 weights, fp32 replica
 * gradients).  A step:
 *   1. moonep_ep_count: histogram of the rank's ids into counts [N + 1]
 *      (device int32: copies per expert, then the rank's status bits), plus
 *      the per-range scratch dispatch needs, into the rank's workspace
 *      (moonep_ep_workspace_bytes; layout from moonep_ep_ws_layout).
 *   2. all-gather of every rank's counts into counts_all [R][N + 1] on every
 *      rank, by the caller (for example NCCL's all-gather).
 *   3. moonep_ep_plan: every rank plans from the same counts, so every rank
 *      derives the same tables (identical to moonep_plan's for the R*S
 *      tokens); the rank's copy numbers start after the lower ranks' copies.
 *   4. moonep_ep_prefetch, moonep_ep_dispatch, (experts), moonep_ep_combine,
 *      and for training moonep_ep_combine_backward, (experts' backward),
 *      moonep_ep_dispatch_backward, moonep_ep_reduce_grad, each on the
 *      rank's own stream.
 * Between steps the caller orders the ranks (a barrier on every rank after
 * its dispatch and before any combine reads the expert outputs; likewise
 * around prefetch and reduce_grad): the kernels never wait on one another.
 * Peer tables (recv_peers, y_peers, grad_y_peers, grad_recv_peers,
 * w_home_peers, g_rep_peers) are device
 * arrays of R device pointers, entry q pointing at rank q's buffer as this
 * GPU addresses it (peer-mapped memory, CUDA IPC or symmetric allocations;
 * the rank's own buffer at entry r).  `dest` holds global flat rows
 * q*C_max + row as in moonep_dispatch.  Copies use plain loads and bulk
 * copies, never a multicast load.  The workspace status of every call
 * behaves as in the single-GPU calls; a bad id on any rank makes every
 * rank's plan fail (the status travels in counts). */

/* Workspace layout and size of one rank's plan (the dispatch scratch
 * covers the rank's S tokens). */
MOONEP_API int moonep_ep_ws_layout(const moonep_cfg_t *cfg, moonep_ws_layout_t *out);
MOONEP_API size_t moonep_ep_workspace_bytes(const moonep_cfg_t *cfg);

/* Step 1.  topk_idx: device int32 [S][K], rank `rank`'s ids.  counts:
 * device int32 [N + 1], written.  Clears the workspace header; no host
 * sync. */
MOONEP_API int moonep_ep_count(const moonep_cfg_t *cfg, int32_t rank, const int32_t *topk_idx, void *ws,
                               int32_t *counts, void *stream);

/* Steps 1 and 2 in one launch: moonep_ep_count, and the rank's finished
 * counts [N + 1] stored into row `rank` of every rank's counts_all.
 * counts_all_peers: device table of R pointers, entry q to rank q's
 * counts_all (device int32 [R][N + 1]) as this GPU addresses it.  The last
 * counting CTA to finish stores the row (plain stores, no multicast; no CTA
 * waits for another); once every rank's launch has completed (the caller's
 * barrier), each rank's counts_all is what the all-gather of step 2 would
 * have left.  Also launches with S = 0, to store the rank's zero row. */
MOONEP_API int moonep_ep_count_exchange(const moonep_cfg_t *cfg, int32_t rank, const int32_t *topk_idx, void *ws,
                                        int32_t *counts, int32_t *const *counts_all_peers, void *stream);

/* Step 3.  counts_all: device int32 [R][N + 1], row q = rank q's counts.
 * flags as in moonep_plan_ex.  The tables equal moonep_plan_ex's on the
 * concatenated ids. */
MOONEP_API int moonep_ep_plan(const moonep_cfg_t *cfg, int32_t flags, int32_t rank, const int32_t *counts_all,
                              void *ws, void *stream);

/* Dispatch of rank `rank`'s tokens: x device bf16 [S][H], topk_idx [S][K];
 * row q*C_max + row of the plan goes to recv_peers[q] + row*H; dest [S][K]
 * written with the flat rows. */
MOONEP_API int moonep_ep_dispatch(const moonep_cfg_t *cfg, int32_t rank, void *ws, const void *x,
                                  const int32_t *topk_idx, void *const *recv_peers, int32_t *dest, void *stream);

/* Combine of rank `rank`'s tokens: out [S][H] from y_peers[q] (rank q's
 * expert outputs [C_max][H]), dest and topk_w [S][K] of this rank; the
 * arithmetic of moonep_combine. */
MOONEP_API int moonep_ep_combine(const moonep_cfg_t *cfg, int32_t rank, void *ws, const void *const *y_peers,
                                 const int32_t *dest, const float *topk_w, void *out, void *stream);

/* Combine backward of rank `rank`'s tokens: grad_out [S][H] (bf16) and
 * dest, topk_w [S][K] of this rank; grad_y_peers[q] + row*H receives
 * grad_y of row q*C_max + row (rank q's [C_max][H] bf16 buffer), and
 * grad_w [S][K] (fp32, or NULL) reads y from y_peers as moonep_ep_combine
 * does; the arithmetic, the order of the grad_w sums and the rows written
 * are those of moonep_combine_backward.  y_peers may be NULL when grad_w is
 * NULL. */
MOONEP_API int moonep_ep_combine_backward(const moonep_cfg_t *cfg, int32_t rank, void *ws, const void *grad_out,
                                          const void *const *y_peers, const int32_t *dest, const float *topk_w,
                                          void *const *grad_y_peers, float *grad_w, void *stream);

/* Dispatch backward of rank `rank`'s tokens: grad_x [S][H] (bf16) from
 * grad_recv_peers[q] (rank q's [C_max][H] gradient of the dispatched rows)
 * and this rank's dest [S][K]; the arithmetic of moonep_dispatch_backward. */
MOONEP_API int moonep_ep_dispatch_backward(const moonep_cfg_t *cfg, int32_t rank, void *ws,
                                           const void *const *grad_recv_peers, const int32_t *dest, void *grad_x,
                                           void *stream);

/* Prefetch into rank `rank`'s slots: w_slot [B][elems] (bf16); slot b of
 * the rank gets expert e's weights from w_home_peers[e / L] + (e % L)*elems. */
MOONEP_API int moonep_ep_prefetch(const moonep_cfg_t *cfg, int32_t rank, void *ws, const void *const *w_home_peers,
                                  void *w_slot, int64_t elems_per_expert, void *stream);

/* reduce_grad for rank `rank`'s own experts: g_home [L][elems] (fp32) of
 * this rank; each replica is read from and cleared in
 * g_rep_peers[receiver] + slot*elems, added in ascending receiver order. */
MOONEP_API int moonep_ep_reduce_grad(const moonep_cfg_t *cfg, int32_t rank, void *ws, float *g_home,
                                     void *const *g_rep_peers, int64_t elems_per_expert, void *stream);

/* Upper bound on polls of every bounded device wait (default 1 << 22).  A
 * wait that runs out sets MOONEP_ST_TIMEOUT and the kernel returns. */
MOONEP_API int moonep_set_wait_limit(int64_t polls);

/* Token ranges (dispatch CTAs) used for T tokens and N experts: a whole
 * number w >= 1 of waves of 296 ranges (two per SM of a B200), w = T / 1184
 * rounded to the nearest (about 4 tokens per range) and at most
 * 2^22 / (296 N); T itself if T is smaller. */
MOONEP_API int64_t moonep_num_ranges(int64_t T, int64_t N);

/* Description of the last host error on this thread ("" if none). */
MOONEP_API const char *moonep_last_error(void);

/* Library version string. */
MOONEP_API const char *moonep_version(void);

#ifdef __cplusplus
}
#endif
#endif /* MOONEP_H */
