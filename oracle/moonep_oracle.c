/*
 * moonep_oracle.c -- plain, slow, single-threaded CPU oracle for the MoonEP
 * hot path.  TEST INFRASTRUCTURE ONLY: it is called by the tests, by the
 * smoke check and by the benchmark's CPU-baseline leg, never by the product
 * path.  It shares no code, header or table with the CUDA library.
 *
 * What it computes, and where that is stated:
 *  - every expert-parallel rank receives exactly C = S*K rows whatever the
 *    router skew ("Moonshot AI Open-Sources MoonEP", TL;DR; "The Busiest Rank
 *    Sets Your Step Time", section "What the technique is");
 *  - the planner's allocation table alloc[e][r] never exceeds capacity per
 *    rank ("The Busiest Rank Sets Your Step Time", section "What we measured",
 *    the planning-balance table and the paragraph after it);
 *  - redundant copies of hot experts are placed on ranks with spare room and
 *    the overflow is routed there (same page, "What the technique is");
 *  - the sender computes the receiver's final expert-grouped row and writes
 *    there (same page, "What the technique is": zero copy; agentlenshq
 *    "MoonshotAI/MoonEP", "How it works");
 *  - combine gathers the expert outputs back into token order (same page,
 *    flowchart);
 *  - prefetch copies the duplicated experts' weights into slots [E, E+B) and
 *    reduce_grad adds the replica gradients to the home expert's gradient,
 *    then clears the used slots (twodots.gr "MoonEP balances AI experts in
 *    MoE models", the memory-contract paragraphs);
 *  - the plan's two variants: remote weights beyond B slots and one home
 *    group per receiver (or_plan_ex modes 1 and 2, with their citations);
 *  - copy-out for zero_copy = false (or_copy_out) and the backward pair
 *    (or_combine_backward, or_dispatch_backward).
 *
 * The pages give no planning algorithm.  The spill rule implemented here is
 * the library's documented rule: each home rank keeps its rows in expert
 * order up to C; the overflow, taken expert by expert in ascending global
 * expert order, goes to the lowest-index ranks that still have room and a
 * free replica slot, one slot per (expert, receiver) piece; what no receiver
 * can take stays on its home rank in a headroom region starting at row C.
 *
 * Floating point: combine accumulates in fp32 with fmaf in fixed k order and
 * rounds once to bf16 (round to nearest even, written from the bit pattern);
 * reduce_grad adds fp32 values in ascending receiver order.  Both orders are
 * part of the library contract, so the oracle uses them rather than fp64.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int32_t R, L, S, K, H, B, C, C_max;
} or_cfg;

/* status bits (same meaning as the library's, defined independently) */
#define OR_ST_EXPERT_ID 0x1
#define OR_ST_CAPACITY 0x2
#define OR_ST_FALLBACK 0x100

typedef struct {
    int32_t status, fallback_rows, n_replicas, migrated_rows;
    int32_t *cnt, *keep, *spill, *home_off, *fb_cnt, *fb_off;  /* [N]          */
    int32_t *load, *deficit, *fill, *slots_used;               /* [R]          */
    int32_t *slot_expert, *slot_cnt, *slot_off, *slot_first_j; /* [R*B]        */
    int32_t *rep_ptr;                                          /* [N+1]        */
    int32_t *rep_expert, *rep_recv, *rep_slot, *rep_first_j, *rep_cnt; /* [N+R] */
    int32_t *rep_off;                                          /* [N+R] row on the receiver */
    int32_t *recv_ptr;                                         /* [R+1] pieces by receiver */
    int32_t *seg_off, *seg_len;                                /* [R*(2L+B)]   */
    int32_t *alloc;                                            /* [N*R]        */
    int32_t *dest;                                             /* [R*S*K]      */
} or_plan_t;

static int64_t or_min64(int64_t a, int64_t b) { return a < b ? a : b; }

/* ------------------------------------------------------------------------ */
/* Plan: O1 validate, O2 histogram, O3 keep, O4 spill, O5 layout, O6 dest.  */
/* ------------------------------------------------------------------------ */
/* mode 0: the library's headroom rule (above).  mode 1, remote weights (the
 * pages' inference fallback: when a rank would need more replicas than it has
 * prefetch slots, the group GEMM reads the weights from the home rank,
 * twodots.gr "MoonEP balances AI experts in MoE models", memory-contract
 * paragraphs; "The Busiest Rank Sets Your Step Time", "Installation and
 * integration"): a receiver takes spilled rows while it has room whatever its
 * slots; its first B pieces get slots, later ones are remote (slot -1), so no
 * row ever falls back and every rank holds exactly C rows.
 * mode 2, one home group per receiver ("The Busiest Rank Sets Your Step
 * Time", section "Installation and integration", the paragraph on B after
 * the weight-tensor figure: a rank duplicates experts of at most one remote
 * home group, which is why B = E/R slots always suffice): the headroom rule
 * with one more condition on the receiver -- once it holds a piece of an
 * expert of home group h, it takes rows of group h only. */
int or_plan_ex(const or_cfg *c, int mode, const int32_t *topk_idx, or_plan_t *p)
{
    const int R = c->R, L = c->L, B = c->B;
    const int N = R * L;
    const int64_t T = (int64_t)R * c->S;
    const int64_t G = T * c->K;          /* number of routed (token, k) copies */
    const int64_t C = c->C;
    const int SEG = 2 * L + B;

    p->status = 0;
    p->fallback_rows = 0;
    p->n_replicas = 0;
    p->migrated_rows = 0;

    /* O1: every id must name an expert */
    for (int64_t g = 0; g < G; ++g)
        if (topk_idx[g] < 0 || topk_idx[g] >= N) {
            p->status |= OR_ST_EXPERT_ID;
            return p->status;
        }

    /* O2: tokens_per_expert histogram and per-home-rank load */
    for (int e = 0; e < N; ++e) p->cnt[e] = 0;
    for (int64_t g = 0; g < G; ++g) p->cnt[topk_idx[g]] += 1;
    for (int h = 0; h < R; ++h) {
        int64_t s = 0;
        for (int loc = 0; loc < L; ++loc) s += p->cnt[h * L + loc];
        p->load[h] = (int32_t)s;
    }

    /* O3: each home rank keeps rows in local-expert order up to C */
    for (int h = 0; h < R; ++h) {
        int64_t kept = 0;
        for (int loc = 0; loc < L; ++loc) {
            int e = h * L + loc;
            int64_t room = C - kept;
            int64_t k = or_min64(p->cnt[e], room);
            p->keep[e] = (int32_t)k;
            p->spill[e] = p->cnt[e] - (int32_t)k;
            p->home_off[e] = (int32_t)kept;
            kept += k;
        }
        p->deficit[h] = (int32_t)(C - or_min64(p->load[h], C));
    }

    /* O4: spilled chunks in ascending expert order go to the lowest-index
     * rank that still has a deficit and a free slot; each (expert, receiver)
     * piece takes one slot; what is left falls back to the home rank. */
    int32_t *def = (int32_t *)malloc(sizeof(int32_t) * (size_t)(R > 0 ? R : 1));
    for (int r = 0; r < R; ++r) {
        def[r] = p->deficit[r];
        p->slots_used[r] = 0;
    }
    for (int i = 0; i < R * B; ++i) {
        p->slot_expert[i] = -1;
        p->slot_cnt[i] = 0;
        p->slot_first_j[i] = 0;
    }
    int npieces = 0;
    int32_t *on_r = (int32_t *)calloc((size_t)(R > 0 ? R : 1), sizeof(int32_t)); /* pieces per receiver */
    int32_t *lock = (int32_t *)malloc(sizeof(int32_t) * (size_t)(R > 0 ? R : 1)); /* mode 2: home group */
    for (int r = 0; r < R; ++r) lock[r] = -1;
    for (int e = 0; e < N; ++e) {
        p->rep_ptr[e] = npieces;
        int64_t a = p->spill[e];
        int64_t spilled = 0;
        while (a > 0) {
            int r = -1;
            for (int q = 0; q < R; ++q)
                if (def[q] > 0 && (mode == 1 || p->slots_used[q] < B) &&
                    (mode != 2 || lock[q] < 0 || lock[q] == e / L)) {
                    r = q;
                    break;
                }
            if (r < 0) break;
            int64_t t = or_min64(a, def[r]);
            int b = on_r[r] < B ? on_r[r] : -1;   /* modes 0 and 2 always have a free slot here */
            on_r[r]++;
            lock[r] = e / L;
            if (b >= 0) p->slots_used[r]++;
            p->rep_expert[npieces] = e;
            p->rep_recv[npieces] = r;
            p->rep_slot[npieces] = b;
            p->rep_first_j[npieces] = (int32_t)(p->keep[e] + spilled);
            p->rep_cnt[npieces] = (int32_t)t;
            if (b >= 0) {
                p->slot_expert[r * B + b] = e;
                p->slot_cnt[r * B + b] = (int32_t)t;
                p->slot_first_j[r * B + b] = (int32_t)(p->keep[e] + spilled);
            }
            ++npieces;
            def[r] -= (int32_t)t;
            a -= t;
            spilled += t;
        }
        p->fb_cnt[e] = (int32_t)a;
        p->fallback_rows += (int32_t)a;
        p->migrated_rows += (int32_t)spilled;
    }
    p->rep_ptr[N] = npieces;
    p->n_replicas = npieces;
    free(def);
    free(on_r);
    free(lock);

    /* O5: layout of rank r: kept local segments, then slots in slot order,
     * then (from row C) the fallback segments of r's own experts. */
    for (int r = 0; r < R; ++r) {
        int64_t off = 0;
        for (int loc = 0; loc < L; ++loc) {
            int e = r * L + loc;
            p->seg_off[r * SEG + loc] = (int32_t)off;
            p->seg_len[r * SEG + loc] = p->keep[e];
            off += p->keep[e];
        }
        for (int b = 0; b < B; ++b) {
            p->slot_off[r * B + b] = (int32_t)off;
            p->seg_off[r * SEG + L + b] = (int32_t)off;
            p->seg_len[r * SEG + L + b] = p->slot_cnt[r * B + b];
            off += p->slot_cnt[r * B + b];
        }
        /* remote pieces (mode 1) follow the slots, in piece order */
        for (int q = 0; q < npieces; ++q)
            if (p->rep_recv[q] == r && p->rep_slot[q] < 0) {
                p->rep_off[q] = (int32_t)off;
                off += p->rep_cnt[q];
            }
        p->fill[r] = (int32_t)off;
        int64_t fo = C;
        for (int loc = 0; loc < L; ++loc) {
            int e = r * L + loc;
            p->fb_off[e] = (int32_t)fo;
            p->seg_off[r * SEG + L + B + loc] = (int32_t)fo;
            p->seg_len[r * SEG + L + B + loc] = p->fb_cnt[e];
            fo += p->fb_cnt[e];
        }
        if (fo > c->C_max) p->status |= OR_ST_CAPACITY;
    }
    for (int q = 0; q < npieces; ++q)
        if (p->rep_slot[q] >= 0) p->rep_off[q] = p->slot_off[p->rep_recv[q] * B + p->rep_slot[q]];
    /* pieces grouped by receiver; pieces are created in receiver order within
     * an expert, and receivers are filled in ascending order, so counting is
     * enough (checked by the tests) */
    for (int r = 0; r <= R; ++r) p->recv_ptr[r] = 0;
    for (int q = 0; q < npieces; ++q) p->recv_ptr[p->rep_recv[q] + 1]++;
    for (int r = 0; r < R; ++r) p->recv_ptr[r + 1] += p->recv_ptr[r];
    if (p->fallback_rows > 0) p->status |= OR_ST_FALLBACK;
    if (p->status & OR_ST_CAPACITY) return p->status;

    /* allocation table: rows of expert e on rank r (fallback rows are on the
     * home rank, in its headroom) */
    for (int64_t i = 0; i < (int64_t)N * R; ++i) p->alloc[i] = 0;
    for (int e = 0; e < N; ++e) p->alloc[(int64_t)e * R + e / L] = p->keep[e] + p->fb_cnt[e];
    for (int q = 0; q < npieces; ++q)
        p->alloc[(int64_t)p->rep_expert[q] * R + p->rep_recv[q]] += p->rep_cnt[q];

    /* O6: the copies of expert e are numbered j = 0, 1, ... in ascending
     * global order g = (r*S + s)*K + k; copy j goes home while j < keep[e],
     * then through e's replica pieces in creation order, then to fallback. */
    int32_t *seen = (int32_t *)calloc((size_t)(N > 0 ? N : 1), sizeof(int32_t));
    for (int64_t g = 0; g < G; ++g) {
        int e = topk_idx[g];
        int h = e / L;
        int64_t j = seen[e]++;
        int64_t rank, row;
        if (j < p->keep[e]) {
            rank = h;
            row = p->home_off[e] + j;
        } else {
            rank = -1;
            row = -1;
            for (int q = p->rep_ptr[e]; q < p->rep_ptr[e + 1]; ++q)
                if (j >= p->rep_first_j[q] && j < p->rep_first_j[q] + p->rep_cnt[q]) {
                    rank = p->rep_recv[q];
                    row = p->rep_off[q] + (j - p->rep_first_j[q]);
                    break;
                }
            if (rank < 0) {
                int64_t moved = p->cnt[e] - p->fb_cnt[e]; /* keep + replica rows */
                rank = h;
                row = p->fb_off[e] + (j - moved);
            }
        }
        p->dest[g] = (int32_t)(rank * c->C_max + row);
    }
    free(seen);
    return p->status;
}

int or_plan(const or_cfg *c, const int32_t *topk_idx, or_plan_t *p) { return or_plan_ex(c, 0, topk_idx, p); }

/* ------------------------------------------------------------------------ */
/* Independent row-at-a-time simulator of the same rule (for brute force).  */
/* Places overflow rows one by one: a row goes home while the home rank has */
/* room; else to the receiver of the expert's current piece while that      */
/* receiver has room; else to the lowest rank with room and a free slot,    */
/* opening a new slot (mode 2: and, once it holds a piece, whose pieces are */
/* all of this row's home group).  Offsets are assigned only after every row */
/* has a place.  Outputs: alloc, slot_expert, slot_cnt, fb_cnt, dest,       */
/* status.                                                                   */
/* ------------------------------------------------------------------------ */
int or_plan_unitwise_ex(const or_cfg *c, int mode, const int32_t *topk_idx, int32_t *alloc,
                        int32_t *slot_expert, int32_t *slot_cnt, int32_t *fb_cnt, int32_t *dest,
                        int32_t *status_out)
{
    const int R = c->R, L = c->L, B = c->B, N = R * L;
    const int64_t G = (int64_t)R * c->S * c->K;
    const int64_t C = c->C;
    int status = 0;
    for (int64_t g = 0; g < G; ++g)
        if (topk_idx[g] < 0 || topk_idx[g] >= N) {
            *status_out = OR_ST_EXPERT_ID;
            return OR_ST_EXPERT_ID;
        }
    /* copies of each expert in ascending g */
    int64_t *count = (int64_t *)calloc((size_t)N + 1, sizeof(int64_t));
    for (int64_t g = 0; g < G; ++g) count[topk_idx[g] + 1]++;
    for (int e = 0; e < N; ++e) count[e + 1] += count[e];
    int64_t *order = (int64_t *)malloc(sizeof(int64_t) * (size_t)(G > 0 ? G : 1));
    int64_t *fillpos = (int64_t *)malloc(sizeof(int64_t) * (size_t)N);
    for (int e = 0; e < N; ++e) fillpos[e] = count[e];
    for (int64_t g = 0; g < G; ++g) order[fillpos[topk_idx[g]]++] = g;

    /* placement per row: kind 0 home, 1 piece (index in the piece list), 2 fallback */
    int *kind = (int *)malloc(sizeof(int) * (size_t)(G > 0 ? G : 1));
    int *pidx = (int *)malloc(sizeof(int) * (size_t)(G > 0 ? G : 1));
    int64_t *rows = (int64_t *)calloc((size_t)R, sizeof(int64_t)); /* rows in [0,C) */
    int *npc_r = (int *)calloc((size_t)R, sizeof(int));            /* pieces per receiver */
    int *grp_r = (int *)malloc(sizeof(int) * (size_t)(R > 0 ? R : 1)); /* home group of its pieces */
    for (int r = 0; r < R; ++r) grp_r[r] = -1;
    int maxp = (int)(N + R + 1);
    int *pc_rank = (int *)malloc(sizeof(int) * (size_t)maxp);
    int *pc_slot = (int *)malloc(sizeof(int) * (size_t)maxp);
    int *pc_exp = (int *)malloc(sizeof(int) * (size_t)maxp);
    int64_t *pc_n = (int64_t *)calloc((size_t)maxp, sizeof(int64_t));
    int np = 0;
    for (int i = 0; i < R * B; ++i) { slot_expert[i] = -1; slot_cnt[i] = 0; }
    for (int e = 0; e < N; ++e) fb_cnt[e] = 0;

    /* pass 1: every home rank keeps rows in expert order while it has room */
    for (int e = 0; e < N; ++e) {
        int h = e / L;
        for (int64_t q = count[e]; q < count[e + 1]; ++q) {
            if (rows[h] < C) { kind[q] = 0; rows[h]++; }
            else kind[q] = -1;
        }
    }
    /* pass 2: overflow rows one at a time, expert by expert */
    for (int e = 0; e < N; ++e) {
        int cur = -1;
        for (int64_t q = count[e]; q < count[e + 1]; ++q) {
            if (kind[q] == 0) continue;
            if (cur >= 0 && rows[pc_rank[cur]] < C) {
                kind[q] = 1; pidx[q] = cur; pc_n[cur]++; rows[pc_rank[cur]]++;
                continue;
            }
            int pick = -1;
            for (int r = 0; r < R; ++r)
                if (rows[r] < C && (mode == 1 || npc_r[r] < B) &&
                    (mode != 2 || grp_r[r] < 0 || grp_r[r] == e / L)) { pick = r; break; }
            if (pick >= 0) {
                cur = np++;
                pc_rank[cur] = pick;
                pc_slot[cur] = npc_r[pick] < B ? npc_r[pick] : -1;
                pc_exp[cur] = e;
                npc_r[pick]++;
                grp_r[pick] = e / L;
                kind[q] = 1; pidx[q] = cur; pc_n[cur] = 1; rows[pick]++;
            } else {
                cur = -1;
                kind[q] = 2;
                fb_cnt[e]++;
            }
        }
    }
    /* offsets: home rows per rank in expert order, then slotted pieces by
     * slot, then remote pieces in creation order; fallback from C */
    int64_t *home_base = (int64_t *)calloc((size_t)N, sizeof(int64_t));
    int64_t *home_n = (int64_t *)calloc((size_t)N, sizeof(int64_t));
    int64_t *pc_base = (int64_t *)calloc((size_t)maxp, sizeof(int64_t));
    int64_t *fb_base = (int64_t *)calloc((size_t)N, sizeof(int64_t));
    for (int e = 0; e < N; ++e)
        for (int64_t q = count[e]; q < count[e + 1]; ++q)
            if (kind[q] == 0) home_n[e]++;
    for (int r = 0; r < R; ++r) {
        int64_t off = 0;
        for (int loc = 0; loc < L; ++loc) { home_base[r * L + loc] = off; off += home_n[r * L + loc]; }
        for (int b = 0; b < B; ++b)
            for (int k = 0; k < np; ++k)
                if (pc_rank[k] == r && pc_slot[k] == b) {
                    pc_base[k] = off; off += pc_n[k];
                    slot_expert[r * B + b] = pc_exp[k];
                    slot_cnt[r * B + b] = (int32_t)pc_n[k];
                }
        for (int k = 0; k < np; ++k)
            if (pc_rank[k] == r && pc_slot[k] < 0) { pc_base[k] = off; off += pc_n[k]; }
        int64_t fo = C;
        for (int loc = 0; loc < L; ++loc) { fb_base[r * L + loc] = fo; fo += fb_cnt[r * L + loc]; }
        if (fo > c->C_max) status |= OR_ST_CAPACITY;
    }
    for (int64_t i = 0; i < (int64_t)N * R; ++i) alloc[i] = 0;
    int64_t *pc_used = (int64_t *)calloc((size_t)maxp, sizeof(int64_t));
    for (int e = 0; e < N; ++e) {
        int h = e / L;
        int64_t nh = 0, nf = 0;
        for (int64_t q = count[e]; q < count[e + 1]; ++q) {
            int64_t row;
            int rank;
            if (kind[q] == 0) { rank = h; row = home_base[e] + nh++; }
            else if (kind[q] == 1) { rank = pc_rank[pidx[q]]; row = pc_base[pidx[q]] + pc_used[pidx[q]]++; }
            else { rank = h; row = fb_base[e] + nf++; }
            alloc[(int64_t)e * R + rank]++;
            dest[order[q]] = (int32_t)(rank * (int64_t)c->C_max + row);
        }
    }
    int64_t fb_total = 0;
    for (int e = 0; e < N; ++e) fb_total += fb_cnt[e];
    if (fb_total > 0) status |= OR_ST_FALLBACK;
    free(count); free(order); free(fillpos); free(kind); free(pidx); free(rows); free(npc_r); free(grp_r);
    free(pc_rank); free(pc_slot); free(pc_exp); free(pc_n); free(home_base); free(home_n);
    free(pc_base); free(fb_base); free(pc_used);
    *status_out = status;
    return status;
}

int or_plan_unitwise(const or_cfg *c, const int32_t *topk_idx, int32_t *alloc, int32_t *slot_expert,
                     int32_t *slot_cnt, int32_t *fb_cnt, int32_t *dest, int32_t *status_out)
{
    return or_plan_unitwise_ex(c, 0, topk_idx, alloc, slot_expert, slot_cnt, fb_cnt, dest, status_out);
}

/* ------------------------------------------------------------------------ */
/* bf16 helpers (bit patterns as uint16)                                    */
/* ------------------------------------------------------------------------ */
static float or_bf16_to_f32(uint16_t u)
{
    uint32_t b = (uint32_t)u << 16;
    float f;
    memcpy(&f, &b, 4);
    return f;
}

/* round to nearest even; NaN stays a (quiet) NaN */
static uint16_t or_f32_to_bf16(float f)
{
    uint32_t b;
    memcpy(&b, &f, 4);
    if ((b & 0x7F800000u) == 0x7F800000u && (b & 0x007FFFFFu))
        return (uint16_t)((b >> 16) | 0x0040u);
    uint32_t lsb = (b >> 16) & 1u;
    b += 0x7FFFu + lsb;
    return (uint16_t)(b >> 16);
}

/* O7 dispatch: recv[dest[g]] = x[token(g)] bitwise, for tokens [0, n_tokens) */
void or_dispatch(const or_cfg *c, const int32_t *dest, const uint16_t *x, uint16_t *recv,
                 int64_t n_tokens)
{
    const int64_t H = c->H;
    for (int64_t t = 0; t < n_tokens; ++t)
        for (int k = 0; k < c->K; ++k) {
            int64_t d = dest[t * c->K + k];
            memcpy(recv + d * H, x + t * H, (size_t)H * 2);
        }
}

/* O7b copy-out (zero_copy = false): the rows the plan put in the receive
 * buffer -- every segment of every rank (local, slot, fallback) and every
 * remote piece -- copied bitwise to the same rows of a buffer of the
 * caller's; other rows of `out` are left alone.  The application normally
 * works on views of the communication buffer, which the next dispatch or
 * combine overwrites; a caller that keeps rows beyond that (autograd, for
 * one) asks for zero_copy = false and gets its own copy ("MoonEP balances AI
 * experts in MoE models", twodots.gr: the paragraph on zero-copy
 * communication and static shapes, and the one on the lifetime of zero-copy
 * views).  Returns the number of rows copied. */
int64_t or_copy_out(const or_cfg *c, const int32_t *seg_off, const int32_t *seg_len, int n_rep,
                    const int32_t *rep_recv, const int32_t *rep_slot, const int32_t *rep_off,
                    const int32_t *rep_cnt, const uint16_t *recv, uint16_t *out)
{
    const int64_t H = c->H, Cm = c->C_max;
    const int SEG = 2 * c->L + c->B;
    int64_t rows = 0;
    for (int r = 0; r < c->R; ++r) {
        for (int s = 0; s < SEG; ++s) {
            int64_t row0 = (int64_t)r * Cm + seg_off[r * SEG + s];
            int64_t n = seg_len[r * SEG + s];
            memcpy(out + row0 * H, recv + row0 * H, (size_t)(n * H * 2));
            rows += n;
        }
    }
    for (int q = 0; q < n_rep; ++q)
        if (rep_slot[q] < 0) {
            int64_t row0 = (int64_t)rep_recv[q] * Cm + rep_off[q];
            memcpy(out + row0 * H, recv + row0 * H, (size_t)((int64_t)rep_cnt[q] * H * 2));
            rows += rep_cnt[q];
        }
    return rows;
}

/* O8 stand-in expert: y[row] = bf16(float(recv[row]) * scale[expert(row)]),
 * one fp32 multiply; expert(row) from the segment tables. */
static void or_scale_rows(const or_cfg *c, int64_t row0, int64_t n, int e, const uint16_t *recv,
                          const float *scale, uint16_t *y)
{
    const int64_t H = c->H;
    for (int64_t i = 0; i < n; ++i)
        for (int64_t h = 0; h < H; ++h) {
            float v = or_bf16_to_f32(recv[(row0 + i) * H + h]) * scale[e];
            y[(row0 + i) * H + h] = or_f32_to_bf16(v);
        }
}

/* remote pieces (slot -1, remote-weights mode) are not in the segment
 * tables: rep_* describe them (n_rep pieces; may be 0) */
void or_expert_scale(const or_cfg *c, const int32_t *seg_off, const int32_t *seg_len,
                     const int32_t *slot_expert, const uint16_t *recv, const float *scale,
                     uint16_t *y, int n_rep, const int32_t *rep_expert, const int32_t *rep_recv,
                     const int32_t *rep_slot, const int32_t *rep_off, const int32_t *rep_cnt)
{
    const int R = c->R, L = c->L, B = c->B, SEG = 2 * L + B;
    for (int q = 0; q < n_rep; ++q)
        if (rep_slot[q] < 0)
            or_scale_rows(c, (int64_t)rep_recv[q] * c->C_max + rep_off[q], rep_cnt[q], rep_expert[q], recv, scale, y);
    for (int r = 0; r < R; ++r)
        for (int s = 0; s < SEG; ++s) {
            int e;
            if (s < L) e = r * L + s;
            else if (s < L + B) e = slot_expert[r * B + (s - L)];
            else e = r * L + (s - L - B);
            if (seg_len[r * SEG + s] == 0 || e < 0) continue;
            or_scale_rows(c, (int64_t)r * c->C_max + seg_off[r * SEG + s], seg_len[r * SEG + s], e, recv, scale, y);
        }
}

/* O9 combine: acc = 0; acc = fmaf(w[t,k], float(y[dest[t,k]]), acc) for
 * k = 0..K-1; out = bf16(acc).  acc_out (may be NULL) keeps the fp32 sums. */
void or_combine(const or_cfg *c, const int32_t *dest, const uint16_t *y, const float *w,
                uint16_t *out, float *acc_out, int64_t n_tokens)
{
    const int64_t H = c->H;
    for (int64_t t = 0; t < n_tokens; ++t)
        for (int64_t h = 0; h < H; ++h) {
            float acc = 0.0f;
            for (int k = 0; k < c->K; ++k) {
                int64_t d = dest[t * c->K + k];
                acc = fmaf(w[t * c->K + k], or_bf16_to_f32(y[d * H + h]), acc);
            }
            out[t * H + h] = or_f32_to_bf16(acc);
            if (acc_out) acc_out[t * H + h] = acc;
        }
}

/* O10a prefetch: w_slot[r][b] = w_home[slot_expert[r][b]] for used slots */
void or_prefetch(const or_cfg *c, const int32_t *slot_expert, const uint16_t *w_home,
                 uint16_t *w_slot, int64_t elems)
{
    for (int i = 0; i < c->R * c->B; ++i) {
        int e = slot_expert[i];
        if (e < 0) continue;
        memcpy(w_slot + (int64_t)i * elems, w_home + (int64_t)e * elems, (size_t)elems * 2);
    }
}

/* O10b reduce_grad: for each expert with replicas, in ascending receiver
 * order, g_home[e] = g_home[e] + g_rep[r][b] (fp32); then zero the used
 * replica slots.  The reduce buffer is [R, B, H, H'] (twodots.gr): only
 * pieces that hold a slot have a replica gradient; a piece without one
 * (remote weights) contributes nothing here. */
void or_reduce_grad(const or_cfg *c, const int32_t *rep_ptr, const int32_t *rep_recv,
                    const int32_t *rep_slot, float *g_home, float *g_rep, int64_t elems)
{
    const int N = c->R * c->L;
    for (int e = 0; e < N; ++e) {
        for (int q = rep_ptr[e]; q < rep_ptr[e + 1]; ++q) {
            if (rep_slot[q] < 0) continue;
            const float *src = g_rep + ((int64_t)rep_recv[q] * c->B + rep_slot[q]) * elems;
            float *dst = g_home + (int64_t)e * elems;
            for (int64_t i = 0; i < elems; ++i) dst[i] = dst[i] + src[i];
        }
        for (int q = rep_ptr[e]; q < rep_ptr[e + 1]; ++q) {
            if (rep_slot[q] < 0) continue;
            float *src = g_rep + ((int64_t)rep_recv[q] * c->B + rep_slot[q]) * elems;
            for (int64_t i = 0; i < elems; ++i) src[i] = 0.0f;
        }
    }
}

/* exported bf16 conversions, so tests can pin them against numpy/torch */
uint16_t or_f32_to_bf16_export(float f) { return or_f32_to_bf16(f); }
float or_bf16_to_f32_export(uint16_t u) { return or_bf16_to_f32(u); }

/* ------------------------------------------------------------------------ */
/* Backward of the data path (training; combine's and dispatch's adjoints).  */
/* The forward steps are linear: combine gives out[t] = sum_k w[t,k] *       */
/* y[dest[t,k]], dispatch gives recv[dest[t,k]] = x[t].  Their gradients:    */
/*   combine backward:  grad_y[dest[t,k]] = w[t,k] * grad_out[t]             */
/*                      grad_w[t,k]       = sum_h grad_out[t,h] * y[dest,h]  */
/*   dispatch backward: grad_x[t]         = sum_k grad_recv[dest[t,k]]       */
/* grad_y is one fp32 multiply rounded to bf16; grad_w is summed in fp64     */
/* (its order is not part of any contract); grad_x accumulates fp32 adds in  */
/* k order and rounds once to bf16, like combine.                            */
/* ------------------------------------------------------------------------ */
void or_combine_backward(const or_cfg *c, const int32_t *dest, const uint16_t *grad_out, const uint16_t *y,
                         const float *w, uint16_t *grad_y, double *grad_w, int64_t n_tokens)
{
    const int64_t H = c->H;
    for (int64_t t = 0; t < n_tokens; ++t)
        for (int k = 0; k < c->K; ++k) {
            int64_t d = dest[t * c->K + k];
            float wk = w[t * c->K + k];
            double dot = 0.0;
            for (int64_t h = 0; h < H; ++h) {
                float g = or_bf16_to_f32(grad_out[t * H + h]);
                grad_y[d * H + h] = or_f32_to_bf16(wk * g);
                if (grad_w) dot += (double)g * (double)or_bf16_to_f32(y[d * H + h]);
            }
            if (grad_w) grad_w[t * c->K + k] = dot;
        }
}

void or_dispatch_backward(const or_cfg *c, const int32_t *dest, const uint16_t *grad_recv, uint16_t *grad_x,
                          float *acc_out, int64_t n_tokens)
{
    const int64_t H = c->H;
    for (int64_t t = 0; t < n_tokens; ++t)
        for (int64_t h = 0; h < H; ++h) {
            float acc = 0.0f;
            for (int k = 0; k < c->K; ++k) {
                int64_t d = dest[t * c->K + k];
                acc = acc + or_bf16_to_f32(grad_recv[d * H + h]);
            }
            grad_x[t * H + h] = or_f32_to_bf16(acc);
            if (acc_out) acc_out[t * H + h] = acc;
        }
}
