// api.cu -- the C ABI of the MoonEP hot path: argument validation, workspace
// layout, launch configuration and error reporting.  Every compute step runs
// in the kernels of plan.cu, dispatch.cu, combine.cu and weights.cu; this
// file only checks arguments and launches them.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <string>
#include <unordered_map>

#include "moonep_internal.cuh"

#ifndef MOONEP_DISPATCH_MAX_CTAS
#define MOONEP_DISPATCH_MAX_CTAS 2  // resident dispatch CTAs per SM the shared memory is sized for
                                    // (4 and 5 give smaller pieces and ran 3-4% slower)
#endif

using namespace moonep;

namespace {

thread_local std::string g_err;
std::atomic<int64_t> g_wait_limit{int64_t(1) << 22};

int fail(int code, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return code;
}

int cuda_fail(cudaError_t e, const char *what) {
    return fail(MOONEP_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

struct DeviceInfo {
    bool ready = false;
    bool ok = false;
    int sms = 0;
    int plan_grid = 0;
    int combine_grid = 0;
    int backward_grid = 0;
    size_t plan_smem = 0;
};

std::mutex g_dev_mu;
DeviceInfo g_dev[64];

// zero-copy view generations: dispatch and combine launches per workspace
std::mutex g_gen_mu;
std::unordered_map<const void *, int64_t> g_gen;

void bump_generation(const void *ws) {
    std::lock_guard<std::mutex> lk(g_gen_mu);
    ++g_gen[ws];
}

// Checks the current device once (sm_100, cooperative launch) and caches
// launch sizes that depend on it.
int device_info(int N, DeviceInfo **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= 64) return fail(MOONEP_ERR_DEVICE, "device index %d out of range", dev);
    std::lock_guard<std::mutex> lk(g_dev_mu);
    DeviceInfo &d = g_dev[dev];
    if (!d.ready) {
        int major = 0, minor = 0, coop = 0;
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
        cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev);
        cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
        d.ok = (major == 10 && minor == 0 && coop != 0);
        d.ready = true;
        d.combine_grid = d.sms;  // one persistent combine CTA per SM
        d.backward_grid = d.sms;  // one persistent combine_backward CTA per SM
    }
    if (!d.ok) return fail(MOONEP_ERR_DEVICE, "device %d is not an sm_100 GPU with cooperative launch", dev);
    // plan kernel: shared memory depends on N
    const size_t smem = plan_smem_bytes(N);
    if (smem != d.plan_smem) {
        static std::atomic<size_t> plan_smem_set[64];
        e = set_smem_limit(plan_kernel_ptr(), smem, plan_smem_set);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(plan)");
        int nb = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, plan_kernel_ptr(), 512, smem);
        if (e != cudaSuccess) return cuda_fail(e, "occupancy(plan)");
        if (nb < 1) return fail(MOONEP_ERR_DEVICE, "plan kernel does not fit an SM");
        d.plan_grid = d.sms;  // one CTA per SM; co-resident by the cooperative launch
        d.plan_smem = smem;
    }
    *out = &d;
    return MOONEP_OK;
}

int check_cfg(const moonep_cfg_t *c) {
    if (!c) return fail(MOONEP_ERR_ARG, "cfg is NULL");
    if (c->R < 1 || c->R > 64) return fail(MOONEP_ERR_ARG, "R=%d outside [1, 64]", c->R);
    if (c->L < 1) return fail(MOONEP_ERR_ARG, "L=%d < 1", c->L);
    const int64_t N = (int64_t)c->R * c->L;
    if (N > 4096) return fail(MOONEP_ERR_ARG, "N=R*L=%lld above 4096", (long long)N);
    if (c->S < 0) return fail(MOONEP_ERR_ARG, "S=%d < 0", c->S);
    if (c->K < 1 || c->K > 64) return fail(MOONEP_ERR_ARG, "K=%d outside [1, 64]", c->K);
    if (c->H < 8 || c->H > (1 << 20) || (c->H % 8) != 0)
        return fail(MOONEP_ERR_ARG, "H=%d must be a multiple of 8 in [8, 2^20]", c->H);
    if (c->B < 0 || c->B > 1024 || (int64_t)c->R * c->B > 65536)
        return fail(MOONEP_ERR_ARG, "B=%d outside [0, 1024] or R*B above 65536", c->B);
    const int64_t C = (int64_t)c->S * c->K;
    if (c->C != C) return fail(MOONEP_ERR_ARG, "C=%d must equal S*K=%lld", c->C, (long long)C);
    if (c->C_max < c->C) return fail(MOONEP_ERR_ARG, "C_max=%d below C=%d", c->C_max, c->C);
    const int64_t T = (int64_t)c->R * c->S;
    if (T * c->K > INT32_MAX) return fail(MOONEP_ERR_ARG, "T*K above 2^31-1");
    if ((int64_t)c->R * c->C_max > INT32_MAX) return fail(MOONEP_ERR_ARG, "R*C_max above 2^31-1");
    return MOONEP_OK;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int check_ptr(const void *p, uintptr_t a, const char *name, bool needed) {
    if (!needed) return MOONEP_OK;
    if (!p) return fail(MOONEP_ERR_ARG, "%s is NULL", name);
    if (!aligned(p, a)) return fail(MOONEP_ERR_ARG, "%s is not %d-byte aligned", name, (int)a);
    return MOONEP_OK;
}

}  // namespace

namespace moonep {
// records a host error for moonep_last_error (used by other translation units)
int set_error(int code, const char *msg) { return fail(code, "%s", msg); }
}  // namespace moonep

namespace {

#define TRY(x)                        \
    do {                              \
        int _rc = (x);                \
        if (_rc != MOONEP_OK) return _rc; \
    } while (0)

}  // namespace

extern "C" {

int moonep_ws_layout(const moonep_cfg_t *cfg, moonep_ws_layout_t *out) {
    TRY(check_cfg(cfg));
    if (!out) return fail(MOONEP_ERR_ARG, "out is NULL");
    compute_layout(*cfg, *out);
    return MOONEP_OK;
}

size_t moonep_plan_workspace_bytes(const moonep_cfg_t *cfg) {
    if (check_cfg(cfg) != MOONEP_OK) return 0;
    moonep_ws_layout_t l;
    compute_layout(*cfg, l);
    return (size_t)l.words * 4;
}

int moonep_rank_bytes(const moonep_cfg_t *cfg, int64_t elems_per_expert, moonep_rank_bytes_t *out) {
    TRY(check_cfg(cfg));
    if (!out) return fail(MOONEP_ERR_ARG, "out is NULL");
    if (elems_per_expert < 0) return fail(MOONEP_ERR_ARG, "elems_per_expert < 0");
    out->dispatch_bytes = (int64_t)cfg->C_max * cfg->H * 2;
    out->prefetch_bytes = (int64_t)cfg->B * elems_per_expert * 2;
    out->reduce_bytes = (int64_t)cfg->B * elems_per_expert * 4;
    return MOONEP_OK;
}

int64_t moonep_num_ranges(int64_t T, int64_t N) { return T < 0 || N < 0 ? 0 : num_ranges(T, N); }

int moonep_set_wait_limit(int64_t polls) {
    if (polls < 0) return fail(MOONEP_ERR_ARG, "wait limit < 0");
    g_wait_limit.store(polls);
    return MOONEP_OK;
}

const char *moonep_last_error(void) { return g_err.c_str(); }

const char *moonep_version(void) { return "moonep-b200 0.1 (sm_100a)"; }

int moonep_plan(const moonep_cfg_t *cfg, const int32_t *topk_idx, void *ws, void *stream) {
    return moonep_plan_ex(cfg, 0, topk_idx, ws, stream);
}

int moonep_plan_ex(const moonep_cfg_t *cfg, int32_t flags, const int32_t *topk_idx, void *ws, void *stream) {
    TRY(check_cfg(cfg));
    if (flags & ~(MOONEP_PLAN_REMOTE_WEIGHTS | MOONEP_PLAN_ONE_GROUP))
        return fail(MOONEP_ERR_ARG, "unknown plan flags 0x%x", flags);
    if ((flags & MOONEP_PLAN_REMOTE_WEIGHTS) && (flags & MOONEP_PLAN_ONE_GROUP))
        return fail(MOONEP_ERR_ARG, "plan flags 0x%x: remote weights and one group exclude each other", flags);
    const int64_t T = (int64_t)cfg->R * cfg->S;
    TRY(check_ptr(topk_idx, 4, "topk_idx", T > 0));
    TRY(check_ptr(ws, 16, "ws", true));
    const int N = cfg->R * cfg->L;
    DeviceInfo *d = nullptr;
    TRY(device_info(N, &d));
    cudaStream_t s = (cudaStream_t)stream;
    PlanParams p{};
    p.cfg = *cfg;
    p.flags = flags;
    p.N = N;
    p.T = T;
    compute_layout(*cfg, p.lay);
    p.Q = p.lay.n_ranges;
    {
        // phase A holds one block's (range, expert) histogram and its totals
        // per expert in shared memory
        const int64_t rpb = p.lay.n_blocks > 0 ? (p.Q + p.lay.n_blocks - 1) / p.lay.n_blocks : 0;
        if ((size_t)((rpb + 1) * N) * sizeof(int) > d->plan_smem)
            return fail(MOONEP_ERR_ARG, "plan: %lld ranges per block of %d experts exceed shared memory",
                        (long long)rpb, N);
    }
    p.ids = topk_idx;
    p.ws = (int32_t *)ws;
    p.wait_limit = g_wait_limit.load();
    cudaError_t e = cudaMemsetAsync(ws, 0, (size_t)(MOONEP_WS_HEADER_WORDS + N) * 4, s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(plan header)");
    e = launch_plan(p, d->plan_grid, d->plan_smem, s);
    if (e != cudaSuccess) return cuda_fail(e, "plan kernel launch");
    return MOONEP_OK;
}

int moonep_dispatch(const moonep_cfg_t *cfg, void *ws, const void *x, const int32_t *topk_idx, void *recv,
                    int32_t *dest, void *stream) {
    TRY(check_cfg(cfg));
    const int64_t T = (int64_t)cfg->R * cfg->S;
    TRY(check_ptr(ws, 16, "ws", true));
    TRY(check_ptr(x, 16, "x", T > 0));
    TRY(check_ptr(topk_idx, 4, "topk_idx", T > 0));
    TRY(check_ptr(recv, 16, "recv", T > 0));
    TRY(check_ptr(dest, 4, "dest", T > 0));
    const int N = cfg->R * cfg->L;
    DeviceInfo *d = nullptr;
    TRY(device_info(N, &d));
    if (T == 0) return MOONEP_OK;
    DispatchParams p{};
    p.cfg = *cfg;
    p.N = N;
    p.T = T;
    compute_layout(*cfg, p.lay);
    p.Q = p.lay.n_ranges;
    p.row_bytes = (uint32_t)cfg->H * 2;
    size_t smem = 0;
    // shared memory sized for two resident CTAs per SM (at H = 7168 this
    // comes to 66 KB, so the SM holds three); ranges beyond those run in
    // later waves
    int ctas_per_sm = (int)((p.Q + d->sms - 1) / d->sms);
    if (ctas_per_sm > MOONEP_DISPATCH_MAX_CTAS) ctas_per_sm = MOONEP_DISPATCH_MAX_CTAS;
    cudaError_t e = dispatch_smem_config(N, p.row_bytes, ctas_per_sm < 1 ? 1 : ctas_per_sm, &p.piece_bytes, &p.npc,
                                         &smem);
    if (e != cudaSuccess) return fail(MOONEP_ERR_ARG, "dispatch: no shared-memory configuration for H=%d", cfg->H);
    p.x = (const uint8_t *)x;
    p.ids = topk_idx;
    p.recv = (uint8_t *)recv;
    p.dest = dest;
    p.ws = (int32_t *)ws;
    p.wait_limit = g_wait_limit.load();
    e = launch_dispatch(p, smem, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "dispatch kernel launch");
    bump_generation(ws);
    return MOONEP_OK;
}

// combine and dispatch backward share the TMA gather kernel; the backward
// has no weights (each one is 1)
static int combine_impl(const moonep_cfg_t *cfg, void *ws, const void *y, const int32_t *dest, const float *topk_w,
                        void *out, void *stream, bool weighted) {
    TRY(check_cfg(cfg));
    const int64_t T = (int64_t)cfg->R * cfg->S;
    TRY(check_ptr(ws, 16, "ws", true));
    TRY(check_ptr(y, 16, weighted ? "y" : "grad_recv", T > 0));
    TRY(check_ptr(dest, 4, "dest", T > 0));
    TRY(check_ptr(topk_w, 4, "topk_w", weighted && T > 0));
    TRY(check_ptr(out, 16, weighted ? "out" : "grad_x", T > 0));
    DeviceInfo *d = nullptr;
    TRY(device_info(cfg->R * cfg->L, &d));
    if (T == 0) return MOONEP_OK;
    CombineParams p{};
    p.cfg = *cfg;
    p.T = T;
    p.hv = cfg->H / 8;
    size_t smem = 0;
    if (combine_config(cfg->K, p.hv, &p.chunk_bytes, &p.upt, &p.stages, &smem) != cudaSuccess)
        return fail(MOONEP_ERR_ARG, "combine: no shared-memory configuration for K=%d H=%d", cfg->K, cfg->H);
    p.units = T * p.upt;
    p.rows_total = (int64_t)cfg->R * cfg->C_max;
    p.y = (const uint4 *)y;
    p.dest = dest;
    p.w = weighted ? topk_w : nullptr;
    p.out = (uint4 *)out;
    p.ws = (int32_t *)ws;
    p.wait_limit = g_wait_limit.load();
    int64_t grid = d->combine_grid;
    if (grid > p.units) grid = p.units;
    if (grid < 1) grid = 1;
    cudaError_t e = launch_combine(p, (int)grid, smem, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "combine kernel launch");
    if (weighted) bump_generation(ws);
    return MOONEP_OK;
}

int moonep_combine(const moonep_cfg_t *cfg, void *ws, const void *y, const int32_t *dest, const float *topk_w,
                   void *out, void *stream) {
    return combine_impl(cfg, ws, y, dest, topk_w, out, stream, true);
}

int moonep_dispatch_backward(const moonep_cfg_t *cfg, void *ws, const void *grad_recv, const int32_t *dest,
                             void *grad_x, void *stream) {
    return combine_impl(cfg, ws, grad_recv, dest, nullptr, grad_x, stream, false);
}

int moonep_combine_backward(const moonep_cfg_t *cfg, void *ws, const void *grad_out, const void *y,
                            const int32_t *dest, const float *topk_w, void *grad_y, float *grad_w, void *stream) {
    TRY(check_cfg(cfg));
    const int64_t T = (int64_t)cfg->R * cfg->S;
    TRY(check_ptr(ws, 16, "ws", true));
    TRY(check_ptr(grad_out, 16, "grad_out", T > 0));
    TRY(check_ptr(dest, 4, "dest", T > 0));
    TRY(check_ptr(topk_w, 4, "topk_w", T > 0));
    TRY(check_ptr(grad_y, 16, "grad_y", T > 0));
    if (grad_w) {
        TRY(check_ptr(grad_w, 4, "grad_w", true));
        TRY(check_ptr(y, 16, "y (needed for grad_w)", T > 0));
    }
    DeviceInfo *d = nullptr;
    TRY(device_info(cfg->R * cfg->L, &d));
    if (T == 0) return MOONEP_OK;
    BackwardParams p{};
    p.cfg = *cfg;
    p.T = T;
    p.hv = cfg->H / 8;
    size_t smem = 0;
    if (combine_backward_config(cfg->K, p.hv, grad_w != nullptr, &p.chunk_bytes, &p.upt, &p.stages, &smem) !=
        cudaSuccess)
        return fail(MOONEP_ERR_ARG, "combine_backward: no shared-memory configuration for K=%d H=%d", cfg->K, cfg->H);
    p.rows_total = (int64_t)cfg->R * cfg->C_max;
    p.wait_limit = g_wait_limit.load();
    p.grad_out = (const uint4 *)grad_out;
    p.y = (const uint4 *)y;
    p.dest = dest;
    p.w = topk_w;
    p.grad_y = (uint4 *)grad_y;
    p.grad_w = grad_w;
    p.ws = (int32_t *)ws;
    int64_t grid = d->backward_grid;
    if (grid > T) grid = T;
    if (grid < 1) grid = 1;
    cudaError_t e = launch_combine_backward(p, (int)grid, smem, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "combine_backward kernel launch");
    return MOONEP_OK;
}

int moonep_copy_out(const moonep_cfg_t *cfg, void *ws, const void *recv, void *out, void *stream) {
    TRY(check_cfg(cfg));
    const int64_t rows = (int64_t)cfg->R * cfg->C_max;
    TRY(check_ptr(ws, 16, "ws", true));
    TRY(check_ptr(recv, 16, "recv", rows > 0));
    TRY(check_ptr(out, 16, "out", rows > 0));
    const int64_t bytes = rows * cfg->H * 2;
    const char *a = (const char *)recv, *b = (const char *)out;
    if (rows > 0 && a < b + bytes && b < a + bytes) return fail(MOONEP_ERR_ARG, "copy_out: recv and out overlap");
    DeviceInfo *d = nullptr;
    TRY(device_info(cfg->R * cfg->L, &d));
    if (rows == 0 || (int64_t)cfg->R * cfg->S == 0) return MOONEP_OK;
    CopyOutParams p{};
    p.cfg = *cfg;
    compute_layout(*cfg, p.lay);
    p.Q = p.lay.n_ranges;
    p.row_vecs = cfg->H / 8;
    p.src = (const uint4 *)recv;
    p.dst = (uint4 *)out;
    p.ws = (int32_t *)ws;
    p.wait_limit = g_wait_limit.load();
    cudaError_t e = launch_copy_out(p, d->sms, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "copy_out kernel launch");
    return MOONEP_OK;
}

int64_t moonep_view_generation(const void *ws) {
    std::lock_guard<std::mutex> lk(g_gen_mu);
    auto it = g_gen.find(ws);
    return it == g_gen.end() ? 0 : it->second;
}

int moonep_prefetch(const moonep_cfg_t *cfg, void *ws, const void *w_home, void *w_slot, int64_t elems_per_expert,
                    void *stream) {
    TRY(check_cfg(cfg));
    if (elems_per_expert <= 0 || (elems_per_expert % 8) != 0)
        return fail(MOONEP_ERR_ARG, "elems_per_expert=%lld must be a positive multiple of 8",
                    (long long)elems_per_expert);
    TRY(check_ptr(ws, 16, "ws", true));
    TRY(check_ptr(w_home, 16, "w_home", true));
    TRY(check_ptr(w_slot, 16, "w_slot", cfg->B > 0));
    DeviceInfo *d = nullptr;
    TRY(device_info(cfg->R * cfg->L, &d));
    if (cfg->B == 0) return MOONEP_OK;
    CopyParams p{};
    p.cfg = *cfg;
    p.vecs = elems_per_expert * 2 / 16;
    p.src = (const uint4 *)w_home;
    p.dst = (uint4 *)w_slot;
    p.ws = (int32_t *)ws;
    compute_layout(*cfg, p.lay);
    p.wait_limit = g_wait_limit.load();
    cudaError_t e = launch_prefetch(p, d->sms, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "prefetch kernel launch");
    return MOONEP_OK;
}

int moonep_reduce_grad(const moonep_cfg_t *cfg, void *ws, float *g_home, float *g_rep, int64_t elems_per_expert,
                       void *stream) {
    TRY(check_cfg(cfg));
    if (elems_per_expert <= 0 || (elems_per_expert % 4) != 0)
        return fail(MOONEP_ERR_ARG, "elems_per_expert=%lld must be a positive multiple of 4",
                    (long long)elems_per_expert);
    TRY(check_ptr(ws, 16, "ws", true));
    TRY(check_ptr(g_home, 16, "g_home", true));
    TRY(check_ptr(g_rep, 16, "g_rep", cfg->B > 0));
    DeviceInfo *d = nullptr;
    TRY(device_info(cfg->R * cfg->L, &d));
    if (cfg->B == 0) return MOONEP_OK;
    CopyParams p{};
    p.cfg = *cfg;
    p.vecs = elems_per_expert * 4 / 16;
    p.src = (const uint4 *)g_home;
    p.dst = (uint4 *)g_rep;
    p.ws = (int32_t *)ws;
    compute_layout(*cfg, p.lay);
    p.wait_limit = g_wait_limit.load();
    cudaError_t e = launch_reduce_grad(p, d->sms, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "reduce_grad kernel launch");
    return MOONEP_OK;
}

// ---------------------------------------------------------------------------
// expert parallelism: one rank's calls
// ---------------------------------------------------------------------------

static int check_rank(const moonep_cfg_t *cfg, int32_t rank) {
    if (rank < 0 || rank >= cfg->R) return fail(MOONEP_ERR_ARG, "rank=%d outside [0, R=%d)", rank, cfg->R);
    return MOONEP_OK;
}

int moonep_ep_ws_layout(const moonep_cfg_t *cfg, moonep_ws_layout_t *out) {
    TRY(check_cfg(cfg));
    if (!out) return fail(MOONEP_ERR_ARG, "out is NULL");
    compute_layout_tokens(*cfg, cfg->S, *out);
    return MOONEP_OK;
}

size_t moonep_ep_workspace_bytes(const moonep_cfg_t *cfg) {
    if (check_cfg(cfg) != MOONEP_OK) return 0;
    moonep_ws_layout_t l;
    compute_layout_tokens(*cfg, cfg->S, l);
    return (size_t)l.words * 4;
}

// the plan kernel in one of its expert-parallel modes
static int ep_plan_launch(const moonep_cfg_t *cfg, int32_t mode, int32_t flags, int32_t rank, const int32_t *ids,
                          void *ws, int32_t *counts_out, const int32_t *counts_all, void *stream,
                          int32_t *const *counts_peers = nullptr) {
    const int N = cfg->R * cfg->L;
    DeviceInfo *d = nullptr;
    TRY(device_info(N, &d));
    PlanParams p{};
    p.cfg = *cfg;
    p.flags = flags;
    p.N = N;
    p.T = cfg->S;
    compute_layout_tokens(*cfg, cfg->S, p.lay);
    p.Q = p.lay.n_ranges;
    const int64_t rpb = p.lay.n_blocks > 0 ? (p.Q + p.lay.n_blocks - 1) / p.lay.n_blocks : 0;
    if ((size_t)((rpb + 1) * N) * sizeof(int) > d->plan_smem)
        return fail(MOONEP_ERR_ARG, "plan: %lld ranges per block of %d experts exceed shared memory", (long long)rpb, N);
    p.ids = ids;
    p.ws = (int32_t *)ws;
    p.wait_limit = g_wait_limit.load();
    p.mode = mode;
    p.rank = rank;
    p.counts_out = counts_out;
    p.counts_all = counts_all;
    p.counts_peers = counts_peers;
    cudaError_t e = launch_plan(p, d->plan_grid, d->plan_smem, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "plan kernel launch");
    return MOONEP_OK;
}

static int ep_count_impl(const moonep_cfg_t *cfg, int32_t rank, const int32_t *topk_idx, void *ws, int32_t *counts,
                         int32_t *const *counts_all_peers, void *stream) {
    TRY(check_cfg(cfg));
    TRY(check_rank(cfg, rank));
    TRY(check_ptr(topk_idx, 4, "topk_idx", cfg->S > 0));
    TRY(check_ptr(ws, 16, "ws", true));
    TRY(check_ptr(counts, 4, "counts", true));
    const int N = cfg->R * cfg->L;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = cudaMemsetAsync(ws, 0, (size_t)MOONEP_WS_HEADER_WORDS * 4, s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(header)");
    e = cudaMemsetAsync(counts, 0, (size_t)(N + 1) * 4, s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(counts)");
    if (cfg->S == 0 && !counts_all_peers) {
        DeviceInfo *d = nullptr;
        return device_info(N, &d);
    }
    // with peers the launch runs even without tokens: it stores the rank's
    // (zero) counts into every rank's counts_all
    return ep_plan_launch(cfg, kPlanCount, 0, rank, topk_idx, ws, counts, nullptr, stream, counts_all_peers);
}

int moonep_ep_count(const moonep_cfg_t *cfg, int32_t rank, const int32_t *topk_idx, void *ws, int32_t *counts,
                    void *stream) {
    return ep_count_impl(cfg, rank, topk_idx, ws, counts, nullptr, stream);
}

int moonep_ep_count_exchange(const moonep_cfg_t *cfg, int32_t rank, const int32_t *topk_idx, void *ws,
                             int32_t *counts, int32_t *const *counts_all_peers, void *stream) {
    TRY(check_ptr(counts_all_peers, 8, "counts_all_peers", true));
    return ep_count_impl(cfg, rank, topk_idx, ws, counts, counts_all_peers, stream);
}

int moonep_ep_plan(const moonep_cfg_t *cfg, int32_t flags, int32_t rank, const int32_t *counts_all, void *ws,
                   void *stream) {
    TRY(check_cfg(cfg));
    TRY(check_rank(cfg, rank));
    if (flags & ~(MOONEP_PLAN_REMOTE_WEIGHTS | MOONEP_PLAN_ONE_GROUP))
        return fail(MOONEP_ERR_ARG, "unknown plan flags 0x%x", flags);
    if ((flags & MOONEP_PLAN_REMOTE_WEIGHTS) && (flags & MOONEP_PLAN_ONE_GROUP))
        return fail(MOONEP_ERR_ARG, "plan flags 0x%x: remote weights and one group exclude each other", flags);
    TRY(check_ptr(counts_all, 4, "counts_all", true));
    TRY(check_ptr(ws, 16, "ws", true));
    return ep_plan_launch(cfg, kPlanFromCounts, flags, rank, nullptr, ws, nullptr, counts_all, stream);
}

int moonep_ep_dispatch(const moonep_cfg_t *cfg, int32_t rank, void *ws, const void *x, const int32_t *topk_idx,
                       void *const *recv_peers, int32_t *dest, void *stream) {
    TRY(check_cfg(cfg));
    TRY(check_rank(cfg, rank));
    const int64_t T = cfg->S;
    TRY(check_ptr(ws, 16, "ws", true));
    TRY(check_ptr(x, 16, "x", T > 0));
    TRY(check_ptr(topk_idx, 4, "topk_idx", T > 0));
    TRY(check_ptr(recv_peers, 8, "recv_peers", T > 0));
    TRY(check_ptr(dest, 4, "dest", T > 0));
    const int N = cfg->R * cfg->L;
    DeviceInfo *d = nullptr;
    TRY(device_info(N, &d));
    if (T == 0) return MOONEP_OK;
    DispatchParams p{};
    p.cfg = *cfg;
    p.N = N;
    p.T = T;
    compute_layout_tokens(*cfg, T, p.lay);
    p.Q = p.lay.n_ranges;
    p.row_bytes = (uint32_t)cfg->H * 2;
    size_t smem = 0;
    int ctas_per_sm = (int)((p.Q + d->sms - 1) / d->sms);
    if (ctas_per_sm > MOONEP_DISPATCH_MAX_CTAS) ctas_per_sm = MOONEP_DISPATCH_MAX_CTAS;
    cudaError_t e = dispatch_smem_config(N, p.row_bytes, ctas_per_sm < 1 ? 1 : ctas_per_sm, &p.piece_bytes, &p.npc,
                                         &smem, true);
    if (e != cudaSuccess) return fail(MOONEP_ERR_ARG, "dispatch: no shared-memory configuration for H=%d", cfg->H);
    p.x = (const uint8_t *)x;
    p.ids = topk_idx;
    p.recv_peers = (uint8_t *const *)recv_peers;
    p.dest = dest;
    p.ws = (int32_t *)ws;
    p.wait_limit = g_wait_limit.load();
    p.ep_tag = rank + 1;
    e = launch_dispatch(p, smem, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "dispatch kernel launch");
    bump_generation(ws);
    return MOONEP_OK;
}

static int ep_combine_impl(const moonep_cfg_t *cfg, int32_t rank, void *ws, const void *const *y_peers,
                           const int32_t *dest, const float *topk_w, void *out, void *stream, bool weighted) {
    TRY(check_cfg(cfg));
    TRY(check_rank(cfg, rank));
    const int64_t T = cfg->S;
    TRY(check_ptr(ws, 16, "ws", true));
    TRY(check_ptr(y_peers, 8, weighted ? "y_peers" : "grad_recv_peers", T > 0));
    TRY(check_ptr(dest, 4, "dest", T > 0));
    TRY(check_ptr(topk_w, 4, "topk_w", weighted && T > 0));
    TRY(check_ptr(out, 16, weighted ? "out" : "grad_x", T > 0));
    DeviceInfo *d = nullptr;
    TRY(device_info(cfg->R * cfg->L, &d));
    if (T == 0) return MOONEP_OK;
    CombineParams p{};
    p.cfg = *cfg;
    p.T = T;
    p.hv = cfg->H / 8;
    size_t smem = 0;
    if (combine_config(cfg->K, p.hv, &p.chunk_bytes, &p.upt, &p.stages, &smem, true) != cudaSuccess)
        return fail(MOONEP_ERR_ARG, "combine: no shared-memory configuration for K=%d H=%d", cfg->K, cfg->H);
    p.units = T * p.upt;
    p.rows_total = (int64_t)cfg->R * cfg->C_max;
    p.y = nullptr;
    p.y_peers = (const uint8_t *const *)y_peers;
    p.dest = dest;
    p.w = weighted ? topk_w : nullptr;
    p.out = (uint4 *)out;
    p.ws = (int32_t *)ws;
    p.wait_limit = g_wait_limit.load();
    p.ep_tag = rank + 1;
    int64_t grid = d->combine_grid;
    if (grid > p.units) grid = p.units;
    if (grid < 1) grid = 1;
    cudaError_t e = launch_combine(p, (int)grid, smem, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "combine kernel launch");
    if (weighted) bump_generation(ws);
    return MOONEP_OK;
}

int moonep_ep_combine(const moonep_cfg_t *cfg, int32_t rank, void *ws, const void *const *y_peers,
                      const int32_t *dest, const float *topk_w, void *out, void *stream) {
    return ep_combine_impl(cfg, rank, ws, y_peers, dest, topk_w, out, stream, true);
}

int moonep_ep_dispatch_backward(const moonep_cfg_t *cfg, int32_t rank, void *ws, const void *const *grad_recv_peers,
                                const int32_t *dest, void *grad_x, void *stream) {
    return ep_combine_impl(cfg, rank, ws, grad_recv_peers, dest, nullptr, grad_x, stream, false);
}

int moonep_ep_combine_backward(const moonep_cfg_t *cfg, int32_t rank, void *ws, const void *grad_out,
                               const void *const *y_peers, const int32_t *dest, const float *topk_w,
                               void *const *grad_y_peers, float *grad_w, void *stream) {
    TRY(check_cfg(cfg));
    TRY(check_rank(cfg, rank));
    const int64_t T = cfg->S;
    TRY(check_ptr(ws, 16, "ws", true));
    TRY(check_ptr(grad_out, 16, "grad_out", T > 0));
    TRY(check_ptr(dest, 4, "dest", T > 0));
    TRY(check_ptr(topk_w, 4, "topk_w", T > 0));
    TRY(check_ptr(grad_y_peers, 8, "grad_y_peers", T > 0));
    if (grad_w) {
        TRY(check_ptr(grad_w, 4, "grad_w", true));
        TRY(check_ptr(y_peers, 8, "y_peers (needed for grad_w)", T > 0));
    }
    DeviceInfo *d = nullptr;
    TRY(device_info(cfg->R * cfg->L, &d));
    if (T == 0) return MOONEP_OK;
    BackwardParams p{};
    p.cfg = *cfg;
    p.T = T;
    p.hv = cfg->H / 8;
    size_t smem = 0;
    if (combine_backward_config(cfg->K, p.hv, grad_w != nullptr, &p.chunk_bytes, &p.upt, &p.stages, &smem) !=
        cudaSuccess)
        return fail(MOONEP_ERR_ARG, "combine_backward: no shared-memory configuration for K=%d H=%d", cfg->K, cfg->H);
    p.rows_total = (int64_t)cfg->R * cfg->C_max;
    p.wait_limit = g_wait_limit.load();
    p.grad_out = (const uint4 *)grad_out;
    p.y = nullptr;
    p.y_peers = grad_w ? (const uint8_t *const *)y_peers : nullptr;
    p.dest = dest;
    p.w = topk_w;
    p.grad_y = nullptr;
    p.grad_y_peers = (uint8_t *const *)grad_y_peers;
    p.grad_w = grad_w;
    p.ws = (int32_t *)ws;
    p.ep_tag = rank + 1;
    int64_t grid = d->backward_grid;
    if (grid > T) grid = T;
    if (grid < 1) grid = 1;
    cudaError_t e = launch_combine_backward(p, (int)grid, smem, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "combine_backward kernel launch");
    return MOONEP_OK;
}

int moonep_ep_prefetch(const moonep_cfg_t *cfg, int32_t rank, void *ws, const void *const *w_home_peers, void *w_slot,
                       int64_t elems_per_expert, void *stream) {
    TRY(check_cfg(cfg));
    TRY(check_rank(cfg, rank));
    if (elems_per_expert <= 0 || (elems_per_expert % 8) != 0)
        return fail(MOONEP_ERR_ARG, "elems_per_expert=%lld must be a positive multiple of 8",
                    (long long)elems_per_expert);
    TRY(check_ptr(ws, 16, "ws", true));
    TRY(check_ptr(w_home_peers, 8, "w_home_peers", true));
    TRY(check_ptr(w_slot, 16, "w_slot", cfg->B > 0));
    DeviceInfo *d = nullptr;
    TRY(device_info(cfg->R * cfg->L, &d));
    if (cfg->B == 0) return MOONEP_OK;
    CopyParams p{};
    p.cfg = *cfg;
    p.vecs = elems_per_expert * 2 / 16;
    p.src = nullptr;
    p.dst = (uint4 *)w_slot;
    p.ws = (int32_t *)ws;
    compute_layout_tokens(*cfg, cfg->S, p.lay);
    p.wait_limit = g_wait_limit.load();
    p.peers = (uint8_t *const *)w_home_peers;
    p.ep_tag = rank + 1;
    cudaError_t e = launch_prefetch(p, d->sms, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "prefetch kernel launch");
    return MOONEP_OK;
}

int moonep_ep_reduce_grad(const moonep_cfg_t *cfg, int32_t rank, void *ws, float *g_home, void *const *g_rep_peers,
                          int64_t elems_per_expert, void *stream) {
    TRY(check_cfg(cfg));
    TRY(check_rank(cfg, rank));
    if (elems_per_expert <= 0 || (elems_per_expert % 4) != 0)
        return fail(MOONEP_ERR_ARG, "elems_per_expert=%lld must be a positive multiple of 4",
                    (long long)elems_per_expert);
    TRY(check_ptr(ws, 16, "ws", true));
    TRY(check_ptr(g_home, 16, "g_home", true));
    TRY(check_ptr(g_rep_peers, 8, "g_rep_peers", cfg->B > 0));
    DeviceInfo *d = nullptr;
    TRY(device_info(cfg->R * cfg->L, &d));
    if (cfg->B == 0) return MOONEP_OK;
    CopyParams p{};
    p.cfg = *cfg;
    p.vecs = elems_per_expert * 4 / 16;
    p.src = (const uint4 *)g_home;
    p.dst = nullptr;
    p.ws = (int32_t *)ws;
    compute_layout_tokens(*cfg, cfg->S, p.lay);
    p.wait_limit = g_wait_limit.load();
    p.peers = (uint8_t *const *)g_rep_peers;
    p.ep_tag = rank + 1;
    cudaError_t e = launch_reduce_grad(p, d->sms, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "reduce_grad kernel launch");
    return MOONEP_OK;
}

int moonep_plan_read(const moonep_cfg_t *cfg, const void *ws, moonep_plan_info_t *info, int32_t *host_tables,
                     void *stream) {
    TRY(check_cfg(cfg));
    TRY(check_ptr(ws, 16, "ws", true));
    if (!info && !host_tables) return fail(MOONEP_ERR_ARG, "nothing to read");
    moonep_ws_layout_t l;
    compute_layout(*cfg, l);
    cudaStream_t s = (cudaStream_t)stream;
    int32_t hdr[MOONEP_WS_HEADER_WORDS];
    cudaError_t e = cudaMemcpyAsync(hdr, ws, sizeof hdr, cudaMemcpyDeviceToHost, s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyAsync(header)");
    if (host_tables) {
        e = cudaMemcpyAsync(host_tables, (const int32_t *)ws + l.cnt, (size_t)(l.tables_end - l.cnt) * 4,
                            cudaMemcpyDeviceToHost, s);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyAsync(tables)");
    }
    e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    if (info) {
        info->status = hdr[HDR_STATUS];
        info->fallback_rows = hdr[HDR_FALLBACK];
        info->n_replicas = hdr[HDR_NREP];
        info->migrated_rows = hdr[HDR_MIGRATED];
    }
    return MOONEP_OK;
}

}  // extern "C"
