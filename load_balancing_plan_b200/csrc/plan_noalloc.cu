// plan_noalloc.cu -- moonep_plan_noalloc: the planning step for callers that
// cannot allocate device memory themselves.
//
// moonep_plan needs a caller-allocated workspace: besides the plan tables it
// holds scratch the planner uses while it runs (per-token-range counts of
// every expert, grid-barrier counters).  Some callers cannot get such a
// buffer: a plug-in that a host framework hands tensors to but no
// allocator, or a process whose device memory is owned by a pooled
// allocator that must not see extra cudaMalloc calls or grow in the middle
// of a step.  For them this variant keeps the whole workspace in a fixed,
// file-scope device array of kStaticWsBytes (2 MiB, held by every GPU that
// loads the library until the process exits) and copies the plan header and
// tables into the caller's output buffer.  It runs the same plan kernel as
// moonep_plan and allocates nothing.  The copy lacks the dispatch scratch
// that follows the tables in a full workspace, so its header is marked
// (word HDR_TABLES_ONLY) and moonep_dispatch refuses it; the calls that read
// only the header and tables (plan_read, prefetch, reduce_grad, copy_out,
// combine and the backward pair) accept it.
//
// The cached device address stays valid for the life of the CUDA context;
// after cudaDeviceReset on that device it is stale, and the library must not
// be called on that device again in this process.
//
// The array's name is only a host-side handle; its device address comes from
// cudaGetSymbolAddress, taken once per device, with that device current, by
// the first call made on that device.  All calls share the array, which
// keeps the last call's contents; each call clears the parts that must start
// at zero (the header and the per-expert counters), as moonep_plan does.
// Calls that overlap on the GPU (on different streams, or from different
// host threads on one device) race on the array: the caller must serialise
// them.
#include <cstdio>
#include <mutex>

#include "moonep_internal.cuh"

namespace {

constexpr size_t kStaticWsBytes = size_t(2) << 20;  // 2 MiB

__device__ __align__(256) int32_t g_static_ws[kStaticWsBytes / sizeof(int32_t)];

std::mutex g_mu;
void *g_ptr[64] = {};

// device address of g_static_ws on the current device (set up once per device)
int static_ws(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return moonep::set_error(MOONEP_ERR_CUDA, "cudaGetDevice failed");
    if (dev < 0 || dev >= 64) return moonep::set_error(MOONEP_ERR_DEVICE, "device index out of range");
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_ws);
        if (e != cudaSuccess || !p) {
            char msg[256];
            snprintf(msg, sizeof msg, "cudaGetSymbolAddress(static workspace): %s", cudaGetErrorString(e));
            return moonep::set_error(MOONEP_ERR_CUDA, msg);
        }
        g_ptr[dev] = p;
    }
    *out = g_ptr[dev];
    return MOONEP_OK;
}

}  // namespace

extern "C" MOONEP_API int moonep_plan_noalloc(const moonep_cfg_t *cfg, const int32_t *topk_idx, int32_t *tables_out,
                                              void *stream) {
    moonep_ws_layout_t lay;
    int rc = moonep_ws_layout(cfg, &lay);
    if (rc != MOONEP_OK) return rc;
    const size_t need = (size_t)lay.words * sizeof(int32_t);
    if (need > kStaticWsBytes) {
        char msg[256];
        snprintf(msg, sizeof msg,
                 "moonep_plan_noalloc: this configuration needs a %zu-byte workspace, above the %zu-byte "
                 "static workspace; use moonep_plan with a caller-allocated workspace",
                 need, kStaticWsBytes);
        return moonep::set_error(MOONEP_ERR_ARG, msg);
    }
    if (!tables_out || (reinterpret_cast<uintptr_t>(tables_out) & 15))
        return moonep::set_error(MOONEP_ERR_ARG, "moonep_plan_noalloc: tables_out is NULL or not 16-byte aligned");
    void *ws = nullptr;
    rc = static_ws(&ws);
    if (rc != MOONEP_OK) return rc;
    rc = moonep_plan(cfg, topk_idx, ws, stream);
    if (rc != MOONEP_OK) return rc;
    cudaError_t e = cudaMemcpyAsync(tables_out, ws, (size_t)lay.tables_end * sizeof(int32_t),
                                    cudaMemcpyDeviceToDevice, (cudaStream_t)stream);
    if (e != cudaSuccess) {
        char msg[256];
        snprintf(msg, sizeof msg, "moonep_plan_noalloc: copy of the tables: %s", cudaGetErrorString(e));
        return moonep::set_error(MOONEP_ERR_CUDA, msg);
    }
    // mark the copy as tables only: it has no dispatch scratch, and dispatch
    // refuses such a workspace (MOONEP_ST_CFG) instead of reading past its end
    e = cudaMemsetAsync(tables_out + moonep::HDR_TABLES_ONLY, moonep::kTablesOnlyMark & 0xFF, sizeof(int32_t),
                        (cudaStream_t)stream);
    if (e != cudaSuccess) {
        char msg[256];
        snprintf(msg, sizeof msg, "moonep_plan_noalloc: marking the copy: %s", cudaGetErrorString(e));
        return moonep::set_error(MOONEP_ERR_CUDA, msg);
    }
    return MOONEP_OK;
}
