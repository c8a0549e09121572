// Host side of the C ABI declared in include/ssa.h: argument validation,
// workspace sizing, kernel-path choice and status reporting.  Every compute
// step runs in the kernels of the sibling .cu files.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <cmath>

#include "ssa_internal.h"

namespace ssa {

namespace {
thread_local char g_last_error[512] = "";
constexpr unsigned long long kDefaultWaitLimitNs = 2000000000ull;
std::atomic<unsigned long long> g_wait_limit_ns{kDefaultWaitLimitNs};
std::atomic<void*> g_kernel_events[kKernelEvents];
constexpr unsigned long long kDefaultDsBudget = 4ull << 30;
std::atomic<unsigned long long> g_ds_budget{kDefaultDsBudget};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shape/method checks shared by every entry point.
int validate(const ssa_params_t* p) {
    if (!p) return fail(SSA_ERR_INVALID_ARG, "params is NULL");
    if (p->B <= 0 || p->H <= 0 || p->T <= 0 || p->D <= 0)
        return fail(SSA_ERR_INVALID_ARG, "B, H, T, D must be positive (got %d, %d, %d, %d)", p->B,
                    p->H, p->T, p->D);
    if (p->dtype != SSA_F32 && p->dtype != SSA_BF16)
        return fail(SSA_ERR_INVALID_ARG, "unknown dtype %d", p->dtype);
    if (p->block != 64 && p->block != 128)
        return fail(SSA_ERR_UNSUPPORTED, "block must be 64 or 128 (got %d)", p->block);
    if (p->T % p->block != 0)
        return fail(SSA_ERR_INVALID_ARG, "T (%d) must be a multiple of block (%d)", p->T, p->block);
    if (p->D != 64 && p->D != 128)
        return fail(SSA_ERR_UNSUPPORTED, "head dim D must be 64 or 128 (got %d)", p->D);
    const int n = p->T / p->block;
    if (p->topk < 1 || p->topk > n)
        return fail(SSA_ERR_INVALID_ARG, "topk must be in [1, T/block = %d] (got %d)", n, p->topk);
    if ((p->flags & SSA_FLAG_FORCE_SINK) && p->topk < 2)
        return fail(SSA_ERR_INVALID_ARG, "FORCE_SINK needs topk >= 2 (got %d)", p->topk);
    if (p->flags & ~(unsigned)(SSA_FLAG_FORCE_SINK | SSA_FLAG_FORCE_SIMT))
        return fail(SSA_ERR_INVALID_ARG, "unknown flag bits 0x%x", p->flags);
    if (!(p->sm_scale > 0.f) || !std::isfinite(p->sm_scale))
        return fail(SSA_ERR_INVALID_ARG, "sm_scale must be positive and finite");
    if ((double)p->B * p->H * p->T * p->D > 9.0e15)
        return fail(SSA_ERR_INVALID_ARG, "tensor too large");
    return SSA_OK;
}

int need_ptr(const void* ptr, const char* name) {
    if (!ptr) return fail(SSA_ERR_INVALID_ARG, "%s is NULL", name);
    if (!aligned16(ptr)) return fail(SSA_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
    return SSA_OK;
}

int opt_ptr(const void* ptr, const char* name) {
    if (ptr && !aligned16(ptr)) return fail(SSA_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
    return SSA_OK;
}

int need_ws(void* ws, size_t have, size_t need, const char* what) {
    if (need == 0) return SSA_OK;
    if (have < need)
        return fail(SSA_ERR_WORKSPACE, "%s needs %zu workspace bytes, got %zu", what, need, have);
    if (!ws) return fail(SSA_ERR_WORKSPACE, "%s: workspace pointer is NULL", what);
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
        return fail(SSA_ERR_INVALID_ARG, "%s: workspace must be 256-byte aligned", what);
    return SSA_OK;
}

bool use_tc(const ssa_params_t& p) {
    return !(p.flags & SSA_FLAG_FORCE_SIMT) && fwd_tc_supported(p) && bwd_tc_supported(p);
}

size_t fwd_workspace(const ssa_params_t& p) { return use_tc(p) ? fwd_tc_workspace(p) : 0; }
// CUDA-core path of the sparse-only forward: the dual kernel's other outputs
// (h_full in dtype, then delta, lse_full, sqdiff as float32 rows)
size_t fwd_sparse_workspace(const ssa_params_t& p) {
    if (use_tc(p)) return 0;
    const size_t esz = p.dtype == SSA_BF16 ? 2 : 4;
    return align_up(num_elems(p) * esz, 256) + 3 * align_up(num_rows(p) * 4, 256);
}
size_t bwd_workspace(const ssa_params_t& p) {
    return use_tc(p) ? bwd_tc_workspace(p) : bwd_simt_workspace(p);
}

}  // namespace

unsigned long long wait_limit_ns() { return g_wait_limit_ns.load(std::memory_order_relaxed); }
unsigned long long ds_budget_bytes() { return g_ds_budget.load(std::memory_order_relaxed); }

void mark_kernel_event(int i, cudaStream_t s) {
    void* e = g_kernel_events[i].load(std::memory_order_relaxed);
    if (e) cudaEventRecord(static_cast<cudaEvent_t>(e), s);
}

int fail(int status, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
    return status;
}

int check_launch(const char* what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(SSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    return SSA_OK;
}

}  // namespace ssa

using namespace ssa;

#define SSA_TRY(expr)              \
    do {                           \
        int _st = (expr);          \
        if (_st != SSA_OK) return _st; \
    } while (0)

extern "C" {

size_t ssa_workspace_size(const ssa_params_t* p, int which) {
    if (validate(p) != SSA_OK) return (size_t)-1;
    switch (which) {
        case SSA_WS_SELECT: return select_workspace(*p);
        case SSA_WS_FWD: return fwd_workspace(*p);
        case SSA_WS_LOSS: return loss_workspace(*p);
        case SSA_WS_BWD: return bwd_workspace(*p);
        case SSA_WS_FWD_SPARSE: return fwd_sparse_workspace(*p);
        case SSA_WS_DECODE: return decode_workspace(*p);
        default: fail(SSA_ERR_INVALID_ARG, "unknown workspace id %d", which); return (size_t)-1;
    }
}

int ssa_select_blocks(const ssa_params_t* p, const void* q, const void* k, int32_t* idx,
                      int32_t* cnt, uint32_t* mask, void* ws, size_t ws_bytes, void* stream) {
    g_last_error[0] = 0;
    SSA_TRY(validate(p));
    SSA_TRY(need_ptr(q, "q"));
    SSA_TRY(need_ptr(k, "k"));
    SSA_TRY(need_ptr(idx, "idx"));
    SSA_TRY(need_ptr(cnt, "cnt"));
    SSA_TRY(need_ptr(mask, "mask"));
    SSA_TRY(need_ws(ws, ws_bytes, select_workspace(*p), "ssa_select_blocks"));
    return launch_select(*p, q, k, idx, cnt, mask, ws, static_cast<cudaStream_t>(stream));
}

int ssa_attn_fwd_dual(const ssa_params_t* p, const void* q, const void* k, const void* v,
                      const int32_t* idx, const int32_t* cnt, const uint32_t* mask,
                      void* h_full, void* h_sparse, float* delta, float* lse_full,
                      float* lse_sparse, float* sqdiff, void* ws, size_t ws_bytes,
                      void* stream) {
    g_last_error[0] = 0;
    SSA_TRY(validate(p));
    SSA_TRY(need_ptr(q, "q"));
    SSA_TRY(need_ptr(k, "k"));
    SSA_TRY(need_ptr(v, "v"));
    SSA_TRY(opt_ptr(idx, "idx"));
    SSA_TRY(opt_ptr(cnt, "cnt"));
    SSA_TRY(need_ptr(mask, "mask"));
    SSA_TRY(need_ptr(h_full, "h_full"));
    SSA_TRY(need_ptr(h_sparse, "h_sparse"));
    SSA_TRY(need_ptr(delta, "delta"));
    SSA_TRY(need_ptr(lse_full, "lse_full"));
    SSA_TRY(need_ptr(lse_sparse, "lse_sparse"));
    SSA_TRY(need_ptr(sqdiff, "sqdiff_rows"));
    SSA_TRY(need_ws(ws, ws_bytes, fwd_workspace(*p), "ssa_attn_fwd_dual"));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (use_tc(*p))
        return launch_fwd_tc(*p, q, k, v, mask, h_full, h_sparse, delta, lse_full, lse_sparse,
                             sqdiff, nullptr, ws, s);
    return launch_fwd_simt(*p, q, k, v, mask, h_full, h_sparse, delta, lse_full, lse_sparse,
                           sqdiff, s);
}

int ssa_attn_fwd_dual_diag(const ssa_params_t* p, const void* q, const void* k, const void* v,
                           const int32_t* idx, const int32_t* cnt, const uint32_t* mask,
                           void* h_full, void* h_sparse, float* delta, float* lse_full,
                           float* lse_sparse, float* sqdiff, float* sink_rows, float* head_stats,
                           void* ws, size_t ws_bytes, void* stream) {
    g_last_error[0] = 0;
    SSA_TRY(validate(p));
    SSA_TRY(need_ptr(sink_rows, "sink_rows"));
    SSA_TRY(need_ptr(head_stats, "head_stats"));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (!use_tc(*p)) {  // CUDA-core path: the dual forward, then the diagnostics pass
        SSA_TRY(ssa_attn_fwd_dual(p, q, k, v, idx, cnt, mask, h_full, h_sparse, delta, lse_full,
                                  lse_sparse, sqdiff, ws, ws_bytes, stream));
        return launch_diagnostics(*p, q, k, lse_full, delta, sink_rows, head_stats, s);
    }
    SSA_TRY(need_ptr(q, "q"));
    SSA_TRY(need_ptr(k, "k"));
    SSA_TRY(need_ptr(v, "v"));
    SSA_TRY(opt_ptr(idx, "idx"));
    SSA_TRY(opt_ptr(cnt, "cnt"));
    SSA_TRY(need_ptr(mask, "mask"));
    SSA_TRY(need_ptr(h_full, "h_full"));
    SSA_TRY(need_ptr(h_sparse, "h_sparse"));
    SSA_TRY(need_ptr(delta, "delta"));
    SSA_TRY(need_ptr(lse_full, "lse_full"));
    SSA_TRY(need_ptr(lse_sparse, "lse_sparse"));
    SSA_TRY(need_ptr(sqdiff, "sqdiff_rows"));
    SSA_TRY(need_ws(ws, ws_bytes, fwd_workspace(*p), "ssa_attn_fwd_dual_diag"));
    SSA_TRY(launch_fwd_tc(*p, q, k, v, mask, h_full, h_sparse, delta, lse_full, lse_sparse, sqdiff,
                          sink_rows, ws, s));
    return launch_diag_heads(*p, delta, sink_rows, head_stats, s);
}

int ssa_attn_fwd_sparse(const ssa_params_t* p, const void* q, const void* k, const void* v,
                        const int32_t* idx, const int32_t* cnt, const uint32_t* mask,
                        void* h_sparse, float* lse_sparse, void* ws, size_t ws_bytes, void* stream) {
    g_last_error[0] = 0;
    SSA_TRY(validate(p));
    SSA_TRY(need_ptr(q, "q"));
    SSA_TRY(need_ptr(k, "k"));
    SSA_TRY(need_ptr(v, "v"));
    SSA_TRY(opt_ptr(idx, "idx"));
    SSA_TRY(opt_ptr(cnt, "cnt"));
    SSA_TRY(need_ptr(mask, "mask"));
    SSA_TRY(need_ptr(h_sparse, "h_sparse"));
    SSA_TRY(need_ptr(lse_sparse, "lse_sparse"));
    const size_t need = fwd_sparse_workspace(*p);
    SSA_TRY(need_ws(ws, ws_bytes, need, "ssa_attn_fwd_sparse"));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (use_tc(*p)) return launch_fwd_sparse_tc(*p, q, k, v, mask, h_sparse, lse_sparse, s);
    // CUDA-core path: the dual kernel, its full-stream outputs kept in the workspace
    const size_t esz = p->dtype == SSA_BF16 ? 2 : 4;
    const size_t rows = align_up(num_rows(*p) * 4, 256);
    char* w = static_cast<char*>(ws);
    void* h_full = w;
    char* r = w + align_up(num_elems(*p) * esz, 256);
    float* delta = reinterpret_cast<float*>(r);
    float* lse_full = reinterpret_cast<float*>(r + rows);
    float* sqdiff = reinterpret_cast<float*>(r + 2 * rows);
    return launch_fwd_simt(*p, q, k, v, mask, h_full, h_sparse, delta, lse_full, lse_sparse, sqdiff,
                           s);
}

static int decode_shape(const ssa_params_t* p) {
    SSA_TRY(validate(p));
    if (p->D != 64 && p->D != 128) return fail(SSA_ERR_UNSUPPORTED, "decode: D must be 64 or 128");
    if (p->topk > 64) return fail(SSA_ERR_UNSUPPORTED, "decode: topk must be <= 64");
    return SSA_OK;
}

int ssa_decode_pool(const ssa_params_t* p, int j0, int j1, const void* k_cache, double* kbar,
                    void* stream) {
    g_last_error[0] = 0;
    SSA_TRY(decode_shape(p));
    SSA_TRY(need_ptr(k_cache, "k_cache"));
    SSA_TRY(need_ptr(kbar, "kbar"));
    if (j0 < 0 || j1 < j0 || j1 > num_blocks(*p))
        return fail(SSA_ERR_INVALID_ARG, "decode_pool: blocks [%d, %d) outside [0, %d]", j0, j1,
                    num_blocks(*p));
    return launch_decode_pool(*p, j0, j1, k_cache, kbar, static_cast<cudaStream_t>(stream));
}

int ssa_decode_step(const ssa_params_t* p, int t, const void* q, const void* k_cache,
                    const void* v_cache, const double* kbar, void* h, float* lse, int32_t* idx,
                    void* ws, size_t ws_bytes, void* stream) {
    g_last_error[0] = 0;
    SSA_TRY(decode_shape(p));
    if (t < 0 || t >= p->T) return fail(SSA_ERR_INVALID_ARG, "decode_step: t = %d outside [0, %d)", t, p->T);
    SSA_TRY(need_ptr(q, "q"));
    SSA_TRY(need_ptr(k_cache, "k_cache"));
    SSA_TRY(need_ptr(v_cache, "v_cache"));
    SSA_TRY(need_ptr(kbar, "kbar"));
    SSA_TRY(need_ptr(h, "h"));
    SSA_TRY(need_ptr(lse, "lse"));
    SSA_TRY(opt_ptr(idx, "idx"));
    SSA_TRY(need_ws(ws, ws_bytes, decode_workspace(*p), "ssa_decode_step"));
    return launch_decode_step(*p, t, q, k_cache, v_cache, kbar, h, lse, idx, ws,
                              static_cast<cudaStream_t>(stream));
}

int ssa_attn_diagnostics(const ssa_params_t* p, const void* q, const void* k,
                         const float* lse_full, const float* delta, float* sink_rows,
                         float* head_stats, void* stream) {
    g_last_error[0] = 0;
    SSA_TRY(validate(p));
    SSA_TRY(need_ptr(q, "q"));
    SSA_TRY(need_ptr(k, "k"));
    SSA_TRY(need_ptr(lse_full, "lse_full"));
    SSA_TRY(need_ptr(delta, "delta"));
    SSA_TRY(need_ptr(sink_rows, "sink_rows"));
    SSA_TRY(need_ptr(head_stats, "head_stats"));
    return launch_diagnostics(*p, q, k, lse_full, delta, sink_rows, head_stats,
                              static_cast<cudaStream_t>(stream));
}

int ssa_align_loss(const ssa_params_t* p, const float* sqdiff, float w_s, float w_c,
                   float* loss_out, void* ws, size_t ws_bytes, void* stream) {
    g_last_error[0] = 0;
    SSA_TRY(validate(p));
    SSA_TRY(need_ptr(sqdiff, "sqdiff_rows"));
    SSA_TRY(need_ptr(loss_out, "loss_out"));
    if (!std::isfinite(w_s) || !std::isfinite(w_c))
        return fail(SSA_ERR_INVALID_ARG, "loss weights must be finite");
    SSA_TRY(need_ws(ws, ws_bytes, loss_workspace(*p), "ssa_align_loss"));
    return launch_loss(*p, sqdiff, w_s, w_c, loss_out, ws, static_cast<cudaStream_t>(stream));
}

int ssa_attn_bwd(const ssa_params_t* p, const void* q, const void* k, const void* v,
                 const int32_t* idx, const int32_t* cnt, const uint32_t* mask,
                 const void* h_full, const void* h_sparse, const float* lse_full,
                 const float* lse_sparse, const void* dh_full, const void* dh_sparse,
                 float w_s, float w_c, void* dq, void* dk, void* dv, void* ws,
                 size_t ws_bytes, void* stream) {
    g_last_error[0] = 0;
    SSA_TRY(validate(p));
    SSA_TRY(need_ptr(q, "q"));
    SSA_TRY(need_ptr(k, "k"));
    SSA_TRY(need_ptr(v, "v"));
    SSA_TRY(opt_ptr(idx, "idx"));
    SSA_TRY(opt_ptr(cnt, "cnt"));
    SSA_TRY(need_ptr(mask, "mask"));
    SSA_TRY(need_ptr(h_full, "h_full"));
    SSA_TRY(need_ptr(h_sparse, "h_sparse"));
    SSA_TRY(need_ptr(lse_full, "lse_full"));
    SSA_TRY(need_ptr(lse_sparse, "lse_sparse"));
    SSA_TRY(opt_ptr(dh_full, "dh_full"));
    SSA_TRY(opt_ptr(dh_sparse, "dh_sparse"));
    SSA_TRY(need_ptr(dq, "dq"));
    SSA_TRY(need_ptr(dk, "dk"));
    SSA_TRY(need_ptr(dv, "dv"));
    if (!std::isfinite(w_s) || !std::isfinite(w_c))
        return fail(SSA_ERR_INVALID_ARG, "loss weights must be finite");
    SSA_TRY(need_ws(ws, ws_bytes, bwd_workspace(*p), "ssa_attn_bwd"));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (use_tc(*p))
        return launch_bwd_tc(*p, q, k, v, mask, h_full, h_sparse, lse_full, lse_sparse, dh_full,
                             dh_sparse, w_s, w_c, dq, dk, dv, ws, s);
    return launch_bwd_simt(*p, q, k, v, mask, h_full, h_sparse, lse_full, lse_sparse, dh_full,
                           dh_sparse, w_s, w_c, dq, dk, dv, ws, s);
}

int ssa_device_status(void* stream) {
    g_last_error[0] = 0;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return fail(SSA_ERR_CUDA, "stream: %s", cudaGetErrorString(e));
    int st = fwd_tc_take_status(s);
    if (st == SSA_OK) st = bwd_tc_take_status(s);
    if (st == SSA_OK) st = selftest_take_status();
    if (st == SSA_OK) st = decode_take_status();
    if (st == SSA_OK) st = select_take_status();
    if (st != SSA_OK) return st;
    return check_launch("pending");
}

const char* ssa_status_string(int status) {
    switch (status) {
        case SSA_OK: return "ok";
        case SSA_ERR_INVALID_ARG: return "invalid argument";
        case SSA_ERR_UNSUPPORTED: return "unsupported configuration";
        case SSA_ERR_WORKSPACE: return "workspace too small or missing";
        case SSA_ERR_CUDA: return "CUDA error";
        case SSA_ERR_TIMEOUT: return "device wait timed out";
        default: return "unknown status";
    }
}

const char* ssa_last_error(void) { return g_last_error; }

int ssa_kernel_path(const ssa_params_t* p) {
    if (validate(p) != SSA_OK) return -1;
    return use_tc(*p) ? 1 : 0;
}

int ssa_version(void) { return (1 << 16) | 0; }

int ssa_bwd_heads_per_group(const ssa_params_t* p) {
    if (validate(p) != SSA_OK || !use_tc(*p)) return -1;
    return ssa::bwd_tc_heads_per_group(*p);
}

void ssa_debug_set_wait_limit_ns(unsigned long long ns) {
    g_wait_limit_ns.store(ns ? ns : kDefaultWaitLimitNs, std::memory_order_relaxed);
}

void ssa_debug_set_ds_budget_bytes(unsigned long long bytes) {
    g_ds_budget.store(bytes ? bytes : kDefaultDsBudget, std::memory_order_relaxed);
}

int ssa_debug_set_kernel_events(void* const* events, int n) {
    if (n == 0) {
        for (auto& e : ssa::g_kernel_events) e.store(nullptr, std::memory_order_relaxed);
        return SSA_OK;
    }
    if (n != ssa::kKernelEvents || !events) return ssa::fail(SSA_ERR_INVALID_ARG, "need %d events", ssa::kKernelEvents);
    for (int i = 0; i < n; ++i)
        ssa::g_kernel_events[i].store(events[i], std::memory_order_relaxed);
    return SSA_OK;
}

}  // extern "C"
