// Internal declarations shared by the host-side translation units of libssa.
// Kernels live in their own .cu files; each exposes one host launcher here.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stddef.h>
#include <stdint.h>

#include <mutex>

#include "ssa.h"

namespace ssa {

// Records a detail message for ssa_last_error() and returns `status`.
int fail(int status, const char* fmt, ...);

// Turns a pending launch/runtime error into SSA_ERR_CUDA (with detail).
int check_launch(const char* what);

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Shared memory a CTA may hold on sm_100 (227 KB).
constexpr size_t kMaxSmemPerCta = 232448;

// Lets kernel K take dynamic shared memory up to the per-CTA maximum less its
// static shared memory (once per process; launches above the default 48 KB
// of dynamic plus static shared memory fail without it).  Call it before any
// stream capture.  Returns an SSA status; *dyn_limit receives the limit.
template <auto K>
int opt_in_max_smem(const char* what, size_t* dyn_limit = nullptr) {
    static std::once_flag once;
    static cudaError_t err = cudaSuccess;
    static size_t limit = 0;
    std::call_once(once, [] {
        cudaFuncAttributes fa;
        err = cudaFuncGetAttributes(&fa, K);
        if (err == cudaSuccess) {
            limit = kMaxSmemPerCta - fa.sharedSizeBytes;
            err = cudaFuncSetAttribute(K, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)limit);
        }
    });
    if (dyn_limit) *dyn_limit = limit;
    if (err != cudaSuccess) return fail(SSA_ERR_CUDA, "%s: shared memory attribute: %s", what, cudaGetErrorString(err));
    return SSA_OK;
}

// Wall-clock limit of the kernels' bounded waits (default 2 s; tests shorten it).
unsigned long long wait_limit_ns();

// Byte budget of the tensor-core backward's dS workspace (default 4 GiB;
// tests shrink it so that small problems run in several head groups).
unsigned long long ds_budget_bytes();

// Measurement hook (ssa_debug_set_kernel_events): records caller event i on
// stream s when the hook is enabled, else does nothing.
constexpr int kKernelEvents = 4;
void mark_kernel_event(int i, cudaStream_t s);

inline size_t num_rows(const ssa_params_t& p) {
    return (size_t)p.B * p.H * p.T;
}
inline size_t num_elems(const ssa_params_t& p) { return num_rows(p) * p.D; }
inline int num_blocks(const ssa_params_t& p) { return p.T / p.block; }
inline int mask_words(const ssa_params_t& p) { return (num_blocks(p) + 31) / 32; }

// ---- selection (select.cu)
size_t select_workspace(const ssa_params_t& p);
int launch_select(const ssa_params_t& p, const void* q, const void* k, int32_t* idx,
                  int32_t* cnt, uint32_t* mask, void* ws, cudaStream_t s);

// ---- forward, CUDA-core path (fwd_simt.cu)
int launch_fwd_simt(const ssa_params_t& p, const void* q, const void* k, const void* v,
                    const uint32_t* mask, void* h_full, void* h_sparse, float* delta,
                    float* lse_full, float* lse_sparse, float* sqdiff, cudaStream_t s);

// ---- forward, tcgen05 path (fwd_tc.cu)
bool fwd_tc_supported(const ssa_params_t& p);
size_t fwd_tc_workspace(const ssa_params_t& p);
int launch_fwd_tc(const ssa_params_t& p, const void* q, const void* k, const void* v,
                  const uint32_t* mask, void* h_full, void* h_sparse, float* delta,
                  float* lse_full, float* lse_sparse, float* sqdiff, float* sink, void* ws,
                  cudaStream_t s);  // sink: optional block-0 mass per row
int fwd_tc_take_status(cudaStream_t s);  // SSA_ERR_TIMEOUT if a wait expired
// the sparse stream alone (inference): h_sparse and lse_sparse only
int launch_fwd_sparse_tc(const ssa_params_t& p, const void* q, const void* k, const void* v,
                         const uint32_t* mask, void* h_sparse, float* lse_sparse, cudaStream_t s);

// ---- decode over a key/value cache (decode.cu)
size_t decode_workspace(const ssa_params_t& p);
int launch_decode_pool(const ssa_params_t& p, int j0, int j1, const void* k, double* kbar,
                       cudaStream_t s);
int launch_decode_step(const ssa_params_t& p, int t, const void* q, const void* k, const void* v,
                       const double* kbar, void* h, float* lse, int32_t* idx, void* ws,
                       cudaStream_t s);

// ---- attention diagnostics (diag.cu)
int launch_diagnostics(const ssa_params_t& p, const void* q, const void* k, const float* lse_full,
                       const float* delta, float* sink, float* stats, cudaStream_t s);
// per-head means of delta and of the sink mass from the row vectors (fixed-order float64)
int launch_diag_heads(const ssa_params_t& p, const float* delta, const float* sink, float* stats,
                      cudaStream_t s);

// ---- alignment loss (loss.cu)
size_t loss_workspace(const ssa_params_t& p);
int launch_loss(const ssa_params_t& p, const float* sqdiff, float w_s, float w_c,
                float* loss_out, void* ws, cudaStream_t s);

// ---- backward, CUDA-core path (bwd_simt.cu)
size_t bwd_simt_workspace(const ssa_params_t& p);
int launch_bwd_simt(const ssa_params_t& p, const void* q, const void* k, const void* v,
                    const uint32_t* mask, const void* h_full, const void* h_sparse,
                    const float* lse_full, const float* lse_sparse, const void* dh_full,
                    const void* dh_sparse, float w_s, float w_c, void* dq, void* dk,
                    void* dv, void* ws, cudaStream_t s);

// ---- backward, tcgen05 path (bwd_tc.cu)
bool bwd_tc_supported(const ssa_params_t& p);
size_t bwd_tc_workspace(const ssa_params_t& p);
int launch_bwd_tc(const ssa_params_t& p, const void* q, const void* k, const void* v,
                  const uint32_t* mask, const void* h_full, const void* h_sparse,
                  const float* lse_full, const float* lse_sparse, const void* dh_full,
                  const void* dh_sparse, float w_s, float w_c, void* dq, void* dk, void* dv,
                  void* ws, cudaStream_t s);
int bwd_tc_take_status(cudaStream_t s);  // SSA_ERR_TIMEOUT if a wait expired
int bwd_tc_heads_per_group(const ssa_params_t& p);  // heads sharing the dS workspace

// ---- self-tests (selftest.cu)
int select_take_status();  // SSA_ERR_TIMEOUT if a pooling wait expired
int decode_take_status();  // SSA_ERR_TIMEOUT if a decode-step wait expired
int selftest_take_status();  // SSA_ERR_TIMEOUT if the self-test wait expired

}  // namespace ssa
