/*
 * ssa.h -- C ABI of libssa: the per-layer dual-stream causal attention of
 * SSA ("SSA: Sparse Sparse Attention by Aligning Full and Sparse Attention
 * Outputs in Feature Space", arXiv 2511.20102) on NVIDIA B200 (sm_100a).
 *
 * For one layer and the same Q, K, V the library computes
 *   - the full-attention output h_full (causal softmax over every past token),
 *   - the block-sparse output h_sparse (softmax over the selected key blocks
 *     only; the sparse stream normalises over its own subset),
 *   - the discarded attention mass delta(t) (full-softmax weight on keys the
 *     sparse rule did not select),
 *   - the alignment losses L_sparsity and L_commit,
 *   - and the backward pass through both streams.
 * Sources: gist.science technical summaries of the paper (Italian
 * "Sintesi Tecnica", French "Resume technique"), section 1 (problem
 * statement: normalisation over the selected subset, error linear in the
 * discarded mass), section 2 (methodology: sparse and full streams,
 * counterpart output computed only for alignment, L_sparsity and L_commit,
 * total objective E_mode[L_ce] + alpha L_align), section 4 ("Efficienza":
 * inference runs the same operations as MoBA).
 *
 * Conventions for every entry point
 *   - Tensors are row-major contiguous [B, H, T, D] (q, k, v, h_*, dh_*, d*),
 *     in the element type given by params->dtype.  Row statistics (delta,
 *     lse_*, sqdiff_rows) are float32 [B, H, T].  Selection outputs are
 *     idx int32 [B, H, n, topk], cnt int32 [B, H, n] and mask uint32
 *     [B, H, n, ceil(n/32)] with n = T / block.
 *   - Every pointer except `params` is DEVICE memory owned by the caller.
 *     The library allocates nothing.  Scratch memory is passed as `ws`
 *     (device, 256-byte aligned) of at least ssa_workspace_size(...) bytes;
 *     it may be NULL when that size is 0.  The library keeps no pointer
 *     after a call returns.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream).  Argument errors are returned synchronously before
 *     anything is launched; launch errors return SSA_ERR_CUDA.  A kernel
 *     whose bounded wait expired records SSA_ERR_TIMEOUT in a device status
 *     word that ssa_device_status() reports after synchronising; the outputs
 *     of the calls made since the last check are then undefined (nothing
 *     outside their outputs and workspaces is written, and later calls run
 *     normally).
 *   - Alignment: every device pointer 16-byte aligned; the bf16 tensor-core
 *     path takes D == 64 or 128.
 */
#ifndef SSA_H
#define SSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SSA_OK = 0,
    SSA_ERR_INVALID_ARG = -1, /* null pointer, bad shape, misaligned pointer */
    SSA_ERR_UNSUPPORTED = -2, /* valid but not implemented (dtype/D/block)   */
    SSA_ERR_WORKSPACE = -3,   /* ws smaller than ssa_workspace_size()        */
    SSA_ERR_CUDA = -4,        /* a CUDA runtime call or launch failed         */
    SSA_ERR_TIMEOUT = -5      /* a device-side bounded wait gave up           */
} ssa_status_t;

typedef enum { SSA_F32 = 0, SSA_BF16 = 1 } ssa_dtype_t;

/* SSA_FLAG_FORCE_SINK: block 0 (the "sink") is always selected; it counts
 * inside topk.
 * SSA_FLAG_FORCE_SIMT: run the CUDA-core (SIMT) kernels even where the
 * tcgen05 tensor-core kernels apply; a slower comparator with the same
 * results up to float32 rounding order. */
enum { SSA_FLAG_FORCE_SINK = 1u, SSA_FLAG_FORCE_SIMT = 2u };

/*
 * Layer shape and method parameters.
 *   B, H, T, D : batch, heads, tokens, head dim.  T % block == 0.
 *                D in {64, 128}.
 *   block      : tokens per query block and per key block, 64 or 128.
 *   topk       : selected key blocks per query block, counting the always
 *                selected current block (and block 0 under FORCE_SINK);
 *                1 <= topk <= n, topk >= 2 with FORCE_SINK.
 *   dtype      : ssa_dtype_t of every [B,H,T,D] tensor.
 *   sm_scale   : softmax scale sigma (logit = sigma * q.k), > 0.
 *   flags      : OR of SSA_FLAG_*.
 */
typedef struct {
    int B, H, T, D, block, topk;
    int dtype;
    float sm_scale;
    unsigned flags;
} ssa_params_t;

enum {
    SSA_WS_SELECT = 0,
    SSA_WS_FWD = 1,
    SSA_WS_LOSS = 2,
    SSA_WS_BWD = 3,
    SSA_WS_FWD_SPARSE = 4,
    SSA_WS_DECODE = 5
};

/* Bytes of scratch the named entry point needs for these params (0 if none,
 * (size_t)-1 if the params are invalid). */
size_t ssa_workspace_size(const ssa_params_t* params, int which);

/*
 * Block selection of the sparse stream (section 2, "Sparse Attention
 * Stream": block-sparse attention; section 4: MoBA-identical operations).
 * Per (b, h, query block i):
 *   Qbar_i = mean of q over block i, Kbar_j = mean of k over block j,
 *   score s_ij = Qbar_i . Kbar_j, formed in float64 (block sums are exact);
 *   S_i = {i} (plus {0} under FORCE_SINK) and the best topk - |forced|
 *   blocks j < i by (score descending, j ascending), or all j < i if fewer.
 * Writes idx (S_i ascending, -1 padded), cnt (|S_i|) and mask (bit j%32 of
 * word j/32 set iff j in S_i).  Workspace: SSA_WS_SELECT.
 */
int ssa_select_blocks(const ssa_params_t* params, const void* q, const void* k,
                      int32_t* idx, int32_t* cnt, uint32_t* mask,
                      void* ws, size_t ws_bytes, void* stream);

/*
 * ssa_select_blocks without a workspace argument, for callers that cannot
 * allocate device memory where they run selection (for example a plugin
 * inside a serving process whose memory pool owns all device memory, or a
 * latency-critical loop that must not call cudaMalloc after start-up).  The
 * paper has no counterpart; this is a packaging variant of the call above
 * with identical results.
 *   - Scratch comes from a 16 MiB array in the library's own device memory,
 *     held by every GPU that loads the library until the process exits.
 *     Shapes needing more (B*H*(T/block)*D > 1,048,576) are rejected with
 *     SSA_ERR_UNSUPPORTED before anything is launched.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture begins.  The address is cached per CUDA
 *     context: after a cudaDeviceReset the first call in the new context
 *     looks it up again (so it too should come before any capture).
 *   - All calls share the one array: calls that overlap on the GPU (other
 *     streams, other host threads) race and give undefined results; order
 *     them on one stream.  Nothing in the array needs clearing between calls.
 */
int ssa_select_blocks_noalloc(const ssa_params_t* params, const void* q, const void* k,
                              int32_t* idx, int32_t* cnt, uint32_t* mask, void* stream);

/*
 * Both attention streams in one pass over K/V (section 2: the full stream
 * and the counterpart sparse output of the same layer).  For query t in
 * block i, keys s <= t, x = sm_scale * q_t . k_s, sel(t,s) = block(s) in S_i
 * (read from `mask`; idx/cnt may be NULL and are not read):
 *   h_full   = sum_s e^x v_s / sum_s e^x
 *   h_sparse = sum_{sel} e^x v_s / sum_{sel} e^x
 *   delta    = sum_{not sel} e^x / sum_s e^x
 *   lse_full = log sum_s e^x,   lse_sparse = log sum_{sel} e^x
 *   sqdiff_rows[t] = sum_c (h_full - h_sparse)_c^2 from the float32 values
 *                    before rounding to dtype.
 * Accumulation is float32.  Workspace: SSA_WS_FWD.
 */
int ssa_attn_fwd_dual(const ssa_params_t* params, const void* q, const void* k,
                      const void* v, const int32_t* idx, const int32_t* cnt,
                      const uint32_t* mask, void* h_full, void* h_sparse,
                      float* delta, float* lse_full, float* lse_sparse,
                      float* sqdiff_rows, void* ws, size_t ws_bytes, void* stream);

/*
 * The sparse stream alone, as run at inference (section 4, "Efficienza":
 * at inference SSA runs the same operations as MoBA).  For query t in block
 * i and the keys s <= t whose block is in S_i (read from `mask`; idx/cnt
 * may be NULL and are not read), x = sm_scale * q_t . k_s:
 *   h_sparse = sum_{sel} e^x v_s / sum_{sel} e^x,  lse_sparse = log sum_{sel} e^x
 * — the same quantities as ssa_attn_fwd_dual's, from a kernel that visits
 * only the selected key blocks (work proportional to the selected pairs).
 * h_sparse is [B,H,T,D] in dtype, lse_sparse [B,H,T] float32.  Workspace:
 * SSA_WS_FWD_SPARSE (0 on the tensor-core path; the CUDA-core path runs the
 * dual kernel and keeps the full-stream outputs there).
 */
int ssa_attn_fwd_sparse(const ssa_params_t* params, const void* q, const void* k,
                        const void* v, const int32_t* idx, const int32_t* cnt,
                        const uint32_t* mask, void* h_sparse, float* lse_sparse,
                        void* ws, size_t ws_bytes, void* stream);

/*
 * Decoding over a key/value cache (section 4, "Efficienza": at inference SSA
 * runs MoBA's operations; the pages do not describe decoding itself, and the
 * rule below is MoBA's).  params->T is the cache capacity (a multiple of
 * block); k_cache, v_cache are [B,H,T,D] in dtype, keys 0..t valid; D is 64
 * or 128 and topk <= 64 here.
 *
 * ssa_decode_pool: kbar[b,h,j,:] = mean of the keys of block j, float64, for
 *   j0 <= j < j1 (call it once a block is complete; kbar is [B,H,T/block,D]).
 * ssa_decode_step: one step at position t.  i = t / block; the current query
 *   q_t ([B,H,D]) is scored against kbar_j of the completed blocks j < i in
 *   float64; S = {i} (+ {0} with SSA_FLAG_FORCE_SINK), plus the best-scoring
 *   completed blocks (ties to the lower index) up to topk places in all (all
 *   of them when there are fewer); then h = softmax attention of q_t over
 *   every key of S that is <= t ([B,H,D] in dtype) and lse its log-sum-exp
 *   (float32 [B,H]).  idx, if not NULL, receives S ascending, -1 padded
 *   ([B,H,topk] int32).  kbar must hold blocks 0..i-1.  Workspace:
 *   SSA_WS_DECODE (0 bytes: the step runs as one launch of a cluster of 4 or
 *   8 CTAs per head whose hand-offs stay in shared memory; the argument is
 *   kept so that callers need no change if a later version needs scratch).
 *   k_cache and v_cache must be 16-byte aligned (the selected blocks are
 *   copied with bulk copies).  A bulk copy or a hand-off that does not
 *   complete within the wait limit makes ssa_device_status return
 *   SSA_ERR_TIMEOUT; h and lse of the heads concerned are then undefined
 *   (left unwritten, or formed without the blocks whose copies expired; idx
 *   is still exact), and the launch still ends only after every CTA of each
 *   cluster has stopped writing into the others' shared memory.
 */
int ssa_decode_pool(const ssa_params_t* params, int j0, int j1, const void* k_cache,
                    double* kbar, void* stream);
int ssa_decode_step(const ssa_params_t* params, int t, const void* q, const void* k_cache,
                    const void* v_cache, const double* kbar, void* h, float* lse, int32_t* idx,
                    void* ws, size_t ws_bytes, void* stream);

/*
 * Attention diagnostics, from the dual forward's lse_full and delta for the
 * same q, k.  The sparse approximation error grows with the discarded mass
 * delta ("Sintesi Tecnica: SSA", section 1); the paper's abstract (the
 * chatpaper.ai summary and the arXiv 2511.20102 listing, "Abstract") ties
 * long-context extrapolation to too much attention going to sink areas, the
 * first block here, and discusses how sparse learned attention is:
 *   sink_rows[t]  = sum_{s <= t, s < block} exp(sm_scale q_t . k_s - lse_full(t))
 *                   (full-softmax mass on block 0), float32 [B,H,T];
 *   head_stats    = float32 [B,H,2]: mean over t of delta, mean over t of sink.
 * The means are fixed-order float64 sums (bitwise repeatable).  No workspace.
 */
int ssa_attn_diagnostics(const ssa_params_t* params, const void* q, const void* k,
                         const float* lse_full, const float* delta, float* sink_rows,
                         float* head_stats, void* stream);

/*
 * ssa_attn_fwd_dual and ssa_attn_diagnostics in one call: the same outputs
 * as the first (same arguments and workspace, SSA_WS_FWD) plus sink_rows and
 * head_stats as the second defines them.  On the tensor-core path the
 * forward kernel accumulates each row's weight on block 0 while it walks key
 * tile 0 (rescaled with the running max like the row sums) and divides by
 * the full normaliser at the end, so q and block 0 of k are not read again;
 * one small kernel then forms the per-head means.  On the CUDA-core path it
 * runs the two calls one after the other.
 */
int ssa_attn_fwd_dual_diag(const ssa_params_t* params, const void* q, const void* k,
                           const void* v, const int32_t* idx, const int32_t* cnt,
                           const uint32_t* mask, void* h_full, void* h_sparse, float* delta,
                           float* lse_full, float* lse_sparse, float* sqdiff_rows,
                           float* sink_rows, float* head_stats, void* ws, size_t ws_bytes,
                           void* stream);

/*
 * Alignment losses (section 2, "Allineamento Bidirezionale"): with
 * N = B*H*T*D and L = sum(sqdiff_rows) / N (the mean squared difference of
 * the two outputs), writes loss_out[0] = w_sparsity * L (L_sparsity) and
 * loss_out[1] = w_commit * L (L_commit), float32, device memory.  The sum
 * is a fixed-order float64 reduction: repeated calls give identical bits.
 * Workspace: SSA_WS_LOSS.
 */
int ssa_align_loss(const ssa_params_t* params, const float* sqdiff_rows,
                   float w_sparsity, float w_commit, float* loss_out,
                   void* ws, size_t ws_bytes, void* stream);

/*
 * Backward of  <dh_full, h_full> + <dh_sparse, h_sparse>
 *            + w_sparsity * L_sparsity + w_commit * L_commit
 * with respect to q, k, v; L_sparsity reaches h_full only and L_commit
 * h_sparse only (stop-gradient on the opposite stream); no gradient flows
 * through selection or delta.  The full stream carries gradient to every
 * causal key (section 2, "Full Attention Stream").  h_full, h_sparse,
 * lse_full and lse_sparse are the forward's outputs for the same inputs.
 * dh_full / dh_sparse may be NULL (read as zero).  dq, dk, dv are written
 * (not accumulated).  Workspace: SSA_WS_BWD; on the tensor-core path it
 * holds the bf16 dS blocks of the causal triangle for up to 4 GiB worth of
 * (batch, head) pairs at a time (about 2 * T^2 / 2 bytes per pair), so long
 * sequences are processed a group of heads at a time.
 */
int ssa_attn_bwd(const ssa_params_t* params, const void* q, const void* k,
                 const void* v, const int32_t* idx, const int32_t* cnt,
                 const uint32_t* mask, const void* h_full, const void* h_sparse,
                 const float* lse_full, const float* lse_sparse,
                 const void* dh_full, const void* dh_sparse,
                 float w_sparsity, float w_commit,
                 void* dq, void* dk, void* dv,
                 void* ws, size_t ws_bytes, void* stream);

/* Synchronises `stream`, then returns SSA_ERR_TIMEOUT if any kernel since the
 * previous call recorded an expired wait (and clears the record), else
 * SSA_ERR_CUDA on a pending CUDA error, else SSA_OK. */
int ssa_device_status(void* stream);

/* Static text for a status code. */
const char* ssa_status_string(int status);

/* Detail of the last error returned on the calling host thread ("" if none). */
const char* ssa_last_error(void);

/* Heads per group of the tensor-core backward (the dS workspace holds one
 * group; the groups run one after another; B*H when all fit), or -1 when
 * the params are invalid or select the CUDA-core path. */
int ssa_bwd_heads_per_group(const ssa_params_t* params);

/* Which kernel family the params select: 0 = CUDA-core (SIMT) kernels
 * (float32, or SSA_FLAG_FORCE_SIMT), 1 = bf16 tcgen05 tensor-core kernels
 * (D = 64 or 128), -1 = invalid or unsupported params. */
int ssa_kernel_path(const ssa_params_t* params);

/* Self-test of the element-wise arithmetic inside the tensor-core kernels
 * (not part of the method; for tests).  For n device floats x, writes the
 * FMA-pipe polynomial 2^x, the MUFU 2^x and the bf16 bit patterns produced
 * by the integer-ALU packing, each exactly as the kernels compute them. */
int ssa_selftest_math(const float* x, int n, float* exp2_poly, float* exp2_mufu,
                      uint16_t* bf16_alu, void* stream);

/* Self-test of the bounded wait the tensor-core kernels use for every
 * mbarrier (not part of the method; for tests): one thread waits on an
 * mbarrier that nothing ever arrives at.  The wait gives up after limit_ns
 * (1 ns .. 10 s), *gave_up (device int) is set to 1 and the expiry is
 * recorded, so the next ssa_device_status returns SSA_ERR_TIMEOUT. */
int ssa_selftest_wait_timeout(unsigned long long limit_ns, int* gave_up, void* stream);

/* Test hook: wall-clock limit of every bounded wait inside the tensor-core
 * kernels, in nanoseconds, for launches made after the call (0 restores the
 * default of 2 s).  A wait that runs past it makes the kernel stop, let
 * copies and MMAs in flight land, free TMEM and return; ssa_device_status
 * then reports SSA_ERR_TIMEOUT and the outputs of that call are undefined.
 * Process-wide; not synchronised with calls running on other threads. */
void ssa_debug_set_wait_limit_ns(unsigned long long ns);

/* Test hook: byte budget of the tensor-core backward's dS workspace, which
 * sets how many heads form one group (ssa_bwd_heads_per_group: the largest
 * count whose dS blocks fit, at least 1).  0 restores the default of 4 GiB.
 * Affects ssa_workspace_size(SSA_WS_BWD), ssa_bwd_heads_per_group and
 * ssa_attn_bwd calls made after it, so a caller sizes the workspace after
 * setting it.  A smaller budget makes small problems run the grouped path
 * (several launches of the dK/dV kernel and the dQ GEMM, one per group)
 * that otherwise only very long sequences reach.  Process-wide, like the
 * hook above. */
void ssa_debug_set_ds_budget_bytes(unsigned long long bytes);

/* Measurement hook: makes later ssa_attn_bwd calls on the tensor-core path
 * record the caller's CUDA events (cudaEvent_t, passed as void*) on the call's
 * stream at kernel boundaries: events[0] before the preprocess kernel,
 * events[1] after it, events[2] after the dK/dV kernel and events[3] after
 * the dQ GEMM of the first group of heads (ssa_bwd_heads_per_group; the
 * only group unless the dS buffer is split).  n must be 4 to enable, 0 to disable; the events stay
 * owned by the caller, who must disable the hook before destroying them.
 * Returns SSA_OK or SSA_ERR_INVALID_ARG.  Process-wide, like the hook above. */
int ssa_debug_set_kernel_events(void* const* events, int n);

/* ABI version, (major << 16) | minor. */
int ssa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SSA_H */
