// Backward through both SSA attention streams on the sm_100a tensor cores
// (bf16 operands, fp32 accumulate, head dim 128).
//
// Math ("Sintesi Tecnica: SSA", section 2: the full stream carries gradient
// to every token; L_sparsity and L_commit with stop-gradient on the opposite
// stream).  For query t, key s <= t, x = sigma q_t.k_s:
//   P_f = exp(x - lse_full(t));  P_s = c_t P_f on selected (t,s), else 0,
//   with c_t = exp(lse_full(t) - lse_sparse(t)) (the sparse stream's own
//   normaliser);
//   dS  = P_f (G_f(t).v_s - D_f(t)) + P_s (G_s(t).v_s - D_s(t))
//   dv_s = sum_t P_f G_f(t) + P_s G_s(t),  dk_s = sigma sum_t dS q_t,
//   dq_t = sigma sum_s dS k_s,
// where G_f, G_s are the upstream gradients of h_full, h_sparse plus the
// alignment terms and D_f = G_f.h_full, D_s = G_s.h_sparse.  Since P_s = c_t P_f
// on selected pairs, the kernels use G_s' = c_t G_s and D_s' = c_t D_s:
//   dS = P_f (G_f.v - D_f + sel (G_s'.v - D_s')),  dv_s += P_f (G_f + sel G_s'),
// so c_t never appears past the preprocess and P_s^T is P_f^T with the
// unselected key rows zeroed.
//
// Three kernels, no atomics (bitwise repeatable):
//   bwd_tc_pre_kernel   one warp per row: G_f, G_s' rounded to bf16, D_f and
//                       D_s' from the rounded values, lse_full*log2(e)
//                       (the three scalars stored negated).
//   bwd_dkdv_tc_kernel  CTA = 128 keys of one head; steps of 64 queries.
//                       K and V are copied into TMEM once; per step
//                       S^T = K Q^T and dP_f^T = V G_f^T (TS, N = 64), and
//                       dP_s^T = V G_s'^T on steps the sparse stream
//                       touches.  The compute warpgroups form P_f^T (bf16,
//                       back into TMEM, plus a row-masked copy for the sparse
//                       stream on mixed steps) and dS^T (bf16, to a swizzled
//                       shared-memory tile); then dV += P_f^T G_f + P_s^T G_s'
//                       (TS) and dK += dS^T Q (SS).  Warp 2 stores each dS^T
//                       tile to the workspace by TMA.
//                       TMEM: dV | dK | K | V | S range | dP_f^T = 512 cols.
//   bwd_dq_gemm_kernel  dQ = sigma dS K over the stored dS^T blocks: CTA =
//                       128 queries of one head, a 3-stage TMA ring of two
//                       dS^T blocks and a key tile per stage, the
//                       accumulator in 128 TMEM columns.
// The sparse-stream MMAs are skipped on steps where no (query block, key
// block) pair is selected.  Every wait is bounded; an expiry sets a device
// status word and the CTA drains its tensor-core work and frees TMEM.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "ssa_internal.h"
#include "tc_util.cuh"

namespace ssa {
namespace {

using namespace tc;

constexpr int TILE = 128;  // keys per dK/dV CTA, queries per dQ CTA
constexpr int STEP = 64;   // queries per dK/dV step, keys per dQ step
constexpr uint32_t BOX_T = TILE * 128;  // [128 rows x 64 d] bf16 = 16 KB (head dims 64, 128: 1 or 2 boxes)
constexpr uint32_t BOX_S = STEP * 128;  // [64 rows x 64 d] bf16 = 8 KB
constexpr uint32_t TILE_BYTES = 2 * BOX_T;
constexpr uint32_t STEP_BYTES = 2 * BOX_S;
constexpr float kLog2e = 1.4426950408889634f;

__device__ unsigned int g_bwd_tc_status;

struct BwdArgs {
    __nv_bfloat16* dq;
    __nv_bfloat16* dk;
    __nv_bfloat16* dv;
    const float* neg_lse2;  // -lse_full * log2(e)
    const float* neg_Df;    // -D_f
    const float* neg_Ds;    // -D_s of the c_t-scaled G_s
    const uint32_t* mask;
    int BH, T, block, words, n_blocks;
    int ds_blocks;  // dS^T blocks per (batch, head): one per (key tile, 64-query step)
    float scale_log2;  // sigma * log2(e)
    float sm_scale;
    unsigned long long timeout_ns;
};

__device__ __forceinline__ bool bit(const uint32_t* row, int j) {
    return (row[j >> 5] >> (j & 31)) & 1u;
}

__device__ __forceinline__ bool wait_drain(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(bar, parity))
        if (globaltimer() - t0 > limit_ns) return false;
    return true;
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(dst), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
        : "memory");
}

// ============================================================ preprocess
// One warp per row, lane owns D/32 consecutive columns.
template <int D>
__global__ void __launch_bounds__(256)
bwd_tc_pre_kernel(const __nv_bfloat16* __restrict__ hf, const __nv_bfloat16* __restrict__ hs,
                  const __nv_bfloat16* __restrict__ dhf, const __nv_bfloat16* __restrict__ dhs,
                  const float* __restrict__ lse_f, const float* __restrict__ lse_s, size_t rows,
                  float cf, float cs, __nv_bfloat16* __restrict__ gf, __nv_bfloat16* __restrict__ gs,
                  float* __restrict__ neg_lse2, float* __restrict__ neg_Df,
                  float* __restrict__ neg_Ds) {
    constexpr int NP = D / 64;  // bf16 pairs per lane
    const size_t row = (size_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const size_t e = row * D + 2 * NP * lane;
    auto ld = [](const __nv_bfloat16* p, float (&o)[2 * NP]) {
#pragma unroll
        for (int i = 0; i < NP; ++i) {
            const __nv_bfloat162 x = reinterpret_cast<const __nv_bfloat162*>(p)[i];
            o[2 * i] = __low2float(x);
            o[2 * i + 1] = __high2float(x);
        }
    };
    // c_t = exp(lse_full - lse_sparse) carries P_f to P_s on selected pairs; it is
    // folded into G_s here (0 where the sparse stream has no mass)
    const float lf = lse_f[row], ls = lse_s[row];
    const float c = ls > -INFINITY ? expf(lf - ls) : 0.f;
    float f[2 * NP], s[2 * NP], uf[2 * NP], us[2 * NP];
#pragma unroll
    for (int i = 0; i < 2 * NP; ++i) uf[i] = us[i] = 0.f;
    ld(hf + e, f);
    ld(hs + e, s);
    if (dhf) ld(dhf + e, uf);
    if (dhs) ld(dhs + e, us);
    float sf = 0.f, ss = 0.f;
    uint32_t pf[NP], ps[NP];
#pragma unroll
    for (int i = 0; i < NP; ++i) {
        const float gf0 = uf[2 * i] + cf * (f[2 * i] - s[2 * i]);
        const float gf1 = uf[2 * i + 1] + cf * (f[2 * i + 1] - s[2 * i + 1]);
        const float gs0 = c * (us[2 * i] + cs * (s[2 * i] - f[2 * i]));
        const float gs1 = c * (us[2 * i + 1] + cs * (s[2 * i + 1] - f[2 * i + 1]));
        pf[i] = pack_bf16(gf0, gf1);
        ps[i] = pack_bf16(gs0, gs1);
        // D from the rounded values the tensor cores will see
        const __nv_bfloat162 rf = *reinterpret_cast<__nv_bfloat162*>(&pf[i]);
        const __nv_bfloat162 rs = *reinterpret_cast<__nv_bfloat162*>(&ps[i]);
        sf = fmaf(__low2float(rf), f[2 * i], fmaf(__high2float(rf), f[2 * i + 1], sf));
        ss = fmaf(__low2float(rs), s[2 * i], fmaf(__high2float(rs), s[2 * i + 1], ss));
    }
#pragma unroll
    for (int i = 0; i < NP; ++i) {
        reinterpret_cast<uint32_t*>(gf + e)[i] = pf[i];
        reinterpret_cast<uint32_t*>(gs + e)[i] = ps[i];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        sf += __shfl_xor_sync(0xffffffffu, sf, o);
        ss += __shfl_xor_sync(0xffffffffu, ss, o);
    }
    if (lane == 0) {  // negated: the consumers add them
        neg_lse2[row] = -(lf * kLog2e);
        neg_Df[row] = -sf;
        neg_Ds[row] = -ss;
    }
}

// ============================================================ dK / dV
#ifndef SSA_KV_POLY_PAIRS
#define SSA_KV_POLY_PAIRS 0
#endif
#ifndef SSA_KV_PACK_CVT
#define SSA_KV_PACK_CVT 0
#endif
namespace kv {
// K and V of the tile live in TMEM: the A operands of S^T = K Q^T and
// dP^T = V G^T (TS form: only the 64-query B tiles are read from shared
// memory).  Q, G_f, G_s' steps stream through a ring.  The S range holds S^T
// and then, on sparse steps, dP_s^T; once the compute warps have read them
// the next step's S^T goes there.  The dP range holds dP_f^T and then the
// bf16 P^T that feeds dV += P^T G_f (+ the sparse stream's row-masked copy
// next to it on mixed steps); the next step's dP_f^T is issued behind the dV
// MMAs, and is needed only after the next step's exponentials.  dS^T goes
// to a double-buffered swizzled shared tile: the A operand of dK += dS^T Q
// and the source of its TMA store for the dQ GEMM.
constexpr int COLS = 32;  // query columns per compute warpgroup (two warpgroups)
// of a thread's 16 exponential pairs per step, this many (the last ones) run
// as a polynomial on the FMA pipe instead of the MUFU unit
constexpr int kPolyPairs = SSA_KV_POLY_PAIRS;
static_assert(kPolyPairs >= 0 && kPolyPairs <= COLS / 2 && kPolyPairs % 2 == 0, "whole float4 groups");
// bf16 packing of dS: integer ALU (add half an ulp, byte permute) or the conversion unit
__device__ __forceinline__ uint32_t pack_ds(float lo, float hi) {
#if SSA_KV_PACK_CVT
    return pack_bf16(lo, hi);
#else
    return pack_bf16_alu(lo, hi);
#endif
}
constexpr int kThr = 384;  // warp 0 TMA, 1 MMA, 2 dS^T stores, 3 idle, 4-11 compute
constexpr int kComp = 256;
constexpr uint32_t OFF_STAGE = 0;
constexpr uint32_t ST_Q = 0, ST_GF = STEP_BYTES, ST_GS = 2 * STEP_BYTES;
constexpr uint32_t STAGE_BYTES = 3 * STEP_BYTES;
constexpr int NSTAGE = 3;
// dS^T, bf16 [128 keys x 64 queries], K-major with 128-byte swizzle, x2
constexpr uint32_t T_BYTES = 128 * 128;
constexpr uint32_t OFF_DS = OFF_STAGE + NSTAGE * STAGE_BYTES;
// per stage, fp32 over the step's 64 queries: -lse_full*log2(e) | -D_f | -D_s
constexpr uint32_t ROW_BYTES = 3 * STEP * 4;
constexpr uint32_t OFF_ROWS = OFF_DS + 2 * T_BYTES;
constexpr int NBAR = 24;
constexpr uint32_t OFF_BAR = OFF_ROWS + NSTAGE * ROW_BYTES;
// TMEM slot, abort flag, then one selection word per stage (bit 0: the step's
// query block selects key block kb0, bit 1: selects kb1)
constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;
constexpr uint32_t SMEM_BYTES = OFF_MISC + 32 + 1024;  // + slack for 1024-byte alignment
static_assert(SMEM_BYTES <= 232448, "227 KB of shared memory per CTA");
enum : int {  // barrier indices, derived from the ring depth
    B_FULL = 0, B_EMPTY = B_FULL + NSTAGE,
    B_OPS = B_EMPTY + NSTAGE,  // K and V are in TMEM
    B_SREADY = B_OPS + 1,      // S^T of the step is in TMEM
    B_SFREE = B_SREADY + 1,    // ... and has been read (the range may be overwritten)
    B_PSREADY = B_SFREE + 1,   // dP_s^T of a sparse step is in the S range
    B_PSFREE = B_PSREADY + 1,  // ... and has been read
    B_PREADY = B_PSFREE + 1,   // dP_f^T of the step is in the dP range
    B_PTREADY = B_PREADY + 1,  // ... has been read and P^T (bf16) written over it
    B_DSREADY = B_PTREADY + 1, // x2: dS^T buffer written
    B_TFREE = B_DSREADY + 2,   // x2: dS^T buffer read by the dK MMAs and the store
    B_DONE = B_TFREE + 2, B_DRAIN = B_DONE + 1, B_COUNT = B_DRAIN + 1
};
static_assert(B_COUNT <= NBAR, "barrier area");
// TMEM columns for head dim D: dV | dK (D each) | K | V (bf16, D/2 each) | S | dP (64 each);
// 512 at D = 128, 320 at D = 64
template <int D> struct Tm {
    static constexpr uint32_t DV = 0, DK = D, K = 2 * D, V = 2 * D + D / 2, S = 3 * D, DPF = 3 * D + 64;
};
// bf16 P^T of warpgroup w over the first 16 of its 32 dP columns, the masked
// copy in the other 16: TMEM column of the A operand's k-step kk (16 queries)
__device__ __forceinline__ uint32_t acol(int kk) { return 32u * (kk >> 1) + 8u * (kk & 1); }
}  // namespace kv

template <int D>
__global__ void __launch_bounds__(kv::kThr, 1)
bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_gf,
                   const __grid_constant__ CUtensorMap tm_gs, const __grid_constant__ CUtensorMap tm_ds,
                   const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
                   const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
                   const BwdArgs a) {
    using namespace kv;
    static_assert(D == 64 || D == 128, "head dim 64 or 128");
    constexpr uint32_t TM_DV = Tm<D>::DV, TM_DK = Tm<D>::DK, TM_K = Tm<D>::K, TM_V = Tm<D>::V,
                       TM_S = Tm<D>::S, TM_DPF = Tm<D>::DPF;
    constexpr uint32_t kStep = STEP * D * 2;  // bytes of one step tile (Q, G_f or G_s')
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);
    unsigned int* status = &g_bwd_tc_status;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + OFF_MISC + 4);
    uint32_t* flags = reinterpret_cast<uint32_t*>(gbase + OFF_MISC + 8);
    const float* rows_s = reinterpret_cast<const float*>(gbase + OFF_ROWS);
    const uint64_t lim = a.timeout_ns;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int J = (int)(blockIdx.x / a.BH);  // key tile; J = 0 has the most steps: first
    const int bh = (int)(blockIdx.x % a.BH);
    const int s0 = J * TILE;
    const int ns = (a.T - s0) / STEP;
    const int kb0 = s0 / a.block;
    const int kb1 = (s0 + 64 < a.T) ? (s0 + 64) / a.block : kb0;
    auto BAR = [&](int i) { return base + OFF_BAR + 8u * (uint32_t)i; };
    const size_t rowbase = (size_t)bh * a.T;
    // first dS^T block of this key tile: tiles J' < J hold (T - 128 J') / 64 blocks each
    const int ds_blk0 = bh * a.ds_blocks + J * (a.T / STEP) - J * (J - 1);

    if (threadIdx.x == 0) {
        for (int s = 0; s < NSTAGE; ++s) {
            mbar_init(BAR(B_FULL + s), 1);
            mbar_init(BAR(B_EMPTY + s), 1);
        }
        mbar_init(BAR(B_OPS), kComp);
        mbar_init(BAR(B_SREADY), 1);
        mbar_init(BAR(B_SFREE), kComp);
        mbar_init(BAR(B_PSREADY), 1);
        mbar_init(BAR(B_PSFREE), kComp);
        mbar_init(BAR(B_PREADY), 1);
        mbar_init(BAR(B_PTREADY), kComp);
        for (int b = 0; b < 2; ++b) {
            mbar_init(BAR(B_DSREADY + b), kComp);
            mbar_init(BAR(B_TFREE + b), 2);  // MMA commit + the dS^T store's source read
        }
        mbar_init(BAR(B_DONE), 1);
        mbar_init(BAR(B_DRAIN), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(base + OFF_MISC, 512);
        tmem_relinquish();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    const unsigned FULL = 0xffffffffu;
    auto wait = [&](int bar, uint32_t parity) {
        const bool r = __all_sync(FULL, mbar_wait(BAR(bar), parity, abort_flag, status, lim));
        fence_after_sync();
        return r;
    };
    if (warp == 0) {
        // -------------------------------------------- TMA producer (whole warp)
        if (elect_one()) {
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_gf);
            prefetch_tmap(&tm_gs);
            prefetch_tmap(&tm_ds);
        }
        __syncwarp();
        int issued[NSTAGE];
        for (int s = 0; s < NSTAGE; ++s) issued[s] = -1;
        for (int i = 0; i < ns; ++i) {
            const int s = i % NSTAGE;
            const int t0 = s0 + STEP * i;
            // selection of the tile's key blocks by the step's query block
            const uint32_t* m = a.mask + ((size_t)bh * a.n_blocks + t0 / a.block) * a.words;
            const uint32_t fl = (uint32_t)bit(m, kb0) | ((uint32_t)bit(m, kb1) << 1);
            if (i >= NSTAGE &&
                !__all_sync(FULL, mbar_wait(BAR(B_EMPTY + s), ((i / NSTAGE) + 1) & 1, abort_flag, status,
                                            lim)))
                break;
            const uint32_t st = base + OFF_STAGE + s * STAGE_BYTES;
            const uint32_t rw = base + OFF_ROWS + s * ROW_BYTES;
            if (elect_one()) {
                const bool sp = fl != 0u;
                flags[s] = fl;  // published by the arrive below
                mbar_expect_tx(BAR(B_FULL + s), 2 * kStep + 2 * STEP * 4 + (sp ? kStep + STEP * 4 : 0u));
#pragma unroll
                for (int x = 0; x < D / 64; ++x) {
                    tma_load_3d(st + ST_Q + x * BOX_S, &tm_q, BAR(B_FULL + s), 64 * x, t0, bh);
                    tma_load_3d(st + ST_GF + x * BOX_S, &tm_gf, BAR(B_FULL + s), 64 * x, t0, bh);
                }
                bulk_load(rw, a.neg_lse2 + rowbase + t0, STEP * 4, BAR(B_FULL + s));
                bulk_load(rw + STEP * 4, a.neg_Df + rowbase + t0, STEP * 4, BAR(B_FULL + s));
                if (sp) {  // the sparse stream's operands only where it has work
#pragma unroll
                    for (int x = 0; x < D / 64; ++x)
                        tma_load_3d(st + ST_GS + x * BOX_S, &tm_gs, BAR(B_FULL + s), 64 * x, t0, bh);
                    bulk_load(rw + 2 * STEP * 4, a.neg_Ds + rowbase + t0, STEP * 4, BAR(B_FULL + s));
                }
            }
            __syncwarp();
            issued[s] = i;
        }
        // every copy issued lands before the CTA exits, also when another role gives
        // up after this warp left its loop (the last load of each stage; earlier
        // ones completed before their stage was refilled)
        for (int s = 0; s < NSTAGE; ++s)
            if (issued[s] >= 0) wait_drain(BAR(B_FULL + s), (issued[s] / NSTAGE) & 1, kDrainLimitNs);
    } else if (warp == 1) {
        {  // ------------------------------------------ MMA issuer (whole warp)
            // descriptors formed once, advanced by constant offsets; each MMA group
            // and its commits are issued by one elected lane
            constexpr uint32_t id_s = idesc_bf16_f32(TILE, STEP, false);  // S^T, dP^T
            constexpr uint32_t id_a = idesc_bf16_f32(TILE, D, true);      // dV, dK
            const uint64_t st_k0 = smem_desc_sw128(base + OFF_STAGE, 16, 1024);      // K-major
            const uint64_t st_m0 = smem_desc_sw128(base + OFF_STAGE, BOX_S, 1024);   // MN-major
            const uint64_t ds_0 = smem_desc_sw128(base + OFF_DS, 16, 1024);          // K-major A
            auto ks = [](int kk) { return (uint32_t)((kk >> 2) * BOX_S + (kk & 3) * 32); };
            // D (TMEM) += A (TMEM, K or V) x B^T (64 rows of the stage, K-major)
            auto issue_tn = [&](uint32_t d, uint32_t a_col, uint32_t st_off) {
                const uint64_t bd = desc_add(st_k0, st_off);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    mma_ts(tmem + d, tmem + a_col + 8 * kk, desc_add(bd, ks(kk)), id_s, kk > 0);
            };
            auto stage_off = [&](int i) { return (uint32_t)((i % NSTAGE) * STAGE_BYTES); };
            bool ok = wait(B_OPS, 0) && wait(B_FULL, 0);
            if (ok) {
                if (elect_one()) {
                    issue_tn(TM_S, TM_K, stage_off(0) + ST_Q);  // S^T_0
                    mma_commit(BAR(B_SREADY));
                    issue_tn(TM_DPF, TM_V, stage_off(0) + ST_GF);  // dP_f^T_0
                    mma_commit(BAR(B_PREADY));
                }
                __syncwarp();
            }
            int nsp = 0;  // sparse steps so far (phase of B_PSREADY / B_PSFREE)
            for (int i = 0; ok && i < ns; ++i) {
                const int s = i % NSTAGE, b = i & 1;
                const uint32_t fl = flags[s];
                const bool sp = fl != 0u;
                const bool more = i + 1 < ns;
                // (a) S range: dP_s^T once S^T has been read (sparse steps), then the
                // next step's S^T once that has been read too
                if (sp || more) {
                    if (!wait(B_SFREE, i & 1)) {
                        ok = false;
                        break;
                    }
                }
                if (sp) {
                    if (elect_one()) {
                        issue_tn(TM_S, TM_V, stage_off(i) + ST_GS);
                        mma_commit(BAR(B_PSREADY));
                    }
                    __syncwarp();
                    if (more && !wait(B_PSFREE, nsp & 1)) {
                        ok = false;
                        break;
                    }
                    ++nsp;
                }
                if (more) {
                    if (!wait(B_FULL + (i + 1) % NSTAGE, ((i + 1) / NSTAGE) & 1)) {
                        ok = false;
                        break;
                    }
                    if (elect_one()) {
                        issue_tn(TM_S, TM_K, stage_off(i + 1) + ST_Q);
                        mma_commit(BAR(B_SREADY));
                    }
                    __syncwarp();
                }
                // (b) dP range: dV += P_f^T G_f (+ P_s^T G_s') once P^T has replaced
                // dP_f^T there, then dP_f^T of the next step (the MMAs run in order)
                if (!wait(B_PTREADY, i & 1)) {
                    ok = false;
                    break;
                }
                // P_s^T = P_f^T on selected key rows (c_t is folded into G_s'); the
                // row-masked copy is needed only when the tile's two key blocks differ
                const uint32_t ps_off = (fl == 1u || fl == 2u) ? 16u : 0u;
                if (elect_one()) {
                    const uint64_t gfm = desc_add(st_m0, stage_off(i) + ST_GF);
                    const uint64_t gsm = desc_add(st_m0, stage_off(i) + ST_GS);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_ts(tmem + TM_DV, tmem + TM_DPF + acol(kk), desc_add(gfm, kk * 2048), id_a,
                               (i > 0 || kk > 0) ? 1u : 0u);
                    if (sp) {
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_ts(tmem + TM_DV, tmem + TM_DPF + acol(kk) + ps_off, desc_add(gsm, kk * 2048),
                                   id_a, 1u);
                    }
                    if (more) {
                        issue_tn(TM_DPF, TM_V, stage_off(i + 1) + ST_GF);
                        mma_commit(BAR(B_PREADY));
                    }
                }
                __syncwarp();
                // (c) dK += dS^T Q once dS^T is in shared memory
                if (!wait(B_DSREADY + b, (i >> 1) & 1)) {
                    ok = false;
                    break;
                }
                if (elect_one()) {
                    const uint64_t qm = desc_add(st_m0, stage_off(i) + ST_Q);
                    const uint64_t dd = desc_add(ds_0, b * T_BYTES);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_ss(tmem + TM_DK, desc_add(dd, kk * 32), desc_add(qm, kk * 2048), id_a,
                               (i > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(BAR(B_EMPTY + s));
                    mma_commit(BAR(B_TFREE + b));
                }
                __syncwarp();
            }
            (void)nsp;
            if (elect_one()) {
                mma_commit(BAR(B_DONE));
                mma_commit(BAR(B_DRAIN));
            }
            __syncwarp();
            wait_drain(BAR(B_DRAIN), 0, kDrainLimitNs);
        }
    } else if (warp == 2) {
        // ------------------------------------------ dS^T stores for the dQ GEMM
        // (lane 0 owns the bulk group; off the MMA issuer's path)
        for (int i = 0; i < ns; ++i) {
            const int b = i & 1;
            if (!wait(B_DSREADY + b, (i >> 1) & 1)) break;
            if (lane == 0) {
                tma_store_3d(&tm_ds, base + OFF_DS + b * T_BYTES, 0, 0, ds_blk0 + i);
                bulk_commit_group();
                bulk_wait_group_read0();
                mbar_arrive(BAR(B_TFREE + b));
            }
            __syncwarp();
        }
        if (lane == 0) bulk_wait_group0();  // the dS^T stores are complete
        __syncwarp();
    } else if (warp >= 4) {
        // ------------------------------------------ two compute warpgroups
        // warpgroup wg handles query columns [32 wg, 32 wg + 32) of every step
        const int wg = (warp - 4) >> 2, sw = (warp - 4) & 3;
        const int r = sw * 32 + lane;  // key row of the tile == TMEM lane
        const int s_tok = s0 + r;
        const uint32_t trow = tmem + ((uint32_t)(sw * 32) << 16);
        const float sl2 = a.scale_log2;
        const bool in_kb1 = r >= 64 && a.block == 64;  // warp-uniform
        const bool key_ok = s_tok < a.T;                // warp-uniform (T is a multiple of 64)
        const int c0 = COLS * wg;
        bool ok = true;
        {  // K and V rows of the tile (this warpgroup's D/2 columns of each) into TMEM
            const size_t row = rowbase + (key_ok ? s_tok : 0);
            constexpr int W = D / 4;  // 32-bit TMEM columns per warpgroup and operand
            auto fill = [&](const __nv_bfloat16* src, uint32_t col) {
                uint32_t u[W];
                const uint4* p4 = reinterpret_cast<const uint4*>(src + row * D + 2 * W * wg);
#pragma unroll
                for (int v4 = 0; v4 < W / 4; ++v4) {
                    const uint4 x = key_ok ? __ldg(p4 + v4) : make_uint4(0u, 0u, 0u, 0u);
                    u[4 * v4] = x.x;
                    u[4 * v4 + 1] = x.y;
                    u[4 * v4 + 2] = x.z;
                    u[4 * v4 + 3] = x.w;
                }
                tmem_st<W>(trow + col + W * wg, u);
            };
            fill(k, TM_K);
            fill(v, TM_V);
            tmem_wait_st();
            fence_before_sync();
            mbar_arrive(BAR(B_OPS));
        }
        const uint32_t rowoff = (uint32_t)(r >> 3) * 1024 + (uint32_t)(r & 7) * 128;
        int nsp = 0;
        for (int i = 0; i < ns; ++i) {
            const int t0 = s0 + STEP * i;
            const int s = i % NSTAGE, b = i & 1;
            // the stage's row vectors and selection word (already landed: the MMA
            // warp waited for them before issuing this step's S^T)
            if (!wait(B_FULL + s, (i / NSTAGE) & 1) || !wait(B_SREADY, i & 1)) {
                ok = false;
                break;
            }
            const uint32_t fl = flags[s];
            const bool sp = fl != 0u;
            const bool use_s = in_kb1 ? (fl >> 1) & 1u : fl & 1u;
            const bool mixed = fl == 1u || fl == 2u;
            const bool diag = t0 < s0 + TILE;
            const float* rw = rows_s + s * (3 * STEP);
            float pf[COLS];
            uint32_t pfk[COLS / 2];
            {
                uint32_t su[COLS];
                tmem_ld32(trow + TM_S + c0, su);
                tmem_wait_ld();
                fence_before_sync();
                mbar_arrive(BAR(B_SFREE));  // the S range may now take dP_s^T
                const float4* L4 = reinterpret_cast<const float4*>(rw + c0);
                const f32x2 sl2x2 = mk2(sl2, sl2);
#pragma unroll
                for (int j4 = 0; j4 < COLS / 4; ++j4) {
                    const float4 L = L4[j4];  // -lse_full * log2(e) of the four queries
                    const f32x2 x01 = fma2(mk2(__uint_as_float(su[4 * j4]), __uint_as_float(su[4 * j4 + 1])),
                                           sl2x2, mk2(L.x, L.y));
                    const f32x2 x23 = fma2(mk2(__uint_as_float(su[4 * j4 + 2]), __uint_as_float(su[4 * j4 + 3])),
                                           sl2x2, mk2(L.z, L.w));
                    if (2 * j4 >= COLS / 2 - kPolyPairs) {
                        un2(exp2_poly2(x01), pf[4 * j4], pf[4 * j4 + 1]);
                        un2(exp2_poly2(x23), pf[4 * j4 + 2], pf[4 * j4 + 3]);
                    } else {
                        float x0, x1, x2, x3;
                        un2(x01, x0, x1);
                        un2(x23, x2, x3);
                        pf[4 * j4] = ex2(x0);
                        pf[4 * j4 + 1] = ex2(x1);
                        pf[4 * j4 + 2] = ex2(x2);
                        pf[4 * j4 + 3] = ex2(x3);
                    }
                }
                if (diag) {  // causal: query t0 + c0 + j sees key s_tok only if t >= s
#pragma unroll
                    for (int j = 0; j < COLS; ++j)
                        if (t0 + c0 + j < s_tok) pf[j] = 0.f;
                }
#pragma unroll
                for (int j2 = 0; j2 < COLS / 2; ++j2) pfk[j2] = pack_bf16_alu(pf[2 * j2], pf[2 * j2 + 1]);
            }
            // dP_s^T (sparse steps) comes through the S range after S^T
            uint32_t pu[COLS];
            if (sp) {
                if (!wait(B_PSREADY, nsp & 1)) {
                    ok = false;
                    break;
                }
                ++nsp;
                if (use_s) {
                    tmem_ld32(trow + TM_S + c0, pu);
                    tmem_wait_ld();
                }
                fence_before_sync();
                mbar_arrive(BAR(B_PSFREE));  // the S range may take the next S^T
            }
            if (!wait(B_PREADY, i & 1)) {
                ok = false;
                break;
            }
            uint32_t dsk[COLS / 2];
            {
                uint32_t fu[COLS];
                tmem_ld32(trow + TM_DPF + c0, fu);
                tmem_wait_ld();
                // P^T (bf16) over this warpgroup's dP_f^T columns, now read; on a mixed
                // step the sparse stream's copy, zero on unselected key rows, beside it
                tmem_st<16>(trow + TM_DPF + c0, pfk);
                if (mixed) {
                    if (!use_s)
#pragma unroll
                        for (int e = 0; e < COLS / 2; ++e) pfk[e] = 0u;
                    tmem_st<16>(trow + TM_DPF + c0 + 16, pfk);
                }
                tmem_wait_st();
                fence_before_sync();
                mbar_arrive(BAR(B_PTREADY));
                const float4* F4 = reinterpret_cast<const float4*>(rw + STEP + c0);
                const float4* S4 = reinterpret_cast<const float4*>(rw + 2 * STEP + c0);
#pragma unroll
                for (int j4 = 0; j4 < COLS / 4; ++j4) {
                    const float4 F = F4[j4];  // -D_f
                    f32x2 g01 = add2(mk2(__uint_as_float(fu[4 * j4]), __uint_as_float(fu[4 * j4 + 1])),
                                     mk2(F.x, F.y));
                    f32x2 g23 = add2(mk2(__uint_as_float(fu[4 * j4 + 2]), __uint_as_float(fu[4 * j4 + 3])),
                                     mk2(F.z, F.w));
                    if (use_s) {
                        const float4 S = S4[j4];  // -D_s'
                        g01 = add2(g01, add2(mk2(__uint_as_float(pu[4 * j4]), __uint_as_float(pu[4 * j4 + 1])),
                                             mk2(S.x, S.y)));
                        g23 = add2(g23, add2(mk2(__uint_as_float(pu[4 * j4 + 2]), __uint_as_float(pu[4 * j4 + 3])),
                                             mk2(S.z, S.w)));
                    }
                    float d0, d1, d2, d3;
                    un2(mul2(mk2(pf[4 * j4], pf[4 * j4 + 1]), g01), d0, d1);
                    un2(mul2(mk2(pf[4 * j4 + 2], pf[4 * j4 + 3]), g23), d2, d3);
                    dsk[2 * j4] = pack_ds(d0, d1);
                    dsk[2 * j4 + 1] = pack_ds(d2, d3);
                }
                if (!key_ok) {  // stored dS^T rows past T stay zero
#pragma unroll
                    for (int e = 0; e < COLS / 2; ++e) dsk[e] = 0u;
                }
            }
            // dS^T row r into buffer b once the dK MMAs and the store of step i-2 read it
            if (i >= 2 && !wait(B_TFREE + b, ((i >> 1) + 1) & 1)) {
                ok = false;
                break;
            }
            {
                uint8_t* dsb = gbase + OFF_DS + b * T_BYTES + rowoff;
#pragma unroll
                for (int q4 = 0; q4 < COLS / 8; ++q4) {
                    const uint32_t chunk = (uint32_t)((c0 >> 3) + q4) ^ (uint32_t)(r & 7);
                    *reinterpret_cast<uint4*>(dsb + chunk * 16) =
                        make_uint4(dsk[4 * q4], dsk[4 * q4 + 1], dsk[4 * q4 + 2], dsk[4 * q4 + 3]);
                }
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // visible to the MMAs
            mbar_arrive(BAR(B_DSREADY + b));
        }
        if (ok) ok = wait(B_DONE, 0);
        // dV and dK leave through shared memory (the stage ring, idle once every
        // MMA has completed) and TMA stores: a thread owns a key row, so direct
        // stores would scatter each warp's writes over 32 rows.  Rows past T are
        // clipped by the tensor maps.
        const bool all_ok = bar_and(ok, 1, kComp);
        uint8_t* stage = gbase + OFF_STAGE;
        constexpr uint32_t kOutBytes = TILE * D * 2;
        if (all_ok) {
            constexpr int OC = D / 2;  // output columns per warpgroup
            stage_row_cols<OC / 32>(trow + TM_DV + OC * wg, 1.f, stage, OC * wg, r);
            stage_row_cols<OC / 32>(trow + TM_DK + OC * wg, a.sm_scale, stage + kOutBytes, OC * wg, r);
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        bar_sync(1, kComp);
        if (all_ok && warp == 4 && lane == 0) {
#pragma unroll
            for (int x = 0; x < D / 64; ++x) {
                tma_store_3d(&tm_dv, base + OFF_STAGE + x * BOX_T, 64 * x, s0, bh);
                tma_store_3d(&tm_dk, base + OFF_STAGE + kOutBytes + x * BOX_T, 64 * x, s0, bh);
            }
            bulk_commit_group();
            bulk_wait_group_read0();  // the staging area stays valid until read
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        fence_after_sync();
        tmem_dealloc(tmem, 512);
    }
}

// ============================================================ dQ
// dQ = sigma dS K as a GEMM over the dS^T blocks the dK/dV kernel stored:
// CTA = 128 queries (M), K-dim = keys in tiles of 128, N = head dim.  A is the
// pair of [128 keys x 64 queries] dS^T blocks of the query tile (MN-major),
// B the key tile (MN-major); both arrive by TMA into a 3-stage ring.
namespace dq {
constexpr int NSTAGE = 3;
constexpr uint32_t BLK_BYTES = 128 * 128;            // one dS^T block
constexpr uint32_t ST_B = 2 * BLK_BYTES;             // K tile after the two blocks
constexpr uint32_t STAGE_BYTES = 2 * BLK_BYTES + TILE_BYTES;
constexpr uint32_t OFF_BAR = NSTAGE * STAGE_BYTES;
constexpr uint32_t OFF_MISC = OFF_BAR + 16 * 8;
constexpr uint32_t SMEM_BYTES = OFF_MISC + 16 + 1024;
static_assert(SMEM_BYTES <= 232448, "227 KB of shared memory per CTA");
constexpr int kThr = 192;  // warp 0 TMA, 1 MMA, 2-5 epilogue
enum : int {
    B_FULL = 0, B_EMPTY = B_FULL + NSTAGE, B_DONE = B_EMPTY + NSTAGE, B_DRAIN = B_DONE + 1,
    B_COUNT = B_DRAIN + 1
};
static_assert(B_COUNT <= 16, "barrier area holds 16");
}  // namespace dq

template <int D>
__global__ void __launch_bounds__(dq::kThr, 1)
bwd_dq_gemm_kernel(const __grid_constant__ CUtensorMap tm_ds, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_dq, const BwdArgs a) {
    using namespace dq;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + OFF_MISC + 4);
    unsigned int* status = &g_bwd_tc_status;
    const uint64_t lim = a.timeout_ns;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ntq = (a.T + TILE - 1) / TILE;
    const int I = ntq - 1 - (int)(blockIdx.x / a.BH);  // longest rows first
    const int bh = (int)(blockIdx.x % a.BH);
    const int t0 = I * TILE;
    const bool two = t0 + 64 < a.T;  // the tile's second 64-query step exists
    const int nj = I + 1;            // key tiles 0..I
    auto BAR = [&](int i) { return base + OFF_BAR + 8u * (uint32_t)i; };

    if (threadIdx.x == 0) {
        for (int s = 0; s < NSTAGE; ++s) {
            mbar_init(BAR(B_FULL + s), 1);
            mbar_init(BAR(B_EMPTY + s), 1);
        }
        mbar_init(BAR(B_DONE), 1);
        mbar_init(BAR(B_DRAIN), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(base + OFF_MISC, 128);
        tmem_relinquish();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    const unsigned FULL = 0xffffffffu;
    if (warp == 0) {
        // -------------------------------------------- TMA producer (whole warp)
        if (elect_one()) {
            prefetch_tmap(&tm_ds);
            prefetch_tmap(&tm_k);
        }
        __syncwarp();
        int issued[NSTAGE];
        for (int s = 0; s < NSTAGE; ++s) issued[s] = -1;
        for (int j = 0; j < nj; ++j) {
            const int s = j % NSTAGE;
            if (j >= NSTAGE &&
                !__all_sync(FULL, mbar_wait(BAR(B_EMPTY + s), ((j / NSTAGE) + 1) & 1, abort_flag, status,
                                            lim)))
                break;
            const uint32_t st = base + s * STAGE_BYTES;
            // blocks of key tile j for query steps 2(I - j) and 2(I - j) + 1
            const int blk = bh * a.ds_blocks + j * (a.T / STEP) - j * (j - 1) + 2 * (I - j);
            if (elect_one()) {
                mbar_expect_tx(BAR(B_FULL + s), (two ? 2 : 1) * BLK_BYTES + TILE * D * 2);
                tma_load_3d(st, &tm_ds, BAR(B_FULL + s), 0, 0, blk);
                if (two) tma_load_3d(st + BLK_BYTES, &tm_ds, BAR(B_FULL + s), 0, 0, blk + 1);
#pragma unroll
                for (int x = 0; x < D / 64; ++x)
                    tma_load_3d(st + ST_B + x * BOX_T, &tm_k, BAR(B_FULL + s), 64 * x, TILE * j, bh);
            }
            __syncwarp();
            issued[s] = j;
        }
        for (int s = 0; s < NSTAGE; ++s)  // every issued copy lands before the CTA exits
            if (issued[s] >= 0) wait_drain(BAR(B_FULL + s), (issued[s] / NSTAGE) & 1, kDrainLimitNs);
    } else if (warp == 1) {
        // ------------------------------------------ MMA issuer (whole warp)
        constexpr uint32_t id = idesc_bf16_f32(TILE, D, true, true);  // A and B MN-major
        const uint64_t a0 = smem_desc_sw128(base, BLK_BYTES, 1024);
        const uint64_t b0 = smem_desc_sw128(base + ST_B, BOX_T, 1024);
        for (int j = 0; j < nj; ++j) {
            const int s = j % NSTAGE;
            if (!__all_sync(FULL, mbar_wait(BAR(B_FULL + s), (j / NSTAGE) & 1, abort_flag, status, lim)))
                break;
            fence_after_sync();
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)  // 16 keys per k-step
                    mma_ss(tmem, desc_add(a0, s * STAGE_BYTES + kk * 2048),
                           desc_add(b0, s * STAGE_BYTES + kk * 2048), id, (j > 0 || kk > 0) ? 1u : 0u);
                mma_commit(BAR(B_EMPTY + s));
            }
            __syncwarp();
        }
        if (elect_one()) {
            mma_commit(BAR(B_DONE));
            mma_commit(BAR(B_DRAIN));
        }
        __syncwarp();
        wait_drain(BAR(B_DRAIN), 0, kDrainLimitNs);
    } else {
        // ------------------------------------------ epilogue: warps 2-5 cover TMEM lanes
        const int sw = warp & 3;
        const int r = sw * 32 + lane;
        const uint32_t trow = tmem + ((uint32_t)(sw * 32) << 16);
        // dQ leaves through shared memory (the ring, idle once every MMA has
        // completed) and TMA stores; rows past T are clipped by the tensor map
        const bool ok = __all_sync(FULL, mbar_wait(BAR(B_DONE), 0, abort_flag, status, lim));
        const bool all_ok = bar_and(ok, 1, 128);
        if (all_ok) {
            fence_after_sync();
            stage_row_cols<D / 32>(trow, a.sm_scale, gbase, 0, r);
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        bar_sync(1, 128);
        if (all_ok && warp == 2 && lane == 0) {
#pragma unroll
            for (int x = 0; x < D / 64; ++x) tma_store_3d(&tm_dq, base + x * BOX_T, 64 * x, t0, bh);
            bulk_commit_group();
            bulk_wait_group_read0();  // the staging area stays valid until read
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        fence_after_sync();
        tmem_dealloc(tmem, 128);
    }
}

// ============================================================ host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// [BH, T, D] bf16 as a 3-D tensor (d, t, bh); box 64 d x `rows` t; 128B swizzle.
int make_map(CUtensorMap* m, const void* ptr, int BH, int T, int rows, int D) {
    auto fn = encode_fn();
    if (!fn) return fail(SSA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)T, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)T * D * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)rows, 1};
    cuuint32_t es[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides,
                    box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(SSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return SSA_OK;
}

// dS^T blocks [128 keys x 64 queries] bf16 as a 3-D tensor (query, key, block);
// box = one block; 128B swizzle (the layout the dK/dV kernel writes in smem).
int make_ds_map(CUtensorMap* m, void* ptr, size_t nblk) {
    auto fn = encode_fn();
    if (!fn) return fail(SSA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    cuuint64_t dims[3] = {(cuuint64_t)STEP, (cuuint64_t)TILE, (cuuint64_t)nblk};
    cuuint64_t strides[2] = {(cuuint64_t)STEP * 2, (cuuint64_t)STEP * TILE * 2};
    cuuint32_t box[3] = {(cuuint32_t)STEP, (cuuint32_t)TILE, 1};
    cuuint32_t es[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, ptr, dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(SSA_ERR_CUDA, "cuTensorMapEncodeTiled (dS) failed (%d)", (int)r);
    return SSA_OK;
}

// dS^T blocks per (batch, head): key tile J holds (T - 128 J) / 64 steps.
size_t ds_blocks_per_bh(int T) {
    const size_t ntk = (size_t)(T + TILE - 1) / TILE;
    return ntk * (size_t)(T / STEP) - ntk * (ntk - 1);
}
// Heads per launch so that the dS^T buffer stays within a byte budget
// (4 GiB unless a test sets another through ssa_debug_set_ds_budget_bytes).
int heads_per_chunk(const ssa_params_t& p) {
    const size_t per = ds_blocks_per_bh(p.T) * (size_t)STEP * TILE * 2;
    const size_t bh = (size_t)p.B * p.H;
    size_t hc = (size_t)ds_budget_bytes() / per;
    if (hc < 1) hc = 1;
    if (hc > bh) hc = bh;
    return (int)hc;
}

struct TcWs {
    __nv_bfloat16* gf;
    __nv_bfloat16* gs;
    float *neg_lse2, *neg_Df, *neg_Ds;
    __nv_bfloat16* ds;
};

TcWs carve(const ssa_params_t& p, void* ws) {
    const size_t big = align_up(num_elems(p) * 2, 256);
    const size_t small = align_up(num_rows(p) * 4, 256);
    char* b = static_cast<char*>(ws);
    TcWs w;
    w.gf = reinterpret_cast<__nv_bfloat16*>(b);
    w.gs = reinterpret_cast<__nv_bfloat16*>(b + big);
    w.neg_lse2 = reinterpret_cast<float*>(b + 2 * big);
    w.neg_Df = reinterpret_cast<float*>(b + 2 * big + small);
    w.neg_Ds = reinterpret_cast<float*>(b + 2 * big + 2 * small);
    w.ds = reinterpret_cast<__nv_bfloat16*>(b + 2 * big + 3 * small);
    return w;
}

}  // namespace

int bwd_tc_heads_per_group(const ssa_params_t& p) { return heads_per_chunk(p); }

bool bwd_tc_supported(const ssa_params_t& p) {
    return p.dtype == SSA_BF16 && (p.D == 64 || p.D == 128) && (p.block == 64 || p.block == 128) &&
           (size_t)p.B * p.H * ((p.T + TILE - 1) / TILE) <= 0x7fffffffull &&
           ds_blocks_per_bh(p.T) <= 0x7fffffffull;
}

size_t bwd_tc_workspace(const ssa_params_t& p) {
    return 2 * align_up(num_elems(p) * 2, 256) + 3 * align_up(num_rows(p) * 4, 256) +
           (size_t)heads_per_chunk(p) * ds_blocks_per_bh(p.T) * STEP * TILE * 2;
}

namespace {
template <int D>
int launch_bwd_tc_impl(const ssa_params_t& p, const void* q, const void* k, const void* v,
                       const void* hf, const void* hs, const float* lf, const float* ls,
                       const void* dhf, const void* dhs, float w_s, float w_c, const uint32_t* mask,
                       void* dq, void* dk, void* dv, void* ws, cudaStream_t s) {
    const int BH = p.B * p.H;
    const TcWs w = carve(p, ws);
    const size_t rows = num_rows(p);
    const double two_over_n = 2.0 / (double)num_elems(p);
    mark_kernel_event(0, s);
    bwd_tc_pre_kernel<D><<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(hf), static_cast<const __nv_bfloat16*>(hs),
        static_cast<const __nv_bfloat16*>(dhf), static_cast<const __nv_bfloat16*>(dhs), lf, ls, rows,
        (float)(w_s * two_over_n), (float)(w_c * two_over_n), w.gf, w.gs, w.neg_lse2, w.neg_Df, w.neg_Ds);
    int st = check_launch("bwd_tc_pre_kernel");
    if (st != SSA_OK) return st;
    mark_kernel_event(1, s);

    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once, [] {
        attr_err = cudaFuncSetAttribute(bwd_dkdv_tc_kernel<D>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kv::SMEM_BYTES);
        if (attr_err == cudaSuccess)
            attr_err = cudaFuncSetAttribute(bwd_dq_gemm_kernel<D>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            (int)dq::SMEM_BYTES);
    });
    if (attr_err != cudaSuccess)
        return fail(SSA_ERR_CUDA, "bwd_tc: smem attribute: %s", cudaGetErrorString(attr_err));

    const int ntile = (p.T + TILE - 1) / TILE;
    const size_t nb = ds_blocks_per_bh(p.T);
    const int hc = heads_per_chunk(p);
    const size_t head_elems = (size_t)p.T * D;
    const size_t head_mask = (size_t)num_blocks(p) * mask_words(p);
    // every (batch, head) is independent: chunks of hc heads share the dS^T buffer
    for (int h0 = 0; h0 < BH && st == SSA_OK; h0 += hc) {
        const int nh = BH - h0 < hc ? BH - h0 : hc;
        auto off = [&](const void* ptr) {
            return static_cast<const void*>(static_cast<const __nv_bfloat16*>(ptr) + h0 * head_elems);
        };
        CUtensorMap k128, q64, gf64, gs64, ds_map, dq128, dk128, dv128;
        st = make_map(&k128, off(k), nh, p.T, TILE, D);
        if (st == SSA_OK) st = make_map(&dq128, off(dq), nh, p.T, TILE, D);
        if (st == SSA_OK) st = make_map(&dk128, off(dk), nh, p.T, TILE, D);
        if (st == SSA_OK) st = make_map(&dv128, off(dv), nh, p.T, TILE, D);
        if (st == SSA_OK) st = make_map(&q64, off(q), nh, p.T, STEP, D);
        if (st == SSA_OK) st = make_map(&gf64, off(w.gf), nh, p.T, STEP, D);
        if (st == SSA_OK) st = make_map(&gs64, off(w.gs), nh, p.T, STEP, D);
        if (st == SSA_OK) st = make_ds_map(&ds_map, w.ds, (size_t)nh * nb);
        if (st != SSA_OK) break;

        BwdArgs a;
        a.dq = static_cast<__nv_bfloat16*>(dq) + h0 * head_elems;
        a.dk = static_cast<__nv_bfloat16*>(dk) + h0 * head_elems;
        a.dv = static_cast<__nv_bfloat16*>(dv) + h0 * head_elems;
        a.neg_lse2 = w.neg_lse2 + (size_t)h0 * p.T;
        a.neg_Df = w.neg_Df + (size_t)h0 * p.T;
        a.neg_Ds = w.neg_Ds + (size_t)h0 * p.T;
        a.mask = mask + h0 * head_mask;
        a.BH = nh;
        a.T = p.T;
        a.block = p.block;
        a.words = mask_words(p);
        a.n_blocks = num_blocks(p);
        a.ds_blocks = (int)nb;
        a.scale_log2 = p.sm_scale * kLog2e;
        a.sm_scale = p.sm_scale;
        a.timeout_ns = wait_limit_ns();
        const unsigned grid = (unsigned)((size_t)nh * ntile);
        bwd_dkdv_tc_kernel<D><<<grid, kv::kThr, kv::SMEM_BYTES, s>>>(
            q64, gf64, gs64, ds_map, dk128, dv128, static_cast<const __nv_bfloat16*>(off(k)),
            static_cast<const __nv_bfloat16*>(off(v)), a);
        st = check_launch("bwd_dkdv_tc_kernel");
        if (st != SSA_OK) break;
        if (h0 == 0) mark_kernel_event(2, s);
        bwd_dq_gemm_kernel<D><<<grid, dq::kThr, dq::SMEM_BYTES, s>>>(ds_map, k128, dq128, a);
        st = check_launch("bwd_dq_gemm_kernel");
        if (h0 == 0) mark_kernel_event(3, s);
    }
    return st;
}
}  // namespace

int launch_bwd_tc(const ssa_params_t& p, const void* q, const void* k, const void* v,
                  const uint32_t* mask, const void* hf, const void* hs, const float* lf,
                  const float* ls, const void* dhf, const void* dhs, float w_s, float w_c,
                  void* dq, void* dk, void* dv, void* ws, cudaStream_t s) {
    if (p.D == 64)
        return launch_bwd_tc_impl<64>(p, q, k, v, hf, hs, lf, ls, dhf, dhs, w_s, w_c, mask, dq, dk,
                                      dv, ws, s);
    return launch_bwd_tc_impl<128>(p, q, k, v, hf, hs, lf, ls, dhf, dhs, w_s, w_c, mask, dq, dk,
                                   dv, ws, s);
}

int bwd_tc_take_status(cudaStream_t) {
    unsigned int v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_bwd_tc_status, sizeof v);
    if (e != cudaSuccess) return fail(SSA_ERR_CUDA, "status read: %s", cudaGetErrorString(e));
    if (v) {
        const unsigned int zero = 0;
        cudaMemcpyToSymbol(g_bwd_tc_status, &zero, sizeof zero);
        return fail(SSA_ERR_TIMEOUT, "bwd tcgen05 kernels: a bounded mbarrier wait expired");
    }
    return SSA_OK;
}

}  // namespace ssa
