// Fused dual-stream forward on the sm_100a tensor cores (bf16 in, fp32
// accumulate, head dim 64 or 128): one pass over the causal K/V of a 128-row query
// tile produces the full-attention output, the block-sparse output, the
// discarded mass delta(t) and both log-sum-exps ("Sintesi Tecnica: SSA",
// section 2: the sparse stream and its full-attention counterpart of the
// same layer; section 1: the sparse stream normalises over the selected
// subset only).
//
// CTA = (query tile of 128 rows, batch*head), 384 threads:
//   warps 0, 2  TMA producers: Q once and K_j (warp 0), V_j (warp 2), into
//               2-stage rings
//   warp 1      TMEM owner and MMA issuer (one thread):
//                 S_j = Q K_j^T          (tcgen05 SS, into S buffer j%2)
//                 O_sel/O_uns += P_j V_j  (tcgen05 TS, P read from TMEM)
//   warps 4..11 two softmax warpgroups, warpgroup h taking keys
//               [64h, 64h + 64) of every tile: thread = query row = TMEM
//               lane.  They read S_j, keep one running max for both streams
//               (combined through shared memory once per tile), split the row
//               sum into l_sel / l_uns by the selection mask and write P_j
//               (bf16) back into the S buffer for the PV product.
// TMEM (512 columns): S0 [0,128) S1 [128,256) O_sel [256,384) O_uns [384,512).
//
// A 128-key tile holds one or two key blocks and the 128 query rows one or
// two query blocks.  For each 64-key half the selection is read for both
// query blocks; when they agree the half's PV goes to one accumulator, when
// they differ ("mixed") P is written twice with complementary rows zeroed
// and both accumulators receive one MMA each.
//
// The running max is only raised (and O rescaled) when a row's tile max
// exceeds it by more than 2^8; the final normalisation divides by sums taken
// against the same stale max, so the result is unchanged.
//
// Optionally (ssa_attn_fwd_dual_diag) each row's weight on block 0 is summed
// while key tile 0 is processed, rescaled with the row sums, and divided by
// the full normaliser in the epilogue: the attention-sink mass.
//
// Every mbarrier wait is bounded (wall-clock limit); on expiry the kernel
// records SSA_ERR_TIMEOUT in a device status word, the other roles stop,
// in-flight tensor-core work is drained and TMEM is released.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "ssa_internal.h"
#include "tc_util.cuh"

namespace ssa {
namespace {

using namespace tc;

constexpr int BM = 128;  // query rows per tile
constexpr int BN = 128;  // keys per tile
constexpr int HD = 128;  // largest head dim (the shared-memory layout is sized for it)
constexpr int kThreads = 384;  // warps 0-2 roles, 3 idle, 4-11 two softmax warpgroups
constexpr int kSoftmax = 256;
constexpr uint32_t TILE_BYTES = BM * HD * 2;  // 32 KB ring slot (half used at d = 64)
constexpr uint32_t HALF_BYTES = 128 * 128;    // [128 rows x 64 cols] bf16 box, 16 KB
constexpr int kMaxWords = 256;                // mask words per query block (n <= 8192)

constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_K = OFF_Q + TILE_BYTES;
constexpr uint32_t OFF_V = OFF_K + 2 * TILE_BYTES;
constexpr uint32_t OFF_BAR = OFF_V + 2 * TILE_BYTES;
constexpr int NBAR = 16;
constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;  // [0] tmem base, [1] abort flag
constexpr uint32_t OFF_MASK = OFF_MISC + 16;       // mask rows of the two query blocks
// warpgroup exchange area, 1024 f32: row maxima [parity][wg][row] (512), then in
// the epilogue l_sel/l_uns [wg][2][row] (512), squared-difference sums [wg][row]
// at offset 512 (256) and block-0 weights [wg][row] at offset 768 (256)
constexpr uint32_t OFF_XCH = OFF_MASK + 2 * kMaxWords * 4;
// sparse-only forward: the key tiles the CTA uses, ascending (int16), and the
// per-warp counts of the list compaction
constexpr int kMaxTiles = kMaxWords * 32 * 128 / BN;  // T <= kMaxWords * 32 blocks of 128
constexpr uint32_t OFF_LIST = OFF_XCH + 1024 * 4;
constexpr uint32_t OFF_LCNT = OFF_LIST + kMaxTiles * 2;
constexpr uint32_t SMEM_USED = OFF_LCNT + 16 * 4;
static_assert(SMEM_USED + 1024 <= 232448, "shared memory per CTA");
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // slack for 1024-byte alignment

enum : int {  // barrier indices (two-stage K / V rings, two S buffers)
    B_QFULL = 0, B_KFULL = 1, B_KEMPTY = 3, B_VFULL = 5, B_VEMPTY = 7,
    B_SREADY = 9, B_PREADY = 11, B_PVDONE = 13, B_DRAIN = 14, B_COUNT = 15
};
static_assert(B_COUNT <= NBAR, "barrier area");

constexpr uint32_t TM_S0 = 0, TM_S1 = 128, TM_OSEL = 256, TM_OUNS = 384;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
// pairs c with c % 8 in {1, 4, 6} (three eighths) use the FMA-pipe exponential
__device__ __forceinline__ bool poly_pair(int c) {
    return (c & 7) == 1 || (c & 7) == 4 || (c & 7) == 6;
}
constexpr float kLn2 = 0.693147180559945309f;

__device__ unsigned int g_fwd_tc_status;

struct FwdArgs {
    __nv_bfloat16* h_full;
    __nv_bfloat16* h_sparse;
    float* delta;
    float* lse_full;
    float* lse_sparse;
    float* sqdiff;
    float* sink;  // optional (dual forward only): full-softmax mass on block 0 per row
    const uint32_t* mask;
    int BH, T, block, words, n_blocks;
    float scale_log2;  // sm_scale * log2(e)
    unsigned long long timeout_ns;
};

__device__ __forceinline__ bool bit(const uint32_t* row, int j) {
    return (row[j >> 5] >> (j & 31)) & 1u;
}

// Selection of key-tile J, half h, for the tile's two query blocks (rows
// 0-63 and 64-127), with don't-care rows made to agree: query rows that see
// none of the half's keys (diagonal tile, block 64, h = 1) and rows past T.
__device__ __forceinline__ void half_sel(const uint32_t* mrow, int J, int I, int h, int block,
                                         bool ragged1, bool& s0, bool& s1) {
    const int kb = (J * BN + 64 * h) >> (block == 64 ? 6 : 7);  // block is 64 or 128
    s0 = bit(mrow, kb);
    s1 = bit(mrow + kMaxWords, kb);
    if (block == 64 && J == I && h == 1) s0 = s1;
    if (ragged1) s1 = s0;
}

__device__ __forceinline__ bool wait_drain(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(bar, parity))
        if (globaltimer() - t0 > limit_ns) return false;
    return true;
}

// D: head dim, 64 or 128 (one or two 64-column boxes per tile; an S tile
// takes D/16 MMA k-steps; each softmax warpgroup owns D/2 output columns).
// kSparse = false: the dual forward (both streams).  kSparse = true: the
// sparse stream alone (inference, the same operations as MoBA): every role
// walks only the CTA's list of selected keys (with blocks of 64, the
// off-diagonal selected blocks packed two to a tile, each half loaded as its
// own 64-row box), the running max is taken over selected keys only,
// unselected (row, half) pairs get P = 0, one accumulator (O_sel), and the
// epilogue writes h_sparse and lse_sparse only.
template <int D, bool kSparse>
__global__ void __launch_bounds__(kThreads, 1)
fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_k64,
              const __grid_constant__ CUtensorMap tm_v64, const __grid_constant__ CUtensorMap tm_hf,
              const __grid_constant__ CUtensorMap tm_hs, const FwdArgs a) {
    static_assert(D == 64 || D == 128, "head dim 64 or 128");
    constexpr uint32_t kTileBytes = BM * D * 2;  // bytes a Q / K / V tile load brings
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + OFF_MISC + 4);
    uint32_t* mrow = reinterpret_cast<uint32_t*>(gbase + OFF_MASK);
    unsigned int* status = &g_fwd_tc_status;
    const uint64_t lim = a.timeout_ns;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ntq = (a.T + BM - 1) / BM;
    const int I = ntq - 1 - (int)(blockIdx.x / a.BH);  // longest rows first
    const int bh = (int)(blockIdx.x % a.BH);
    const int t0 = I * BM;
    const int ntk = I + 1;
    const bool ragged1 = t0 + 64 >= a.T;
    const int qb0 = t0 / a.block;
    const int qb1 = ragged1 ? qb0 : (t0 + 64) / a.block;
    auto BAR = [&](int i) { return base + OFF_BAR + 8u * (uint32_t)i; };

    if (threadIdx.x == 0) {
        mbar_init(BAR(B_QFULL), 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(BAR(B_KFULL + s), 1);
            mbar_init(BAR(B_KEMPTY + s), 1);
            mbar_init(BAR(B_VFULL + s), 1);
            mbar_init(BAR(B_VEMPTY + s), 1);
            mbar_init(BAR(B_SREADY + s), 1);
            mbar_init(BAR(B_PREADY + s), kSoftmax);
        }
        mbar_init(BAR(B_PVDONE), 1);
        mbar_init(BAR(B_DRAIN), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    {
        const uint32_t* m0 = a.mask + ((size_t)bh * a.n_blocks + qb0) * a.words;
        const uint32_t* m1 = a.mask + ((size_t)bh * a.n_blocks + qb1) * a.words;
        for (int w = threadIdx.x; w < a.words; w += kThreads) {
            mrow[w] = m0[w];
            mrow[kMaxWords + w] = m1[w];
        }
    }
    if (warp == 1) {
        tmem_alloc(base + OFF_MISC, 512);
        tmem_relinquish();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    // key tiles the CTA processes: every causal one for the dual forward.  For
    // the sparse stream alone, blocks of 128 keys: the tiles that the query
    // block selects (the diagonal tile always: the current block is always
    // selected).  Blocks of 64 keys: the off-diagonal key blocks that either
    // query block selects, paired in ascending order into tiles of two
    // 64-key halves (a last odd block leaves its second half empty), then the
    // diagonal tile.  Either list is built once, ascending, by a ballot
    // compaction over all threads, so that no role walks unselected tiles.
    int16_t* tlist = reinterpret_cast<int16_t*>(gbase + OFF_LIST);
    int ntiles = ntk;
    const bool packed = kSparse && a.block == 64;
    int nsel_off = 0;  // packed: selected off-diagonal key blocks
    if constexpr (kSparse) {
        int* lcnt = reinterpret_cast<int*>(gbase + OFF_LCNT);
        const int nitems = packed ? 2 * I : ntk;  // key blocks below the diagonal, or tiles
        int total = 0;
        for (int c = 0; c < nitems; c += kThreads) {  // the same trip count in every thread
            const int j = c + (int)threadIdx.x;
            bool used = false;
            if (j < nitems) {
                if (packed) {
                    used = bit(mrow, j) || bit(mrow + kMaxWords, j);
                } else {
                    bool a0, a1, b0, b1;
                    half_sel(mrow, j, I, 0, a.block, ragged1, a0, a1);
                    half_sel(mrow, j, I, 1, a.block, ragged1, b0, b1);
                    used = a0 || a1 || b0 || b1;
                }
            }
            const uint32_t bal = __ballot_sync(0xffffffffu, used);
            if (lane == 0) lcnt[warp] = __popc(bal);
            __syncthreads();
            int before = 0, all = 0;
            for (int w = 0; w < kThreads / 32; ++w) {
                const int cw = lcnt[w];
                before += w < warp ? cw : 0;
                all += cw;
            }
            if (used) tlist[total + before + __popc(bal & ((1u << lane) - 1u))] = (int16_t)j;
            total += all;
            __syncthreads();  // lcnt is reused by the next chunk; the list is complete after the last
        }
        if (packed) {
            nsel_off = total;
            ntiles = (total + 1) / 2 + 1;
        } else {
            ntiles = total;
        }
    }
    // tile jj: natural key tile j (j >= 0), or (packed) the key blocks kb0, kb1
    // of its two halves (kb1 = -1: empty half)
    struct TileDesc {
        int j, kb0, kb1;
    };
    auto tile_desc = [&](int jj) -> TileDesc {
        if (kSparse && packed) {
            if (jj == ntiles - 1) return {I, 0, 0};
            return {-1, (int)tlist[2 * jj], 2 * jj + 1 < nsel_off ? (int)tlist[2 * jj + 1] : -1};
        }
        return {kSparse ? (int)tlist[jj] : jj, 0, 0};
    };
    // selection of half h of a tile by the tile's two query blocks
    auto sel_half = [&](const TileDesc& td, int h, bool& s0, bool& s1) {
        if (td.j >= 0) {
            half_sel(mrow, td.j, I, h, a.block, ragged1, s0, s1);
            return;
        }
        const int kb = h ? td.kb1 : td.kb0;
        s0 = kb >= 0 && bit(mrow, kb);
        s1 = kb >= 0 && bit(mrow + kMaxWords, kb);
        if (ragged1) s1 = s0;
    };

    // Roles 0 and 1 run their loops with the whole warp (warp-uniform address and
    // descriptor arithmetic); one elected lane issues each TMA / tcgen05 op.
    const unsigned FULL = 0xffffffffu;
    if (warp == 0 || warp == 2) {
        // ------------------------------------------------ TMA producers
        // warp 0: Q once, then the K ring; warp 2: the V ring.  Separate
        // producers keep a K load from queueing behind a V slot that waits
        // for the other warpgroup's PV product.
        const bool is_k = warp == 0;
        const CUtensorMap* tm = is_k ? &tm_k : &tm_v;
        const CUtensorMap* tm64 = is_k ? &tm_k64 : &tm_v64;  // 64-row boxes: packed halves
        const int FULLB = is_k ? B_KFULL : B_VFULL, EMPTYB = is_k ? B_KEMPTY : B_VEMPTY;
        const uint32_t ring = base + (is_k ? OFF_K : OFF_V);
        if (elect_one()) {
            prefetch_tmap(tm);
            if (is_k) {
                prefetch_tmap(&tm_q);
                mbar_expect_tx(BAR(B_QFULL), kTileBytes);
#pragma unroll
                for (int x = 0; x < D / 64; ++x)
                    tma_load_3d(base + OFF_Q + x * HALF_BYTES, &tm_q, BAR(B_QFULL), 64 * x, t0, bh);
            }
        }
        __syncwarp();
        int issued[2] = {-1, -1};
        for (int jj = 0; jj < ntiles; ++jj) {
            const TileDesc td = tile_desc(jj);
            const int s = jj & 1;  // ring slot of the jj-th processed tile
            const uint32_t ph = ((jj >> 1) + 1) & 1;
            const uint32_t dst = ring + s * TILE_BYTES;
            if (jj >= 2 && !__all_sync(FULL, mbar_wait(BAR(EMPTYB + s), ph, abort_flag, status, lim)))
                break;
            if (elect_one()) {
                mbar_expect_tx(BAR(FULLB + s), kTileBytes);
                if (td.j >= 0 || (td.kb1 == td.kb0 + 1 && (td.kb0 & 1) == 0)) {
                    // a natural key tile (or a packed pair that is one): one 128-row box
                    const int row0 = td.j >= 0 ? td.j * BN : td.kb0 * 64;
#pragma unroll
                    for (int x = 0; x < D / 64; ++x)
                        tma_load_3d(dst + x * HALF_BYTES, tm, BAR(FULLB + s), 64 * x, row0, bh);
                } else {
                    // two 64-row boxes per 64-column box: the same swizzled layout as
                    // one 128-row box; an empty half repeats the first block (its
                    // selection bits are clear, so it takes no part)
#pragma unroll
                    for (int x = 0; x < D / 64; ++x)
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int kb = (h && td.kb1 >= 0) ? td.kb1 : td.kb0;
                            tma_load_3d(dst + x * HALF_BYTES + h * (64 * 128), tm64, BAR(FULLB + s), 64 * x,
                                        kb * 64, bh);
                        }
                }
            }
            __syncwarp();
            if (s == 0) issued[0] = jj;
            else issued[1] = jj;
        }
        // Every copy this warp issued lands before the CTA exits, whether or not a
        // wait gave up (another role may abort after this warp left its loop): the
        // Q tile, then the last load of each ring slot (earlier ones completed
        // before their slot was refilled).  Free on the normal path.
        if (is_k) wait_drain(BAR(B_QFULL), 0, kDrainLimitNs);
        if (issued[0] >= 0) wait_drain(BAR(FULLB), (issued[0] >> 1) & 1, kDrainLimitNs);
        if (issued[1] >= 0) wait_drain(BAR(FULLB + 1), (issued[1] >> 1) & 1, kDrainLimitNs);
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        // Descriptors are formed once and advanced by constant offsets; each group
        // of MMAs (and its commits) is issued by one elected lane.
        constexpr uint32_t idesc_qk = idesc_bf16_f32(BM, BN, false);
        constexpr uint32_t idesc_pv = idesc_bf16_f32(BM, D, true);
        const uint64_t qdesc = smem_desc_sw128(base + OFF_Q, 16, 1024);          // K-major Q
        const uint64_t kdesc0 = smem_desc_sw128(base + OFF_K, 16, 1024);         // K-major K
        // V is MN-major: 64-wide column boxes LBO = 16 KB apart, 8-key row groups
        // SBO = 1 KB apart; 16 keys (2 KB) per MMA
        const uint64_t vdesc0 = smem_desc_sw128(base + OFF_V, HALF_BYTES, 1024);
        bool ok = __all_sync(FULL, mbar_wait(BAR(B_QFULL), 0, abort_flag, status, lim));
        auto issue_pv = [&](const TileDesc& td, int ii) -> bool {  // the ii-th processed tile
            const int b = ii & 1;
            const uint32_t ph = (ii >> 1) & 1;
            if (!__all_sync(FULL, mbar_wait(BAR(B_PREADY + b), ph, abort_flag, status, lim))) return false;
            if (!__all_sync(FULL, mbar_wait(BAR(B_VFULL + b), ph, abort_flag, status, lim))) return false;
            fence_after_sync();
            const uint64_t vd = desc_add(vdesc0, b * TILE_BYTES);
            const uint32_t sb = tmem + (b ? TM_S1 : TM_S0);
            bool s0[2], s1[2];
            sel_half(td, 0, s0[0], s1[0]);
            sel_half(td, 1, s0[1], s1[1]);
            if (elect_one()) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t bd = desc_add(vd, (4 * h + kk) * 2048);
                        // half h's P sits in the first 32 columns of its own S range,
                        // the complementary ("alt") copy of a mixed half in the next 32
                        const uint32_t pa = sb + 64 * h + 8 * kk;
                        if (kSparse) {  // rows that do not select the half hold P = 0
                            if (s0[h] || s1[h]) mma_ts(tmem + TM_OSEL, pa, bd, idesc_pv, 1);
                        } else if (s0[h] == s1[h]) {
                            mma_ts(tmem + (s0[h] ? TM_OSEL : TM_OUNS), pa, bd, idesc_pv, 1);
                        } else {
                            mma_ts(tmem + TM_OSEL, pa, bd, idesc_pv, 1);
                            mma_ts(tmem + TM_OUNS, pa + 32, bd, idesc_pv, 1);
                        }
                    }
                }
                mma_commit(BAR(B_VEMPTY + b));
                mma_commit(BAR(B_PVDONE));
            }
            __syncwarp();
            return true;
        };
        int jj = 0;
        TileDesc tdprev = {0, 0, 0};
        for (; ok && jj < ntiles; ++jj) {
            const TileDesc td = tile_desc(jj);
            const int s = jj & 1;
            if (!__all_sync(FULL, mbar_wait(BAR(B_KFULL + s), (jj >> 1) & 1, abort_flag, status, lim))) {
                ok = false;
                break;
            }
            fence_after_sync();
            const uint64_t kd = desc_add(kdesc0, s * TILE_BYTES);
            const uint32_t sd = tmem + (s ? TM_S1 : TM_S0);
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    // K-major, 128B swizzle: 16 bf16 of d = 32 bytes per MMA step
                    const uint32_t off = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
                    mma_ss(sd, desc_add(qdesc, off), desc_add(kd, off), idesc_qk, kk > 0 ? 1u : 0u);
                }
                mma_commit(BAR(B_SREADY + s));
                mma_commit(BAR(B_KEMPTY + s));
            }
            __syncwarp();
            if (jj >= 1 && !issue_pv(tdprev, jj - 1)) ok = false;
            tdprev = td;
        }
        if (ok && jj > 0) issue_pv(tdprev, jj - 1);
        if (elect_one()) mma_commit(BAR(B_DRAIN));  // all MMAs complete before teardown
        __syncwarp();
        wait_drain(BAR(B_DRAIN), 0, kDrainLimitNs);
    } else if (warp >= 4) {
        // ------------------------------------------- two softmax warpgroups
        // Warpgroup h (= wg) owns keys [64h, 64h+64) of every tile and the
        // columns [64h, 64h+64) of O_sel / O_uns.  The row max is combined
        // through shared memory once per tile; l_sel / l_uns and the squared
        // difference are combined in the epilogue.
        const int wg = (warp - 4) >> 2, sw = (warp - 4) & 3;
        const int r = sw * 32 + lane;  // row of the tile == TMEM lane
        const uint32_t trow = tmem + ((uint32_t)(sw * 32) << 16);
        const int c0 = 64 * wg;          // this warpgroup's S columns (keys)
        constexpr int OC = D / 2;        // and its O columns
        const int oc0 = OC * wg;
        float* xch = reinterpret_cast<float*>(gbase + OFF_XCH);  // [parity][wg][row]
        // named barrier of the two warpgroups; the votes also OR a flag across the
        // warps they join, so that they leave the tile loop at the same tile (same
        // barrier counts)
        auto wg_sync = [] { asm volatile("bar.sync 1, 256;" ::: "memory"); };
        // the per-tile row-max exchange only needs the two warps that hold the same
        // 32 rows (warps 4 + sw and 8 + sw, on the same scheduler): barrier 2 + sw
        auto pair_vote = [sw](bool flag) -> bool {
            uint32_t out;
            asm volatile(
                "{\n\t.reg .pred p, q;\n\t"
                "setp.ne.u32 q, %1, 0;\n\t"
                "bar.red.or.pred p, %2, 64, q;\n\t"
                "selp.u32 %0, 1, 0, p;\n\t}"
                : "=r"(out)
                : "r"((uint32_t)flag), "r"(2 + sw)
                : "memory");
            return out != 0;
        };
        auto wg_vote = [](bool flag) -> bool {
            uint32_t out;
            asm volatile(
                "{\n\t.reg .pred p, q;\n\t"
                "setp.ne.u32 q, %1, 0;\n\t"
                "bar.red.or.pred p, 1, 256, q;\n\t"
                "selp.u32 %0, 1, 0, p;\n\t}"
                : "=r"(out)
                : "r"((uint32_t)flag)
                : "memory");
            return out != 0;
        };
        {
            uint32_t z[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) z[i] = 0u;
#pragma unroll
            for (int x = 0; x < OC / 32; ++x) {
                tmem_st32(trow + TM_OSEL + oc0 + 32 * x, z);
                tmem_st32(trow + TM_OUNS + oc0 + 32 * x, z);
            }
            tmem_wait_st();
        }
        const float sl2 = a.scale_log2;
        float m2 = -INFINITY, lsel = 0.f, luns = 0.f;
        // this warpgroup's share of the row's weight on block 0 (keys < block of
        // key tile 0), rescaled with l_sel / l_uns: the attention-sink mass
        float lsink = 0.f;
        const bool sink_keys = !kSparse && a.sink != nullptr && c0 < a.block;
        bool ok = true;
        for (int jj = 0; jj < ntiles; ++jj) {  // jj: tiles processed so far (ring slot / phase)
            const TileDesc td = tile_desc(jj);
            const int j = td.j;  // -1 for a packed tile (never the diagonal)
            const int b = jj & 1;
            // warp-uniform outcome: the TMEM loads below are warp-collective
            const bool got = __all_sync(
                0xffffffffu, mbar_wait(BAR(B_SREADY + b), (jj >> 1) & 1, abort_flag, status, lim));
            const uint32_t sb = trow + (b ? TM_S1 : TM_S0) + c0;
            float s[64];
            if (got) {
                fence_after_sync();
                uint32_t u0[32], u1[32];
                tmem_ld32(sb, u0);
                tmem_ld32(sb + 32, u1);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    s[c] = __uint_as_float(u0[c]);
                    s[32 + c] = __uint_as_float(u1[c]);
                }
            } else {
#pragma unroll
                for (int c = 0; c < 64; ++c) s[c] = 0.f;
            }
            if (j == I) {  // diagonal tile: keys after the row are masked (and keys >= T)
#pragma unroll
                for (int c = 0; c < 64; ++c)
                    if (c0 + c > r) s[c] = -INFINITY;
            }
            bool s0, s1;
            sel_half(td, wg, s0, s1);
            const bool mixed = s0 != s1;
            const bool row_sel = mixed ? ((r < 64 || a.block == 128) ? s0 : s1) : s0;
            if (kSparse && !row_sel) {  // the sparse stream alone: this half is not attended
#pragma unroll
                for (int c = 0; c < 64; ++c) s[c] = -INFINITY;
            }
            float mx8[8];  // independent partial maxima (short dependency chains)
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                mx8[k] = max3(s[k], s[8 + k], s[16 + k]);
                mx8[k] = max3(mx8[k], s[24 + k], s[32 + k]);
                mx8[k] = max3(mx8[k], s[40 + k], s[48 + k]);
                mx8[k] = fmaxf(mx8[k], s[56 + k]);
            }
            float mx = max3(max3(mx8[0], mx8[1], mx8[2]), max3(mx8[3], mx8[4], mx8[5]),
                            fmaxf(mx8[6], mx8[7]));
            // The two warps holding these rows exchange their halves' maxima only
            // when the running max must move: on the first tile, or when either
            // half of some row exceeds it by more than the lazy-rescale threshold
            // (the same rows rescale as with an exchange on every tile, since
            // max(a, b) > t exactly when a > t or b > t).
            const bool moved = jj == 0 || mx * sl2 > m2 + kRescaleThreshold;
            if (pair_vote(moved || !got || *abort_flag)) {
                float* xm = xch + (jj & 1) * 256;
                xm[wg * 128 + r] = mx;
                if (pair_vote(!got || *abort_flag)) {  // a wait expired somewhere: both leave here
                    ok = false;
                    break;
                }
                mx = fmaxf(mx, xm[(1 - wg) * 128 + r]);
                const float mnew = mx * sl2;
                if (jj == 0) {
                    m2 = mnew;
                } else {
                const bool need = mnew > m2 + kRescaleThreshold;
                // PV_{j-1} must have landed in O before it is rescaled.  If that wait
                // expires the rescale is skipped and the abort flag ends the loop at
                // the next vote.
                if (__any_sync(0xffffffffu, need) &&
                    __all_sync(0xffffffffu, mbar_wait(BAR(B_PVDONE), (jj - 1) & 1, abort_flag,
                                                      status, lim))) {
                    fence_after_sync();
                    const float mup = fmaxf(m2, mnew);
                    const float alpha = ex2(m2 - mup);
                    m2 = mup;
                    lsel *= alpha;
                    luns *= alpha;
                    lsink *= alpha;
                    constexpr int NCH = OC / 32;  // 32-column chunks per accumulator
#pragma unroll 1
                    for (int c = 0; c < (kSparse ? NCH : 2 * NCH); ++c) {
                        const uint32_t col = (c < NCH ? TM_OSEL : TM_OUNS) + oc0 + 32 * (c % NCH);
                        uint32_t u[32];
                        tmem_ld32(trow + col, u);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(__uint_as_float(u[i]) * alpha);
                        tmem_st32(trow + col, u);
                    }
                    tmem_wait_st();
                }
                }
            }
            const float negm = -m2;
            // sparse stream alone: rows with no attended key yet, or whose half is not
            // attended, contribute P = 0 (no exponentials)
            const bool zero_p = kSparse && (!row_sel || !(m2 > -INFINITY));
            // p = 2^(s*sigma*log2e - m), two columns at a time (packed f32x2).  Off
            // the diagonal three eighths of the pairs take the FMA-pipe exponential so
            // that the MUFU unit is not the limit; on the diagonal every pair uses
            // the MUFU, whose 2^-inf = 0 keeps masked keys exact.
            const f32x2 sl2x2 = mk2(sl2, sl2), nm2 = mk2(negm, negm);
            f32x2 acc[4] = {mk2(0.f, 0.f), mk2(0.f, 0.f), mk2(0.f, 0.f), mk2(0.f, 0.f)};
            uint32_t pk[32];
            if (zero_p) {
#pragma unroll
                for (int c = 0; c < 32; ++c) pk[c] = 0u;
            } else if (j == I) {
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    float x0, x1;
                    un2(fma2(mk2(s[2 * c], s[2 * c + 1]), sl2x2, nm2), x0, x1);
                    const float p0 = ex2(x0), p1 = ex2(x1);
                    acc[c & 3] = add2(acc[c & 3], mk2(p0, p1));
                    pk[c] = pack_bf16(p0, p1);
                }
            } else {
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    const f32x2 x2 = fma2(mk2(s[2 * c], s[2 * c + 1]), sl2x2, nm2);
                    float p0, p1;
                    if (poly_pair(c)) {
                        un2(exp2_poly2(x2), p0, p1);
                    } else {
                        float x0, x1;
                        un2(x2, x0, x1);
                        p0 = ex2(x0);
                        p1 = ex2(x1);
                    }
                    acc[c & 3] = add2(acc[c & 3], mk2(p0, p1));
                    pk[c] = pack_bf16(p0, p1);
                }
            }
            float a0, a1, b0, b1;
            un2(add2(acc[0], acc[1]), a0, a1);
            un2(add2(acc[2], acc[3]), b0, b1);
            const float sum = (a0 + a1) + (b0 + b1);
            if (kSparse || !mixed) {
                tmem_st32(sb, pk);
            } else {
                uint32_t main_[32], alt[32];
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    main_[c] = row_sel ? pk[c] : 0u;
                    alt[c] = row_sel ? 0u : pk[c];
                }
                tmem_st32(sb, main_);
                tmem_st32(sb + 32, alt);
            }
            if (row_sel) lsel += sum;
            else luns += sum;
            if (j == 0 && sink_keys) lsink = sum;
            tmem_wait_st();
            fence_before_sync();
            mbar_arrive(BAR(B_PREADY + b));
        }
        // Every MMA (the last PV included) has completed once B_DRAIN has.  A
        // parity wait on B_PVDONE for the last tile is not enough: the softmax
        // only knows that the PV two tiles back has landed, and a barrier one
        // phase behind reports the wanted parity as complete.
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(BAR(B_DRAIN), 0, abort_flag, status, lim));
        // both warpgroups take the same decision and the same barriers below
        ok = !wg_vote(!ok || *abort_flag);
        float* xl = xch;  // [wg][sel|uns][row] reuses the max exchange area
        xl[(wg * 2) * 128 + r] = lsel;
        xl[(wg * 2 + 1) * 128 + r] = luns;
        wg_sync();
        const float Ls = lsel + xl[((1 - wg) * 2) * 128 + r];
        const int t = t0 + r;
        const bool valid = t < a.T;
        const size_t row = (size_t)bh * a.T + (valid ? t : 0);
        // The output tiles go through shared memory (the K ring, free once every
        // MMA has completed) in the 128-byte-swizzled [128 rows x 64 columns]
        // boxes of the output tensor maps, and leave by TMA stores: a thread owns
        // a row, so direct stores would scatter each warp's writes over 32 rows.
        // Rows past T are clipped by the tensor map.
        uint8_t* stage = gbase + OFF_K;  // h_sparse boxes, then h_full boxes (dual)
        constexpr uint32_t kOutBytes = BM * D * 2;
        const uint32_t rowoff = (uint32_t)(r >> 3) * 1024 + (uint32_t)(r & 7) * 128;
        // 16-byte chunk v (8 columns) of output columns [col0, col0 + 32): box col/64
        auto put = [&](uint8_t* tile, int col0, const uint32_t (&h)[16]) {
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                const int col = col0 + 8 * v;
                const uint32_t chunk = (uint32_t)((col & 63) >> 3) ^ (uint32_t)(r & 7);
                *reinterpret_cast<uint4*>(tile + (col >> 6) * HALF_BYTES + rowoff + chunk * 16) =
                    make_uint4(h[4 * v], h[4 * v + 1], h[4 * v + 2], h[4 * v + 3]);
            }
        };
        // one thread stores the staged tile(s) once every row is written
        auto store_tiles = [&](bool dual) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            wg_sync();
            if (warp == 4 && lane == 0 && ok) {
#pragma unroll
                for (int x = 0; x < D / 64; ++x) {
                    tma_store_3d(&tm_hs, base + OFF_K + x * HALF_BYTES, 64 * x, t0, bh);
                    if (dual) tma_store_3d(&tm_hf, base + OFF_K + kOutBytes + x * HALF_BYTES, 64 * x, t0, bh);
                }
                bulk_commit_group();
                bulk_wait_group_read0();  // the staging area stays valid until read
            }
        };
        if constexpr (kSparse) {
            // the diagonal block holds key t itself, so Ls > 0 on valid rows
            if (ok) {
                fence_after_sync();
                const float inv_ls = Ls > 0.f ? 1.f / Ls : 0.f;
#pragma unroll 1
                for (int c = 0; c < OC / 32; ++c) {
                    uint32_t os[32];
                    tmem_ld32(trow + TM_OSEL + oc0 + 32 * c, os);
                    tmem_wait_ld();
                    uint32_t hs[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        hs[e] = pack_bf16(__uint_as_float(os[2 * e]) * inv_ls,
                                          __uint_as_float(os[2 * e + 1]) * inv_ls);
                    put(stage, oc0 + 32 * c, hs);
                }
                if (wg == 0 && valid)
                    a.lse_sparse[row] = Ls > 0.f ? (m2 + log2f(Ls)) * kLn2 : -INFINITY;
            }
            store_tiles(false);
        } else {
            const float Lu = luns + xl[((1 - wg) * 2 + 1) * 128 + r];
            float sq = 0.f;
            if (ok) {
                fence_after_sync();
                const float l = Ls + Lu;
                const float inv_l = 1.f / l;
                const float inv_ls = Ls > 0.f ? 1.f / Ls : 0.f;
#pragma unroll 1
                for (int c = 0; c < OC / 32; ++c) {
                    uint32_t os[32], ou[32];
                    tmem_ld32(trow + TM_OSEL + oc0 + 32 * c, os);
                    tmem_ld32(trow + TM_OUNS + oc0 + 32 * c, ou);
                    tmem_wait_ld();
                    uint32_t hf[16], hs[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const float sa = __uint_as_float(os[2 * e]), sb2 = __uint_as_float(os[2 * e + 1]);
                        const float ua = __uint_as_float(ou[2 * e]), ub = __uint_as_float(ou[2 * e + 1]);
                        const float fa = (sa + ua) * inv_l, fb = (sb2 + ub) * inv_l;
                        const float pa = sa * inv_ls, pb = sb2 * inv_ls;
                        sq = fmaf(fa - pa, fa - pa, sq);
                        sq = fmaf(fb - pb, fb - pb, sq);
                        hf[e] = pack_bf16(fa, fb);
                        hs[e] = pack_bf16(pa, pb);
                    }
                    put(stage, oc0 + 32 * c, hs);
                    put(stage + kOutBytes, oc0 + 32 * c, hf);
                }
            }
            float* xs = xch + 512;  // [wg][row] squared-difference partials
            float* xk = xch + 768;  // [wg][row] block-0 weight partials
            xs[wg * 128 + r] = sq;
            xk[wg * 128 + r] = lsink;
            store_tiles(true);  // (its barrier also publishes xs, xk)
            if (ok && wg == 0 && valid) {
                const float l = Ls + Lu;
                a.delta[row] = Lu / l;
                a.lse_full[row] = (m2 + log2f(l)) * kLn2;
                a.lse_sparse[row] = Ls > 0.f ? (m2 + log2f(Ls)) * kLn2 : -INFINITY;
                a.sqdiff[row] = sq + xs[128 + r];
                if (a.sink) a.sink[row] = (lsink + xk[128 + r]) / l;
            }
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        fence_after_sync();
        tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------- host side
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

// [BH, T, D] bf16 viewed as a 3-D tensor (d, t, bh); box = 64 d x `rows` t
// (128 by default), 128-byte swizzle; rows past T are zero-filled by the TMA
// unit.
int make_map(CUtensorMap* m, const void* ptr, int BH, int T, int D, int rows = BM) {
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

}  // namespace

bool fwd_tc_supported(const ssa_params_t& p) {
    return p.dtype == SSA_BF16 && (p.D == 64 || p.D == 128) && (p.block == 64 || p.block == 128) &&
           mask_words(p) <= kMaxWords && (size_t)p.B * p.H * ((p.T + BM - 1) / BM) <= 0x7fffffffull;
}

size_t fwd_tc_workspace(const ssa_params_t&) { return 0; }

namespace {
template <int D, bool kSparse>
int launch_fwd_tc_impl(const ssa_params_t& p, const void* q, const void* k, const void* v,
                       const uint32_t* mask, const FwdArgs& outs, cudaStream_t s) {
    const int BH = p.B * p.H;
    CUtensorMap mq, mk, mv, mk64, mv64, mhf, mhs;
    int st = make_map(&mq, q, BH, p.T, D);
    if (st == SSA_OK) st = make_map(&mk, k, BH, p.T, D);
    if (st == SSA_OK) st = make_map(&mv, v, BH, p.T, D);
    // 64-row boxes: the halves of the sparse-only forward's packed tiles
    if (st == SSA_OK) st = make_map(&mk64, k, BH, p.T, D, 64);
    if (st == SSA_OK) st = make_map(&mv64, v, BH, p.T, D, 64);
    if (st == SSA_OK) st = make_map(&mhs, outs.h_sparse, BH, p.T, D);
    // the sparse-only kernel writes h_sparse alone (the h_full map is not used)
    if (st == SSA_OK) st = make_map(&mhf, kSparse ? outs.h_sparse : outs.h_full, BH, p.T, D);
    if (st != SSA_OK) return st;
    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once, [] {
        attr_err = cudaFuncSetAttribute(fwd_tc_kernel<D, kSparse>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    });
    if (attr_err != cudaSuccess)
        return fail(SSA_ERR_CUDA, "fwd_tc: smem attribute: %s", cudaGetErrorString(attr_err));
    FwdArgs a = outs;
    a.mask = mask;
    a.BH = BH;
    a.T = p.T;
    a.block = p.block;
    a.words = mask_words(p);
    a.n_blocks = num_blocks(p);
    a.scale_log2 = p.sm_scale * 1.4426950408889634f;
    a.timeout_ns = wait_limit_ns();
    const unsigned grid = (unsigned)((size_t)BH * ((p.T + BM - 1) / BM));
    fwd_tc_kernel<D, kSparse><<<grid, kThreads, SMEM_BYTES, s>>>(mq, mk, mv, mk64, mv64, mhf, mhs, a);
    return check_launch(kSparse ? "fwd_tc_kernel<sparse>" : "fwd_tc_kernel");
}
}  // namespace

int launch_fwd_tc(const ssa_params_t& p, const void* q, const void* k, const void* v,
                  const uint32_t* mask, void* hf, void* hs, float* delta, float* lf, float* ls,
                  float* sq, float* sink, void*, cudaStream_t s) {
    FwdArgs o{};
    o.h_full = static_cast<__nv_bfloat16*>(hf);
    o.h_sparse = static_cast<__nv_bfloat16*>(hs);
    o.delta = delta;
    o.lse_full = lf;
    o.lse_sparse = ls;
    o.sqdiff = sq;
    o.sink = sink;
    return p.D == 64 ? launch_fwd_tc_impl<64, false>(p, q, k, v, mask, o, s)
                     : launch_fwd_tc_impl<128, false>(p, q, k, v, mask, o, s);
}

int launch_fwd_sparse_tc(const ssa_params_t& p, const void* q, const void* k, const void* v,
                         const uint32_t* mask, void* hs, float* ls, cudaStream_t s) {
    FwdArgs o{};
    o.h_sparse = static_cast<__nv_bfloat16*>(hs);
    o.lse_sparse = ls;
    return p.D == 64 ? launch_fwd_tc_impl<64, true>(p, q, k, v, mask, o, s)
                     : launch_fwd_tc_impl<128, true>(p, q, k, v, mask, o, s);
}

int fwd_tc_take_status(cudaStream_t) {
    unsigned int v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_fwd_tc_status, sizeof v);
    if (e != cudaSuccess) return fail(SSA_ERR_CUDA, "status read: %s", cudaGetErrorString(e));
    if (v) {
        const unsigned int zero = 0;
        cudaMemcpyToSymbol(g_fwd_tc_status, &zero, sizeof zero);
        return fail(SSA_ERR_TIMEOUT, "fwd_tc_kernel: a bounded mbarrier wait expired");
    }
    return SSA_OK;
}

}  // namespace ssa
