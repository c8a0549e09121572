// One generation step of the sparse stream over a key/value cache ("Sintesi
// Tecnica: SSA", section 4, "Efficienza": at inference SSA runs the same
// operations as MoBA).  The pages do not describe decoding itself; the
// reading here is MoBA's inference rule: the current query q_t is scored
// against the pooled keys Kbar_j of the completed blocks j < i = t / block
// (float64, like the training-time scores), the current block i is always
// attended (keys 0..t of it) and counts inside the budget k, block 0 is
// forced only with SSA_FLAG_FORCE_SINK, the remaining places go to the best
// scores (ties to the lower index), and the step attends over every key of
// the selected blocks up to t.
//
// Launches (CUDA cores: one query per head is matrix-vector work, bound by
// the key/value bytes it reads and, at this size, by latency):
//   decode_pool_kernel   Kbar_j = mean of block j's keys (float64, exact)
//   decode_step_kernel   one cluster of 8 (or 4) CTAs per head; distributed
//                        shared memory carries the hand-offs, one cluster
//                        barrier in all:
//     1. every CTA scores its share of the completed blocks (warp per block,
//        lanes over d, float64) and stores each score into every CTA of the
//        cluster; cluster barrier;
//     2. every CTA takes the same selection from the same scores (each
//        candidate counts the candidates ahead of it under (score desc,
//        index asc), several lanes per candidate) and builds the ascending
//        list;
//     3. every CTA streams the keys and values of its selected blocks (list
//        slots rank, rank + cluster, ...) into shared memory with bulk copies,
//        all of a pass in flight at once, and runs one online softmax over
//        them: the partial (max, sum, o) goes to the leader, followed by a
//        release arrival on the leader's mbarrier;
//     4. the leader waits for the other CTAs' arrivals (bounded) and merges
//        the partials into h and the log-sum-exp.
#include <cooperative_groups.h>
#include <type_traits>

#include "device_util.cuh"
#include "ssa_internal.h"
#include "tc_util.cuh"

namespace cg = cooperative_groups;

namespace ssa {
namespace {

using namespace tc;

constexpr int kThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kThreads)
decode_pool_kernel(const T* __restrict__ k, int Tcap, int D, int block, int j0,
                   double* __restrict__ kbar, int nb) {
    const int j = j0 + blockIdx.x;
    const size_t bh = blockIdx.y;
    const T* src = k + (bh * Tcap + (size_t)j * block) * D;
    for (int c = threadIdx.x; c < D; c += kThreads) {
        double acc = 0.0;
        for (int r = 0; r < block; ++r) acc += (double)to_f32(src[(size_t)r * D + c]);
        kbar[(bh * nb + j) * D + c] = acc / (double)block;  // block is a power of two: exact
    }
}

// 8 consecutive elements of a row as float (16 bytes for bf16, 32 for f32;
// the address is a multiple of 16 bytes)
template <typename T>
__device__ __forceinline__ void load8(const T* p, float (&x)[8]) {
    if constexpr (sizeof(T) == 2) {
        const uint4 u = *reinterpret_cast<const uint4*>(p);
        const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
        for (int z = 0; z < 8; ++z) x[z] = to_f32(e[z]);
    } else {
        const float4 a = *reinterpret_cast<const float4*>(p);
        const float4 b = *reinterpret_cast<const float4*>(p + 4);
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
        x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
    }
}

constexpr int kStepThreads = 512;
constexpr int kStepWarps = kStepThreads / 32;

__device__ unsigned int g_decode_status;

// Shared memory of the step kernel, the same layout in every CTA of a cluster:
//   score [nb] f64 (every CTA holds all scores) | set bitmask [nb / 32 + 1] u32 |
//   selected blocks [topk] i32 | partials [cluster][2 + D] f32 (the leader's
//   are used) | p [nbuf * block] f32 | o partial sums [KG][D] f32 |
//   mbarriers (copies, partials) | keys [nbuf][block][D] T | values likewise.
struct StepSmem {
    size_t score, bits, sel, part, ps, og, bar, kbuf, vbuf, total;
    __host__ __device__ StepSmem(int nb, int topk, int D, int cluster, int nbuf, int block, int esize) {
        auto up = [](size_t x, size_t a) { return (x + a - 1) / a * a; };
        score = 0;
        bits = score + (size_t)nb * 8;
        sel = bits + ((size_t)nb / 32 + 1) * 4;
        part = up(sel + (size_t)topk * 4, 16);
        ps = part + (size_t)cluster * (2 + D) * 4;
        og = up(ps + (size_t)nbuf * block * 4, 16);
        bar = og + (size_t)(kStepThreads / (D / 8)) * D * 4;
        kbuf = up(bar + 16, 128);
        vbuf = kbuf + (size_t)nbuf * block * D * esize;
        total = vbuf + (size_t)nbuf * block * D * esize;
    }
};

__device__ __forceinline__ uint32_t cluster_map(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}
// one-dimensional bulk copy global -> this CTA's shared memory, completing on `bar`
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
        : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// bounded wait (wall clock); on a timeout ORs 1 into the status word
__device__ __forceinline__ bool wait_phase(uint32_t bar, uint32_t parity, bool cluster_scope,
                                           uint64_t limit_ns) {
    const uint64_t t0 = globaltimer();
    for (;;) {
        if (cluster_scope ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity)) return true;
        if (globaltimer() - t0 > limit_ns) {
            atomicOr(&g_decode_status, 1u);
            return false;
        }
    }
}

// kCluster: CTAs per head, 8 or 4 (chosen by the host from the head count).
// nbuf: selected blocks whose keys and values fit in shared memory at once.
template <typename T, int D, int kCluster>
__global__ void __launch_bounds__(kStepThreads, 1)
decode_step_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                   const double* __restrict__ kbar, int nb, int Tcap, int block, int t, int topk,
                   bool force_sink, float scale, int nbuf, uint64_t limit_ns, T* __restrict__ h,
                   float* __restrict__ lse, int32_t* __restrict__ idx_out) {
    constexpr int M = D / 32;                   // pooled-key columns per lane (scores)
    constexpr int U = 4;                        // pooled-key rows in flight per warp
    constexpr int W = 16 / (int)sizeof(T);      // elements of a 16-byte piece
    constexpr int P = D / (8 * W);              // pieces per lane of a key row (8 lanes per key)
    constexpr int CH = D / 8;                   // 8-column chunks of a value row
    constexpr int KG = kStepThreads / CH;       // key groups of P V
    extern __shared__ __align__(128) unsigned char sm[];
    __shared__ float red[2][kStepWarps];
    __shared__ int nsel_s;
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const size_t bh = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int i = t / block;
    const int words = (i >> 5) + 1;  // bits 0 .. i
    const StepSmem L(nb, topk, D, kCluster, nbuf, block, (int)sizeof(T));
    double* score = reinterpret_cast<double*>(sm + L.score);
    uint32_t* bits = reinterpret_cast<uint32_t*>(sm + L.bits);
    int32_t* sel = reinterpret_cast<int32_t*>(sm + L.sel);
    float* part = reinterpret_cast<float*>(sm + L.part);
    float* ps = reinterpret_cast<float*>(sm + L.ps);
    float* og = reinterpret_cast<float*>(sm + L.og);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L.bar);
    T* kbuf = reinterpret_cast<T*>(sm + L.kbuf);
    T* vbuf = reinterpret_cast<T*>(sm + L.vbuf);
    const uint32_t bar_copy = smem_u32(&bars[0]), bar_part = smem_u32(&bars[1]);
    if (tid == 0) {
        mbar_init(bar_copy, 1);
        mbar_init(bar_part, kCluster - 1);  // one arrival per other CTA (used by the leader)
        fence_mbar_init();
    }
    for (int w = tid; w < words; w += kStepThreads) bits[w] = 0u;

    // 1. scores of the completed blocks j < i: block j goes to CTA j % kCluster,
    // warp (j / kCluster) % 16; lane l owns columns l, l + 32, ... (coalesced rows of
    // the float64 pooled keys), U rows in flight per warp.  Lane r < kCluster stores
    // the score into CTA r's array: every CTA ends up with all of them.
    {
        double qr[M];
#pragma unroll
        for (int m = 0; m < M; ++m) qr[m] = (double)to_f32(q[bh * D + lane + 32 * m]);
        const double* kb = kbar + bh * (size_t)nb * D;
        double* score_r = cluster.map_shared_rank(score, lane < kCluster ? lane : 0);
        for (int c0 = rank + kCluster * warp; c0 < i; c0 += kCluster * kStepWarps * U) {
            double a[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int j = c0 + kCluster * kStepWarps * u;
                const double* kr = kb + (size_t)min(j, i - 1) * D + lane;  // past the end: unused
                double acc = 0.0;
#pragma unroll
                for (int m = 0; m < M; ++m) acc = fma(qr[m], kr[32 * m], acc);
                a[u] = acc;
            }
#pragma unroll
            for (int u = 0; u < U; ++u) a[u] = warp_sum(a[u]);
            if (lane < kCluster) {
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int j = c0 + kCluster * kStepWarps * u;
                    if (j < i) score_r[j] = a[u];
                }
            }
        }
    }
    cluster.sync();  // all scores in every CTA; the mbarrier inits visible cluster-wide

    // 2. every CTA selects (the same decision from the same scores): forced
    // blocks, then candidate j (first <= j < i) is kept iff fewer than r
    // candidates come before it in (score desc, index asc).  nseg lanes of a
    // warp count for one candidate, each over every nseg-th rival.
    {
        const bool sink = force_sink && i > 0;
        const int want = topk < i + 1 ? topk : i + 1;  // fewer candidates than places: take all
        const int first = sink ? 1 : 0;                // candidates are first .. i-1
        const int r = want - (sink ? 2 : 1);           // free slots (>= 0: a sink needs topk >= 2)
        const int ncand = i - first;
        if (tid == 0) {  // atomic: other threads may set bits of the same words meanwhile
            atomicOr(&bits[i >> 5], 1u << (i & 31));
            if (sink) atomicOr(&bits[0], 1u);
        }
        int nseg = 1;
        while (nseg < 32 && nseg * 2 * ncand <= kStepThreads) nseg *= 2;
        const int per = kStepThreads / nseg;  // candidates per sweep
        const int seg = tid % nseg;
        for (int base = 0; base < ncand; base += per) {  // the same trip count in every thread
            const int cidx = base + tid / nseg;
            const bool live = cidx < ncand;
            const int j = first + (live ? cidx : 0);
            const double sj = score[j];
            int ahead = 0;
            for (int j2 = first + seg; j2 < i; j2 += nseg) {
                const double a0 = score[j2];
                ahead += (a0 > sj || (a0 == sj && j2 < j)) ? 1 : 0;
            }
            for (int off = nseg >> 1; off > 0; off >>= 1) ahead += __shfl_xor_sync(0xffffffffu, ahead, off);
            if (live && seg == 0 && ahead < r) atomicOr(&bits[j >> 5], 1u << (j & 31));
        }
        __syncthreads();
        if (warp == 0) {  // the ascending list (-1 padded) by popcount prefix
            int32_t* irow = (idx_out && rank == 0) ? idx_out + bh * topk : nullptr;
            int basep = 0;
            for (int w0 = 0; w0 < words; w0 += 32) {
                const int w = w0 + lane;
                const uint32_t wv = w < words ? bits[w] : 0u;
                const int c = __popc(wv);
                int incl = c;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const int o = __shfl_up_sync(0xffffffffu, incl, off);
                    if (lane >= off) incl += o;
                }
                int pos = basep + incl - c;
                for (uint32_t b = wv; b != 0u; b &= b - 1u, ++pos) {
                    if (pos < topk) {  // NaN scores: stay in bounds
                        const int vv = w * 32 + __ffs(b) - 1;
                        sel[pos] = vv;
                        if (irow) irow[pos] = vv;
                    }
                }
                basep += __shfl_sync(0xffffffffu, incl, 31);
            }
            if (irow)
                for (int pp = basep + lane; pp < topk; pp += 32) irow[pp] = -1;
            if (lane == 0) nsel_s = basep < topk ? basep : topk;
        }
        __syncthreads();
    }

    // 3. this CTA's slots rank, rank + kCluster, ... of the list, nbuf blocks per
    // pass: one thread streams the blocks' keys and values into shared memory
    // with bulk copies (every block of the pass in flight at once), then
    //   scores: 8 lanes per key, 16-byte pieces (8m + c) * W of the row;
    //   online softmax over the CTA's keys (running max and sum);
    //   P V: thread (8-column chunk, key group), rescaled with the max.
    const int nsel = nsel_s;
    const int mine = nsel > rank ? (nsel - rank + kCluster - 1) / kCluster : 0;
    float m_run = -INFINITY, l_run = 0.f;
    float o8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    const int kc = lane & 7, kw = lane >> 3;     // score phase: chunk and key within the warp
    const int c8 = tid % CH, g = tid / CH;        // P V phase
    float qv[P][W];
#pragma unroll
    for (int m = 0; m < P; ++m) {
        const T* qp = q + bh * D + (8 * m + kc) * W;
#pragma unroll
        for (int z = 0; z < W; ++z) qv[m][z] = to_f32(qp[z]);
    }
    bool ok = true;
    int pass = 0;
    for (int p0 = 0; p0 < mine && ok; p0 += nbuf, ++pass) {
        const int nbp = min(nbuf, mine - p0);
        auto nks_of = [&](int b) {  // keys <= t of the pass's block b
            const int j = sel[rank + kCluster * (p0 + b)];
            return min((j + 1) * block, t + 1) - j * block;
        };
        if (tid == 0) {
            // the previous pass's reads of the buffers (ordered by the barrier that
            // ended it) come before the copies' writes
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            uint32_t bytes = 0;
            for (int b = 0; b < nbp; ++b) bytes += 2u * (uint32_t)nks_of(b) * D * (uint32_t)sizeof(T);
            mbar_expect_tx(bar_copy, bytes);
            for (int b = 0; b < nbp; ++b) {
                const int j = sel[rank + kCluster * (p0 + b)];
                const uint32_t nbytes = (uint32_t)nks_of(b) * D * (uint32_t)sizeof(T);
                const size_t src = (bh * Tcap + (size_t)j * block) * D;
                bulk_load(smem_u32(kbuf + (size_t)b * block * D), k + src, nbytes, bar_copy);
                bulk_load(smem_u32(vbuf + (size_t)b * block * D), v + src, nbytes, bar_copy);
            }
        }
        if (!__syncthreads_and(wait_phase(bar_copy, pass & 1, false, limit_ns))) {
            // a copy did not land in time: wait (bounded) for it before the
            // buffers are given up, and give no partial
            wait_phase(bar_copy, pass & 1, false, kDrainLimitNs);
            ok = false;
            break;
        }
        const int nkp = nbp * block;
        for (int s0 = 4 * warp; s0 < nkp; s0 += 4 * kStepWarps) {
            const int s = s0 + kw;
            const int b = s / block, rr = s % block;
            const bool valid = s < nkp && rr < nks_of(b < nbp ? b : 0);
            float acc = 0.f;
            if (valid) {
                const T* row = kbuf + (size_t)s * D;
#pragma unroll
                for (int m = 0; m < P; ++m) {
                    float x[8];
                    if constexpr (W == 8) {
                        load8(row + (8 * m + kc) * W, x);
#pragma unroll
                        for (int z = 0; z < 8; ++z) acc = fmaf(qv[m][z], x[z], acc);
                    } else {
                        const float4 a4 = *reinterpret_cast<const float4*>(row + (8 * m + kc) * W);
                        acc = fmaf(qv[m][0], a4.x, acc);
                        acc = fmaf(qv[m][1], a4.y, acc);
                        acc = fmaf(qv[m][2], a4.z, acc);
                        acc = fmaf(qv[m][3], a4.w, acc);
                    }
                }
            }
            acc += __shfl_xor_sync(0xffffffffu, acc, 4);
            acc += __shfl_xor_sync(0xffffffffu, acc, 2);
            acc += __shfl_xor_sync(0xffffffffu, acc, 1);
            if (kc == 0 && s < nkp) ps[s] = valid ? acc * scale : -INFINITY;
        }
        __syncthreads();
        float mx = -INFINITY;
        for (int s = tid; s < nkp; s += kStepThreads) mx = fmaxf(mx, ps[s]);
        mx = warp_max(mx);
        if (lane == 0) red[0][warp] = mx;
        __syncthreads();
        float m_new = m_run;
#pragma unroll
        for (int w = 0; w < kStepWarps; ++w) m_new = fmaxf(m_new, red[0][w]);
        // every pass holds at least one key <= t, so m_new is finite
        const float alpha = m_run > -INFINITY ? expf(m_run - m_new) : 0.f;
        float ls = 0.f;
        for (int s = tid; s < nkp; s += kStepThreads) {
            const float x = ps[s];
            const float pw = x > -INFINITY ? expf(x - m_new) : 0.f;
            ps[s] = pw;
            ls += pw;
        }
        ls = warp_sum(ls);
        if (lane == 0) red[1][warp] = ls;
        __syncthreads();
        float lp = 0.f;
#pragma unroll
        for (int w = 0; w < kStepWarps; ++w) lp += red[1][w];
        l_run = l_run * alpha + lp;
        m_run = m_new;
#pragma unroll
        for (int z = 0; z < 8; ++z) o8[z] *= alpha;
        for (int s = g; s < nkp; s += KG) {
            const int b = s / block, rr = s % block;
            if (rr < nks_of(b)) {
                float x[8];
                load8(vbuf + (size_t)s * D + 8 * c8, x);
                const float pw = ps[s];
#pragma unroll
                for (int z = 0; z < 8; ++z) o8[z] = fmaf(pw, x[z], o8[z]);
            }
        }
        __syncthreads();  // ps, red and the buffers are reused by the next pass
    }

    // the CTA's partial (m, l, o) into the leader's slot `rank`
#pragma unroll
    for (int z = 0; z < 8; ++z) og[g * D + 8 * c8 + z] = o8[z];
    __syncthreads();
    float* part_l = cluster.map_shared_rank(part, 0) + rank * (2 + D);
    for (int c = tid; c < D; c += kStepThreads) {
        float o = 0.f;
        for (int gg = 0; gg < KG; ++gg) o += og[gg * D + c];
        part_l[2 + c] = ok ? o : 0.f;
    }
    if (tid == 0) {
        part_l[0] = ok ? m_run : -INFINITY;
        part_l[1] = ok ? l_run : 0.f;
    }
    __syncthreads();
    if (rank != 0) {
        if (tid == 0) {
            asm volatile("fence.acq_rel.cluster;" ::: "memory");
            asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(
                             cluster_map(bar_part, 0))
                         : "memory");
        }
        return;  // no other CTA reads this CTA's shared memory from here on
    }

    // 4. the leader merges the partials once the other CTAs' have arrived:
    // weights e^{m_r - M}
    if (!__syncthreads_and(wait_phase(bar_part, 0, true, limit_ns))) return;
    __shared__ float wgt[8];
    if (warp == 0) {
        const float mr = lane < kCluster ? part[lane * (2 + D)] : -INFINITY;
        const float Mx = warp_max(mr);
        const float w = (lane < kCluster && mr > -INFINITY) ? expf(mr - Mx) : 0.f;
        if (lane < kCluster) wgt[lane] = w;
        const float Ls = warp_sum(lane < kCluster ? w * part[lane * (2 + D) + 1] : 0.f);
        if (lane == 0) {
            red[0][0] = Ls;
            lse[bh] = Mx + logf(Ls);
        }
    }
    __syncthreads();
    const float inv_L = 1.f / red[0][0];
    for (int c = tid; c < D; c += kStepThreads) {
        float acc = 0.f;
#pragma unroll
        for (int r = 0; r < kCluster; ++r) acc = fmaf(wgt[r], part[r * (2 + D) + 2 + c], acc);
        h[bh * D + c] = from_f32<T>(acc * inv_L);
    }
}

}  // namespace

// the step keeps everything in the clusters' shared memory: no workspace
size_t decode_workspace(const ssa_params_t&) { return 0; }

int launch_decode_pool(const ssa_params_t& p, int j0, int j1, const void* k, double* kbar,
                       cudaStream_t s) {
    if (j1 <= j0) return SSA_OK;
    const dim3 grid((unsigned)(j1 - j0), (unsigned)(p.B * p.H));
    const int nb = num_blocks(p);
    if (p.dtype == SSA_BF16)
        decode_pool_kernel<__nv_bfloat16><<<grid, kThreads, 0, s>>>(
            static_cast<const __nv_bfloat16*>(k), p.T, p.D, p.block, j0, kbar, nb);
    else
        decode_pool_kernel<float><<<grid, kThreads, 0, s>>>(static_cast<const float*>(k), p.T, p.D,
                                                            p.block, j0, kbar, nb);
    return check_launch("decode_pool_kernel");
}

int launch_decode_step(const ssa_params_t& p, int t, const void* q, const void* k, const void* v,
                       const double* kbar, void* h, float* lse, int32_t* idx, void*,
                       cudaStream_t s) {
    const int BH = p.B * p.H;
    const int nb = num_blocks(p);
    const bool sink = (p.flags & SSA_FLAG_FORCE_SINK) != 0;
    const int esize = p.dtype == SSA_BF16 ? 2 : 4;
    // 8 CTAs per head while every head's cluster fits in one wave (a cluster of
    // 8 CTAs of 512 threads takes 8 SMs of one GPC; measured: 8 clusters at a
    // time), else 4
    const int cl = BH <= 8 ? 8 : 4;
    auto run = [&](auto tag, auto dtag, auto ctag) -> int {
        using T = decltype(tag);
        constexpr int D = decltype(dtag)::value;
        constexpr int kCluster = decltype(ctag)::value;
        auto kern = decode_step_kernel<T, D, kCluster>;
        size_t limit = 0;
        int st = opt_in_max_smem<decode_step_kernel<T, D, kCluster>>("decode_step_kernel", &limit);
        if (st != SSA_OK) return st;
        // as many of a CTA's selected blocks per pass as shared memory holds
        const int per_cta = (p.topk + kCluster - 1) / kCluster;
        const size_t fixed = StepSmem(nb, p.topk, D, kCluster, 0, p.block, esize).total;
        const size_t per_block = StepSmem(nb, p.topk, D, kCluster, 1, p.block, esize).total - fixed + 16;
        int nbuf = limit > fixed ? (int)((limit - fixed) / per_block) : 0;
        if (nbuf > per_cta) nbuf = per_cta;
        while (nbuf > 1 && StepSmem(nb, p.topk, D, kCluster, nbuf, p.block, esize).total > limit) --nbuf;
        if (nbuf < 1)
            return fail(SSA_ERR_UNSUPPORTED, "decode: T/block = %d blocks leave no room for a key block in shared memory",
                        nb);
        const size_t smem = StepSmem(nb, p.topk, D, kCluster, nbuf, p.block, esize).total;
        if (smem > limit)
            return fail(SSA_ERR_UNSUPPORTED, "decode: %zu bytes of shared memory needed (limit %zu)", smem, limit);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)kCluster, (unsigned)BH);
        cfg.blockDim = dim3(kStepThreads);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = kCluster;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        cudaError_t e = cudaLaunchKernelEx(&cfg, kern, static_cast<const T*>(q), static_cast<const T*>(k),
                                           static_cast<const T*>(v), kbar, nb, p.T, p.block, t, p.topk,
                                           sink, p.sm_scale, nbuf, (uint64_t)wait_limit_ns(),
                                           static_cast<T*>(h), lse, idx);
        if (e != cudaSuccess) return fail(SSA_ERR_CUDA, "decode_step_kernel: %s", cudaGetErrorString(e));
        return check_launch("decode_step_kernel");
    };
    using D64 = std::integral_constant<int, 64>;
    using D128 = std::integral_constant<int, 128>;
    using C4 = std::integral_constant<int, 4>;
    using C8 = std::integral_constant<int, 8>;
    auto with_cluster = [&](auto tag, auto dtag) -> int {
        return cl == 8 ? run(tag, dtag, C8{}) : run(tag, dtag, C4{});
    };
    if (p.dtype == SSA_BF16)
        return p.D == 64 ? with_cluster(__nv_bfloat16{}, D64{}) : with_cluster(__nv_bfloat16{}, D128{});
    return p.D == 64 ? with_cluster(float{}, D64{}) : with_cluster(float{}, D128{});
}

int decode_take_status() {
    unsigned int v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_decode_status, sizeof v);
    if (e != cudaSuccess) return fail(SSA_ERR_CUDA, "status read: %s", cudaGetErrorString(e));
    if (v != 0) {
        const unsigned int zero = 0;
        cudaMemcpyToSymbol(g_decode_status, &zero, sizeof zero);
        return fail(SSA_ERR_TIMEOUT, "decode step: a wait for copies or partials expired");
    }
    return SSA_OK;
}

}  // namespace ssa
