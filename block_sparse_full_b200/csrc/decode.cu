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
//        lanes over d, float64) and stores each score, as an integer order
//        key, into every CTA of the cluster; cluster barrier;
//     2. the selection: each candidate counts the candidates ahead of it
//        under (score desc, index asc), several lanes per candidate; every
//        CTA ranks all candidates, or, when there are many, the CTAs split
//        them and share the kept bits (one more cluster barrier); then every
//        CTA builds the ascending list;
//     3. every CTA streams the keys and values of its selected blocks (list
//        slots rank, rank + cluster, ...) into shared memory with bulk copies,
//        all of a pass in flight at once, and runs one online softmax over
//        them: the partial (max, sum, o) goes to the leader, followed by a
//        release arrival on the leader's mbarrier;
//     4. the leader waits for the other CTAs' arrivals (bounded) and merges
//        the partials into h and the log-sum-exp.
#include <cooperative_groups.h>
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>
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

// candidates above which the cluster's CTAs split the ranking (each counts for
// every kCluster-th candidate; one more cluster barrier)
constexpr int kSplitRankMin = 192;

__device__ unsigned int g_decode_status;

// Shared memory of the step kernel, the same layout in every CTA of a cluster:
//   order keys of the block scores [nb] u64 (every CTA holds all of them) |
//   set bitmask [nb / 32 + 1] u32 | selected blocks [topk] i32 | popcount
//   prefix of the bitmask words [nb / 32 + 2] i32 | partials [cluster][2 + D]
//   f32 (the leader's are used) | attention scores [nbuf * block] f32 |
//   p [nbuf * block] bf16 | o partial sums [KG][D] f32 | mbarriers (copies,
//   partials) | keys [nbuf][block][D] T (bf16: per block, D / 64 tiles
//   [block][64] in the 128-byte swizzle) | values likewise.
struct StepSmem {
    size_t key, bits, sel, wpre, part, ps, pb, og, bar, kbuf, vbuf, total;
    __host__ __device__ StepSmem(int nb, int topk, int D, int cluster, int nbuf, int block, int esize,
                                 int threads) {
        auto up = [](size_t x, size_t a) { return (x + a - 1) / a * a; };
        key = 0;
        bits = key + (size_t)nb * 8;
        sel = bits + ((size_t)nb / 32 + 1) * 4;
        wpre = sel + (size_t)topk * 4;
        part = up(wpre + ((size_t)nb / 32 + 2) * 4, 16);
        ps = part + (size_t)cluster * (2 + D) * 4;
        pb = ps + (size_t)nbuf * block * 4;
        og = up(pb + (size_t)nbuf * block * 2, 16);
        bar = og + (size_t)(threads / (D / 8)) * D * 4;
        kbuf = up(bar + 16, 1024);
        vbuf = kbuf + (size_t)nbuf * block * D * esize;
        total = vbuf + (size_t)nbuf * block * D * esize + 1024;  // + room to align the base
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

// Tensor-core fragments (mma.sync m16n8k16, bf16 in, f32 accumulate) and the
// shared-memory matrix loads that feed them.
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr)
                 : "memory");
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr)
                 : "memory");
}
__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// The selection order (score desc, index asc) on integers: the float64 score
// mapped to a u64 whose unsigned order is the score's order (-0 taken as +0,
// so that equal scores give equal keys).
__device__ __forceinline__ uint64_t order_key(double x) {
    const uint64_t b = (uint64_t)__double_as_longlong(x == 0.0 ? 0.0 : x);
    return (b >> 63) ? ~b : (b | 0x8000000000000000ull);
}

// kCluster: CTAs per head; NT: threads per CTA (both chosen by the host from
// the head count).
// nbuf: selected blocks whose keys and values fit in shared memory at once.
template <typename T, int D, int kCluster, int NT>
__global__ void __launch_bounds__(NT, 1)
decode_step_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                   const double* __restrict__ kbar, int nb, int Tcap, int block, int t, int topk,
                   bool force_sink, float scale, int nbuf, uint64_t limit_ns, T* __restrict__ h,
                   float* __restrict__ lse, int32_t* __restrict__ idx_out) {
    constexpr int M = D / 32;                   // pooled-key columns per lane (scores)
    constexpr int U = 4;                        // pooled-key rows in flight per warp
    constexpr int W = 16 / (int)sizeof(T);      // elements of a 16-byte piece
    constexpr int P = D / (8 * W);              // pieces per lane of a key row (8 lanes per key)
    constexpr int CH = D / 8;                   // 8-column chunks of a value row
    constexpr int KG = NT / CH;                 // key groups of P V
    constexpr int kStepThreads = NT;
    constexpr int kStepWarps = NT / 32;
    extern __shared__ __align__(128) unsigned char sm_raw[];
    __shared__ float red[2][kStepWarps];
    __shared__ int nsel_s;
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const size_t bh = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int i = t / block;
    const int words = (i >> 5) + 1;  // bits 0 .. i
    const StepSmem L(nb, topk, D, kCluster, nbuf, block, (int)sizeof(T), NT);
    // the 128-byte swizzle of the TMA tiles follows address bits 7-9: the
    // layout starts on a 1024-byte boundary (the same offset in every CTA)
    unsigned char* sm = sm_raw + ((1024u - (smem_u32(sm_raw) & 1023u)) & 1023u);
    uint64_t* key = reinterpret_cast<uint64_t*>(sm + L.key);
    uint32_t* bits = reinterpret_cast<uint32_t*>(sm + L.bits);
    int32_t* sel = reinterpret_cast<int32_t*>(sm + L.sel);
    int32_t* wpre = reinterpret_cast<int32_t*>(sm + L.wpre);
    float* part = reinterpret_cast<float*>(sm + L.part);
    float* ps = reinterpret_cast<float*>(sm + L.ps);
    __nv_bfloat16* pb = reinterpret_cast<__nv_bfloat16*>(sm + L.pb);
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
    // the score's order key into CTA r's array: every CTA ends up with all of them.
    {
        double qr[M];
#pragma unroll
        for (int m = 0; m < M; ++m) qr[m] = (double)to_f32(q[bh * D + lane + 32 * m]);
        const double* kb = kbar + bh * (size_t)nb * D;
        uint64_t* key_r = cluster.map_shared_rank(key, lane < kCluster ? lane : 0);
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
                    if (j < i) key_r[j] = order_key(a[u]);
                }
            }
        }
    }
    cluster.sync();  // all scores in every CTA; the mbarrier inits visible cluster-wide

    // 2. the selection: forced blocks, then candidate j (first <= j < i) is kept
    // iff fewer than r candidates come before it in (key desc, index asc).  nseg
    // lanes of a warp count for one candidate, each over every nseg-th rival, four
    // rivals per iteration.  Past kSplitRankMin candidates the CTAs of the cluster
    // split them (CTA rank counts for candidates rank, rank + kCluster, ...) and
    // OR their bitmask words into every other CTA (one remote reduction per word
    // and CTA, all in flight at once).  Then every thread places the set bits it
    // owns by a popcount prefix of the words: the ascending list.
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
        const bool split = ncand > kSplitRankMin && ncand > r;  // the same in every CTA
        if (ncand <= r) {
            for (int j = first + tid; j < i; j += NT) atomicOr(&bits[j >> 5], 1u << (j & 31));
        } else {
            const int c0 = split ? rank : 0, cstep = split ? kCluster : 1;
            const int mc = (ncand - c0 + cstep - 1) / cstep;  // candidates counted here
            int nseg = 1;
            while (nseg < 32 && nseg * 2 * mc <= NT) nseg *= 2;
            const int per = NT / nseg;  // candidates per sweep
            const int seg = tid % nseg;
            for (int base = 0; base < mc; base += per) {  // the same trip count in every thread
                const int ci = base + tid / nseg;
                const bool live = ci < mc;
                const int j = first + c0 + cstep * (live ? ci : 0);
                const uint64_t kj = key[j];
                int a0 = 0, a1 = 0, a2 = 0, a3 = 0;
                int j2 = first + seg;
                for (; j2 + 3 * nseg < i; j2 += 4 * nseg) {
                    const uint64_t x0 = key[j2], x1 = key[j2 + nseg], x2 = key[j2 + 2 * nseg],
                                   x3 = key[j2 + 3 * nseg];
                    a0 += (int)((x0 > kj) | ((x0 == kj) & (j2 < j)));
                    a1 += (int)((x1 > kj) | ((x1 == kj) & (j2 + nseg < j)));
                    a2 += (int)((x2 > kj) | ((x2 == kj) & (j2 + 2 * nseg < j)));
                    a3 += (int)((x3 > kj) | ((x3 == kj) & (j2 + 3 * nseg < j)));
                }
                for (; j2 < i; j2 += nseg) {
                    const uint64_t x0 = key[j2];
                    a0 += (int)((x0 > kj) | ((x0 == kj) & (j2 < j)));
                }
                int ahead = (a0 + a1) + (a2 + a3);
                for (int off = nseg >> 1; off > 0; off >>= 1) ahead += __shfl_xor_sync(0xffffffffu, ahead, off);
                if (live && seg == 0 && ahead < r) atomicOr(&bits[j >> 5], 1u << (j & 31));
            }
        }
        __syncthreads();  // this CTA's bits are complete
        if (split) {
            for (int e = tid; e < words * (kCluster - 1); e += NT) {
                const int w = e % words, q2 = 1 + e / words;
                const uint32_t wv = bits[w];
                if (wv != 0u) atomicOr(cluster.map_shared_rank(bits, (rank + q2) % kCluster) + w, wv);
            }
            cluster.sync();  // every CTA's kept bits are in every CTA
        }
        if (warp == 0) {  // popcount prefix of the words, 32 at a time
            int basep = 0;
            for (int w0 = 0; w0 < words; w0 += 32) {
                const int w = w0 + lane;
                const int c = w < words ? __popc(bits[w]) : 0;
                int incl = c;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const int o = __shfl_up_sync(0xffffffffu, incl, off);
                    if (lane >= off) incl += o;
                }
                if (w < words) wpre[w] = basep + incl - c;
                basep += __shfl_sync(0xffffffffu, incl, 31);
            }
            if (lane == 0) nsel_s = basep < topk ? basep : topk;
        }
        __syncthreads();
        int32_t* irow = (idx_out && rank == 0) ? idx_out + bh * topk : nullptr;
        for (int j = tid; j <= i; j += NT) {
            const uint32_t wv = bits[j >> 5];
            if ((wv >> (j & 31)) & 1u) {
                const int pos = wpre[j >> 5] + __popc(wv & ((1u << (j & 31)) - 1u));
                if (pos < topk) {  // NaN scores: stay in bounds
                    sel[pos] = j;
                    if (irow) irow[pos] = j;
                }
            }
        }
        if (irow)
            for (int pp = nsel_s + tid; pp < topk; pp += NT) irow[pp] = -1;
        __syncthreads();
    }

    // 3. this CTA's slots rank, rank + kCluster, ... of the list, nbuf blocks per
    // pass: one thread streams the blocks' keys and values into shared memory
    // (every block of the pass in flight at once), then one online softmax over
    // the CTA's keys (running max and sum).
    //   bf16: TMA tiles [block rows x 64 columns], 128-byte swizzle; scores and
    //   P V on the tensor cores (mma.sync m16n8k16, f32 accumulate), with the
    //   keys as the M dimension of the scores (one MMA = 16 keys x 16 columns of
    //   the query) and V^T as the M dimension of P V (ldmatrix.trans); the
    //   diagonal block's value rows past t are zeroed before P V.
    //   f32: bulk copies; scores with 8 lanes per key, P V with a thread per
    //   (8-column chunk, key group), on the CUDA cores.
    const int nsel = nsel_s;
    const int mine = nsel > rank ? (nsel - rank + kCluster - 1) / kCluster : 0;
    float m_run = -INFINITY, l_run = 0.f;
    constexpr bool kMma = sizeof(T) == 2;
    constexpr int DT = D / 16;                  // 16-column tiles of the head dim (MMA path)
    constexpr int KGM = kStepWarps / DT;         // key groups of P V (MMA path)
    const int gq = lane >> 2, tq = lane & 3;     // MMA fragment coordinates
    float oc[4] = {0.f, 0.f, 0.f, 0.f};          // MMA path: o[16 dt + gq], o[16 dt + gq + 8] (tq == 0)
    float o8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};  // CUDA-core path
    const int kc = lane & 7, kw = lane >> 3;     // CUDA-core scores: chunk and key within the warp
    const int c8 = tid % CH, g = tid / CH;        // CUDA-core P V
    uint32_t qb[DT][2];                           // MMA path: B fragments of q (lanes gq == 0)
    float qv[P][W];                               // CUDA-core path
    if constexpr (kMma) {
#pragma unroll
        for (int kk = 0; kk < DT; ++kk) {
            const uint32_t* q32 = reinterpret_cast<const uint32_t*>(q + bh * D + 16 * kk);
            qb[kk][0] = gq == 0 ? q32[tq] : 0u;
            qb[kk][1] = gq == 0 ? q32[4 + tq] : 0u;
        }
    } else {
#pragma unroll
        for (int m = 0; m < P; ++m) {
            const T* qp = q + bh * D + (8 * m + kc) * W;
#pragma unroll
            for (int z = 0; z < W; ++z) qv[m][z] = to_f32(qp[z]);
        }
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
            if constexpr (kMma) {
                mbar_expect_tx(bar_copy, (uint32_t)nbp * 2u * (uint32_t)block * D * 2u);
                for (int b = 0; b < nbp; ++b) {
                    const int j = sel[rank + kCluster * (p0 + b)];
#pragma unroll
                    for (int x = 0; x < D / 64; ++x) {
                        const uint32_t off = (uint32_t)((b * D / 64 + x) * block * 128);
                        tma_load_3d(smem_u32(kbuf) + off, &tm_k, bar_copy, 64 * x, j * block, (int)bh);
                        tma_load_3d(smem_u32(vbuf) + off, &tm_v, bar_copy, 64 * x, j * block, (int)bh);
                    }
                }
            } else {
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
        }
        if (!__syncthreads_and(wait_phase(bar_copy, pass & 1, false, limit_ns))) {
            // a copy did not land in time: wait (bounded) for it before the
            // buffers are given up, and give no partial
            wait_phase(bar_copy, pass & 1, false, kDrainLimitNs);
            ok = false;
            break;
        }
        const int nkp = nbp * block;
        if constexpr (kMma) {
            // scores: warp w takes the 16-key tiles w, w + 16, ...; A = 16 keys x 16
            // columns (ldmatrix), B = q (column 0), lane (gq, 0) gets keys gq, gq + 8
            const uint32_t kb0 = smem_u32(kbuf);
            for (int s0 = 16 * warp; s0 < nkp; s0 += 16 * kStepWarps) {
                const int b = s0 / block, rb0 = s0 % block;
                const int mi = lane >> 3, row = rb0 + (lane & 7) + 8 * (mi & 1);
                const uint32_t rbase = kb0 + (uint32_t)(b * D / 64) * block * 128 + (uint32_t)row * 128;
                float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int kk = 0; kk < DT; ++kk) {
                    const int chunk = 2 * kk + (mi >> 1);
                    const uint32_t addr = rbase + (uint32_t)(chunk >> 3) * block * 128 +
                                          (uint32_t)(((chunk & 7) ^ (row & 7)) << 4);
                    uint32_t a[4];
                    ldsm_x4(addr, a);
                    mma_bf16(c, a, qb[kk]);
                }
                if (tq == 0) {
                    const int nks = nks_of(b);
                    ps[s0 + gq] = rb0 + gq < nks ? c[0] * scale : -INFINITY;
                    ps[s0 + gq + 8] = rb0 + gq + 8 < nks ? c[2] * scale : -INFINITY;
                }
            }
            // the diagonal block's value rows past t hold whatever the cache
            // holds there: zero them (P is 0 there, and 0 * NaN is NaN)
            for (int b = 0; b < nbp; ++b) {
                const int nks = nks_of(b);
                if (nks == block) continue;
                uint4* vb = reinterpret_cast<uint4*>(vbuf + (size_t)b * block * D);
                const int nzero = (block - nks) * (D / 8);  // 16-byte chunks
                for (int e = tid; e < nzero; e += kStepThreads) {
                    const int rr = nks + e / (D / 8), cc = e % (D / 8);
                    vb[((cc >> 3) * block + rr) * 8 + (cc & 7)] = make_uint4(0u, 0u, 0u, 0u);
                }
            }
        } else {
            for (int s0 = 4 * warp; s0 < nkp; s0 += 4 * kStepWarps) {
                const int s = s0 + kw;
                const int b = s / block, rr = s % block;
                const bool valid = s < nkp && rr < nks_of(b < nbp ? b : 0);
                float acc = 0.f;
                if (valid) {
                    const T* row = kbuf + (size_t)s * D;
#pragma unroll
                    for (int m = 0; m < P; ++m) {
                        const float4 a4 = *reinterpret_cast<const float4*>(row + (8 * m + kc) * W);
                        acc = fmaf(qv[m][0], a4.x, acc);
                        acc = fmaf(qv[m][1], a4.y, acc);
                        acc = fmaf(qv[m][2], a4.z, acc);
                        acc = fmaf(qv[m][3], a4.w, acc);
                    }
                }
                acc += __shfl_xor_sync(0xffffffffu, acc, 4);
                acc += __shfl_xor_sync(0xffffffffu, acc, 2);
                acc += __shfl_xor_sync(0xffffffffu, acc, 1);
                if (kc == 0 && s < nkp) ps[s] = valid ? acc * scale : -INFINITY;
            }
        }
        __syncthreads();
        float mx = -INFINITY;
        for (int s2 = tid; s2 < nkp; s2 += kStepThreads) mx = fmaxf(mx, ps[s2]);
        mx = warp_max(mx);
        if (lane == 0) red[0][warp] = mx;
        __syncthreads();
        float m_new = m_run;
#pragma unroll
        for (int w = 0; w < kStepWarps; ++w) m_new = fmaxf(m_new, red[0][w]);
        // every pass holds at least one key <= t, so m_new is finite
        const float alpha = m_run > -INFINITY ? expf(m_run - m_new) : 0.f;
        float ls = 0.f;
        for (int s2 = tid; s2 < nkp; s2 += kStepThreads) {
            const float x = ps[s2];
            const float pw = x > -INFINITY ? expf(x - m_new) : 0.f;
            if constexpr (kMma)
                pb[s2] = __float2bfloat16_rn(pw);
            else
                ps[s2] = pw;
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
        if constexpr (kMma) {
            // P V: warp w takes head-dim tile w % DT and the 16-key steps
            // w / DT, w / DT + KGM, ...; A = V^T (16 columns x 16 keys,
            // ldmatrix.trans), B = p (column 0)
#pragma unroll
            for (int z = 0; z < 4; ++z) oc[z] *= alpha;
            const int dt = warp % DT, kg = warp / DT;
            const uint32_t vb0 = smem_u32(vbuf);
            const uint32_t* p32 = reinterpret_cast<const uint32_t*>(pb);
            for (int s0 = 16 * kg; s0 < nkp; s0 += 16 * KGM) {
                const int b = s0 / block, rb0 = s0 % block;
                const int mi = lane >> 3, row = rb0 + (lane & 7) + 8 * (mi >> 1);
                const int chunk = 2 * dt + (mi & 1);
                const uint32_t addr = vb0 + (uint32_t)(b * D / 64 + (chunk >> 3)) * block * 128 +
                                      (uint32_t)row * 128 + (uint32_t)(((chunk & 7) ^ (row & 7)) << 4);
                uint32_t a[4];
                ldsm_x4_trans(addr, a);
                uint32_t bp[2];
                bp[0] = gq == 0 ? p32[(s0 >> 1) + tq] : 0u;
                bp[1] = gq == 0 ? p32[(s0 >> 1) + 4 + tq] : 0u;
                mma_bf16(oc, a, bp);
            }
        } else {
#pragma unroll
            for (int z = 0; z < 8; ++z) o8[z] *= alpha;
            for (int s2 = g; s2 < nkp; s2 += KG) {
                const int b = s2 / block, rr = s2 % block;
                if (rr < nks_of(b)) {
                    float x[8];
                    load8(vbuf + (size_t)s2 * D + 8 * c8, x);
                    const float pw = ps[s2];
#pragma unroll
                    for (int z = 0; z < 8; ++z) o8[z] = fmaf(pw, x[z], o8[z]);
                }
            }
        }
        __syncthreads();  // ps, red and the buffers are reused by the next pass
    }

    // the CTA's partial (m, l, o) into the leader's slot `rank`
    int ngroups;
    if constexpr (kMma) {
        const int dt = warp % DT, kg = warp / DT;
        if (tq == 0) {
            og[kg * D + 16 * dt + gq] = oc[0];
            og[kg * D + 16 * dt + gq + 8] = oc[2];
        }
        ngroups = KGM;
    } else {
#pragma unroll
        for (int z = 0; z < 8; ++z) og[g * D + 8 * c8 + z] = o8[z];
        ngroups = KG;
    }
    __syncthreads();
    float* part_l = cluster.map_shared_rank(part, 0) + rank * (2 + D);
    for (int c = tid; c < D; c += kStepThreads) {
        float o = 0.f;
        for (int gg = 0; gg < ngroups; ++gg) o += og[gg * D + c];
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
    if (!__syncthreads_and(wait_phase(bar_part, 0, true, limit_ns))) {
        // The others write their partials into this CTA's shared memory before
        // they arrive, so it must not exit while one may still write.  Each of
        // them gives up after at most one expired wait per pass (this CTA has
        // the most passes) and one drain: wait that long again (bounded), then
        // leave with the status already recorded and no output.
        const int npass = (mine + nbuf - 1) / nbuf;
        wait_phase(bar_part, 0, true, (uint64_t)(npass + 1) * limit_ns + kDrainLimitNs);
        return;
    }
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

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult qr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qr) == cudaSuccess &&
            qr == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// the bf16 key or value cache [BH, T, D] as a 3-D tensor (d, t, bh); box 64 d x
// `rows` t; 128-byte swizzle
static int make_kv_map(CUtensorMap* m, const void* ptr, int BH, int T, int rows, int D) {
    auto fn = encode_fn();
    if (!fn) return fail(SSA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)T, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)T * D * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)rows, 1};
    cuuint32_t es[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(SSA_ERR_CUDA, "cuTensorMapEncodeTiled (decode) failed (%d)", (int)r);
    return SSA_OK;
}

// CTAs per head and threads per CTA of the step, by the number of heads and
// the budget.
struct DecodeShape {
    int cluster, threads;
};
// Measured at 8192 to 65536 tokens of context (CUDA graph, L2 flushed): eight
// heads or fewer take clusters of 8 x 512 threads; up to 16 heads with at most
// two selected blocks per CTA take 8 x 256 (16.4 vs 18.4 us at 16 heads,
// top-k 16); up to 32 heads, 4 x 512 (at top-k 64, 16 heads: 32.8 us vs 40.9
// with clusters of 8); more heads, 4 x 256 (128 heads: 28.7 vs 45.1 us).
static DecodeShape decode_shape_for(int BH, int topk) {
    if (BH <= 8) return {8, 512};
    if (BH <= 16 && (topk + 7) / 8 <= 2) return {8, 256};
    if (BH <= 32) return {4, 512};
    return {4, 256};
}

int launch_decode_step(const ssa_params_t& p, int t, const void* q, const void* k, const void* v,
                       const double* kbar, void* h, float* lse, int32_t* idx, void*,
                       cudaStream_t s) {
    const int BH = p.B * p.H;
    const int nb = num_blocks(p);
    const bool sink = (p.flags & SSA_FLAG_FORCE_SINK) != 0;
    const int esize = p.dtype == SSA_BF16 ? 2 : 4;
    const DecodeShape shape = decode_shape_for(BH, p.topk);
    auto run = [&](auto tag, auto dtag, auto ctag, auto ntag) -> int {
        using T = decltype(tag);
        constexpr int D = decltype(dtag)::value;
        constexpr int kCluster = decltype(ctag)::value;
        constexpr int NT = decltype(ntag)::value;
        auto kern = decode_step_kernel<T, D, kCluster, NT>;
        size_t limit = 0;
        int st = opt_in_max_smem<decode_step_kernel<T, D, kCluster, NT>>("decode_step_kernel", &limit);
        if (st != SSA_OK) return st;
        // as many of a CTA's selected blocks per pass as shared memory holds
        const int per_cta = (p.topk + kCluster - 1) / kCluster;
        const size_t fixed = StepSmem(nb, p.topk, D, kCluster, 0, p.block, esize, NT).total;
        const size_t per_block = StepSmem(nb, p.topk, D, kCluster, 1, p.block, esize, NT).total - fixed + 16;
        int nbuf = limit > fixed ? (int)((limit - fixed) / per_block) : 0;
        if (nbuf > per_cta) nbuf = per_cta;
        while (nbuf > 1 && StepSmem(nb, p.topk, D, kCluster, nbuf, p.block, esize, NT).total > limit) --nbuf;
        if (nbuf < 1)
            return fail(SSA_ERR_UNSUPPORTED, "decode: T/block = %d blocks leave no room for a key block in shared memory",
                        nb);
        const size_t smem = StepSmem(nb, p.topk, D, kCluster, nbuf, p.block, esize, NT).total;
        if (smem > limit)
            return fail(SSA_ERR_UNSUPPORTED, "decode: %zu bytes of shared memory needed (limit %zu)", smem, limit);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)kCluster, (unsigned)BH);
        cfg.blockDim = dim3(NT);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = kCluster;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        CUtensorMap mk{}, mv{};  // bf16 only: [B*H, T, D] as (d, t, bh), box 64 x block x 1
        if constexpr (sizeof(T) == 2) {
            st = make_kv_map(&mk, k, BH, p.T, p.block, D);
            if (st == SSA_OK) st = make_kv_map(&mv, v, BH, p.T, p.block, D);
            if (st != SSA_OK) return st;
        }
        cudaError_t e = cudaLaunchKernelEx(&cfg, kern, mk, mv, static_cast<const T*>(q), static_cast<const T*>(k),
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
    using N256 = std::integral_constant<int, 256>;
    using N512 = std::integral_constant<int, 512>;
    auto with_cluster = [&](auto tag, auto dtag) -> int {
        if (shape.cluster == 8)
            return shape.threads == 256 ? run(tag, dtag, C8{}, N256{}) : run(tag, dtag, C8{}, N512{});
        return shape.threads == 256 ? run(tag, dtag, C4{}, N256{}) : run(tag, dtag, C4{}, N512{});
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
