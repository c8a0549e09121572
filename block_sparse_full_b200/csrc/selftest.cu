// Element-wise self-test of the arithmetic the tensor-core kernels build on:
// the FMA-pipe exponential, the MUFU exponential and the integer-ALU bf16
// packing, evaluated exactly as the kernels evaluate them so that a test can
// hold them against float64 exp2 and round-to-nearest-even bf16.
#include "ssa_internal.h"
#include "tc_util.cuh"

namespace ssa {
namespace {

__global__ void selftest_kernel(const float* __restrict__ x, int n, float* __restrict__ e_poly,
                                float* __restrict__ e_mufu, uint16_t* __restrict__ bf) {
    const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
    if (i >= n) return;
    const float x0 = x[i], x1 = i + 1 < n ? x[i + 1] : 0.f;
    float p0, p1;
    tc::un2(tc::exp2_poly2(tc::mk2(x0, x1)), p0, p1);
    const uint32_t packed = tc::pack_bf16_alu(x0, x1);
    e_poly[i] = p0;
    e_mufu[i] = tc::ex2(x0);
    bf[i] = (uint16_t)(packed & 0xFFFFu);
    if (i + 1 < n) {
        e_poly[i + 1] = p1;
        e_mufu[i + 1] = tc::ex2(x1);
        bf[i + 1] = (uint16_t)(packed >> 16);
    }
}

__device__ unsigned int g_selftest_status;

// One thread waits, with the kernels' bounded wait, on an mbarrier that no
// one ever arrives at: the wait must give up after `limit_ns` and record the
// expiry in this file's device status word.
__global__ void wait_timeout_kernel(unsigned long long limit_ns, int* __restrict__ gave_up) {
    __shared__ __align__(8) unsigned long long bar;
    __shared__ int abort_flag;
    const uint32_t b = tc::smem_u32(&bar);
    tc::mbar_init(b, 1);
    tc::fence_mbar_init();
    abort_flag = 0;
    const bool ok = tc::mbar_wait(b, 0, &abort_flag, &g_selftest_status, limit_ns);
    *gave_up = ok ? 0 : 1;
}

}  // namespace

int selftest_take_status() {
    unsigned int v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_selftest_status, sizeof v);
    if (e != cudaSuccess) return fail(SSA_ERR_CUDA, "status read: %s", cudaGetErrorString(e));
    if (v) {
        const unsigned int zero = 0;
        cudaMemcpyToSymbol(g_selftest_status, &zero, sizeof zero);
        return fail(SSA_ERR_TIMEOUT, "self-test: a bounded mbarrier wait expired");
    }
    return SSA_OK;
}

}  // namespace ssa

extern "C" int ssa_selftest_wait_timeout(unsigned long long limit_ns, int* gave_up, void* stream) {
    if (!gave_up || limit_ns == 0 || limit_ns > 10000000000ull)
        return ssa::fail(SSA_ERR_INVALID_ARG, "ssa_selftest_wait_timeout: bad arguments");
    ssa::wait_timeout_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns, gave_up);
    return ssa::check_launch("wait_timeout_kernel");
}

extern "C" int ssa_selftest_math(const float* x, int n, float* exp2_poly, float* exp2_mufu,
                                 uint16_t* bf16_alu, void* stream) {
    if (n < 0 || (n > 0 && (!x || !exp2_poly || !exp2_mufu || !bf16_alu)))
        return ssa::fail(SSA_ERR_INVALID_ARG, "ssa_selftest_math: bad arguments");
    if (n == 0) return SSA_OK;
    const int pairs = (n + 1) / 2;
    ssa::selftest_kernel<<<(pairs + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        x, n, exp2_poly, exp2_mufu, bf16_alu);
    return ssa::check_launch("selftest_kernel");
}
