// Block selection for callers that cannot allocate device memory.
//
// ssa_select_blocks needs a caller-provided scratch buffer (the float64 block
// means of Q and K).  Some host programs cannot produce one at the point
// where they run selection: a plugin loaded into a serving process whose
// memory pool owns all device memory and exposes no allocator to plugins, or
// a latency-critical loop that must not call cudaMalloc after start-up
// (cudaMalloc can synchronise the device and stall every other stream).
// ssa_select_blocks_noalloc serves them with a scratch buffer that lives in
// this library's own device memory: a file-scope array that every GPU which
// loads the library holds until the process exits.
//
// Host code cannot use the array's name as a device address (on the host it
// names a shadow variable), so the device address is looked up once per
// device with cudaGetSymbolAddress, while that device is current, on the
// first call made on it.
#include <mutex>

#include "ssa_internal.h"

namespace {

// 16 MiB: enough for B*H*(T/block)*D <= 1,048,576, e.g. B=4 H=32 T=4096
// block=64 d=128 or B=1 H=8 T=65536 block=128 d=128.
constexpr size_t kScratchBytes = 16u << 20;
static __device__ __align__(256) unsigned char g_select_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_select_scratch on the current device (looked up on
// first use, then cached).  Returns an SSA status.
int scratch_address(void** out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return ssa::fail(SSA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices)
        return ssa::fail(SSA_ERR_UNSUPPORTED, "device index %d beyond %d", dev, kMaxDevices);
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_select_scratch);
        if (e != cudaSuccess || !p)
            return ssa::fail(SSA_ERR_CUDA, "cudaGetSymbolAddress(select scratch): %s",
                             cudaGetErrorString(e));
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return SSA_OK;
}

}  // namespace

extern "C" int ssa_select_blocks_noalloc(const ssa_params_t* p, const void* q, const void* k,
                                         int32_t* idx, int32_t* cnt, uint32_t* mask,
                                         void* stream) {
    const size_t need = ssa_workspace_size(p, SSA_WS_SELECT);
    if (need == (size_t)-1) return SSA_ERR_INVALID_ARG;  // detail already recorded
    if (need > kScratchBytes)
        return ssa::fail(SSA_ERR_UNSUPPORTED,
                         "ssa_select_blocks_noalloc: these shapes need %zu bytes of scratch but the "
                         "built-in scratch holds %zu (B*H*(T/block)*D must be <= %zu); call "
                         "ssa_select_blocks with a caller-allocated workspace instead",
                         need, kScratchBytes, kScratchBytes / (2 * sizeof(double)));
    void* scratch = nullptr;
    const int st = scratch_address(&scratch);
    if (st != SSA_OK) return st;
    // The pooling kernel writes every block mean before the scoring kernel
    // reads it, so leftovers from an earlier call never need clearing.
    return ssa_select_blocks(p, q, k, idx, cnt, mask, scratch, kScratchBytes, stream);
}
