// gptq_quantize_layer_noalloc: the column walk without a caller workspace.
//
// Some callers cannot hand this library a device workspace: a plugin or
// operator interface whose enqueue call is not allowed to allocate, a process
// whose memory pool has already reserved nearly all of HBM, or a latency-
// critical path that must not pay for cudaMalloc / cudaFree (which can
// synchronize the device).  This entry point takes the same inputs and
// outputs as gptq_quantize_layer but no `ws`: its scratch is one file-scope
// __device__ array that every GPU loading this library holds until the
// process exits.
//
// Set-up: the first call on each device (with that device current) looks up
// the array's device address with cudaGetSymbolAddress and caches it; host
// code must never pass the array's name itself to a kernel (in host code it
// is only a stand-in, not a device address).  Make that first call before any
// stream capture on the device.
//
// Sharing: all calls use the same array and it keeps whatever the last call
// left in it.  The column walk writes every scratch element it later reads
// within a call, so nothing needs to start at zero; two calls whose work
// overlaps on the GPU (different streams, no ordering) race on the array.
#include <mutex>

#include "kernels.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t{16} << 20;  // 16 MiB per device

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once
// per device.  Returns nullptr if the lookup fails.
void* scratch_on_current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (g_scratch_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
            return nullptr;
        g_scratch_ptr[dev] = p;
    }
    return g_scratch_ptr[dev];
}

}  // namespace

extern "C" size_t gptq_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

extern "C" gptq_status gptq_quantize_layer_noalloc(float* W, int64_t d_row, int64_t d_col,
                                                   int64_t ldw, const float* U,
                                                   const int32_t* perm, const uint8_t* dead,
                                                   const gptq_config* cfg, uint8_t* codes,
                                                   float* scales, int32_t* zeros,
                                                   int32_t* dev_status, cudaStream_t stream) {
    if (cfg == nullptr || d_row <= 0 || d_col <= 0) return GPTQ_ERR_INVALID_ARG;
    size_t need = 0;
    const gptq_status s = gptq_workspace_size(cfg, d_row, d_col, &need);
    if (s != GPTQ_OK) return s;
    if (gptq::quant_min_workspace_bytes(d_row, cfg->block_size) > kNoAllocScratchBytes)
        return GPTQ_ERR_WORKSPACE;  // the layer needs more scratch than the fixed array holds
    void* ws = scratch_on_current_device();
    if (ws == nullptr) return GPTQ_ERR_CUDA;
    return gptq_quantize_layer(W, d_row, d_col, ldw, U, perm, dead, cfg, codes, scales, zeros,
                               dev_status, ws, kNoAllocScratchBytes, stream);
}
