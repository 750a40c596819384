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
// the array's device address with cudaGetSymbolAddress and caches it with the
// identity of the device's current context; a later call in another context
// (after cudaDeviceReset, the module is loaded anew and the array may move)
// looks it up again.  Host code must never pass the array's name itself to a
// kernel (in host code it is only a stand-in, not a device address).  Make
// the first call on a device before any stream capture on it.
//
// Device: every device pointer of the call must be memory of the current
// device (or managed memory); the scratch belongs to the current device, so
// a W on another GPU is rejected with GPTQ_ERR_INVALID_ARG before anything is
// launched.
//
// Sharing: all calls use the same array and it keeps whatever the last call
// left in it.  The column walk writes every scratch element it later reads
// within a call, so nothing needs to start at zero; two calls whose work
// overlaps on the GPU (different streams, no ordering) race on the array.
//
// Schedule: the lazy update defers the errors of up to 8 blocks of 128
// columns in the scratch (d_row * 128 * 4 bytes per block).  When 8 do not
// fit the 16 MiB (d_row > 4096) it defers fewer (4 up to d_row 8192, 2 up to
// 16384, 1 up to 32768), as gptq_quantize_layer does with a workspace of that
// size: the sums are the same, grouped into more and shorter products.
#include <cuda.h>

#include <mutex>

#include "kernels.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t{16} << 20;  // 16 MiB per device

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
struct ScratchEntry {
    unsigned long long ctx = 0;  // context the address belongs to (0: none yet)
    void* ptr = nullptr;
};
ScratchEntry g_scratch[kMaxDevices];

using CtxGetCurrent = CUresult (*)(CUcontext*);
using CtxGetId = CUresult (*)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current context (0 if unavailable).
unsigned long long current_context_id() {
    static CtxGetCurrent get_current = nullptr;
    static CtxGetId get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrent>(p);
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetId>(p);
    });
    CUcontext c = nullptr;
    unsigned long long id = 0;
    if (get_current == nullptr || get_id == nullptr || get_current(&c) != CUDA_SUCCESS ||
        c == nullptr || get_id(c, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

// Device address of the scratch array in the current device's current
// context, looked up once per context.  Returns nullptr if the lookup fails.
void* scratch_on_current_device(int dev) {
    if (dev < 0 || dev >= kMaxDevices) return nullptr;
    // (the pointer checks before this have made the device's context current;
    // without an id the address is simply looked up again)
    const unsigned long long ctx = current_context_id();
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    ScratchEntry& e = g_scratch[dev];
    if (e.ptr == nullptr || ctx == 0 || e.ctx != ctx) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
            return nullptr;
        e.ptr = p;
        e.ctx = ctx;
    }
    return e.ptr;
}

// p is memory of device `dev` (or managed memory); NULL is accepted when
// `optional` (the status word).
bool on_device(const void* p, int dev, bool optional = false) {
    if (p == nullptr) return optional;
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        (void)cudaGetLastError();  // drop the error the failed query recorded
        return false;
    }
    if (a.type == cudaMemoryTypeManaged) return true;
    return a.type == cudaMemoryTypeDevice && a.device == dev;
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
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GPTQ_ERR_CUDA;
    // the scratch is the current device's: every buffer must live there too
    if (!on_device(W, dev) || !on_device(U, dev) || !on_device(codes, dev) ||
        !on_device(scales, dev) || !on_device(zeros, dev) || !on_device(dead, dev) ||
        (cfg->desc_act != 0 && !on_device(perm, dev)) || !on_device(dev_status, dev, true))
        return GPTQ_ERR_INVALID_ARG;
    void* ws = scratch_on_current_device(dev);
    if (ws == nullptr) return GPTQ_ERR_CUDA;
    return gptq_quantize_layer(W, d_row, d_col, ldw, U, perm, dead, cfg, codes, scales, zeros,
                               dev_status, ws, kNoAllocScratchBytes, stream);
}
