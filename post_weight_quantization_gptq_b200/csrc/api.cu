// C ABI of the GPTQ layer quantizer (declared in include/gptq.h): argument
// validation, workspace carving and the launch sequence of each stage.
// Nothing here allocates device memory.
#include <atomic>
#include <cmath>
#include <cstdint>

#include "kernels.h"

namespace gptq {

namespace {
std::atomic<int64_t> g_launches{0};
std::atomic<uint64_t> g_probe[3] = {};
}

void count_launches(int64_t k) { g_launches.fetch_add(k, std::memory_order_relaxed); }

uint64_t take_wait_probe(int kind) {
    if (kind < 1 || kind > 2) return 0;
    if (g_probe[kind].load(std::memory_order_relaxed) == 0) return 0;
    return g_probe[kind].exchange(0, std::memory_order_acq_rel);
}

void arm_wait_probe(int kind, uint64_t ns) {
    if (kind >= 1 && kind <= 2) g_probe[kind].store(ns, std::memory_order_release);
}

int64_t launches() { return g_launches.load(std::memory_order_relaxed); }

int num_sms() {
    // per device, filled on first use; threads that race to fill it store the
    // same value
    static std::atomic<int> cache[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
    if (dev >= 0 && dev < 64) {
        const int c = cache[dev].load(std::memory_order_relaxed);
        if (c > 0) return c;
    }
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
        v = 148;
    if (dev >= 0 && dev < 64) cache[dev].store(v, std::memory_order_relaxed);
    return v;
}

}  // namespace gptq

namespace {

constexpr int64_t kMaxDim = (int64_t{1} << 31) - 1;
constexpr int64_t kMaxQuantCols = 56 * 1024;  // one row of W must fit in shared memory

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t round256(size_t b) { return (b + 255) / 256 * 256; }

gptq_status check_config(const gptq_config* cfg, int64_t d_col) {
    if (cfg == nullptr) return GPTQ_ERR_INVALID_ARG;
    const int b = cfg->bits;
    if (b != 2 && b != 3 && b != 4 && b != 8) return GPTQ_ERR_INVALID_ARG;
    if (!(cfg->damp >= 0.f) || !std::isfinite(cfg->damp)) return GPTQ_ERR_INVALID_ARG;
    const int g = cfg->group_size;
    if (g == 0 || g < -1) return GPTQ_ERR_INVALID_ARG;
    if (cfg->block_size != 128) return GPTQ_ERR_UNSUPPORTED;
    if (g == -1 || g >= d_col) return GPTQ_OK;
    // below a block: a divisor of it, at least 8 columns (groups of 1 to 4
    // weights would carry a scale per handful of codes, and are not tested)
    if (g < cfg->block_size)
        return (g >= 8 && cfg->block_size % g == 0) ? GPTQ_OK : GPTQ_ERR_UNSUPPORTED;
    return (g % cfg->block_size == 0) ? GPTQ_OK : GPTQ_ERR_UNSUPPORTED;
}

gptq_status launch_status(gptq_status s) {
    if (s != GPTQ_OK) return s;
    return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ERR_CUDA;
}

}  // namespace

extern "C" {

const char* gptq_status_string(int32_t status) {
    switch (status) {
        case GPTQ_OK: return "ok";
        case GPTQ_ERR_INVALID_ARG: return "invalid argument";
        case GPTQ_ERR_UNSUPPORTED: return "unsupported configuration";
        case GPTQ_ERR_NOT_PD: return "damped Hessian is not positive definite";
        case GPTQ_ERR_TIMEOUT: return "a bounded device-side wait timed out";
        case GPTQ_ERR_CUDA: return "CUDA runtime error";
        case GPTQ_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        default: return "unknown status";
    }
}

int32_t gptq_version(void) { return 200; }

gptq_status gptq_debug_arm_wait_probe(int32_t kernel, int64_t limit_ns) {
    if ((kernel != 1 && kernel != 2) || limit_ns <= 0 || limit_ns > 1000000000) return GPTQ_ERR_INVALID_ARG;
    gptq::arm_wait_probe(kernel, static_cast<uint64_t>(limit_ns));
    return GPTQ_OK;
}

int64_t gptq_launch_counter(void) { return gptq::launches(); }

gptq_status gptq_workspace_size(const gptq_config* cfg, int64_t d_row, int64_t d_col,
                                size_t* bytes) {
    if (bytes == nullptr || d_row <= 0 || d_col <= 0) return GPTQ_ERR_INVALID_ARG;
    const gptq_status c = check_config(cfg, d_col);
    if (c != GPTQ_OK) return c;
    size_t need = gptq::prep_workspace_bytes(d_col);
    const size_t q = gptq::quant_workspace_bytes(d_row, d_col, cfg->block_size);
    const size_t ch = gptq::chol_workspace_bytes(d_col);
    if (q > need) need = q;
    if (ch > need) need = ch;
    *bytes = round256(need);
    return GPTQ_OK;
}

gptq_status gptq_hessian_accumulate(const uint16_t* X, int64_t n, int64_t d, int64_t ldx,
                                    float* H, int64_t ldh, int32_t* dev_status, void* ws,
                                    size_t ws_bytes, cudaStream_t stream) {
    (void)ws;
    (void)ws_bytes;
    if (d <= 0 || d > kMaxDim || n < 0 || n > kMaxDim) return GPTQ_ERR_INVALID_ARG;
    if (H == nullptr || ldh < d) return GPTQ_ERR_INVALID_ARG;
    if (n == 0) return GPTQ_OK;
    if (X == nullptr || ldx < d || (ldx % 8) != 0 || !aligned(X, 16)) return GPTQ_ERR_INVALID_ARG;
    return launch_status(gptq::launch_hessian(X, n, d, ldx, H, ldh, dev_status, stream));
}

gptq_status gptq_hessian_accumulate_host(const uint16_t* X_host, int64_t n, int64_t d,
                                         int64_t ldx, float* H, int64_t ldh, int32_t* dev_status,
                                         void* staging, size_t staging_bytes,
                                         cudaStream_t stream) {
    if (d <= 0 || d > kMaxDim || n < 0 || n > kMaxDim) return GPTQ_ERR_INVALID_ARG;
    if (H == nullptr || ldh < d) return GPTQ_ERR_INVALID_ARG;
    if (n == 0) return GPTQ_OK;
    if (X_host == nullptr || ldx < d) return GPTQ_ERR_INVALID_ARG;
    if (staging == nullptr || !aligned(staging, 256) ||
        gptq::hessian_stream_chunk_tokens(d, staging_bytes) <= 0)
        return GPTQ_ERR_WORKSPACE;
    return launch_status(gptq::launch_hessian_from_host(X_host, n, d, ldx, H, ldh, dev_status,
                                                        staging, staging_bytes, stream));
}

size_t gptq_hessian_staging_size(int64_t d, int64_t chunk_tokens) {
    if (d <= 0 || d > kMaxDim || chunk_tokens <= 0) return 0;
    const int64_t c = (chunk_tokens + 63) / 64 * 64;
    return static_cast<size_t>(2 * c * gptq::hessian_stream_row_pitch(d) * 2);
}

gptq_status gptq_prepare_hinv(float* H, int64_t d, int64_t ldh, const gptq_config* cfg, float* U,
                              int32_t* perm, uint8_t* dead, int32_t* dev_status, void* ws,
                              size_t ws_bytes, cudaStream_t stream) {
    if (d <= 0 || d > kMaxDim || H == nullptr || ldh < d || U == nullptr || perm == nullptr ||
        dead == nullptr)
        return GPTQ_ERR_INVALID_ARG;
    if (H == U) return GPTQ_ERR_INVALID_ARG;
    if ((d % 4) != 0 || (ldh % 4) != 0 || !aligned(H, 16) || !aligned(U, 16))
        return GPTQ_ERR_UNSUPPORTED;  // tensor-memory-accelerator tiles need 16-byte rows
    if (d > kMaxQuantCols) return GPTQ_ERR_UNSUPPORTED;  // U only feeds the column walk
    const gptq_status c = check_config(cfg, d);
    if (c != GPTQ_OK) return c;
    if (ws == nullptr || !aligned(ws, 256) || ws_bytes < gptq::prep_workspace_bytes(d) ||
        ws_bytes < gptq::chol_workspace_bytes(d))
        return GPTQ_ERR_WORKSPACE;
    gptq_status s =
        gptq::launch_prep(H, d, ldh, cfg->damp, cfg->desc_act, U, perm, dead, dev_status, ws, stream);
    if (s != GPTQ_OK) return s;
    s = gptq::launch_chol_inverse(U, H, ldh, d, U, dev_status, ws, stream);
    return launch_status(s);
}

gptq_status gptq_quantize_layer(float* W, int64_t d_row, int64_t d_col, int64_t ldw,
                                const float* U, const int32_t* perm, const uint8_t* dead,
                                const gptq_config* cfg, uint8_t* codes, float* scales,
                                int32_t* zeros, int32_t* dev_status, void* ws, size_t ws_bytes,
                                cudaStream_t stream) {
    if (d_row <= 0 || d_row > kMaxDim || d_col <= 0 || W == nullptr || ldw < d_col ||
        U == nullptr || perm == nullptr || dead == nullptr || codes == nullptr ||
        scales == nullptr || zeros == nullptr)
        return GPTQ_ERR_INVALID_ARG;
    if (d_col > kMaxQuantCols || (d_col % 4) != 0 || !aligned(U, 16)) return GPTQ_ERR_UNSUPPORTED;
    const gptq_status c = check_config(cfg, d_col);
    if (c != GPTQ_OK) return c;
    if (ws == nullptr || !aligned(ws, 256) ||
        ws_bytes < gptq::quant_min_workspace_bytes(d_row, cfg->block_size))
        return GPTQ_ERR_WORKSPACE;
    return launch_status(gptq::launch_quantize(W, d_row, d_col, ldw, U, perm, dead, cfg->desc_act, cfg->bits,
                                               cfg->group_size, cfg->block_size, cfg->pure_minmax,
                                               codes, scales,
                                               zeros, dev_status, ws, ws_bytes, stream));
}

gptq_status gptq_pack(const uint8_t* codes, int64_t d_row, int64_t d_col, int32_t bits,
                      uint32_t* packed, cudaStream_t stream) {
    if (codes == nullptr || packed == nullptr || d_row <= 0 || d_col <= 0 || d_row > kMaxDim ||
        d_col > kMaxDim)
        return GPTQ_ERR_INVALID_ARG;
    if (bits != 2 && bits != 3 && bits != 4 && bits != 8) return GPTQ_ERR_INVALID_ARG;
    return launch_status(gptq::launch_pack(codes, d_row, d_col, bits, packed, stream));
}

size_t gptq_dequant_matmul_workspace_size(int64_t n_tok, int64_t d_col) {
    if (n_tok <= 0 || d_col <= 0 || d_col > kMaxDim) return 0;
    return gptq::dequant_matmul_workspace_bytes(n_tok, d_col);
}

gptq_status gptq_dequant_matmul(const uint16_t* X, int64_t n_tok, int64_t d_col, int64_t ldx,
                                const uint32_t* packed, const float* scales, const int32_t* zeros,
                                const int32_t* perm, int64_t d_row, int32_t bits,
                                int32_t group_size, float* Y, int64_t ldy, void* ws,
                                size_t ws_bytes, cudaStream_t stream) {
    if (X == nullptr || packed == nullptr || scales == nullptr || zeros == nullptr || Y == nullptr)
        return GPTQ_ERR_INVALID_ARG;
    if (n_tok < 0 || d_col <= 0 || d_row <= 0 || d_col > kMaxDim || d_row > kMaxDim ||
        ldx < d_col || ldy < d_row)
        return GPTQ_ERR_INVALID_ARG;
    if (bits != 2 && bits != 3 && bits != 4 && bits != 8) return GPTQ_ERR_INVALID_ARG;
    if (group_size == 0 || group_size < -1) return GPTQ_ERR_INVALID_ARG;
    if (!aligned(packed, 4) || !aligned(scales, 4) || !aligned(zeros, 4) || !aligned(Y, 4) ||
        !aligned(X, 2))
        return GPTQ_ERR_INVALID_ARG;
    // whole words per row, and no word shared by two groups
    const int64_t cpw = 32 / bits;
    const int64_t g = (group_size == -1 || group_size > d_col) ? d_col : group_size;
    if (bits == 3 || d_col % cpw != 0 || (g % cpw != 0 && g != d_col)) return GPTQ_ERR_UNSUPPORTED;
    if (n_tok == 0) return GPTQ_OK;
    if (ws == nullptr || !aligned(ws, 256) ||
        ws_bytes < gptq::dequant_matmul_workspace_bytes(n_tok, d_col))
        return GPTQ_ERR_WORKSPACE;
    return launch_status(gptq::launch_dequant_matmul(X, n_tok, d_col, ldx, packed, scales, zeros,
                                                     perm, d_row, bits, group_size, Y, ldy, ws,
                                                     stream));
}

size_t gptq_dequant_gemm_workspace_size(int64_t n_tok, int64_t d_col) {
    if (n_tok <= 0 || d_col <= 0 || d_col > kMaxDim) return 0;
    return gptq::dequant_gemm_workspace_bytes(n_tok, d_col);
}

gptq_status gptq_dequant_gemm(const uint16_t* X, int64_t n_tok, int64_t d_col, int64_t ldx,
                              const uint32_t* packed, const float* scales, const int32_t* zeros,
                              const int32_t* perm, int64_t d_row, int32_t bits, int32_t group_size,
                              float* Y, int64_t ldy, int32_t* dev_status, void* ws,
                              size_t ws_bytes, cudaStream_t stream) {
    if (X == nullptr || packed == nullptr || scales == nullptr || zeros == nullptr || Y == nullptr)
        return GPTQ_ERR_INVALID_ARG;
    if (n_tok < 0 || n_tok > (int64_t{1} << 24) || d_col <= 0 || d_row <= 0 || d_col > kMaxDim ||
        d_row > kMaxDim || ldx < d_col || ldy < d_row)
        return GPTQ_ERR_INVALID_ARG;
    if (bits != 2 && bits != 3 && bits != 4 && bits != 8) return GPTQ_ERR_INVALID_ARG;
    if (group_size == 0 || group_size < -1) return GPTQ_ERR_INVALID_ARG;
    if (!aligned(packed, 16) || !aligned(scales, 4) || !aligned(zeros, 4) || !aligned(Y, 4) ||
        !aligned(X, 2))
        return GPTQ_ERR_INVALID_ARG;
    // whole 64-code stages, 16-byte packed rows, no 8-code chunk across two groups
    const int64_t g = (group_size == -1 || group_size > d_col) ? d_col : group_size;
    if (bits == 3 || d_col % 64 != 0 || (g % 8 != 0 && g != d_col)) return GPTQ_ERR_UNSUPPORTED;
    if (n_tok == 0) return GPTQ_OK;
    const bool gather = perm != nullptr || (ldx % 8) != 0 || !aligned(X, 16);
    if (gather && (ws == nullptr || !aligned(ws, 256) ||
                   ws_bytes < gptq::dequant_gemm_workspace_bytes(n_tok, d_col)))
        return GPTQ_ERR_WORKSPACE;
    return launch_status(gptq::launch_dequant_gemm(X, n_tok, d_col, ldx, packed, scales, zeros, perm,
                                                   d_row, bits, group_size, Y, ldy, dev_status, ws,
                                                   stream));
}

gptq_status gptq_sync_status(cudaStream_t stream, const int32_t* dev_status, int32_t* out) {
    if (dev_status == nullptr || out == nullptr) return GPTQ_ERR_INVALID_ARG;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return GPTQ_ERR_CUDA;
    if (cudaMemcpy(out, dev_status, sizeof(int32_t), cudaMemcpyDeviceToHost) != cudaSuccess)
        return GPTQ_ERR_CUDA;
    return GPTQ_OK;
}

}  // extern "C"
