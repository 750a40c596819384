// Stage 1 from host memory: H += 2 X^T X with X streamed in token chunks.
//
// "GPTQ (GPT Quantization)", "Fondation theorique : OBQ": H = 2 X^T X is a
// sum over calibration tokens, so it can be accumulated chunk by chunk while
// the calibration data is still arriving.  This entry point takes X in host
// memory and moves it through a caller-owned device staging buffer of two
// slots: while the tensor cores accumulate chunk c from one slot, the copy
// engine fills the other slot with chunk c + 1.  With pinned host memory the
// step is bound by the host-to-device link, not by the GEMM.
//
// Ordering: copies run on a library-owned copy stream per device, GEMMs on
// the caller's stream.  The copy stream first waits for everything queued on
// the caller's stream before the call (earlier users of the staging buffer),
// a slot is refilled only after the GEMM that read it, and each GEMM waits
// for its slot's copy; at return every GEMM of the call is queued on the
// caller's stream behind its copy, so later work on that stream is ordered.
#include <mutex>

#include "kernels.h"

namespace gptq {
namespace {

constexpr int64_t kTokenQuantum = 64;       // tokens per MMA k-step (BK of the GEMM)
constexpr int64_t kDrainTokens = 32768;     // the GEMM's own accumulation chunk

struct CopyPipe {
    cudaStream_t copy = nullptr;
    cudaEvent_t start = nullptr;
    cudaEvent_t copied[2] = {};
    cudaEvent_t consumed[2] = {};
    bool ok = false;
};
std::mutex g_pipe_mutex;
CopyPipe g_pipe[64];

// Caller holds g_pipe_mutex.
CopyPipe* pipe_on_current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    CopyPipe& p = g_pipe[dev];
    if (!p.ok) {
        if (cudaStreamCreateWithFlags(&p.copy, cudaStreamNonBlocking) != cudaSuccess) return nullptr;
        cudaEvent_t* all[] = {&p.start, &p.copied[0], &p.copied[1], &p.consumed[0], &p.consumed[1]};
        for (auto* e : all)
            if (cudaEventCreateWithFlags(e, cudaEventDisableTiming) != cudaSuccess) return nullptr;
        p.ok = true;
    }
    return &p;
}

}  // namespace

int64_t hessian_stream_row_pitch(int64_t d) { return (d + 7) / 8 * 8; }

int64_t hessian_stream_chunk_tokens(int64_t d, size_t staging_bytes) {
    const int64_t per_token = 2 * hessian_stream_row_pitch(d) * 2;  // two slots of bf16 rows
    int64_t c = static_cast<int64_t>(staging_bytes / static_cast<size_t>(per_token));
    if (c >= kDrainTokens) return c / kDrainTokens * kDrainTokens;
    return c / kTokenQuantum * kTokenQuantum;
}

gptq_status launch_hessian_from_host(const uint16_t* Xh, int64_t n, int64_t d, int64_t ldx,
                                     float* H, int64_t ldh, int32_t* status, void* staging,
                                     size_t staging_bytes, cudaStream_t stream) {
    const int64_t chunk = hessian_stream_chunk_tokens(d, staging_bytes);
    if (chunk <= 0) return GPTQ_ERR_WORKSPACE;
    const int64_t pitch = hessian_stream_row_pitch(d);
    uint16_t* slot[2] = {static_cast<uint16_t*>(staging),
                         static_cast<uint16_t*>(staging) + chunk * pitch};
    std::lock_guard<std::mutex> lock(g_pipe_mutex);
    CopyPipe* p = pipe_on_current_device();
    if (p == nullptr) return GPTQ_ERR_CUDA;
    if (cudaEventRecord(p->start, stream) != cudaSuccess ||
        cudaStreamWaitEvent(p->copy, p->start, 0) != cudaSuccess)
        return GPTQ_ERR_CUDA;
    int64_t c = 0;
    for (int64_t t0 = 0; t0 < n; t0 += chunk, ++c) {
        const int s = static_cast<int>(c & 1);
        const int64_t rows = (n - t0 < chunk) ? n - t0 : chunk;
        if (c >= 2 && cudaStreamWaitEvent(p->copy, p->consumed[s], 0) != cudaSuccess)
            return GPTQ_ERR_CUDA;
        const uint16_t* src = Xh + t0 * ldx;
        cudaError_t e;
        if (ldx == pitch && d == pitch)
            e = cudaMemcpyAsync(slot[s], src, static_cast<size_t>(rows * pitch) * 2,
                                cudaMemcpyHostToDevice, p->copy);
        else
            e = cudaMemcpy2DAsync(slot[s], static_cast<size_t>(pitch) * 2, src,
                                  static_cast<size_t>(ldx) * 2, static_cast<size_t>(d) * 2,
                                  static_cast<size_t>(rows), cudaMemcpyHostToDevice, p->copy);
        if (e != cudaSuccess || cudaEventRecord(p->copied[s], p->copy) != cudaSuccess ||
            cudaStreamWaitEvent(stream, p->copied[s], 0) != cudaSuccess)
            return GPTQ_ERR_CUDA;
        const gptq_status g = launch_hessian(slot[s], rows, d, pitch, H, ldh, status, stream);
        if (g != GPTQ_OK) return g;
        if (cudaEventRecord(p->consumed[s], stream) != cudaSuccess) return GPTQ_ERR_CUDA;
    }
    return GPTQ_OK;
}

}  // namespace gptq
