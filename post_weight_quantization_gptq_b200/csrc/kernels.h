// Internal launchers of the GPTQ kernels (one per stage), called by the
// C-ABI layer in api.cu after it has validated every argument.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/gptq.h"

namespace gptq {

// Streaming multiprocessors of the current device (cached per device).
int num_sms();

// Host-side count of kernels this library has launched (diagnostics).
void count_launches(int64_t k);
int64_t launches();

// Timeout probes armed by gptq_debug_arm_wait_probe: the limit (ns) for the
// next launch of the kernel kind, 0 when unarmed; taking it disarms it.
enum ProbeKind { kProbeHessian = 1, kProbeGemm = 2 };
uint64_t take_wait_probe(int kind);

// Launch with the programmatic-serialization attribute when pdl is set; an
// ordinary launch otherwise.  Such a kernel calls pdl_wait() before its first
// global memory access, and reads data an earlier kernel wrote only through
// coherent paths (TMA, or plain / L2 loads -- never the read-only
// non-coherent path, which a const __restrict__ pointer the kernel never
// writes may compile to): the earlier kernel may still have been running
// when this one started.  Used only where the predecessor in the stream is
// a kernel (not an event record or wait).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_kernel(bool pdl, void (*kern)(KArgs...), dim3 grid, dim3 block,
                                 size_t smem, cudaStream_t stream, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// Shared-memory swizzle of a TMA box: none, 128-byte (16-byte chunks), or
// 128-byte with 32-byte chunks (the layout 32-bit MN-major MMA operands use).
enum class Swz { kNone, k128, k128Atom32 };

// 2-D TMA tensor map over a row-major matrix of `outer` rows x `inner`
// columns (leading dimension ld_elems), boxes of box_outer x box_inner
// elements, fp32 or bf16 (tmap.cu).
bool make_tmap_2d(CUtensorMap* map, bool bf16, const void* base, uint64_t inner, uint64_t outer,
                  uint64_t ld_elems, uint32_t box_inner, uint32_t box_outer, Swz swizzle);

// ---- stage 1 (hessian.cu)
int hessian_num_tiles(int64_t d);
gptq_status launch_hessian(const uint16_t* X, int64_t n, int64_t d, int64_t ldx, float* H,
                           int64_t ldh, int32_t* status, cudaStream_t stream);

// ---- stage 1 from host memory (hessian_host.cu): copy / GEMM pipeline over
// a two-slot device staging buffer
int64_t hessian_stream_row_pitch(int64_t d);
int64_t hessian_stream_chunk_tokens(int64_t d, size_t staging_bytes);
gptq_status launch_hessian_from_host(const uint16_t* Xh, int64_t n, int64_t d, int64_t ldx,
                                     float* H, int64_t ldh, int32_t* status, void* staging,
                                     size_t staging_bytes, cudaStream_t stream);

// ---- stage 2 (prep.cu): dead columns, lambda, act-order, flipped working copy
size_t prep_workspace_bytes(int64_t d);
gptq_status launch_prep(const float* H, int64_t d, int64_t ldh, float damp, int desc_act,
                        float* P, int32_t* perm, uint8_t* dead, int32_t* status, void* ws,
                        cudaStream_t stream);

// ---- stage 2 (chol.cu): P = L L^T in place, X = L^-1, U = J X J
size_t chol_workspace_bytes(int64_t d);
gptq_status launch_chol_inverse(float* P, float* Xbuf, int64_t ldx, int64_t d, float* U,
                                int32_t* status, void* ws, cudaStream_t stream);

// ---- stages 3-4 (quant.cu)
// Workspace of the fastest schedule, and the least the column walk accepts
// (a smaller workspace shortens the deferred runs of the lazy update).
size_t quant_workspace_bytes(int64_t d_row, int64_t d_col, int block);
size_t quant_min_workspace_bytes(int64_t d_row, int block);
gptq_status launch_quantize(float* W, int64_t d_row, int64_t d_col, int64_t ldw, const float* U,
                            const int32_t* perm, const uint8_t* dead, int desc_act, int bits, int group,
                            int block, int pure_minmax, uint8_t* codes, float* scales, int32_t* zeros,
                            int32_t* status, void* ws, size_t ws_bytes, cudaStream_t stream);

// ---- using the quantized layer (dequant_matmul.cu): Y = X W_hat^T, decode form
int dequant_matmul_tokens_per_launch(int bits);
size_t dequant_matmul_workspace_bytes(int64_t n_tok, int64_t d_col);
gptq_status launch_dequant_matmul(const uint16_t* X, int64_t n_tok, int64_t d_col, int64_t ldx,
                                  const uint32_t* packed, const float* scales,
                                  const int32_t* zeros, const int32_t* perm, int64_t d_row,
                                  int bits, int group, float* Y, int64_t ldy, void* ws,
                                  cudaStream_t stream);

// ---- using the quantized layer, many-token form (dequant_gemm.cu): tcgen05
// bf16 GEMM with the weights dequantized into shared memory per stage
size_t dequant_gemm_workspace_bytes(int64_t n_tok, int64_t d_col);
gptq_status launch_dequant_gemm(const uint16_t* X, int64_t n_tok, int64_t d_col, int64_t ldx,
                                const uint32_t* packed, const float* scales, const int32_t* zeros,
                                const int32_t* perm, int64_t d_row, int bits, int group, float* Y,
                                int64_t ldy, int32_t* status, void* ws, cudaStream_t stream);

// ---- stage 5 (pack.cu)
gptq_status launch_pack(const uint8_t* codes, int64_t d_row, int64_t d_col, int bits,
                        uint32_t* packed, cudaStream_t stream);

}  // namespace gptq
