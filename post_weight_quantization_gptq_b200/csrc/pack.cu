// Stage 5: code packing.  4-bit codes go 8 to a uint32 along d_col (the
// density the "GPTQ" article, "Desempenho e Precisao", gives for OPT-175B:
// 175e9 weights in about 87.5 GB).  Other widths continue the same
// little-endian bit stream: code k of a row occupies bits [b k, b k + b).
#include "common.cuh"
#include "kernels.h"

namespace gptq {
namespace {

// One thread per output word; a word gathers every code that overlaps it.
__global__ void pack_kernel(const uint8_t* __restrict__ codes, int64_t r, int64_t d, int bits,
                            int64_t words, uint32_t* __restrict__ packed) {
    const int64_t total = r * words;
    for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
         idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t row = idx / words, m = idx % words;
        const int64_t bit0 = 32 * m;
        const int64_t k_first = bit0 / bits;
        int64_t k_last = (bit0 + 31) / bits;
        if (k_last > d - 1) k_last = d - 1;
        const uint8_t* c = codes + row * d;
        uint32_t word = 0;
        for (int64_t k = k_first; k <= k_last; ++k) {
            const uint32_t code = c[k];
            const int64_t pos = bits * k - bit0;
            word |= (pos >= 0) ? (code << pos) : (code >> (-pos));
        }
        packed[idx] = word;
    }
}

}  // namespace

gptq_status launch_pack(const uint8_t* codes, int64_t d_row, int64_t d_col, int bits,
                        uint32_t* packed, cudaStream_t stream) {
    const int64_t words = (d_col * bits + 31) / 32;
    const int64_t total = d_row * words;
    int64_t blocks = (total + 255) / 256;
    const int64_t cap = 32LL * num_sms();
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    pack_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(codes, d_row, d_col, bits, words,
                                                                    packed);
    count_launches(1);
    return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ERR_CUDA;
}

}  // namespace gptq
