// Stage 5: code packing.  4-bit codes go 8 to a uint32 along d_col (the
// density the "GPTQ" article, "Desempenho e Precisao", gives for OPT-175B:
// 175e9 weights in about 87.5 GB).  Other widths continue the same
// little-endian bit stream: code k of a row occupies bits [b k, b k + b).
#include "common.cuh"
#include "kernels.h"

namespace gptq {
namespace {

constexpr int kThreads = 256;

// The four codes of a 32-bit lane (byte j = code j), masked to BITS bits,
// as one 4*BITS-bit field (code j at bits BITS*j).
template <int BITS>
__device__ __forceinline__ uint32_t squeeze4(uint32_t x) {
    if constexpr (BITS == 8) {
        return x;
    } else if constexpr (BITS == 4) {
        x &= 0x0F0F0F0Fu;
        const uint32_t t = (x | (x >> 4)) & 0x00FF00FFu;  // bytes 0 and 2: two codes each
        return (t & 0xFFu) | ((t >> 8) & 0xFF00u);
    } else {
        x &= 0x03030303u;
        const uint32_t t = x | (x >> 6);                   // nibbles 0 and 4: two codes each
        return (t & 0xFu) | ((t >> 12) & 0xF0u);
    }
}

// BITS in {2, 4, 8}, d a multiple of 16: every row is a whole number of
// 16-code chunks and of the words they fill, so the flat chunk i of the codes
// becomes the flat words [i * BITS / 2, (i + 1) * BITS / 2): one 16-byte load
// and one 4-, 8- or 16-byte store per chunk.
template <int BITS>
__global__ void __launch_bounds__(kThreads)
pack_chunks_kernel(const uint4* __restrict__ codes, int64_t chunks, uint32_t* __restrict__ packed) {
    for (int64_t i = blockIdx.x * static_cast<int64_t>(kThreads) + threadIdx.x; i < chunks;
         i += static_cast<int64_t>(gridDim.x) * kThreads) {
        const uint4 c = __ldg(codes + i);
        const uint32_t a = squeeze4<BITS>(c.x), b = squeeze4<BITS>(c.y);
        const uint32_t e = squeeze4<BITS>(c.z), f = squeeze4<BITS>(c.w);
        if constexpr (BITS == 8) {
            reinterpret_cast<uint4*>(packed)[i] = make_uint4(a, b, e, f);
        } else if constexpr (BITS == 4) {
            reinterpret_cast<uint2*>(packed)[i] = make_uint2(a | (b << 16), e | (f << 16));
        } else {
            packed[i] = a | (b << 8) | (e << 16) | (f << 24);
        }
    }
}

// Any width and shape: one thread per output word of a row (rows along
// grid y); a word gathers every code that overlaps it.
__global__ void __launch_bounds__(kThreads)
pack_words_kernel(const uint8_t* __restrict__ codes, int64_t r, int64_t d, int bits,
                  int64_t words, uint32_t* __restrict__ packed) {
    const uint32_t mask = (1u << bits) - 1u;
    for (int64_t row = blockIdx.y; row < r; row += gridDim.y) {
        const uint8_t* c = codes + row * d;
        for (int64_t m = blockIdx.x * static_cast<int64_t>(kThreads) + threadIdx.x; m < words;
             m += static_cast<int64_t>(gridDim.x) * kThreads) {
            const int64_t bit0 = 32 * m;
            const int64_t k_first = bit0 / bits;
            int64_t k_last = (bit0 + 31) / bits;
            if (k_last > d - 1) k_last = d - 1;
            uint32_t word = 0;
            for (int64_t k = k_first; k <= k_last; ++k) {
                const uint32_t code = c[k] & mask;
                const int64_t pos = bits * k - bit0;
                word |= (pos >= 0) ? (code << pos) : (code >> (-pos));
            }
            packed[row * words + m] = word;
        }
    }
}

int64_t grid_for(int64_t items) {
    int64_t blocks = (items + kThreads - 1) / kThreads;
    const int64_t cap = 16LL * num_sms();
    if (blocks > cap) blocks = cap;
    return blocks < 1 ? 1 : blocks;
}

}  // namespace

gptq_status launch_pack(const uint8_t* codes, int64_t d_row, int64_t d_col, int bits,
                        uint32_t* packed, cudaStream_t stream) {
    const int64_t words = (d_col * bits + 31) / 32;
    const uintptr_t cp = reinterpret_cast<uintptr_t>(codes), pp = reinterpret_cast<uintptr_t>(packed);
    const int store_align = bits == 8 ? 16 : bits == 4 ? 8 : 4;
    if ((bits == 2 || bits == 4 || bits == 8) && d_col % 16 == 0 && (cp & 15) == 0 &&
        (pp & (store_align - 1)) == 0) {
        const int64_t chunks = d_row * (d_col / 16);
        const unsigned grid = static_cast<unsigned>(grid_for(chunks));
        const uint4* c4 = reinterpret_cast<const uint4*>(codes);
        switch (bits) {
            case 2: pack_chunks_kernel<2><<<grid, kThreads, 0, stream>>>(c4, chunks, packed); break;
            case 4: pack_chunks_kernel<4><<<grid, kThreads, 0, stream>>>(c4, chunks, packed); break;
            default: pack_chunks_kernel<8><<<grid, kThreads, 0, stream>>>(c4, chunks, packed); break;
        }
    } else {
        const int64_t gx = (words + kThreads - 1) / kThreads;
        int64_t gy = d_row < 65535 ? d_row : 65535;
        const int64_t budget = 16LL * num_sms();
        const int64_t gxc = gx < budget ? gx : budget;
        if (gy * gxc > budget && gy > 1) gy = (budget + gxc - 1) / gxc;
        const dim3 grid(static_cast<unsigned>(gxc), static_cast<unsigned>(gy < 1 ? 1 : gy));
        pack_words_kernel<<<grid, kThreads, 0, stream>>>(codes, d_row, d_col, bits, words, packed);
    }
    count_launches(1);
    return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ERR_CUDA;
}

}  // namespace gptq
