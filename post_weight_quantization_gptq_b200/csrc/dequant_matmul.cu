// Using the quantized layer: Y = X W_hat^T with the weights dequantized on
// the fly from the packed codes.
//
// "GPTQ (GPT Quantization)", "Limitations" (items 1-2): GPTQ quantizes the
// weights only -- the activations stay at 16 bits -- and the integer weights
// are dequantized before each product.  This is the decode (few-token) form
// of that product on the layout this library writes: codes packed along d_col
// in quantization order, scales / zeros group-major [groups][d_row], and the
// act-order permutation applied to the activations.
//
//  gather_tokens_kernel  Xq[t][k] = X[t][perm[k]] as fp32 (quantization order),
//                        once per call, into the caller's workspace
//  dequant_matmul_kernel a CTA owns 32 output rows, four per warp; per step a
//                        lane loads runs of four consecutive packed words of
//                        its warp's four rows (512 contiguous bytes per warp
//                        load instruction), all before using any, while the CTA
//                        stages the step's token values in shared memory.
//
// Arithmetic per code: the code's bits are moved into the mantissa of a float
// (f = 1 + q / 2^b, exact: one shift and one LOP3, or at 4 bits one byte
// permute after two shared shifts and masks per word) and multiplied into a
// running dot with the token values (at 4 bits two running dots, even and
// odd codes, in one packed f32x2 FMA per pair); per word the dot d = sum_t x_t f_t and
// the token sum S = sum_t x_t give sum_t x_t q_t = 2^b (d - S), so the word
// adds s 2^b d - s (2^b + z) S to the output (two FMAs, the group's scale s
// and zero point z folded in once per group).  d and S carry the same rounding
// as a plain fp32 dot of x with q (the cancellation costs at most b bits of
// the 24, well inside the parity bound).
#include "kernels.h"

namespace gptq {
namespace {

constexpr int kRows = 32;         // output rows per CTA
constexpr int kRowsPerWarp = 4;
constexpr int kThreads = 256;
constexpr int kMaxTok = 8;        // tokens per launch

__device__ __forceinline__ float bf16_to_f32(uint16_t b) {
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

__global__ void gather_tokens_kernel(const uint16_t* __restrict__ X, int64_t ldx, int n_tok, int K,
                                     const int32_t* __restrict__ perm, float* __restrict__ Xq) {
    const int64_t total = static_cast<int64_t>(n_tok) * K;
    for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < total;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t t = e / K, k = e - t * K;
        int64_t col = perm != nullptr ? perm[k] : k;
        if (col < 0 || col >= K) col = k;  // not a permutation entry: stay inside the row
        Xq[e] = bf16_to_f32(X[t * ldx + col]);
    }
}

// Code t of a word as 1 + q / 2^BITS: the code's bits shifted to the top of
// the mantissa, ORed with the exponent of 1.0 (one shift and one LOP3 once t
// is a constant, as it is inside the unrolled loops below).
template <int BITS>
__device__ __forceinline__ float code_as_float(uint32_t word, int t) {
    const int top = 23 - BITS;       // mantissa bit of the code's lowest bit
    const int sh = top - BITS * t;   // left shift that moves code t there
    const uint32_t mask = ((1u << BITS) - 1u) << top;
    const uint32_t v = sh >= 0 ? (word << sh) : (word >> -sh);
    return __uint_as_float((v & mask) | 0x3F800000u);
}

// Packed f32x2 fused multiply-add (sm_100): d = a * b + c on both halves.
__device__ __forceinline__ uint64_t pk2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ float sum2(uint64_t v) {
    float lo, hi;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
    return lo + hi;
}

// d = sum_t x[t] (1 + q_t / 16) over the eight 4-bit codes of a word, with
// the floats built by byte permutes: each code shifted to bits 3..6 of its
// own byte with the byte's top bit set, then placed as the third byte of a
// float whose top byte is 0x3F (exponent 0, mantissa q / 16; the same value
// as code_as_float).  Two running sums (even and odd codes) as one packed
// f32x2 FMA per code pair.
__device__ __forceinline__ float dot4bit(uint32_t word, const float (&xv)[8]) {
    const uint32_t ev = ((word << 3) & 0x78787878u) | 0x80808080u;  // codes 0, 2, 4, 6
    const uint32_t od = ((word >> 1) & 0x78787878u) | 0x80808080u;  // codes 1, 3, 5, 7
    uint64_t d = 0;
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const float f0 = __uint_as_float(__byte_perm(ev, 0x3F000000u, 0x7044 | (p << 8)));
        const float f1 = __uint_as_float(__byte_perm(od, 0x3F000000u, 0x7044 | (p << 8)));
        d = fma2(pk2(xv[2 * p], xv[2 * p + 1]), pk2(f0, f1), d);
    }
    return sum2(d);
}

template <int BITS, int LW>
struct StepShape {
    static constexpr int CPW = 32 / BITS;                 // codes per word
    static constexpr int RUNS = LW / 4;                   // runs of four words per lane
    static constexpr int RUNLEN = 4 * CPW;                // codes per run
    static constexpr int PITCH = RUNLEN + 4;              // shared-memory floats per run
    static constexpr int WORDS = 128 * RUNS;              // words per step
    static constexpr int CODES = WORDS * CPW;             // codes per step
    static constexpr int SMEM = 32 * RUNS * PITCH;        // floats per token
};

template <int BITS, int MT, int LW>  // LW: words per lane per step
// 4-bit: two CTAs per SM (at most 128 registers; the packed dot otherwise
// takes 140 at two tokens and halves the resident warps)
__global__ void __launch_bounds__(kThreads, BITS == 4 ? 2 : 1)
    dequant_matmul_kernel(const float* __restrict__ Xq, int M, int K,
                          const uint32_t* __restrict__ packed, int64_t P,
                          const float* __restrict__ scales, const int32_t* __restrict__ zeros,
                          int N, int wpg, int wpg_log2, float* __restrict__ Y, int64_t ldy) {
    // wpg: packed words per group (a power of two 2^wpg_log2, or wpg_log2 < 0)
    using S_ = StepShape<BITS, LW>;
    constexpr int CPW = S_::CPW, RUNS = S_::RUNS;
    constexpr float kTwoB = static_cast<float>(1 << BITS);
    extern __shared__ __align__(16) float xs[];  // [MT][32 * RUNS runs][PITCH]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nw0 = blockIdx.x * kRows + warp * kRowsPerWarp;  // this warp's first row
    bool live[kRowsPerWarp];
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) live[r] = nw0 + r < N;
    float acc[kRowsPerWarp][MT];
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[r][m] = 0.f;

    // A step covers WORDS consecutive words of the CTA's rows; lane j takes
    // the runs of four words at base + 128 u + 4 j (u < RUNS), so each load
    // instruction reads 512 contiguous bytes of a row.  The step's token
    // values are staged in shared memory, run by run with a 4-float pad, so a
    // lane's float4 reads of its own run are free of bank conflicts.
    const bool vec = (P & 3) == 0 && (reinterpret_cast<uintptr_t>(packed) & 15) == 0;
    const int Pw = static_cast<int>(P);  // words per row (< 2^31)
    for (int base = 0; base < Pw; base += S_::WORDS) {
        // this step's words first: their loads are in flight during the staging
        uint32_t wd[kRowsPerWarp][LW];
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r)
#pragma unroll
            for (int u = 0; u < RUNS; ++u) {
                const int w = base + 128 * u + 4 * lane;
                const uint32_t* src = packed + (nw0 + r) * P + w;
                if (live[r] && vec && w < Pw) {
                    const uint4 q = __ldcs(reinterpret_cast<const uint4*>(src));
                    wd[r][4 * u] = q.x;
                    wd[r][4 * u + 1] = q.y;
                    wd[r][4 * u + 2] = q.z;
                    wd[r][4 * u + 3] = q.w;
                } else {
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        wd[r][4 * u + i] = (live[r] && w + i < Pw) ? __ldcs(src + i) : 0u;
                }
            }
        const int k0 = base * CPW;
        const int ncodes = K - k0 < S_::CODES ? K - k0 : S_::CODES;
        __syncthreads();  // the previous step's token values are consumed
        for (int e = threadIdx.x * 4; e < MT * S_::CODES; e += kThreads * 4) {
            const int m = e / S_::CODES, c = e - m * S_::CODES;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (m < M && c < ncodes)
                v = __ldg(reinterpret_cast<const float4*>(Xq + static_cast<int64_t>(m) * K + k0 + c));
            *reinterpret_cast<float4*>(xs + m * S_::SMEM + (c / S_::RUNLEN) * S_::PITCH + c % S_::RUNLEN) = v;
        }
        __syncthreads();
        int grp = -1;
        float ga[kRowsPerWarp], gb[kRowsPerWarp];
#pragma unroll
        for (int u = 0; u < RUNS; ++u)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int w = base + 128 * u + 4 * lane + i;
            if (w >= Pw) break;
            const int gi = wpg_log2 >= 0 ? (w >> wpg_log2) : w / wpg;  // a word never spans two groups
            if (gi != grp) {
                grp = gi;
#pragma unroll
                for (int r = 0; r < kRowsPerWarp; ++r) {
                    float s = 0.f, z = 0.f;
                    if (live[r]) {
                        const int64_t at = static_cast<int64_t>(gi) * N + nw0 + r;
                        s = __ldg(scales + at);
                        z = static_cast<float>(__ldg(zeros + at));
                    }
                    ga[r] = s * kTwoB;
                    gb[r] = -s * (kTwoB + z);
                }
            }
            const float* xr = xs + (32 * u + lane) * S_::PITCH + i * CPW;
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                if (m >= M) break;
                float xv[CPW];
#pragma unroll
                for (int t = 0; t < CPW; t += 4) {
                    const float4 x4 = *reinterpret_cast<const float4*>(xr + m * S_::SMEM + t);
                    xv[t] = x4.x;
                    xv[t + 1] = x4.y;
                    xv[t + 2] = x4.z;
                    xv[t + 3] = x4.w;
                }
                float S = 0.f;
#pragma unroll
                for (int t = 0; t < CPW; ++t) S += xv[t];
#pragma unroll
                for (int r = 0; r < kRowsPerWarp; ++r) {
                    float d = 0.f;
                    const uint32_t word = wd[r][4 * u + i];
                    if constexpr (BITS == 4) {
                        d = dot4bit(word, xv);
                    } else {
#pragma unroll
                        for (int t = 0; t < CPW; ++t) d = fmaf(xv[t], code_as_float<BITS>(word, t), d);
                    }
                    acc[r][m] = fmaf(ga[r], d, fmaf(gb[r], S, acc[r][m]));
                }
            }
        }
    }
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            float v = acc[r][m];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == 0 && live[r] && m < M) Y[static_cast<int64_t>(m) * ldy + nw0 + r] = v;
        }
    }
}

template <int BITS, int MT>
cudaError_t launch_one(const float* Xq, int M, int K, const uint32_t* packed, int64_t P,
                       const float* scales, const int32_t* zeros, int N, int g, float* Y,
                       int64_t ldy, cudaStream_t stream) {
    // words in flight per lane: 16 for one or two tokens, fewer as the token
    // values take registers
    constexpr int LW = MT <= 2 ? 16 : (MT <= 4 ? 8 : 4);
    const size_t smem = static_cast<size_t>(MT) * StepShape<BITS, LW>::SMEM * sizeof(float);
    auto kern = dequant_matmul_kernel<BITS, MT, LW>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const int wpg = g / StepShape<BITS, LW>::CPW;
    int wpg_log2 = -1;
    for (int b = 0; b < 31; ++b)
        if ((1 << b) == wpg) wpg_log2 = b;
    kern<<<(N + kRows - 1) / kRows, kThreads, smem, stream>>>(Xq, M, K, packed, P, scales, zeros,
                                                             N, wpg, wpg_log2, Y, ldy);
    return cudaGetLastError();
}

template <int BITS>
cudaError_t launch_bits(const float* Xq, int M, int K, const uint32_t* packed, int64_t P,
                        const float* scales, const int32_t* zeros, int N, int g, float* Y,
                        int64_t ldy, cudaStream_t stream) {
    if (M <= 1) return launch_one<BITS, 1>(Xq, M, K, packed, P, scales, zeros, N, g, Y, ldy, stream);
    if (M <= 2) return launch_one<BITS, 2>(Xq, M, K, packed, P, scales, zeros, N, g, Y, ldy, stream);
    if (M <= 4 || BITS == 2)
        return launch_one<BITS, 4>(Xq, M, K, packed, P, scales, zeros, N, g, Y, ldy, stream);
    return launch_one<BITS, kMaxTok>(Xq, M, K, packed, P, scales, zeros, N, g, Y, ldy, stream);
}

}  // namespace

int dequant_matmul_tokens_per_launch(int bits) { return bits == 2 ? 4 : kMaxTok; }

size_t dequant_matmul_workspace_bytes(int64_t n_tok, int64_t d_col) {
    const int64_t t = n_tok < kMaxTok ? n_tok : kMaxTok;
    return ((static_cast<size_t>(t) * d_col * sizeof(float) + 255) / 256) * 256;
}

gptq_status launch_dequant_matmul(const uint16_t* X, int64_t n_tok, int64_t d_col, int64_t ldx,
                                  const uint32_t* packed, const float* scales,
                                  const int32_t* zeros, const int32_t* perm, int64_t d_row,
                                  int bits, int group, float* Y, int64_t ldy, void* ws,
                                  cudaStream_t stream) {
    const int K = static_cast<int>(d_col), N = static_cast<int>(d_row);
    const int g = (group == -1 || group > K) ? K : group;
    const int64_t P = d_col * bits / 32;
    const int per = dequant_matmul_tokens_per_launch(bits);
    float* Xq = static_cast<float*>(ws);
    int64_t launches = 0;
    for (int64_t t0 = 0; t0 < n_tok; t0 += per) {
        const int M = static_cast<int>(n_tok - t0 < per ? n_tok - t0 : per);
        const int64_t total = static_cast<int64_t>(M) * K;
        const int gblocks = static_cast<int>((total + 255) / 256 < 4 * num_sms() ? (total + 255) / 256 : 4 * num_sms());
        gather_tokens_kernel<<<gblocks, 256, 0, stream>>>(X + t0 * ldx, ldx, M, K, perm, Xq);
        cudaError_t e;
        switch (bits) {
            case 2: e = launch_bits<2>(Xq, M, K, packed, P, scales, zeros, N, g, Y + t0 * ldy, ldy, stream); break;
            case 4: e = launch_bits<4>(Xq, M, K, packed, P, scales, zeros, N, g, Y + t0 * ldy, ldy, stream); break;
            case 8: e = launch_bits<8>(Xq, M, K, packed, P, scales, zeros, N, g, Y + t0 * ldy, ldy, stream); break;
            default: return GPTQ_ERR_UNSUPPORTED;
        }
        if (e != cudaSuccess) return GPTQ_ERR_CUDA;
        launches += 2;
    }
    count_launches(launches);
    return GPTQ_OK;
}

}  // namespace gptq
