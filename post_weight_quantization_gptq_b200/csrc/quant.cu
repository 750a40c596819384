// Stages 3-4: the GPTQ column walk.
//
// "GPTQ (GPT Quantization)", "Algorithme complet", step 3: the columns are
// walked in batches; each batch is quantized and its errors are applied to
// the remaining columns in one product (the "lazy update").  Inside a batch
// every column follows the OBQ step of "Fondation theorique : OBQ":
//   q_i = Quant(w_i),  W_F <- W_F - (w_i - q_i) / (H^-1)_ii * (H^-1)_{i,F}
// which, with U the upper factor of the eliminated inverse, is
//   e_i = (w_i - q_i) / U_ii,  W_F <- W_F - e_i * U_{i,F}.
// The quantizer is the AutoGPTQ guide's group-wise asymmetric one
// ("Quantizacao group-wise"): per row and group, scale and zero point from
// the group's current min / max (range widened to contain 0).
//
// Kernels:
//  permute_rows_kernel  W[:, k] <- W[:, perm[k]] (0 for dead columns), in place
//  block_quant_kernel   one 128-column block: row-parallel, 8 lanes per row,
//                       the block's U in shared memory, the column loop
//                       sequential with one shuffle per column
//  lazy_update_kernel   W[:, c1:] -= Err * U[c0:c1, c1:]
#include <cmath>

#include "common.cuh"
#include "kernels.h"

namespace gptq {
namespace {

constexpr int kBlock = 128;       // columns per block (the only supported block size)
constexpr int kRowsPerWarp = 4;   // 8 lanes per row
constexpr int kWarps = 4;
constexpr int kRowsPerCta = kRowsPerWarp * kWarps;

// ------------------------------------------------------------------------
__global__ void permute_rows_kernel(float* __restrict__ W, int64_t r, int64_t d, int64_t ldw,
                                    const int32_t* __restrict__ perm,
                                    const uint8_t* __restrict__ dead) {
    extern __shared__ float rowbuf[];
    for (int64_t row = blockIdx.x; row < r; row += gridDim.x) {
        float* w = W + row * ldw;
        for (int64_t k = threadIdx.x; k < d; k += blockDim.x) rowbuf[k] = w[k];
        __syncthreads();
        for (int64_t k = threadIdx.x; k < d; k += blockDim.x) {
            const int32_t src = perm[k];
            w[k] = dead[src] ? 0.f : rowbuf[src];
        }
        __syncthreads();
    }
}

// Column j of the block lives in lane ((j % 32) / 4) of its row group, in
// register 4 * (j / 32) + (j % 4): each lane owns four runs of 4 columns, 32
// apart, so the 8 lanes of a row read one 128-byte row segment of the U
// block per vector load without bank conflicts.
__device__ __forceinline__ int col_of(int t, int l) { return 32 * (t >> 2) + 4 * l + (t & 3); }

__global__ void __launch_bounds__(kWarps * 32)
    block_quant_kernel(float* __restrict__ W, int64_t r, int64_t d, int64_t ldw,
                       const float* __restrict__ U, int64_t c0, int bw, int bits, int g,
                       uint8_t* __restrict__ codes, float* __restrict__ scales,
                       int32_t* __restrict__ zeros, float* __restrict__ err_out) {
    extern __shared__ __align__(16) float smem[];
    float* Us = smem;                    // [kBlock][kBlock], strict upper part of U's block
    float* dinv = smem + kBlock * kBlock;  // 1 / U_jj
    const int tid = threadIdx.x;
    for (int e = tid; e < kBlock * kBlock; e += blockDim.x) {
        const int j = e / kBlock, f = e % kBlock;
        Us[e] = (j < bw && f < bw && f > j) ? U[(c0 + j) * d + c0 + f] : 0.f;
    }
    for (int j = tid; j < kBlock; j += blockDim.x)
        dinv[j] = (j < bw) ? 1.f / U[(c0 + j) * d + c0 + j] : 0.f;
    __syncthreads();

    const int lane = tid & 31;
    const int l = lane & 7;
    const int gbase = lane & ~7;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * kRowsPerCta + (tid >> 5) * kRowsPerWarp +
                        (lane >> 3);
    const bool live = row < r;
    const float maxq = static_cast<float>((1 << bits) - 1);

    float w[16], ev[16];
    uint32_t qv[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) {
        const int c = col_of(t, l);
        w[t] = (live && c < bw) ? W[row * ldw + c0 + c] : 0.f;
        ev[t] = 0.f;
        qv[t] = 0;
    }

    float s = 1.f, inv_s = 1.f, zf = 0.f;
    if (live && (c0 % g) != 0) {
        // this block continues a group opened by an earlier block (group
        // size > block): take that group's scale and zero point
        const int64_t grp = c0 / g;
        s = scales[grp * r + row];
        zf = static_cast<float>(zeros[grp * r + row]);
        inv_s = 1.f / s;
    }
#pragma unroll
    for (int j = 0; j < kBlock; ++j) {
        if (j < bw) {
        if (((c0 + j) % g) == 0) {
            // group [c0 + j, c0 + j + g): current weights, range widened to 0
            float lo = 0.f, hi = 0.f;
#pragma unroll
            for (int t = 0; t < 16; ++t) {
                const int c = col_of(t, l);
                if (c >= j && c < j + g && c < bw) {
                    lo = fminf(lo, w[t]);
                    hi = fmaxf(hi, w[t]);
                }
            }
            const int64_t gend = (c0 + j + g < d) ? c0 + j + g : d;
            if (live && gend > c0 + bw) {
                // group continues past this block (group_size > block): those
                // columns already hold every earlier block's feedback
                for (int64_t c = c0 + bw + l; c < gend; c += 8) {
                    const float v = W[row * ldw + c];
                    lo = fminf(lo, v);
                    hi = fmaxf(hi, v);
                }
            }
#pragma unroll
            for (int o = 1; o < 8; o <<= 1) {
                lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
                hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
            }
            if (hi == lo) {
                // all-zero group: range [-1, 1], zero point exactly 2^(bits-1)
                s = 2.f / maxq;
                zf = static_cast<float>(1 << (bits - 1));
            } else {
                s = (hi - lo) / maxq;
                zf = rintf(-lo / s);
            }
            inv_s = 1.f / s;
            if (live && l == 0) {
                const int64_t grp = (c0 + j) / g;
                scales[grp * r + row] = s;
                zeros[grp * r + row] = static_cast<int32_t>(zf);
            }
        }
        const int owner = (j & 31) >> 2;
        const int tj = 4 * (j >> 5) + (j & 3);
        const float wj = __shfl_sync(0xffffffffu, w[tj], gbase + owner);
        const float qf = fminf(fmaxf(rintf(wj * inv_s) + zf, 0.f), maxq);
        const float e = (wj - s * (qf - zf)) * dinv[j];
        if (l == owner) {
            qv[tj] = static_cast<uint32_t>(qf);
            ev[tj] = e;
        }
        // feedback into this block's later columns (U row j is zero at and
        // left of the diagonal, so earlier columns are untouched)
        const float4* urow = reinterpret_cast<const float4*>(Us + j * kBlock);
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const float4 u = urow[8 * m + l];
            w[4 * m + 0] = fmaf(-e, u.x, w[4 * m + 0]);
            w[4 * m + 1] = fmaf(-e, u.y, w[4 * m + 1]);
            w[4 * m + 2] = fmaf(-e, u.z, w[4 * m + 2]);
            w[4 * m + 3] = fmaf(-e, u.w, w[4 * m + 3]);
        }
        }
    }

    if (!live) return;
#pragma unroll
    for (int t = 0; t < 16; ++t) {
        const int c = col_of(t, l);
        if (c < bw) {
            W[row * ldw + c0 + c] = w[t];
            err_out[row * kBlock + c] = ev[t];
            codes[row * d + c0 + c] = static_cast<uint8_t>(qv[t]);
        }
    }
}

// ------------------------------------------------------------------------
// W[:, c1:d] -= Err[:, 0:bw] * U[c0:c0+bw, c1:d]  (fp32 FFMA, 64 x 64 tiles)
constexpr int TS = 64;
__global__ void __launch_bounds__(256)
    lazy_update_kernel(float* __restrict__ W, int64_t r, int64_t d, int64_t ldw,
                       const float* __restrict__ U, int64_t c0, int bw,
                       const float* __restrict__ err) {
    __shared__ float As[TS][TS + 1];  // Err tile: rows, k
    __shared__ float Bs[TS][TS + 1];  // U^T tile: cols, k
    const int tid = threadIdx.x;
    const int64_t c1 = c0 + bw;
    const int64_t col0 = c1 + static_cast<int64_t>(blockIdx.x) * TS;
    const int64_t row0 = static_cast<int64_t>(blockIdx.y) * TS;
    const int tx = tid & 15, ty = tid >> 4;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < bw; k0 += TS) {
        for (int e = tid; e < TS * TS; e += 256) {
            const int i = e / TS, k = e % TS;
            As[i][k] = (row0 + i < r && k0 + k < bw) ? err[(row0 + i) * kBlock + k0 + k] : 0.f;
            const int kk = e / TS, cc = e % TS;
            Bs[cc][kk] = (k0 + kk < bw && col0 + cc < d) ? U[(c0 + k0 + kk) * d + col0 + cc] : 0.f;
        }
        __syncthreads();
#pragma unroll 4
        for (int k = 0; k < TS; ++k) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = As[ty + 16 * i][k];
#pragma unroll
            for (int i = 0; i < 4; ++i) b[i] = Bs[tx + 16 * i][k];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int q = 0; q < 4; ++q) acc[i][q] = fmaf(a[i], b[q], acc[i][q]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int64_t rr = row0 + ty + 16 * i;
        if (rr >= r) continue;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int64_t cc = col0 + tx + 16 * q;
            if (cc < d) W[rr * ldw + cc] -= acc[i][q];
        }
    }
}

}  // namespace

size_t quant_workspace_bytes(int64_t d_row, int64_t, int block) {
    return ((static_cast<size_t>(d_row) * block * sizeof(float) + 255) / 256) * 256;
}

gptq_status launch_quantize(float* W, int64_t d_row, int64_t d_col, int64_t ldw, const float* U,
                            const int32_t* perm, const uint8_t* dead, int bits, int group,
                            int block, uint8_t* codes, float* scales, int32_t* zeros,
                            int32_t* status, void* ws, cudaStream_t stream) {
    (void)status;
    if (block != kBlock) return GPTQ_ERR_UNSUPPORTED;
    const int g = (group == -1 || group > d_col) ? static_cast<int>(d_col) : group;
    float* err = static_cast<float*>(ws);

    const size_t row_smem = static_cast<size_t>(d_col) * sizeof(float);
    if (cudaFuncSetAttribute(permute_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(row_smem)) != cudaSuccess)
        return GPTQ_ERR_CUDA;
    const int prow_grid = static_cast<int>(d_row < 4 * num_sms() ? d_row : 4 * num_sms());
    permute_rows_kernel<<<prow_grid, 256, row_smem, stream>>>(W, d_row, d_col, ldw, perm, dead);
    count_launches(1);

    const size_t q_smem = (kBlock * kBlock + kBlock) * sizeof(float);
    if (cudaFuncSetAttribute(block_quant_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(q_smem)) != cudaSuccess)
        return GPTQ_ERR_CUDA;
    const unsigned qgrid = static_cast<unsigned>((d_row + kRowsPerCta - 1) / kRowsPerCta);
    for (int64_t c0 = 0; c0 < d_col; c0 += kBlock) {
        const int bw = static_cast<int>((d_col - c0 < kBlock) ? d_col - c0 : kBlock);
        block_quant_kernel<<<qgrid, kWarps * 32, q_smem, stream>>>(
            W, d_row, d_col, ldw, U, c0, bw, bits, g, codes, scales, zeros, err);
        count_launches(1);
        const int64_t rest = d_col - c0 - bw;
        if (rest > 0) {
            dim3 grid(static_cast<unsigned>((rest + TS - 1) / TS),
                      static_cast<unsigned>((d_row + TS - 1) / TS));
            lazy_update_kernel<<<grid, 256, 0, stream>>>(W, d_row, d_col, ldw, U, c0, bw, err);
            count_launches(1);
        }
    }
    return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ERR_CUDA;
}

}  // namespace gptq
