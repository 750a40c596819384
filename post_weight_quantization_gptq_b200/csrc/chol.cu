// Stage 2b: the inverse factor U of the damped Hessian.
//
// The pseudo-code of "GPTQ (GPT Quantization)" ("Algorithme complet", step 2)
// inverts H through Cholesky.  What the column walk actually consumes is the
// OBQ-eliminated inverse: row i of (H^-1 reduced to the columns >= i).  Those
// rows, scaled by 1/sqrt(pivot), form the upper triangular U with
// H^-1 = U^T U.  With J the exchange matrix and P = J H J = L L^T (a lower
// Cholesky factor), H = (J L J)(J L J)^T with J L J upper triangular, so
// H^-1 = (J L^-1 J)^T (J L^-1 J) and U = J L^-1 J: one Cholesky factorization
// and one triangular inverse (2/3 d^3 flops) instead of the
// factor / invert / refactor route (4/3 d^3).
//
// The exchange J is folded into the gather that builds P (prep.cu) and into
// the final store here, so no extra pass is spent on it.
//
//   P buffer (d x d, ld d, the caller's U): lower triangle = P on entry,
//            L after the factorization; its upper triangle holds the
//            recursive-inverse temporaries; finally U.
//   X buffer (the caller's consumed H, ld ldx): lower triangle = L^-1.
//
// v1 arithmetic: fp32 FFMA everywhere (no TF32 rounding anywhere in this
// stage), tiles of 64.
#include <cmath>

#include "common.cuh"
#include "kernels.h"

namespace gptq {
namespace {

constexpr int NB = 64;  // panel width / tile edge
constexpr int kThreads = 256;

// ------------------------------------------------------------------------
// Diagonal block: L_kk = chol(A_kk) and its inverse (written into X's
// diagonal block, upper part zeroed).
__global__ void __launch_bounds__(kThreads)
    potrf_diag_kernel(float* __restrict__ P, int64_t ldp, int64_t kb, int kw,
                      float* __restrict__ X, int64_t ldx, int32_t* status) {
    __shared__ float S[NB][NB + 1];
    __shared__ float Xs[NB][NB + 1];
    __shared__ float diag[NB];
    __shared__ int bad;
    const int tid = threadIdx.x;
    if (tid == 0) bad = 0;
    for (int e = tid; e < NB * NB; e += kThreads) {
        const int i = e / NB, j = e % NB;
        float v = 0.f;
        if (i < kw && j <= i) v = P[(kb + i) * ldp + kb + j];
        S[i][j] = v;
        Xs[i][j] = 0.f;
    }
    __syncthreads();
    for (int c = 0; c < kw; ++c) {
        float piv = S[c][c];
        if (!(piv > 0.f)) {  // not positive definite (or NaN): flag it, keep going finite
            bad = 1;
            piv = 1.f;
        }
        const float lcc = sqrtf(piv);
        const float inv = 1.f / lcc;
        if (tid == 0) diag[c] = lcc;
        for (int i = c + 1 + tid; i < kw; i += kThreads) S[i][c] *= inv;
        __syncthreads();
        const int m = kw - c - 1;
        for (int e = tid; e < m * m; e += kThreads) {
            const int i = c + 1 + e / m, j = c + 1 + e % m;
            if (j <= i) S[i][j] -= S[i][c] * S[j][c];
        }
        __syncthreads();
    }
    for (int c = tid; c < kw; c += kThreads) S[c][c] = diag[c];
    __syncthreads();
    // L back into P (lower part of the block)
    for (int e = tid; e < kw * kw; e += kThreads) {
        const int i = e / kw, j = e % kw;
        if (j <= i) P[(kb + i) * ldp + kb + j] = S[i][j];
    }
    // Xs = L^-1 by rows: X_ii = 1/L_ii, X_ij = -(sum_{j<=k<i} L_ik X_kj) / L_ii.
    // Four threads share one column j and split the k-sum.
    const int j = tid >> 2, part = tid & 3;
    for (int i = 0; i < kw; ++i) {
        float acc = 0.f;
        if (j < i) {
            for (int k = j + part; k < i; k += 4) acc = fmaf(S[i][k], Xs[k][j], acc);
        }
        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
        if (part == 0 && j < kw) {
            if (j == i) Xs[i][i] = 1.f / S[i][i];
            else if (j < i) Xs[i][j] = -acc / S[i][i];
        }
        __syncwarp();
        __syncthreads();
    }
    for (int e = tid; e < kw * kw; e += kThreads) {
        const int i = e / kw, jj = e % kw;
        X[(kb + i) * ldx + kb + jj] = (jj <= i) ? Xs[i][jj] : 0.f;
    }
    if (tid == 0 && bad) report(status, GPTQ_ERR_NOT_PD);
}

// 64 x 64 tile product helper: acc[a][b] += sum_k As[ty + 16a][k] * Bs[tx + 16b][k]
__device__ __forceinline__ void tile_fma(float (&acc)[4][4], const float (*As)[NB + 1],
                                         const float (*Bs)[NB + 1], int kmax) {
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
#pragma unroll 4
    for (int k = 0; k < kmax; ++k) {
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
}

// ------------------------------------------------------------------------
// Panel: L[i, kb:kb+kw] = A[i, kb:kb+kw] * (L_kk^-1)^T for rows below the
// diagonal block.
__global__ void __launch_bounds__(kThreads)
    trsm_panel_kernel(float* __restrict__ P, int64_t ldp, int64_t kb, int kw, int64_t d,
                      const float* __restrict__ X, int64_t ldx) {
    __shared__ float As[NB][NB + 1];
    __shared__ float Ls[NB][NB + 1];
    const int tid = threadIdx.x;
    const int64_t r0 = kb + kw + static_cast<int64_t>(blockIdx.x) * NB;
    for (int e = tid; e < NB * NB; e += kThreads) {
        const int i = e / NB, k = e % NB;
        As[i][k] = (r0 + i < d && k < kw) ? P[(r0 + i) * ldp + kb + k] : 0.f;
        Ls[i][k] = (i < kw && k <= i) ? X[(kb + i) * ldx + kb + k] : 0.f;
    }
    __syncthreads();
    float acc[4][4] = {};
    tile_fma(acc, As, Ls, kw);
    const int tx = tid & 15, ty = tid >> 4;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int64_t r = r0 + ty + 16 * i;
        if (r >= d) continue;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int c = tx + 16 * q;
            if (c < kw) P[r * ldp + kb + c] = acc[i][q];
        }
    }
}

// Lower-triangular tile index t -> (I, J), I >= J.
__device__ __forceinline__ void tri_coords(int t, int& I, int& J) {
    int i = static_cast<int>((sqrtf(8.f * static_cast<float>(t) + 1.f) - 1.f) * 0.5f);
    while (i * (i + 1) / 2 > t) --i;
    while ((i + 1) * (i + 2) / 2 <= t) ++i;
    I = i;
    J = t - i * (i + 1) / 2;
}

// ------------------------------------------------------------------------
// Trailing update: A[I, J] -= L[I, panel] L[J, panel]^T for the lower tiles
// of the trailing matrix.
__global__ void __launch_bounds__(kThreads)
    syrk_update_kernel(float* __restrict__ P, int64_t ldp, int64_t kb, int kw, int64_t d) {
    __shared__ float As[NB][NB + 1];
    __shared__ float Bs[NB][NB + 1];
    const int tid = threadIdx.x;
    int I, J;
    tri_coords(blockIdx.x, I, J);
    const int64_t s0 = kb + kw;
    const int64_t ri = s0 + static_cast<int64_t>(I) * NB, rj = s0 + static_cast<int64_t>(J) * NB;
    for (int e = tid; e < NB * NB; e += kThreads) {
        const int i = e / NB, k = e % NB;
        As[i][k] = (ri + i < d && k < kw) ? P[(ri + i) * ldp + kb + k] : 0.f;
        Bs[i][k] = (rj + i < d && k < kw) ? P[(rj + i) * ldp + kb + k] : 0.f;
    }
    __syncthreads();
    float acc[4][4] = {};
    tile_fma(acc, As, Bs, kw);
    const int tx = tid & 15, ty = tid >> 4;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int64_t r = ri + ty + 16 * i;
        if (r >= d) continue;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int64_t c = rj + tx + 16 * q;
            if (c < d && c <= r) P[r * ldp + c] -= acc[i][q];
        }
    }
}

// ------------------------------------------------------------------------
// Triangular inverse by recursive doubling.  With the diagonal blocks of
// size s already inverted, each pair (A = [A0, A0+s), C = [C0, C0+s) clipped
// to d) gets
//   X_CA = -X_CC (L_CA X_AA).
// Step 1: T = L_CA X_AA, stored transposed into the P buffer's (free) upper
// triangle: T[c][a] at P[a][c] (a < C0 <= c, so it never touches L).
__global__ void __launch_bounds__(kThreads)
    trinv_step1_kernel(float* __restrict__ P, int64_t ldp, const float* __restrict__ X,
                       int64_t ldx, int64_t d, int64_t s, int ctiles, int atiles) {
    __shared__ float As[NB][NB + 1];  // X_AA^T tile: rows a, cols k (= X[k][a])
    __shared__ float Bs[NB][NB + 1];  // L_CA tile:   rows c, cols k
    const int tid = threadIdx.x;
    const int per_pair = ctiles * atiles;
    const int pair = blockIdx.x / per_pair;
    const int rem = blockIdx.x % per_pair;
    const int ct = rem / atiles, at = rem % atiles;
    const int64_t A0 = 2 * s * pair, C0 = A0 + s;
    const int64_t c0 = C0 + static_cast<int64_t>(ct) * NB;
    const int64_t a0 = A0 + static_cast<int64_t>(at) * NB;
    if (c0 >= d) return;
    float acc[4][4] = {};
    // k runs over A with k >= a: from this a-tile to the end of A (the
    // diagonal 64-blocks of X have a zeroed upper part)
    for (int64_t k0 = a0; k0 < C0; k0 += NB) {
        for (int e = tid; e < NB * NB; e += kThreads) {
            const int lo = e % NB, hi = e / NB;
            As[lo][hi] = X[(k0 + hi) * ldx + a0 + lo];                        // X[k][a]
            Bs[hi][lo] = (c0 + hi < d) ? P[(c0 + hi) * ldp + k0 + lo] : 0.f;  // L[c][k]
        }
        __syncthreads();
        tile_fma(acc, As, Bs, NB);
        __syncthreads();
    }
    const int tx = tid & 15, ty = tid >> 4;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int64_t a = a0 + ty + 16 * i;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int64_t c = c0 + tx + 16 * q;
            if (c < d) P[a * ldp + c] = acc[i][q];
        }
    }
}

// Step 2: X_CA = -X_CC T, with T[k][a] read back from P[a][k].
__global__ void __launch_bounds__(kThreads)
    trinv_step2_kernel(const float* __restrict__ P, int64_t ldp, float* __restrict__ X,
                       int64_t ldx, int64_t d, int64_t s, int ctiles, int atiles) {
    __shared__ float As[NB][NB + 1];  // X_CC tile: rows c, cols k
    __shared__ float Bs[NB][NB + 1];  // T^T tile:  rows a, cols k (= P[a][k])
    const int tid = threadIdx.x;
    const int per_pair = ctiles * atiles;
    const int pair = blockIdx.x / per_pair;
    const int rem = blockIdx.x % per_pair;
    const int ct = rem / atiles, at = rem % atiles;
    const int64_t A0 = 2 * s * pair, C0 = A0 + s;
    const int64_t c0 = C0 + static_cast<int64_t>(ct) * NB;
    const int64_t a0 = A0 + static_cast<int64_t>(at) * NB;
    if (c0 >= d) return;
    float acc[4][4] = {};
    // k runs over C with k <= c: from the start of C to this c-tile
    for (int64_t k0 = C0; k0 <= c0; k0 += NB) {
        for (int e = tid; e < NB * NB; e += kThreads) {
            const int k = e % NB, i = e / NB;
            const bool kin = k0 + k < d;
            As[i][k] = (c0 + i < d && kin) ? X[(c0 + i) * ldx + k0 + k] : 0.f;
            Bs[i][k] = kin ? P[(a0 + i) * ldp + k0 + k] : 0.f;
        }
        __syncthreads();
        tile_fma(acc, As, Bs, NB);
        __syncthreads();
    }
    const int tx = tid & 15, ty = tid >> 4;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int64_t c = c0 + ty + 16 * i;
        if (c >= d) continue;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int64_t a = a0 + tx + 16 * q;
            X[c * ldx + a] = -acc[i][q];
        }
    }
}

// U[i][j] = X[d-1-i][d-1-j] for j >= i, 0 below the diagonal.
__global__ void flip_kernel(const float* __restrict__ X, int64_t ldx, float* __restrict__ U,
                            int64_t d) {
    const int64_t i = blockIdx.y;
    for (int64_t j = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; j < d;
         j += static_cast<int64_t>(gridDim.x) * blockDim.x)
        U[i * d + j] = (j >= i) ? X[(d - 1 - i) * ldx + (d - 1 - j)] : 0.f;
}

}  // namespace

size_t chol_workspace_bytes(int64_t) { return 0; }

gptq_status launch_chol_inverse(float* P, float* X, int64_t ldx, int64_t d, float* U,
                                int32_t* status, void*, cudaStream_t stream) {
    const int64_t ldp = d;
    for (int64_t kb = 0; kb < d; kb += NB) {
        const int kw = static_cast<int>((d - kb < NB) ? d - kb : NB);
        potrf_diag_kernel<<<1, kThreads, 0, stream>>>(P, ldp, kb, kw, X, ldx, status);
        count_launches(1);
        const int64_t m = d - kb - kw;
        if (m > 0) {
            const int mt = static_cast<int>((m + NB - 1) / NB);
            trsm_panel_kernel<<<mt, kThreads, 0, stream>>>(P, ldp, kb, kw, d, X, ldx);
            syrk_update_kernel<<<mt * (mt + 1) / 2, kThreads, 0, stream>>>(P, ldp, kb, kw, d);
            count_launches(2);
        }
    }
    for (int64_t s = NB; s < d; s *= 2) {
        const int64_t pairs = (d + 2 * s - 1) / (2 * s);
        const int ctiles = static_cast<int>(s / NB), atiles = static_cast<int>(s / NB);
        const int64_t grid = pairs * ctiles * atiles;
        trinv_step1_kernel<<<static_cast<unsigned>(grid), kThreads, 0, stream>>>(P, ldp, X, ldx, d,
                                                                                 s, ctiles, atiles);
        trinv_step2_kernel<<<static_cast<unsigned>(grid), kThreads, 0, stream>>>(P, ldp, X, ldx, d,
                                                                                 s, ctiles, atiles);
        count_launches(2);
    }
    dim3 grid(static_cast<unsigned>((d + 255) / 256 < 8 ? (d + 255) / 256 : 8),
              static_cast<unsigned>(d));
    flip_kernel<<<grid, 256, 0, stream>>>(X, ldx, U, d);
    count_launches(1);
    return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ERR_CUDA;
}

}  // namespace gptq
