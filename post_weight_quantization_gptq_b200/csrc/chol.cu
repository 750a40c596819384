// Stage 2b: the inverse factor U of the damped Hessian.
//
// The pseudo-code of "GPTQ (GPT Quantization)" ("Algorithme complet", step 2)
// inverts H through Cholesky.  What the column walk consumes is the
// OBQ-eliminated inverse: row i of (H^-1 reduced to the columns >= i).  Those
// rows, scaled by 1/sqrt(pivot), form the upper triangular U with
// H^-1 = U^T U.  With J the exchange matrix and P = J H J = L L^T (a lower
// Cholesky factor), H = (J L J)(J L J)^T with J L J upper triangular, so
// H^-1 = (J L^-1 J)^T (J L^-1 J) and U = J L^-1 J: one Cholesky factorization
// and one triangular inverse (2/3 d^3 flops) instead of the
// factor / invert / refactor route (4/3 d^3).  The exchange J is folded into
// the gather that builds P (prep.cu) and into the final store here.
//
//   P buffer (d x d, ld d, the caller's U): lower triangle = P on entry, L
//            after the factorization; its strict upper triangle holds the
//            recursive-inverse temporaries; finally U.
//   X buffer (the caller's consumed H, ld ldx): lower triangle = L^-1, with
//            every 128 x 128 diagonal block's strict upper part zeroed.
//
// Blocked right-looking Cholesky with 128-wide panels:
//   potrf_inv_128_kernel  L_kk = chol(A_kk) and L_kk^-1 (one CTA)
//   panel solve           L_ik = A_ik L_kk^-T          (3xTF32 tcgen05 GEMM)
//   trailing update       A_ij -= L_ik L_jk^T, i >= j  (3xTF32 tcgen05 GEMM)
// then L^-1 by recursive doubling (X_CA = -X_CC (L_CA X_AA)) on the same GEMM.
#include <cmath>

#include "common.cuh"
#include "gemm_tf32x3.cuh"
#include "kernels.h"

namespace gptq {
namespace {

constexpr int NB = 128;      // panel width
constexpr int LDA = NB + 1;  // shared-memory row pitch of the diagonal block
constexpr int kDiagThreads = 256;
constexpr int kDiagSmem = (2 * NB * LDA + 64 * 65 + NB) * 4;
constexpr unsigned kFull = 0xffffffffu;

// ------------------------------------------------------------------------
// Diagonal block: L = chol(A) and X = L^-1 for a kw x kw (kw <= 128) block,
// padded with the identity.  Four 32-wide strips: one warp factors and
// inverts the strip's 32 x 32 diagonal block in registers, then the CTA
// solves the strip below and updates the trailing part; finally the four
// 32 x 32 inverses are joined by two levels of recursive doubling.
__global__ void __launch_bounds__(kDiagThreads, 1)
    potrf_inv_128_kernel(float* __restrict__ P, int64_t ldp, int64_t kb, int kw,
                         float* __restrict__ X, int64_t ldx, int32_t* status) {
    extern __shared__ float sm[];
    float* A = sm;              // [128][129] the block, L in its lower part
    float* Xs = A + NB * LDA;   // [128][129] L^-1
    float* T = Xs + NB * LDA;   // [64][65] doubling temporary
    float* dinv = T + 64 * 65;  // [128] 1 / L_ii
    __shared__ int bad;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) bad = 0;
    for (int e = tid; e < NB * NB; e += kDiagThreads) {
        const int i = e >> 7, j = e & (NB - 1);
        float v = (i == j) ? 1.f : 0.f;
        if (i < kw && j <= i) v = P[(kb + i) * ldp + kb + j];
        A[i * LDA + j] = v;
        Xs[i * LDA + j] = 0.f;
    }
    __syncthreads();

    for (int b = 0; b < 4; ++b) {
        const int o = 32 * b;
        if (warp == 0) {
            // -- 32 x 32 Cholesky in registers: lane i holds row o + i
            float a[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) a[j] = (j <= lane) ? A[(o + lane) * LDA + o + j] : 0.f;
#pragma unroll
            for (int c = 0; c < 32; ++c) {
                float piv = __shfl_sync(kFull, a[c], c);
                if (!(piv > 0.f)) {  // not positive definite (or NaN): flag, stay finite
                    bad = 1;
                    piv = 1.f;
                }
                const float lcc = sqrtf(piv);
                const float inv = 1.f / lcc;
                if (lane == c) a[c] = lcc;
                else if (lane > c) a[c] *= inv;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    if (j > c) {
                        const float ljc = __shfl_sync(kFull, a[c], j);
                        if (lane >= j) a[j] = fmaf(-a[c], ljc, a[j]);
                    }
                }
            }
            float dl = 1.f;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                if (j <= lane) A[(o + lane) * LDA + o + j] = a[j];
                if (j == lane) dl = a[j];
            }
            dinv[o + lane] = 1.f / dl;
            __syncwarp();
            // -- its inverse: lane j owns column j
            float x[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                float acc = 0.f;
#pragma unroll
                for (int k = 0; k < 32; ++k)
                    if (k < i) acc = fmaf(A[(o + i) * LDA + o + k], x[k], acc);
                const float di = dinv[o + i];
                x[i] = (i == lane) ? di : ((i > lane) ? -acc * di : 0.f);
            }
#pragma unroll
            for (int i = 0; i < 32; ++i) Xs[(o + i) * LDA + o + lane] = x[i];
        }
        __syncthreads();
        const int r0 = o + 32;
        if (r0 < NB) {
            // -- strip solve: L[i][o+j] = sum_{k<=j} A[i][o+k] Xs[o+j][o+k], i >= r0
            const int j = lane;
            float out[12];
#pragma unroll
            for (int q = 0; q < 12; ++q) {
                const int i = r0 + warp + 8 * q;
                float acc = 0.f;
                if (i < NB) {
                    for (int k = 0; k <= j; ++k)
                        acc = fmaf(A[i * LDA + o + k], Xs[(o + j) * LDA + o + k], acc);
                }
                out[q] = acc;
            }
            __syncthreads();
#pragma unroll
            for (int q = 0; q < 12; ++q) {
                const int i = r0 + warp + 8 * q;
                if (i < NB) A[i * LDA + o + j] = out[q];
            }
            __syncthreads();
            // -- trailing update of the lower part, 4 x 4 register blocks
            const int mb = (NB - r0) / 4;
            const int units = mb * (mb + 1) / 2;
            for (int u = tid; u < units; u += kDiagThreads) {
                int bi = static_cast<int>((sqrtf(8.f * u + 1.f) - 1.f) * 0.5f);
                while (bi * (bi + 1) / 2 > u) --bi;
                while ((bi + 1) * (bi + 2) / 2 <= u) ++bi;
                const int bj = u - bi * (bi + 1) / 2;
                const int i0 = r0 + 4 * bi, j0 = r0 + 4 * bj;
                float acc[4][4] = {};
#pragma unroll 4
                for (int k = 0; k < 32; ++k) {
                    float li[4], lj[4];
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        li[t] = A[(i0 + t) * LDA + o + k];
                        lj[t] = A[(j0 + t) * LDA + o + k];
                    }
#pragma unroll
                    for (int t = 0; t < 4; ++t)
#pragma unroll
                        for (int w = 0; w < 4; ++w) acc[t][w] = fmaf(li[t], lj[w], acc[t][w]);
                }
#pragma unroll
                for (int t = 0; t < 4; ++t)
#pragma unroll
                    for (int w = 0; w < 4; ++w)
                        if (j0 + w <= i0 + t) A[(i0 + t) * LDA + j0 + w] -= acc[t][w];
            }
        }
        __syncthreads();
    }

    // -- join the 32 x 32 inverses: X_CA = -X_CC (L_CA X_AA); T[p*s + c][a]
    for (int s = 32; s < NB; s *= 2) {
        const int pairs = NB / (2 * s);
        const int outs = pairs * s * s;
        for (int e = tid; e < outs; e += kDiagThreads) {
            const int p = e / (s * s), c = (e / s) % s, a = e % s;
            const int A0 = 2 * s * p, C0 = A0 + s;
            float acc = 0.f;
            for (int k = a; k < s; ++k)
                acc = fmaf(A[(C0 + c) * LDA + A0 + k], Xs[(A0 + k) * LDA + A0 + a], acc);
            T[(p * s + c) * 65 + a] = acc;
        }
        __syncthreads();
        for (int e = tid; e < outs; e += kDiagThreads) {
            const int p = e / (s * s), c = (e / s) % s, a = e % s;
            const int A0 = 2 * s * p, C0 = A0 + s;
            float acc = 0.f;
            for (int k = 0; k <= c; ++k)
                acc = fmaf(Xs[(C0 + c) * LDA + C0 + k], T[(p * s + k) * 65 + a], acc);
            Xs[(C0 + c) * LDA + A0 + a] = -acc;
        }
        __syncthreads();
    }

    for (int e = tid; e < kw * kw; e += kDiagThreads) {
        const int i = e / kw, j = e % kw;
        if (j <= i) P[(kb + i) * ldp + kb + j] = A[i * LDA + j];
    }
    // X's diagonal block, zeros above the diagonal included (the tensor-core
    // GEMMs read it as a full tile)
    for (int e = tid; e < kw * kw; e += kDiagThreads) {
        const int i = e / kw, j = e % kw;
        X[(kb + i) * ldx + kb + j] = (j <= i) ? Xs[i * LDA + j] : 0.f;
    }
    if (tid == 0 && bad) report(status, GPTQ_ERR_NOT_PD);
}

// Lower-triangular tile index t -> (I, J), I >= J.
__device__ __forceinline__ void tri_coords(int t, int& I, int& J) {
    int i = static_cast<int>((sqrtf(8.f * static_cast<float>(t) + 1.f) - 1.f) * 0.5f);
    while (i * (i + 1) / 2 > t) --i;
    while ((i + 1) * (i + 2) / 2 <= t) ++i;
    I = i;
    J = t - i * (i + 1) / 2;
}

// ---------------------------------------------------------------- schedulers
// Panel solve: L[m0.., kb..kb+kw) = A[m0.., kb..) (L_kk^-1)^T   (in place)
struct TrsmSched {
    float* P;
    int64_t ldp;
    int d, kb, kw;
    __device__ g3::Job job(int t) const { return {kb + kw + NB * t, kb, kb, kb, (kw + 31) / 32}; }
    __device__ void store(const g3::Job& jb, int row, int col0, const float (&v)[32]) const {
        const int r = jb.m0 + row;
        if (r >= d) return;
        float* dst = P + static_cast<int64_t>(r) * ldp + kb + col0;
#pragma unroll
        for (int j = 0; j < 32; ++j)
            if (col0 + j < kw) dst[j] = v[j];
    }
};

// Trailing update: P[I, J] -= L[I, panel] L[J, panel]^T on lower tiles.
struct SyrkSched {
    float* P;
    int64_t ldp;
    int d, kb, kw, s0;
    __device__ g3::Job job(int t) const {
        int I, J;
        tri_coords(t, I, J);
        return {s0 + NB * I, s0 + NB * J, kb, kb, (kw + 31) / 32};
    }
    __device__ void store(const g3::Job& jb, int row, int col0, const float (&v)[32]) const {
        const int r = jb.m0 + row;
        if (r >= d) return;
        float* dst = P + static_cast<int64_t>(r) * ldp + jb.n0 + col0;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const int c = jb.n0 + col0 + j;
            if (c < d && c <= r) dst[j] -= v[j];
        }
    }
};

// Recursive doubling, step 1: T^T[a][c] = sum_k X[k][a] L[c][k] into P[a][c].
struct Trinv1Sched {
    float* P;
    int64_t ldp;
    int d, s, tiles;  // tiles = s / NB per side
    __device__ g3::Job job(int t) const {
        const int per = tiles * tiles;
        const int pair = t / per, rem = t % per;
        const int ct = rem / tiles, at = rem % tiles;
        const int A0 = 2 * s * pair, C0 = A0 + s;
        const int c0 = C0 + NB * ct, a0 = A0 + NB * at;
        if (c0 >= d) return {0, 0, 0, 0, 0};
        return {a0, c0, a0, a0, (C0 - a0) / 32};
    }
    __device__ void store(const g3::Job& jb, int row, int col0, const float (&v)[32]) const {
        float* dst = P + static_cast<int64_t>(jb.m0 + row) * ldp + jb.n0 + col0;
#pragma unroll
        for (int j = 0; j < 32; ++j)
            if (jb.n0 + col0 + j < d) dst[j] = v[j];
    }
};

// Step 2: X[c][a] = -sum_{C0 <= k <= c} X[c][k] T[k][a], T[k][a] = P[a][k].
struct Trinv2Sched {
    float* X;
    int64_t ldx;
    int d, s, tiles;
    __device__ g3::Job job(int t) const {
        const int per = tiles * tiles;
        const int pair = t / per, rem = t % per;
        const int ct = rem / tiles, at = rem % tiles;
        const int A0 = 2 * s * pair, C0 = A0 + s;
        const int c0 = C0 + NB * ct, a0 = A0 + NB * at;
        if (c0 >= d) return {0, 0, 0, 0, 0};
        return {c0, a0, C0, C0, (c0 + NB - C0) / 32};
    }
    __device__ void store(const g3::Job& jb, int row, int col0, const float (&v)[32]) const {
        const int r = jb.m0 + row;
        if (r >= d) return;
        float* dst = X + static_cast<int64_t>(r) * ldx + jb.n0 + col0;
#pragma unroll
        for (int j = 0; j < 32; ++j) dst[j] = -v[j];
    }
};

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
    const int di = static_cast<int>(d);
    CUtensorMap tP, tX, tXmn;
    if (!make_tmap_2d(&tP, false, P, d, d, ldp, 32, 128, Swz::k128) ||
        !make_tmap_2d(&tX, false, X, d, d, ldx, 32, 128, Swz::k128) ||
        !make_tmap_2d(&tXmn, false, X, d, d, ldx, 32, 32, Swz::k128Atom32))
        return GPTQ_ERR_INVALID_ARG;
    if (cudaFuncSetAttribute(potrf_inv_128_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kDiagSmem) != cudaSuccess)
        return GPTQ_ERR_CUDA;
    int64_t launches = 0;
    for (int64_t kb = 0; kb < d; kb += NB) {
        const int kw = static_cast<int>((d - kb < NB) ? d - kb : NB);
        potrf_inv_128_kernel<<<1, kDiagThreads, kDiagSmem, stream>>>(P, ldp, kb, kw, X, ldx, status);
        ++launches;
        const int64_t m = d - kb - kw;
        if (m > 0) {
            const int mt = static_cast<int>((m + NB - 1) / NB);
            TrsmSched ts{P, ldp, di, static_cast<int>(kb), kw};
            if (g3::launch<TrsmSched, false, false>(tP, tX, ts, mt, status, stream) != cudaSuccess)
                return GPTQ_ERR_CUDA;
            SyrkSched ss{P, ldp, di, static_cast<int>(kb), kw, static_cast<int>(kb + kw)};
            if (g3::launch<SyrkSched, false, false>(tP, tP, ss, mt * (mt + 1) / 2, status, stream) !=
                cudaSuccess)
                return GPTQ_ERR_CUDA;
            launches += 2;
        }
    }
    for (int64_t s = NB; s < d; s *= 2) {
        const int64_t pairs = (d + 2 * s - 1) / (2 * s);
        const int tiles = static_cast<int>(s / NB);
        const int grid = static_cast<int>(pairs * tiles * tiles);
        Trinv1Sched t1{P, ldp, di, static_cast<int>(s), tiles};
        Trinv2Sched t2{X, ldx, di, static_cast<int>(s), tiles};
        if (g3::launch<Trinv1Sched, true, false>(tXmn, tP, t1, grid, status, stream) != cudaSuccess ||
            g3::launch<Trinv2Sched, false, false>(tX, tP, t2, grid, status, stream) != cudaSuccess)
            return GPTQ_ERR_CUDA;
        launches += 2;
    }
    dim3 grid(static_cast<unsigned>((d + 255) / 256 < 8 ? (d + 255) / 256 : 8),
              static_cast<unsigned>(d));
    flip_kernel<<<grid, 256, 0, stream>>>(X, ldx, U, d);
    count_launches(launches + 1);
    return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ERR_CUDA;
}

}  // namespace gptq
