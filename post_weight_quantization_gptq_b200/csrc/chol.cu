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
//            below the diagonal blocks after the factorization; finally U.
//   X buffer (the caller's consumed H, ld ldx): lower triangle = L^-1, with
//            every 128 x 128 diagonal block's strict upper part zeroed.
//
// Blocked right-looking Cholesky with 128-wide panels:
//   potrf_inv_128_kernel  L_kk = chol(A_kk) and L_kk^-1 (one CTA)
//   panel solve           L_ik = A_ik L_kk^-T          (3xTF32 tcgen05 GEMM)
//   trailing update       A_ij -= L_ik L_jk^T, i >= j  (3xTF32 tcgen05 GEMM)
// and L^-1 by right-looking forward substitution on the identity, on the
// same GEMM: with B the strictly lower block part of X (zero at the start),
// after panel k
//   X[k, :k] = L_kk^-1 B[k, :k]                (row k of L^-1 is then final)
//   B[i, :k+1] -= L[i, k] X[k, :k+1],  i > k   (its share of the later rows)
// in the shadow of the panel chain (see launch_chol_inverse).
#include <cmath>
#include <mutex>

#include "common.cuh"
#include "gemm_tf32x3.cuh"
#include "kernels.h"

namespace gptq {
namespace {

constexpr int NB = 128;      // panel width
constexpr int LDA = NB + 4;  // shared-memory row pitch: float4-aligned rows, rows 4 banks apart
constexpr int TP = 68;       // pitch of the doubling temporary
constexpr int kDiagThreads = 256;
constexpr int kDiagSmem = (2 * NB * LDA + 64 * TP + 32 * 32 + 32 * LDA + NB) * 4;

__device__ __forceinline__ float4 lds4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ void sts4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }

// ------------------------------------------------------------------------
// Diagonal block: L = chol(A) and X = L^-1 for a kw x kw (kw <= 128) block,
// padded with the identity.  Four 32-wide strips; for each, one warp factors
// the strip's 32 x 32 diagonal block, then four warps run one forward
// substitution on 128 right-hand sides (the identity -> the strip's inverse,
// and the rows below -> the strip of L), then the CTA updates the trailing
// part; finally the four 32 x 32 inverses are joined by two levels of
// recursive doubling.
//
// Column c of the strip's L below the diagonal is also kept as a row of Lc
// (Lc[c][m] = L[o+c+1+m][o+c], zero past the strip), so each elimination
// step reads it with eight broadcast float4 loads; the strip's rows below
// the diagonal block are kept transposed in Ls for the trailing update.  The factor warp keeps its
// rows in registers and rotates them after every column step, so the pivot
// column is always register 0: the step loop stays rolled (small code, the
// kernel runs once per panel on a cold SM) while every register index is a
// compile-time constant.
__global__ void __launch_bounds__(kDiagThreads, 1)
    potrf_inv_128_kernel(float* __restrict__ P, int64_t ldp, int64_t kb, int kw,
                         float* __restrict__ X, int64_t ldx, int32_t* status) {
    extern __shared__ __align__(16) float sm[];
    float* A = sm;              // [128][LDA] the block, L in its lower part
    float* Xs = A + NB * LDA;   // [128][LDA] L^-1
    float* T = Xs + NB * LDA;   // [64][TP] doubling temporary
    float* Lc = T + 64 * TP;    // [32][32] the current strip's columns of L, shifted
    float* Ls = Lc + 32 * 32;   // [32][LDA] the current strip of L below it, transposed
    float* dinv = Ls + 32 * LDA; // [128] 1 / L_ii
    __shared__ int bad;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) bad = 0;
    pdl_trigger();
    pdl_wait();
    {
        // rows of the block: 16 float4 loads per thread, all in flight
        // (ldp, kb and kw are multiples of 4, so a float4 never crosses kw).
        // Coherent (L2) loads: with a programmatic launch the kernel before
        // this one in the stream may still have been writing P when this one
        // started, so the read-only (non-coherent) path must not be used.
        float4 v[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) {
            const int e = tid + q * kDiagThreads;
            const int i = e >> 5, j = (e & 31) * 4;
            v[q] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (i < kw && j <= i) v[q] = __ldcg(reinterpret_cast<const float4*>(P + (kb + i) * ldp + kb + j));
        }
#pragma unroll
        for (int q = 0; q < 16; ++q) {
            const int e = tid + q * kDiagThreads;
            const int i = e >> 5, j = (e & 31) * 4;
            float vv[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
#pragma unroll
            for (int t = 0; t < 4; ++t)
                vv[t] = (j + t <= i && i < kw) ? vv[t] : (i == j + t ? 1.f : 0.f);
            sts4(A + i * LDA + j, make_float4(vv[0], vv[1], vv[2], vv[3]));
            sts4(Xs + i * LDA + j, make_float4(0.f, 0.f, 0.f, 0.f));
        }
    }
    __syncthreads();

    // -- 32 x 32 Cholesky of the diagonal block at o, by warp 0: lane i holds
    //    row o + i, register r = column c + r
    auto chol32 = [&](int o) {
        float a[32];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const float4 t = lds4(A + (o + lane) * LDA + o + 4 * q);
            a[4 * q] = t.x; a[4 * q + 1] = t.y; a[4 * q + 2] = t.z; a[4 * q + 3] = t.w;
        }
#pragma unroll
        for (int r = 0; r < 32; ++r) a[r] = (r <= lane) ? a[r] : 0.f;
#pragma unroll 1
        for (int c = 0; c < 32; ++c) {
            float piv = __shfl_sync(0xffffffffu, a[0], c);
            if (!(piv > 0.f)) {  // not positive definite (or NaN): flag, stay finite
                bad = 1;
                piv = 1.f;
            }
            const float inv = rsqrtf(piv);
            const float a0 = (lane == c) ? piv * inv : ((lane > c) ? a[0] * inv : 0.f);
            if (lane >= c) A[(o + lane) * LDA + o + c] = a0;
            if (lane == c) dinv[o + c] = inv;
            // lane i > c holds L[o+i][o+c] -> Lc[c][i-c-1]; lanes <= c fill the tail with 0
            Lc[c * 32 + ((lane - c - 1) & 31)] = a0 * (lane > c ? 1.f : 0.f);
            __syncwarp();
#pragma unroll
            for (int q = 0; q < 8; ++q) {  // update and rotate
                const float4 l = lds4(Lc + c * 32 + 4 * q);
                a[4 * q] = fmaf(-a0, l.x, a[4 * q + 1]);
                a[4 * q + 1] = fmaf(-a0, l.y, a[4 * q + 2]);
                a[4 * q + 2] = fmaf(-a0, l.z, a[4 * q + 3]);
                a[4 * q + 3] = (q < 7) ? fmaf(-a0, l.w, a[4 * q + 4]) : 0.f;
            }
        }
    };
    // -- trailing update of the lower part below strip o, 4 x 4 register blocks
    //    u in [u0, u1) (triangular numbering from row r0), read from the
    //    transposed strip (consecutive blocks -> consecutive float4)
    auto trail = [&](int r0, int u0, int u1, int t, int stride) {
        for (int u = u0 + t; u < u1; u += stride) {
            int bi = static_cast<int>((sqrtf(8.f * u + 1.f) - 1.f) * 0.5f);
            while (bi * (bi + 1) / 2 > u) --bi;
            while ((bi + 1) * (bi + 2) / 2 <= u) ++bi;
            const int bj = u - bi * (bi + 1) / 2;
            const int i0 = r0 + 4 * bi, j0 = r0 + 4 * bj;
            float acc2[4][4] = {};
#pragma unroll 8
            for (int k = 0; k < 32; ++k) {
                const float4 li = lds4(Ls + k * LDA + i0), lj = lds4(Ls + k * LDA + j0);
                const float a4[4] = {li.x, li.y, li.z, li.w}, b4[4] = {lj.x, lj.y, lj.z, lj.w};
#pragma unroll
                for (int t4 = 0; t4 < 4; ++t4)
#pragma unroll
                    for (int w = 0; w < 4; ++w) acc2[t4][w] = fmaf(a4[t4], b4[w], acc2[t4][w]);
            }
#pragma unroll
            for (int t4 = 0; t4 < 4; ++t4) {
                float* dst = A + (i0 + t4) * LDA + j0;
                if (j0 + 3 <= i0 + t4) {
                    float4 d4 = lds4(dst);
                    d4.x -= acc2[t4][0]; d4.y -= acc2[t4][1]; d4.z -= acc2[t4][2]; d4.w -= acc2[t4][3];
                    sts4(dst, d4);
                } else {
#pragma unroll
                    for (int w = 0; w < 4; ++w)
                        if (j0 + w <= i0 + t4) dst[w] -= acc2[t4][w];
                }
            }
        }
    };

    if (warp == 0) chol32(0);
    __syncthreads();
    for (int b = 0; b < 4; ++b) {
        const int o = 32 * b;
        const int r0 = o + 32;
        if (warp < 4) {
            // -- forward substitution with L_bb on 128 right-hand sides at once:
            //    threads 0..31 the identity (-> the strip's inverse, a column per
            //    thread), threads 32..127 the rows below (-> the strip of L)
            const int hs = tid;
            const int i = r0 + hs - 32;  // row for hs >= 32
            const bool act = hs < 32 || i < NB;
            float x[32];
            if (hs >= 32 && act) {
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const float4 t = lds4(A + i * LDA + o + 4 * q);
                    x[4 * q] = t.x; x[4 * q + 1] = t.y; x[4 * q + 2] = t.z; x[4 * q + 3] = t.w;
                }
            } else {
#pragma unroll
                for (int r = 0; r < 32; ++r) x[r] = (r == hs) ? 1.f : 0.f;
            }
#pragma unroll 1
            for (int c = 0; c < 32; ++c) {
                // the step's column of L first: its loads do not wait behind the stores
                float4 l[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) l[q] = lds4(Lc + c * 32 + 4 * q);
                const float xc = x[0] * dinv[o + c];
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    x[4 * q] = fmaf(-l[q].x, xc, x[4 * q + 1]);
                    x[4 * q + 1] = fmaf(-l[q].y, xc, x[4 * q + 2]);
                    x[4 * q + 2] = fmaf(-l[q].z, xc, x[4 * q + 3]);
                    x[4 * q + 3] = (q < 7) ? fmaf(-l[q].w, xc, x[4 * q + 4]) : 0.f;
                }
                if (hs < 32) {
                    Xs[(o + c) * LDA + o + hs] = xc;
                } else if (act) {
                    A[i * LDA + o + c] = xc;
                    Ls[c * LDA + i] = xc;
                }
            }
        }
        __syncthreads();
        if (r0 < NB) {
            // the next strip's 32 x 32 diagonal block first (units 0..35), then
            // warp 0 factors it while warps 1..7 finish the trailing update
            const int mb = (NB - r0) / 4;
            const int units = mb * (mb + 1) / 2;
            trail(r0, 0, 36, tid, kDiagThreads);
            __syncthreads();
            if (warp == 0) chol32(r0);
            else trail(r0, 36, units, tid - 32, kDiagThreads - 32);
            __syncthreads();
        }
    }

    // -- join the 32 x 32 inverses: X_CA = -X_CC (L_CA X_AA), 4 x 4 register
    //    blocks (rows c, columns a); T[p*s + c][a] holds L_CA X_AA.  X_AA and
    //    X_CC are lower triangular, so the sums skip their zero parts.
    for (int s = 32; s < NB; s *= 2) {
        const int pairs = NB / (2 * s);
        const int nb4 = s / 4;
        const int blocks = pairs * nb4 * nb4;
        for (int e = tid; e < blocks; e += kDiagThreads) {
            const int p = e / (nb4 * nb4), c0 = ((e / nb4) % nb4) * 4, a0 = (e % nb4) * 4;
            const int A0 = 2 * s * p, C0 = A0 + s;
            float acc[4][4] = {};
#pragma unroll 2
            for (int k = a0; k < s; k += 4) {  // X_AA[k][a] = 0 for k < a
                float4 l[4];
#pragma unroll
                for (int t = 0; t < 4; ++t) l[t] = lds4(A + (C0 + c0 + t) * LDA + A0 + k);
                float4 xx[4];
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) xx[kk] = lds4(Xs + (A0 + k + kk) * LDA + A0 + a0);
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const float lt[4] = {l[t].x, l[t].y, l[t].z, l[t].w};
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        acc[t][0] = fmaf(lt[kk], xx[kk].x, acc[t][0]);
                        acc[t][1] = fmaf(lt[kk], xx[kk].y, acc[t][1]);
                        acc[t][2] = fmaf(lt[kk], xx[kk].z, acc[t][2]);
                        acc[t][3] = fmaf(lt[kk], xx[kk].w, acc[t][3]);
                    }
                }
            }
#pragma unroll
            for (int t = 0; t < 4; ++t)
                sts4(T + (p * s + c0 + t) * TP + a0, make_float4(acc[t][0], acc[t][1], acc[t][2], acc[t][3]));
        }
        __syncthreads();
        for (int e = tid; e < blocks; e += kDiagThreads) {
            const int p = e / (nb4 * nb4), c0 = ((e / nb4) % nb4) * 4, a0 = (e % nb4) * 4;
            const int A0 = 2 * s * p, C0 = A0 + s;
            float acc[4][4] = {};
#pragma unroll 2
            for (int k = 0; k <= c0; k += 4) {  // X_CC[c][k] = 0 for k > c
                float4 xc[4];
#pragma unroll
                for (int t = 0; t < 4; ++t) xc[t] = lds4(Xs + (C0 + c0 + t) * LDA + C0 + k);
                float4 tt[4];
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) tt[kk] = lds4(T + (p * s + k + kk) * TP + a0);
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const float xt[4] = {xc[t].x, xc[t].y, xc[t].z, xc[t].w};
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        acc[t][0] = fmaf(xt[kk], tt[kk].x, acc[t][0]);
                        acc[t][1] = fmaf(xt[kk], tt[kk].y, acc[t][1]);
                        acc[t][2] = fmaf(xt[kk], tt[kk].z, acc[t][2]);
                        acc[t][3] = fmaf(xt[kk], tt[kk].w, acc[t][3]);
                    }
                }
            }
#pragma unroll
            for (int t = 0; t < 4; ++t)
                sts4(Xs + (C0 + c0 + t) * LDA + A0 + a0,
                     make_float4(-acc[t][0], -acc[t][1], -acc[t][2], -acc[t][3]));
        }
        __syncthreads();
    }

    // -- write X (zeros above the diagonal included: the tensor-core GEMMs read
    //    it as a full tile), float4 per access.  L's diagonal block is not
    //    written back: nothing reads it after this kernel.
#pragma unroll 4
    for (int e = tid; e < NB * NB / 4; e += kDiagThreads) {
        const int i = e >> 5, j = (e & 31) * 4;
        if (i >= kw || j >= kw) continue;
        float4 x4 = lds4(Xs + i * LDA + j);
        if (j + 1 > i) x4.y = 0.f;
        if (j + 2 > i) x4.z = 0.f;
        if (j + 3 > i) x4.w = 0.f;
        if (j > i) x4.x = 0.f;
        *reinterpret_cast<float4*>(X + (kb + i) * ldx + kb + j) = x4;
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

// 32 consecutive floats: dst[j] = sign * v[j], as float4 stores (callers
// guarantee 16-byte alignment and bounds).
__device__ __forceinline__ void put32(float* dst, const float (&v)[32], float sign) {
    float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
    for (int q = 0; q < 8; ++q)
        d4[q] = make_float4(sign * v[4 * q], sign * v[4 * q + 1], sign * v[4 * q + 2],
                            sign * v[4 * q + 3]);
}

// ---------------------------------------------------------------- schedulers
// Panel solve: L[m0.., kb..kb+kw) = A[m0.., kb..) (L_kk^-1)^T   (in place)
struct TrsmSched {
    static constexpr bool kRmw = false;
    float* P;
    int64_t ldp;
    int d, kb, kw;
    __device__ g3::Job job(int t) const { return {kb + kw + NB * t, kb, kb, kb, (kw + 31) / 32}; }
    __device__ void store(const g3::Job& jb, int row, int col0, const float (&v)[32]) const {
        const int r = jb.m0 + row;
        if (r >= d) return;
        float* dst = P + static_cast<int64_t>(r) * ldp + kb + col0;
        if (col0 + 32 <= kw) {
            put32(dst, v, 1.f);
        } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
                if (col0 + j < kw) dst[j] = v[j];
        }
    }
};

// Trailing update: P[I, J] -= L[I, panel] L[J, panel]^T on lower tiles.
// part 0: every lower tile; 1: the first tile column (the next panel);
// 2: the tiles right of it.
struct SyrkSched {
    float* P;
    int64_t ldp;
    int d, kb, kw, s0, part;
    __device__ g3::Job job(int t) const {
        int I, J;
        if (part == 1) {
            I = t;
            J = 0;
        } else {
            tri_coords(t, I, J);
            if (part == 2) {
                ++I;
                ++J;
            }
        }
        return {s0 + NB * I, s0 + NB * J, kb, kb, (kw + 31) / 32};
    }
    static constexpr bool kRmw = true;
    __device__ float* dst(const g3::Job& jb, int row) const {
        const int r = jb.m0 + row;
        return r < d ? P + static_cast<int64_t>(r) * ldp + jb.n0 : nullptr;
    }
    // lower triangle only: columns n0 .. min(r, d - 1) are written; the rest of
    // the row segment inside the matrix may be read
    __device__ int ncols(const g3::Job& jb, int row) const {
        const int lim = min(jb.m0 + row + 1, d) - jb.n0;
        return lim < g3::BN ? lim : g3::BN;
    }
    __device__ int nreadable(const g3::Job& jb) const { return min(d - jb.n0, g3::BN); }
};

// Row k of L^-1 left of the diagonal block, in place:
//   X[kb+m][n] = sum_j X_kk[m][j] B[kb+j][n],  n < kb
// (A = X_kk, K-major; B = the block row of B, MN-major).  A CTA reads its
// whole B tile before its epilogue overwrites that tile.
struct XFinSched {
    static constexpr bool kRmw = false;
    float* X;
    int64_t ldx;
    int kb, kw;
    __device__ g3::Job job(int t) const { return {kb, NB * t, kb, kb, (kw + 31) / 32}; }
    __device__ void store(const g3::Job& jb, int row, int col0, const float (&v)[32]) const {
        if (row >= kw) return;
        put32(X + static_cast<int64_t>(kb + row) * ldx + jb.n0 + col0, v, 1.f);
    }
};

// Panel k's share of the later block rows of L^-1:
//   B[i][n] -= sum_j L[i][kb+j] X[kb+j][n],  i >= kb + 128, n < kb + 128
// (A = the panel of L, K-major; B = block row k of X, MN-major).
struct BUpdSched {
    static constexpr bool kRmw = true;
    float* X;
    int64_t ldx;
    int d, kb, mt;
    __device__ g3::Job job(int t) const {
        return {kb + NB + NB * (t % mt), NB * (t / mt), kb, kb, NB / 32};
    }
    __device__ float* dst(const g3::Job& jb, int row) const {
        const int r = jb.m0 + row;
        return r < d ? X + static_cast<int64_t>(r) * ldx + jb.n0 : nullptr;
    }
    __device__ int ncols(const g3::Job&, int) const { return g3::BN; }
    __device__ int nreadable(const g3::Job&) const { return g3::BN; }
};

// B = 0 on the strictly lower 128 x 128 blocks of X (the diagonal blocks are
// written by potrf_inv_128_kernel).
__global__ void zero_lower_blocks_kernel(float* __restrict__ X, int64_t ldx, int64_t d) {
    const int64_t i = blockIdx.y;
    const int64_t jend = (i / NB) * NB;  // columns left of row i's diagonal block
    for (int64_t j = 4 * (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x); j < jend;
         j += 4 * static_cast<int64_t>(gridDim.x) * blockDim.x)
        *reinterpret_cast<float4*>(X + i * ldx + j) = make_float4(0.f, 0.f, 0.f, 0.f);
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

// Side streams and events of the lookahead schedule (created once per
// device; streams and events, no device memory).
namespace {
struct Lookahead {
    cudaStream_t side = nullptr;   // rest of each trailing update
    cudaStream_t inv = nullptr;    // L^-1
    cudaEvent_t start = nullptr;
    cudaEvent_t solved[4] = {};    // panel k's L_kk^-1 and L[:, k] are final
    cudaEvent_t done[4] = {};      // rest of panel k's trailing update done
    cudaEvent_t side_end = nullptr, inv_end = nullptr;
    bool ok = false;
};
std::mutex g_la_mutex;
Lookahead g_la[64];

// Caller holds g_la_mutex.
Lookahead* lookahead_resources() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    Lookahead& la = g_la[dev];
    if (!la.ok) {
        if (cudaStreamCreateWithFlags(&la.side, cudaStreamNonBlocking) != cudaSuccess ||
            cudaStreamCreateWithFlags(&la.inv, cudaStreamNonBlocking) != cudaSuccess)
            return nullptr;
        cudaEvent_t* all[] = {&la.start, &la.side_end, &la.inv_end};
        for (auto* e : all)
            if (cudaEventCreateWithFlags(e, cudaEventDisableTiming) != cudaSuccess) return nullptr;
        for (int i = 0; i < 4; ++i)
            if (cudaEventCreateWithFlags(&la.solved[i], cudaEventDisableTiming) != cudaSuccess ||
                cudaEventCreateWithFlags(&la.done[i], cudaEventDisableTiming) != cudaSuccess)
                return nullptr;
        la.ok = true;
    }
    return &la;
}
}  // namespace

// Lookahead schedule.  The caller's stream runs the panel chain
//   potrf(k) -> panel solve(k) -> update of panel k+1's column -> potrf(k+1);
// the side stream runs the rest of each trailing update and the inverse
// stream builds L^-1, both in the shadow of the chain.  Ordering: both side
// streams start on panel k once its solve is done; the update of panel k+1's
// column waits for the previous panel's rest-of-update (both touch that
// column), so potrf and the panel solve of k+1 see every update they need;
// the inverse stream is in order with itself; nothing on the chain waits for
// it.  A programmatic (early) launch is used only for a kernel whose
// predecessor in its stream is a kernel.  The SMs are shared out so that the
// chain's one-wave launches find free SMs.
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
    // one enqueue sequence at a time per process: the side streams and the
    // events are shared by every call on a device
    std::lock_guard<std::mutex> lock(g_la_mutex);
    Lookahead* la = lookahead_resources();
    if (la == nullptr) return GPTQ_ERR_CUDA;
    const int sms = num_sms();
    const int inv_sms = sms >= 128 ? 32 : (sms + 3) / 4;
    const int side_sms = sms >= 128 ? sms - 32 - inv_sms : (sms + 1) / 2;
    const int npan = static_cast<int>((d + NB - 1) / NB);
    int64_t launches = 0;
    // the side streams start after everything the caller queued before us
    if (cudaEventRecord(la->start, stream) != cudaSuccess ||
        cudaStreamWaitEvent(la->side, la->start, 0) != cudaSuccess ||
        cudaStreamWaitEvent(la->inv, la->start, 0) != cudaSuccess)
        return GPTQ_ERR_CUDA;
    if (npan > 1) {
        const dim3 zgrid(static_cast<unsigned>((d / 4 + 255) / 256 < 4 ? (d / 4 + 255) / 256 : 4),
                         static_cast<unsigned>(d));
        zero_lower_blocks_kernel<<<zgrid, 256, 0, la->inv>>>(X, ldx, d);
        ++launches;
    }
    for (int k = 0; k < npan; ++k) {
        const int64_t kb = static_cast<int64_t>(k) * NB;
        const int kw = static_cast<int>((d - kb < NB) ? d - kb : NB);
        // directly after the previous panel's column update (programmatic
        // launch); panel 0 follows an event record and is launched plainly
        if (launch_kernel(k > 0, potrf_inv_128_kernel, dim3(1), dim3(kDiagThreads), kDiagSmem, stream,
                          P, ldp, kb, kw, X, ldx, status) != cudaSuccess)
            return GPTQ_ERR_CUDA;
        ++launches;
        const int64_t m = d - kb - kw;
        const int mt = static_cast<int>((m + NB - 1) / NB);
        if (m > 0) {
            TrsmSched ts{P, ldp, di, static_cast<int>(kb), kw};
            if (g3::launch<TrsmSched, false, false>(tP, tX, ts, mt, status, stream, sms, true) !=
                cudaSuccess)
                return GPTQ_ERR_CUDA;
            ++launches;
        }
        // panel k is final: the inverse stream and the rest of the trailing
        // update (whose tiles the next column's update does not touch) may go
        if (cudaEventRecord(la->solved[k & 3], stream) != cudaSuccess ||
            cudaStreamWaitEvent(la->inv, la->solved[k & 3], 0) != cudaSuccess ||
            cudaStreamWaitEvent(la->side, la->solved[k & 3], 0) != cudaSuccess)
            return GPTQ_ERR_CUDA;
        if (m > 0) {
            if (k > 0 && cudaStreamWaitEvent(stream, la->done[(k - 1) & 3], 0) != cudaSuccess)
                return GPTQ_ERR_CUDA;
            SyrkSched nx{P, ldp, di, static_cast<int>(kb), kw, static_cast<int>(kb + kw), 1};
            if (g3::launch<SyrkSched, false, false>(tP, tP, nx, mt, status, stream, sms) != cudaSuccess)
                return GPTQ_ERR_CUDA;
            ++launches;
        }
        if (mt > 1) {
            SyrkSched rs{P, ldp, di, static_cast<int>(kb), kw, static_cast<int>(kb + kw), 2};
            if (g3::launch<SyrkSched, false, false>(tP, tP, rs, mt * (mt + 1) / 2 - mt, status,
                                                    la->side, side_sms) != cudaSuccess)
                return GPTQ_ERR_CUDA;
            ++launches;
        }
        if (cudaEventRecord(la->done[k & 3], la->side) != cudaSuccess) return GPTQ_ERR_CUDA;
        // inverse stream: finish row k of L^-1, then pass panel k on to the rows below
        if (k > 0) {
            XFinSched xf{X, ldx, static_cast<int>(kb), kw};
            if (g3::launch<XFinSched, false, true>(tX, tXmn, xf, k, status, la->inv, inv_sms) !=
                cudaSuccess)
                return GPTQ_ERR_CUDA;
            ++launches;
        }
        if (m > 0) {
            BUpdSched bu{X, ldx, di, static_cast<int>(kb), mt};
            if (g3::launch<BUpdSched, false, true>(tP, tXmn, bu, mt * (k + 1), status, la->inv,
                                                   inv_sms, k > 0) != cudaSuccess)
                return GPTQ_ERR_CUDA;
            ++launches;
        }
    }
    if (cudaEventRecord(la->side_end, la->side) != cudaSuccess ||
        cudaEventRecord(la->inv_end, la->inv) != cudaSuccess ||
        cudaStreamWaitEvent(stream, la->side_end, 0) != cudaSuccess ||
        cudaStreamWaitEvent(stream, la->inv_end, 0) != cudaSuccess)
        return GPTQ_ERR_CUDA;
    dim3 grid(static_cast<unsigned>((d + 255) / 256 < 8 ? (d + 255) / 256 : 8),
              static_cast<unsigned>(d));
    flip_kernel<<<grid, 256, 0, stream>>>(X, ldx, U, d);
    count_launches(launches + 1);
    return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ERR_CUDA;
}

}  // namespace gptq
