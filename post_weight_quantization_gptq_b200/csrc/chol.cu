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
// and L^-1 built block row by block row on the same GEMM,
//   X[k, :k] = -X_kk (L[k, :k] X[:k, :k]),
// in the shadow of the panel chain (see launch_chol_inverse).
#include <cmath>
#include <mutex>

#include "common.cuh"
#include "gemm_tf32x3.cuh"
#include "kernels.h"

namespace gptq {
namespace {

constexpr int NB = 128;      // panel width
constexpr int LDA = NB + 1;  // shared-memory row pitch of the diagonal block
constexpr int kDiagThreads = 256;
constexpr int kDiagSmem = (2 * NB * LDA + 64 * 65 + NB) * 4;

// ------------------------------------------------------------------------
// Diagonal block: L = chol(A) and X = L^-1 for a kw x kw (kw <= 128) block,
// padded with the identity.  Four 32-wide strips; for each, one warp factors
// the strip's 32 x 32 diagonal block, then four warps run one forward
// substitution on 128 right-hand sides (the identity -> the strip's inverse,
// and the rows below -> the strip of L), then the CTA updates the trailing
// part; finally the four 32 x 32 inverses are joined by two levels of
// recursive doubling.
//
// The warp keeps its rows in registers and rotates them after every column
// step, so the pivot column is always register 0: the step loop stays rolled
// (small code, the kernel runs once per panel on a cold SM) while all
// register indices are compile-time constants and each step is 31
// independent shuffle + FMA pairs.
__global__ void __launch_bounds__(kDiagThreads, 1)
    potrf_inv_128_kernel(float* __restrict__ P, int64_t ldp, int64_t kb, int kw,
                         float* __restrict__ X, int64_t ldx, int32_t* status) {
    extern __shared__ float sm[];
    float* A = sm;              // [128][129] the block, L in its lower part
    float* Xs = A + NB * LDA;   // [128][129] L^-1
    float* T = Xs + NB * LDA;   // [64][65] doubling temporary
    float* dinv = T + 64 * 65;  // [128] 1 / L_ii
    __shared__ int bad;
    __shared__ float colbuf[32];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) bad = 0;
    {
        // rows of the block: 16 float4 loads per thread, all in flight
        // (ldp, kb and kw are multiples of 4, so a float4 never crosses kw)
        float4 v[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) {
            const int e = tid + q * kDiagThreads;
            const int i = e >> 5, j = (e & 31) * 4;
            v[q] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (i < kw && j <= i) v[q] = *reinterpret_cast<const float4*>(P + (kb + i) * ldp + kb + j);
        }
#pragma unroll
        for (int q = 0; q < 16; ++q) {
            const int e = tid + q * kDiagThreads;
            const int i = e >> 5, j = (e & 31) * 4;
            const float vv[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const int jj = j + t;
                A[i * LDA + jj] = (jj <= i && i < kw) ? vv[t] : (i == jj ? 1.f : 0.f);
                Xs[i * LDA + jj] = 0.f;
            }
        }
    }
    __syncthreads();

    for (int b = 0; b < 4; ++b) {
        const int o = 32 * b;
        if (warp == 0) {
            // -- 32 x 32 Cholesky: lane i holds row o + i, register r = column c + r
            float a[32];
#pragma unroll
            for (int r = 0; r < 32; ++r) a[r] = (r <= lane) ? A[(o + lane) * LDA + o + r] : 0.f;
#pragma unroll 1
            for (int c = 0; c < 32; ++c) {
                float piv = __shfl_sync(0xffffffffu, a[0], c);
                if (!(piv > 0.f)) {  // not positive definite (or NaN): flag, stay finite
                    bad = 1;
                    piv = 1.f;
                }
                const float inv = rsqrtf(piv);
                const float lcc = piv * inv;
                const float a0 = (lane == c) ? lcc : ((lane > c) ? a[0] * inv : a[0]);
                colbuf[lane] = a0;
                if (lane >= c) A[(o + lane) * LDA + o + c] = a0;
                if (lane == c) dinv[o + c] = inv;
                __syncwarp();
#pragma unroll
                for (int r = 1; r < 32; ++r)
                    a[r - 1] = fmaf(-a0, colbuf[(c + r) & 31], a[r]);  // update and rotate
                a[31] = 0.f;
                __syncwarp();
            }
        }
        __syncthreads();
        const int r0 = o + 32;
        if (warp < 4) {
            // -- forward substitution with L_bb on 128 right-hand sides at once:
            //    lanes 0..31 the identity (-> the strip's inverse, a column per
            //    lane), lanes 32..127 the rows below (-> the strip of L)
            const int hs = tid;
            const int i = r0 + hs - 32;  // row for hs >= 32
            const bool act = hs < 32 || i < NB;
            float x[32];
#pragma unroll
            for (int r = 0; r < 32; ++r)
                x[r] = (hs < 32) ? ((r == hs) ? 1.f : 0.f) : (act ? A[i * LDA + o + r] : 0.f);
#pragma unroll 1
            for (int c = 0; c < 32; ++c) {
                const float xc = x[0] * dinv[o + c];
                if (hs < 32) Xs[(o + c) * LDA + o + hs] = xc;
                else if (act) A[i * LDA + o + c] = xc;
                const float* lcol = A + (o + c) * LDA + o + c;  // L[o+c+r][o+c] at lcol[r * LDA]
#pragma unroll
                for (int r = 1; r < 32; ++r) {
                    const float l = (c + r < 32) ? lcol[r * LDA] : 0.f;
                    x[r - 1] = fmaf(-l, xc, x[r]);
                }
                x[31] = 0.f;
            }
        }
        __syncthreads();
        if (r0 < NB) {
            // -- trailing update of the lower part, 4 x 4 register blocks
            const int mb = (NB - r0) / 4;
            const int units = mb * (mb + 1) / 2;
            for (int u = tid; u < units; u += kDiagThreads) {
                int bi = static_cast<int>((sqrtf(8.f * u + 1.f) - 1.f) * 0.5f);
                while (bi * (bi + 1) / 2 > u) --bi;
                while ((bi + 1) * (bi + 2) / 2 <= u) ++bi;
                const int bj = u - bi * (bi + 1) / 2;
                const int i0 = r0 + 4 * bi, j0 = r0 + 4 * bj;
                float acc2[4][4] = {};
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
                        for (int w = 0; w < 4; ++w) acc2[t][w] = fmaf(li[t], lj[w], acc2[t][w]);
                }
#pragma unroll
                for (int t = 0; t < 4; ++t)
#pragma unroll
                    for (int w = 0; w < 4; ++w)
                        if (j0 + w <= i0 + t) A[(i0 + t) * LDA + j0 + w] -= acc2[t][w];
            }
        }
        __syncthreads();
    }

    // -- join the 32 x 32 inverses: X_CA = -X_CC (L_CA X_AA), 4 x 4 register
    //    blocks (rows c, columns a); T[p*s + c][a] holds L_CA X_AA
    for (int s = 32; s < NB; s *= 2) {
        const int pairs = NB / (2 * s);
        const int nb4 = s / 4;
        const int blocks = pairs * nb4 * nb4;
        for (int e = tid; e < blocks; e += kDiagThreads) {
            const int p = e / (nb4 * nb4), c0 = ((e / nb4) % nb4) * 4, a0 = (e % nb4) * 4;
            const int A0 = 2 * s * p, C0 = A0 + s;
            float acc[4][4] = {};
#pragma unroll 8
            for (int k = 0; k < s; ++k) {  // X_AA is zero above its diagonal
                float l[4], xx[4];
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    l[t] = A[(C0 + c0 + t) * LDA + A0 + k];
                    xx[t] = Xs[(A0 + k) * LDA + A0 + a0 + t];
                }
#pragma unroll
                for (int t = 0; t < 4; ++t)
#pragma unroll
                    for (int w = 0; w < 4; ++w) acc[t][w] = fmaf(l[t], xx[w], acc[t][w]);
            }
#pragma unroll
            for (int t = 0; t < 4; ++t)
#pragma unroll
                for (int w = 0; w < 4; ++w) T[(p * s + c0 + t) * 65 + a0 + w] = acc[t][w];
        }
        __syncthreads();
        for (int e = tid; e < blocks; e += kDiagThreads) {
            const int p = e / (nb4 * nb4), c0 = ((e / nb4) % nb4) * 4, a0 = (e % nb4) * 4;
            const int A0 = 2 * s * p, C0 = A0 + s;
            float acc[4][4] = {};
#pragma unroll 8
            for (int k = 0; k < s; ++k) {  // X_CC is zero above its diagonal
                float xc[4], tt[4];
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    xc[t] = Xs[(C0 + c0 + t) * LDA + C0 + k];
                    tt[t] = T[(p * s + k) * 65 + a0 + t];
                }
#pragma unroll
                for (int t = 0; t < 4; ++t)
#pragma unroll
                    for (int w = 0; w < 4; ++w) acc[t][w] = fmaf(xc[t], tt[w], acc[t][w]);
            }
#pragma unroll
            for (int t = 0; t < 4; ++t)
#pragma unroll
                for (int w = 0; w < 4; ++w) Xs[(C0 + c0 + t) * LDA + A0 + a0 + w] = -acc[t][w];
        }
        __syncthreads();
    }

    // -- write L (lower part) and X (zeros above the diagonal included: the
    //    tensor-core GEMMs read it as a full tile), float4 per access
#pragma unroll 4
    for (int e = tid; e < NB * NB / 4; e += kDiagThreads) {
        const int i = e >> 5, j = (e & 31) * 4;
        if (i >= kw || j >= kw) continue;
        float l4[4], x4[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            l4[t] = A[i * LDA + j + t];
            x4[t] = (j + t <= i) ? Xs[i * LDA + j + t] : 0.f;
        }
        *reinterpret_cast<float4*>(X + (kb + i) * ldx + kb + j) = make_float4(x4[0], x4[1], x4[2], x4[3]);
        if (j + 3 <= i) {
            *reinterpret_cast<float4*>(P + (kb + i) * ldp + kb + j) = make_float4(l4[0], l4[1], l4[2], l4[3]);
        } else if (j <= i) {
#pragma unroll
            for (int t = 0; t < 4; ++t)
                if (j + t <= i) P[(kb + i) * ldp + kb + j + t] = l4[t];
        }
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

// 32 consecutive floats: dst[j] = sign * v[j] (or dst[j] -= v[j] with sub),
// as float4 accesses (callers guarantee 16-byte alignment and bounds).
template <bool kSub>
__device__ __forceinline__ void put32(float* dst, const float (&v)[32], float sign) {
    float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        if (kSub) {
            float4 x = d4[q];
            x.x -= v[4 * q]; x.y -= v[4 * q + 1]; x.z -= v[4 * q + 2]; x.w -= v[4 * q + 3];
            d4[q] = x;
        } else {
            d4[q] = make_float4(sign * v[4 * q], sign * v[4 * q + 1], sign * v[4 * q + 2],
                                sign * v[4 * q + 3]);
        }
    }
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
        if (col0 + 32 <= kw) {
            put32<false>(dst, v, 1.f);
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
    __device__ void store(const g3::Job& jb, int row, int col0, const float (&v)[32]) const {
        const int r = jb.m0 + row;
        if (r >= d) return;
        float* dst = P + static_cast<int64_t>(r) * ldp + jb.n0 + col0;
        const int c = jb.n0 + col0;
        if (c + 31 <= r && c + 32 <= d) {
            put32<true>(dst, v, 1.f);
        } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
                if (c + j < d && c + j <= r) dst[j] -= v[j];
        }
    }
};

// Block row kb of L^-1, left of the diagonal, once L_kk^-1 is known:
//   X[kb.., :kb] = -X_kk (L[kb.., :kb] X[:kb, :kb]).
// Step 1: T^T[a][m] = sum_{a <= j < kb} X[j][a] L[kb+m][j], stored in the
// free upper triangle at P[a][kb+m] (a < kb).
struct XRow1Sched {
    float* P;
    int64_t ldp;
    int d, kb, kw;
    __device__ g3::Job job(int t) const {
        const int a0 = NB * t;
        return {a0, kb, a0, a0, (kb - a0) / 32};
    }
    __device__ void store(const g3::Job& jb, int row, int col0, const float (&v)[32]) const {
        float* dst = P + static_cast<int64_t>(jb.m0 + row) * ldp + kb + col0;
        if (col0 + 32 <= kw) {
            put32<false>(dst, v, 1.f);
        } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
                if (col0 + j < kw) dst[j] = v[j];
        }
    }
};

// Step 2: X[kb+m][a] = -sum_j X[kb+m][kb+j] T[j][a], T[j][a] = P[a][kb+j].
struct XRow2Sched {
    float* X;
    int64_t ldx;
    int d, kb, kw;
    __device__ g3::Job job(int t) const { return {kb, NB * t, kb, kb, (kw + 31) / 32}; }
    __device__ void store(const g3::Job& jb, int row, int col0, const float (&v)[32]) const {
        if (row >= kw) return;
        put32<false>(X + static_cast<int64_t>(kb + row) * ldx + jb.n0 + col0, v, -1.f);
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

// Side stream and events of the lookahead schedule (created once per device;
// streams and events, no device memory).
namespace {
struct Lookahead {
    cudaStream_t side = nullptr;
    cudaEvent_t ev[8] = {};  // [0..3] panel column ready, [4..7] trailing update done
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
        if (cudaStreamCreateWithFlags(&la.side, cudaStreamNonBlocking) != cudaSuccess) return nullptr;
        for (auto& e : la.ev)
            if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return nullptr;
        la.ok = true;
    }
    return &la;
}
}  // namespace

// Lookahead schedule.  The caller's stream runs the panel chain
//   potrf(k) -> panel solve(k) -> update of panel k+1's column -> potrf(k+1)
// while a side stream runs the rest of each trailing update and block row k
// of L^-1 in its shadow.  Ordering: the update of panel k+1's column waits
// for the previous panel's rest-of-update (both touch that column); potrf and
// the panel solve of k+1 then see every update they need.
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
    // one enqueue sequence at a time per process: the side stream and the
    // event ring are shared by every call on a device
    std::lock_guard<std::mutex> lock(g_la_mutex);
    Lookahead* la = lookahead_resources();
    if (la == nullptr) return GPTQ_ERR_CUDA;
    const int sms = num_sms();
    const int side_sms = sms > 32 ? sms - 16 : sms;  // leave SMs for the panel chain
    cudaStream_t side = la->side;
    const int npan = static_cast<int>((d + NB - 1) / NB);
    int64_t launches = 0;
    bool side_used = false;
    // the side stream starts after everything the caller queued before us
    if (cudaEventRecord(la->ev[0], stream) != cudaSuccess ||
        cudaStreamWaitEvent(side, la->ev[0], 0) != cudaSuccess)
        return GPTQ_ERR_CUDA;
    for (int k = 0; k < npan; ++k) {
        const int64_t kb = static_cast<int64_t>(k) * NB;
        const int kw = static_cast<int>((d - kb < NB) ? d - kb : NB);
        potrf_inv_128_kernel<<<1, kDiagThreads, kDiagSmem, stream>>>(P, ldp, kb, kw, X, ldx, status);
        ++launches;
        const int64_t m = d - kb - kw;
        const int mt = static_cast<int>((m + NB - 1) / NB);
        cudaEvent_t ready = la->ev[k & 3], done = la->ev[4 + (k & 3)];
        if (m > 0) {
            TrsmSched ts{P, ldp, di, static_cast<int>(kb), kw};
            if (g3::launch<TrsmSched, false, false>(tP, tX, ts, mt, status, stream, sms) != cudaSuccess)
                return GPTQ_ERR_CUDA;
            if (k > 0 && cudaStreamWaitEvent(stream, la->ev[4 + ((k - 1) & 3)], 0) != cudaSuccess)
                return GPTQ_ERR_CUDA;
            SyrkSched nx{P, ldp, di, static_cast<int>(kb), kw, static_cast<int>(kb + kw), 1};
            if (g3::launch<SyrkSched, false, false>(tP, tP, nx, mt, status, stream, sms) != cudaSuccess)
                return GPTQ_ERR_CUDA;
            launches += 2;
        }
        if (cudaEventRecord(ready, stream) != cudaSuccess ||
            cudaStreamWaitEvent(side, ready, 0) != cudaSuccess)
            return GPTQ_ERR_CUDA;
        if (mt > 1) {
            SyrkSched rs{P, ldp, di, static_cast<int>(kb), kw, static_cast<int>(kb + kw), 2};
            if (g3::launch<SyrkSched, false, false>(tP, tP, rs, mt * (mt + 1) / 2 - mt, status, side,
                                                    side_sms) != cudaSuccess)
                return GPTQ_ERR_CUDA;
            ++launches;
        }
        if (cudaEventRecord(done, side) != cudaSuccess) return GPTQ_ERR_CUDA;
        if (k > 0) {
            XRow1Sched x1{P, ldp, di, static_cast<int>(kb), kw};
            XRow2Sched x2{X, ldx, di, static_cast<int>(kb), kw};
            if (g3::launch<XRow1Sched, true, false>(tXmn, tP, x1, k, status, side, side_sms) !=
                    cudaSuccess ||
                g3::launch<XRow2Sched, false, false>(tX, tP, x2, k, status, side, side_sms) !=
                    cudaSuccess)
                return GPTQ_ERR_CUDA;
            launches += 2;
        }
        side_used = true;
    }
    if (side_used) {
        if (cudaEventRecord(la->ev[4], side) != cudaSuccess ||
            cudaStreamWaitEvent(stream, la->ev[4], 0) != cudaSuccess)
            return GPTQ_ERR_CUDA;
    }
    dim3 grid(static_cast<unsigned>((d + 255) / 256 < 8 ? (d + 255) / 256 : 8),
              static_cast<unsigned>(d));
    flip_kernel<<<grid, 256, 0, stream>>>(X, ldx, U, d);
    count_launches(launches + 1);
    return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ERR_CUDA;
}

}  // namespace gptq
