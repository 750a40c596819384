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
constexpr int kDiagThreads = 256;
// A, X, the strip's column of L, two strips of L below the diagonal, 1 / L_ii
constexpr int kDiagSmem = (2 * NB * LDA + 32 * 32 + 2 * 32 * LDA + NB) * 4;
// Bound of the substitution warps' wait for a published factor step (polls
// of a shared-memory word; the factor warp never waits, so this is a guard).
constexpr int kStepSpinLimit = 1 << 22;

__device__ __forceinline__ float4 lds4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ void sts4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }

// 4 x 4 block of  D[i0.., j0..] -= sum_c Ls[c][i0..] * R[c][j0..]  (32 terms;
// R rows ldr apart), float4 loads and read-modify-write stores.
__device__ __forceinline__ void rank32_update4(float* D, const float* Ls, const float* R, int ldr,
                                               int i0, int j0) {
    float acc[4][4] = {};
#pragma unroll 8
    for (int k = 0; k < 32; ++k) {
        const float4 li = lds4(Ls + k * LDA + i0), rj = lds4(R + k * ldr + j0);
        const float a4[4] = {li.x, li.y, li.z, li.w}, b4[4] = {rj.x, rj.y, rj.z, rj.w};
#pragma unroll
        for (int t = 0; t < 4; ++t)
#pragma unroll
            for (int w = 0; w < 4; ++w) acc[t][w] = fmaf(a4[t], b4[w], acc[t][w]);
    }
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        float* dst = D + (i0 + t) * LDA + j0;
        float4 d4 = lds4(dst);
        d4.x -= acc[t][0]; d4.y -= acc[t][1]; d4.z -= acc[t][2]; d4.w -= acc[t][3];
        sts4(dst, d4);
    }
}

// Release store / acquire load of a shared-memory word at CTA scope: the
// writes before the release are visible to a thread whose acquire load sees
// the stored value.
__device__ __forceinline__ void st_release_cta(int* p, int v) {
    asm volatile("st.release.cta.shared::cta.s32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}
__device__ __forceinline__ int ld_acquire_cta(const int* p) {
    int v;
    asm volatile("ld.acquire.cta.shared::cta.s32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)) : "memory");
    return v;
}

// Barrier among the `count` threads (whole warps) that execute it with this
// id (ids other than 0, which __syncthreads uses).
__device__ __forceinline__ void named_barrier_sync(int id, int count) {
    asm volatile("barrier.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// 4 x 2 block of  D[i0.., j0..j0+1] -= sum_c Ls[c][i0..] * Ls[c][j0..]  (32 terms).
__device__ __forceinline__ void rank32_update4x2(float* D, const float* Ls, int i0, int j0) {
    float acc[4][2] = {};
#pragma unroll 8
    for (int k = 0; k < 32; ++k) {
        const float4 li = lds4(Ls + k * LDA + i0);
        const float2 lj = *reinterpret_cast<const float2*>(Ls + k * LDA + j0);
        const float a4[4] = {li.x, li.y, li.z, li.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            acc[t][0] = fmaf(a4[t], lj.x, acc[t][0]);
            acc[t][1] = fmaf(a4[t], lj.y, acc[t][1]);
        }
    }
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        float2* dst = reinterpret_cast<float2*>(D + (i0 + t) * LDA + j0);
        float2 d2 = *dst;
        d2.x -= acc[t][0];
        d2.y -= acc[t][1];
        *dst = d2;
    }
}

// Triangular index u -> (bi, bj), bi >= bj.
__device__ __forceinline__ void tri_index(int u, int& bi, int& bj) {
    int i = static_cast<int>((sqrtf(8.f * u + 1.f) - 1.f) * 0.5f);
    while (i * (i + 1) / 2 > u) --i;
    while ((i + 1) * (i + 2) / 2 <= u) ++i;
    bi = i;
    bj = u - i * (i + 1) / 2;
}

// ------------------------------------------------------------------------
// Diagonal block: X = L^-1 with L = chol(A), for a kw x kw (kw <= 128) block
// padded with the identity.  (L itself is not needed outside: the panel
// solve and the inverse stream use only L^-1.)
//
// Right-looking over four 32-wide strips, with X built in place of a
// right-hand side B (the identity at the start): for strip b at o = 32 b,
//   factor     L_bb = chol(A_bb)                                  (warp 0)
//   substitute X[o.., :o+32] = L_bb^-1 B[o.., :o+32]  and
//              L[i, o..] = A[i, o..] L_bb^-T for the rows i below  (warps 4-7)
//   update     A[i, j] -= L[i, o..] L[j, o..]^T,  B[i, :o+32] -= L[i, o..] X[o.., :o+32]
//              for the rows i below the strip.
// The substitution has exactly 128 right-hand sides at every strip (o + 32
// columns of B, 96 - o rows below), one per thread of warps 4-7, and runs one
// column step behind the factor: warp 0 publishes each step's column of L in
// shared memory with a step counter, and the substitution warps wait for it
// (bounded).  The update is split so that only what the next strip reads
// first (its diagonal block, its columns below it, its rows of B) sits
// between two strips; the rest runs on warps 1-3 beside the next strip's
// factor, and those warps also store each finished strip of X.
//
// The factor warp keeps its rows in registers and rotates them after every
// pair of column steps, so the pivot column is always register 0: the step
// loop stays rolled while every register index is a compile-time constant.  Column c of
// L below the diagonal is published as a row of Lc (Lc[c][m] = L[o+c+1+m][o+c],
// zero past the strip), read back with eight broadcast float4 loads.
__global__ void __launch_bounds__(kDiagThreads, 1)
    potrf_inv_128_kernel(float* __restrict__ P, int64_t ldp, int64_t kb, int kw,
                         float* __restrict__ X, int64_t ldx, int32_t* status) {
    extern __shared__ __align__(16) float sm[];
    float* A = sm;                // [128][LDA] the block (lower part updated)
    float* Xs = A + NB * LDA;     // [128][LDA] B, becoming L^-1 strip by strip
    float* Lc = Xs + NB * LDA;    // [32][32] the current strip's columns of L, shifted
    float* Lsb = Lc + 32 * 32;    // [2][32][LDA] strips of L below them, transposed
    float* dinv = Lsb + 2 * 32 * LDA;  // [128] 1 / L_ii
    __shared__ int bad, stalled;
    __shared__ int progress;      // factor steps published so far (32 b + c + 1)
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        bad = 0;
        stalled = 0;
        progress = 0;
    }
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
            float id[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                id[t] = (i == j + t) ? 1.f : 0.f;
                vv[t] = (j + t <= i && i < kw) ? vv[t] : id[t];
            }
            sts4(A + i * LDA + j, make_float4(vv[0], vv[1], vv[2], vv[3]));
            sts4(Xs + i * LDA + j, make_float4(id[0], id[1], id[2], id[3]));
        }
    }
    __syncthreads();

    // -- strip factor (warp 0): lane i holds row o + i, register r = column c + r
    auto factor = [&](int o, int b) {
        float a[32];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const float4 t = lds4(A + (o + lane) * LDA + o + 4 * q);
            a[4 * q] = t.x; a[4 * q + 1] = t.y; a[4 * q + 2] = t.z; a[4 * q + 3] = t.w;
        }
#pragma unroll
        for (int r = 0; r < 32; ++r) a[r] = (r <= lane) ? a[r] : 0.f;
        // two columns per pass: column c+1 is formed in registers from column
        // c (its pivot row needs only its own value, the other rows one
        // broadcast), then both are published and applied as one rank-2
        // update -- the same operations in the same order as two rank-1
        // passes, with one shared-memory round trip instead of two
#pragma unroll 1
        for (int c = 0; c < 32; c += 2) {
            float piv = __shfl_sync(0xffffffffu, a[0], c);
            if (!(piv > 0.f)) {  // not positive definite (or NaN): flag, stay finite
                bad = 1;
                piv = 1.f;
            }
            const float inv = rsqrtf(piv);
            const float a0 = (lane > c) ? a[0] * inv : 0.f;           // L[o+lane][o+c]
            const float t = __shfl_sync(0xffffffffu, a0, c + 1);      // L[o+c+1][o+c]
            const float n1 = fmaf(-a0, t, a[1]);                       // column c+1 after column c
            float piv1 = __shfl_sync(0xffffffffu, n1, c + 1);
            if (!(piv1 > 0.f)) {
                bad = 1;
                piv1 = 1.f;
            }
            const float inv1 = rsqrtf(piv1);
            const float a1 = (lane > c + 1) ? n1 * inv1 : 0.f;        // L[o+lane][o+c+1]
            if (lane == c) dinv[o + c] = inv;
            if (lane == c + 1) dinv[o + c + 1] = inv1;
            // lane i > c holds L[o+i][o+c] -> Lc[c][i-c-1]; lanes <= c fill the tail with 0
            Lc[c * 32 + ((lane - c - 1) & 31)] = a0;
            Lc[(c + 1) * 32 + ((lane - c - 2) & 31)] = a1;
            __syncwarp();  // orders the warp's writes above before lane 0's release
            if (lane == 0) st_release_cta(&progress, 32 * b + c + 2);
            // a[r] <- a[r+2] - a0 L[o+c+2+r][o+c] - a1 L[o+c+2+r][o+c+1]
            float l0[32], l1[32];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float4 u = lds4(Lc + c * 32 + 4 * q), v = lds4(Lc + (c + 1) * 32 + 4 * q);
                l0[4 * q] = u.x; l0[4 * q + 1] = u.y; l0[4 * q + 2] = u.z; l0[4 * q + 3] = u.w;
                l1[4 * q] = v.x; l1[4 * q + 1] = v.y; l1[4 * q + 2] = v.z; l1[4 * q + 3] = v.w;
            }
#pragma unroll
            for (int r = 0; r < 30; ++r) a[r] = fmaf(-a1, l1[r], fmaf(-a0, l0[r + 1], a[r + 2]));
            a[30] = 0.f;
            a[31] = 0.f;
        }
    };

    // -- substitution (warps 4-7), one step behind the factor: thread t
    //    solves for column t of B (t < o + 32) or for row t of L below the strip
    auto substitute = [&](int o, int b) {
        const int t = tid - 128;
        const bool rhs = t < o + 32;
        float* Ls = Lsb + (b & 1) * 32 * LDA;
        float x[32];
        if (rhs) {
#pragma unroll
            for (int r = 0; r < 32; ++r) x[r] = Xs[(o + r) * LDA + t];
        } else {
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float4 v4 = lds4(A + t * LDA + o + 4 * q);
                x[4 * q] = v4.x; x[4 * q + 1] = v4.y; x[4 * q + 2] = v4.z; x[4 * q + 3] = v4.w;
            }
        }
        int spins = 0;
        // the factor publishes two columns at a time: one wait per pair
#pragma unroll 1
        for (int c2 = 0; c2 < 32; c2 += 2) {
            const int need = 32 * b + c2 + 2;
            while (ld_acquire_cta(&progress) < need) {
                if (++spins > kStepSpinLimit) {
                    stalled = 1;
                    break;
                }
                __nanosleep(32);  // leave the issue slots to the factor warp (same sub-partition)
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int c = c2 + h;
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
                if (rhs) Xs[(o + c) * LDA + t] = xc;
                else Ls[c * LDA + t] = xc;
            }
        }
    };

    // -- strip b's update of what lies below it.  Units of 4 x 4: the next
    //    strip's diagonal block (36), its columns below it, its rows of B
    //    ("first"), or everything further below ("rest").
    //    part 0: the next strip's diagonal block; part 1: its columns below
    //    it and its rows of B; part 2: everything further below
    auto update = [&](int b, int part, int u0, int stride) {
        const int o = 32 * b, o1 = o + 32;  // o1: the next strip
        const float* Ls = Lsb + (b & 1) * 32 * LDA;
        const float* Xr = Xs + o * LDA;     // strip b's rows of X
        const int nb4 = o1 / 4;             // 4-column blocks of B's live columns
        const int below = (NB - o1 - 32) / 4;  // 4-row blocks below the next strip
        if (part == 0) {
            // 72 units of 4 rows x 2 columns: row block i holds 2 i + 2 of them
            for (int u = u0; u < 72; u += stride) {
                int i = static_cast<int>((sqrtf(4.f * u + 1.f) - 1.f) * 0.5f);
                while (i * (i + 1) > u) --i;
                while ((i + 1) * (i + 2) <= u) ++i;
                const int j = u - i * (i + 1);
                rank32_update4x2(A, Ls, o1 + 4 * i, o1 + 2 * j);
            }
        } else if (part == 1) {
            const int n_panel = below * 8, n_b = 8 * nb4;
            for (int u = u0; u < n_panel + n_b; u += stride) {
                if (u < n_panel) {
                    rank32_update4(A, Ls, Ls, LDA, o1 + 32 + 4 * (u >> 3), o1 + 4 * (u & 7));
                } else {
                    const int v = u - n_panel;
                    rank32_update4(Xs, Ls, Xr, LDA, o1 + 4 * (v / nb4), 4 * (v % nb4));
                }
            }
        } else {
            const int n_a = below * (below + 1) / 2, n_b = below * nb4;
            for (int u = u0; u < n_a + n_b; u += stride) {
                if (u < n_a) {
                    int bi, bj;
                    tri_index(u, bi, bj);
                    rank32_update4(A, Ls, Ls, LDA, o1 + 32 + 4 * bi, o1 + 32 + 4 * bj);
                } else {
                    const int v = u - n_a;
                    rank32_update4(Xs, Ls, Xr, LDA, o1 + 32 + 4 * (v / nb4), 4 * (v % nb4));
                }
            }
        }
    };

    // -- rows [r0, r0 + nr) of X to global memory (zeros above the diagonal
    //    included: the tensor-core GEMMs read it as a full tile)
    auto store_rows = [&](int r0, int nr, int t0, int stride) {
        for (int e = t0; e < nr * (NB / 4); e += stride) {
            const int i = r0 + e / (NB / 4), j = (e % (NB / 4)) * 4;
            if (i >= kw || j >= kw) continue;
            float4 x4 = lds4(Xs + i * LDA + j);
            if (j + 1 > i) x4.y = 0.f;
            if (j + 2 > i) x4.z = 0.f;
            if (j + 3 > i) x4.w = 0.f;
            if (j > i) x4.x = 0.f;
            *reinterpret_cast<float4*>(X + (kb + i) * ldx + kb + j) = x4;
        }
    };

    for (int b = 0; b < 4; ++b) {
        const int o = 32 * b;
        if (warp == 0) {
            factor(o, b);
        } else if (warp >= 4) {
            substitute(o, b);
        } else if (b > 0) {
            update(b - 1, 2, tid - 32, 96);  // the previous strip's rest
            store_rows(o - 32, 32, tid - 32, 96);  // the previous strip of X is final
        }
        __syncthreads();
        if (b < 3) {
            // what the next strip reads first: warps 0-2 update its diagonal
            // block (then warp 0 factors it), warps 3-7 its columns below it
            // and its rows of B (then warps 4-7 substitute); each group goes on
            // as soon as its own part is done
            if (warp < 3) {
                update(b, 0, tid, 96);
                named_barrier_sync(1, 96);
            } else {
                update(b, 1, tid - 96, 160);
                named_barrier_sync(2, 160);
            }
        }
    }
    __syncthreads();
    store_rows(96, 32, tid, kDiagThreads);
    if (tid == 0 && bad) report(status, GPTQ_ERR_NOT_PD);
    if (tid == 0 && stalled) report(status, GPTQ_ERR_TIMEOUT);
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
// Drains (see gemm_tf32x3.cuh).  The read-modify-write updates (the trailing
// update, on the chain and beside it, and the inverse's block rows) hand
// -AB^T to TMA tensor reductions into P and X: the read-modify-write happens
// in L2 and the SMs issue no global loads or stores for it.  prepare_hinv
// with them against a drain in which each lane loaded, updated and stored its
// own tile row: 1.46 vs 1.66 ms at d = 4096, 4.1 vs
// 7.5 ms at 8192, 8.9 vs 19.2 ms at 11008, 146 vs 292 ms at 28672.  Full
// tiles are reduced: the upper part of a diagonal tile of P receives values
// too, which nothing reads (the diagonal factor loads only j <= i, every GEMM
// operand lies below the diagonal blocks).  (The shared-memory staged drain
// measured slower than the direct one here: 1.70 and 1.79 ms at 4096.)
// kChainStore: the plain-store outputs (panel solve, L^-1 block row).
// Every GEMM here uses the rounding operand split (the launch default): U's
// error against a float64 factorization halves with it (max 1.1e-6 -> 5e-7
// relative at d = 4096) for about 0.05 ms more per prepare_hinv.
constexpr int kChainStore = g3::kEpiStore;
// Panel solve: L[m0.., kb..kb+kw) = A[m0.., kb..) (L_kk^-1)^T   (in place)
struct TrsmSched {
    static constexpr bool kRmw = false;
    float* P;
    int64_t ldp;
    int d, kb, kw;
    __device__ g3::Job job(int t) const { return {kb + kw + NB * t, kb, kb, kb, (kw + 31) / 32}; }
    __device__ float* dst(const g3::Job& jb, int row) const {
        const int r = jb.m0 + row;
        return r < d ? P + static_cast<int64_t>(r) * ldp + kb : nullptr;
    }
    __device__ int ncols(const g3::Job&, int) const { return kw; }
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
    __device__ float* dst(const g3::Job& jb, int row) const {
        return row < kw ? X + static_cast<int64_t>(kb + row) * ldx + jb.n0 : nullptr;
    }
    __device__ int ncols(const g3::Job&, int) const { return g3::BN; }
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

// U[i][j] = X[d-1-i][d-1-j] for j >= i, 0 below the diagonal; four columns
// per thread (d and ldx are multiples of 4, so the reversed float4 of X that
// holds them is aligned).
__global__ void flip_kernel(const float* __restrict__ X, int64_t ldx, float* __restrict__ U,
                            int64_t d) {
    const int64_t i = blockIdx.y;
    const float* xr = X + (d - 1 - i) * ldx;
    for (int64_t j = 4 * (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x); j < d;
         j += 4 * static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const float4 x = *reinterpret_cast<const float4*>(xr + (d - 4 - j));  // columns d-4-j .. d-1-j
        float4 u = make_float4(x.w, x.z, x.y, x.x);                           // columns j .. j+3 of U
        if (j < i) u.x = 0.f;
        if (j + 1 < i) u.y = 0.f;
        if (j + 2 < i) u.z = 0.f;
        if (j + 3 < i) u.w = 0.f;
        *reinterpret_cast<float4*>(U + i * d + j) = u;
    }
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
    CUtensorMap tP, tX, tXmn, tPd, tXd;
    if (!make_tmap_2d(&tP, false, P, d, d, ldp, 32, 128, Swz::k128) ||
        !make_tmap_2d(&tX, false, X, d, d, ldx, 32, 128, Swz::k128) ||
        !make_tmap_2d(&tXmn, false, X, d, d, ldx, 32, 32, Swz::k128Atom32) ||
        !make_tmap_2d(&tPd, false, P, d, d, ldp, 32, 32, Swz::k128) ||
        !make_tmap_2d(&tXd, false, X, d, d, ldx, 32, 32, Swz::k128))
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
    // SMs shared by the two side streams (the panel chain keeps the rest:
    // at d = 4096 its launches are one wave of at most 31 tiles), split per
    // panel in proportion to the two streams' tiles (below).  Measured
    // against a split that gave the rest of the trailing update enough SMs
    // for five waves and the inverse the others: the same at d = 4096, 2.3x
    // faster at 8192, 3x at 11008, 3.9x at 28672, where that split starved
    // the inverse stream.
    const int pool = sms >= 128 ? sms - 32 : (3 * sms) / 4;
    const int pool_min = pool / 8 > 1 ? pool / 8 : 1;
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
            if (g3::launch<TrsmSched, false, false, kChainStore>(tP, tX, ts, mt, status, stream, sms, true,
                                                                 &tPd) !=
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
            if (g3::launch<SyrkSched, false, false, g3::kEpiReduce>(tP, tP, nx, mt, status, stream, sms,
                                                                    false, &tPd) != cudaSuccess)
                return GPTQ_ERR_CUDA;
            ++launches;
        }
        // the pool is shared in proportion to this panel's tiles on each
        // stream, so both streams advance one panel in about the same time
        // (the rest of the trailing update dominates early, the inverse's
        // block rows late; both carry d^3 / 3 flops in total)
        const int side_tiles = mt * (mt + 1) / 2 - mt;
        const long long inv_tiles = static_cast<long long>(mt) * (k + 1) + k;
        const long long all_tiles = side_tiles + inv_tiles > 0 ? side_tiles + inv_tiles : 1;
        int side_sms = static_cast<int>((static_cast<long long>(pool) * side_tiles + all_tiles / 2) / all_tiles);
        side_sms = side_sms < pool_min ? pool_min : (side_sms > pool - pool_min ? pool - pool_min : side_sms);
        const int inv_sms = pool - side_sms;
        if (mt > 1) {
            SyrkSched rs{P, ldp, di, static_cast<int>(kb), kw, static_cast<int>(kb + kw), 2};
            const int rt = mt * (mt + 1) / 2 - mt;
            if (g3::launch<SyrkSched, false, false, g3::kEpiReduce>(tP, tP, rs, rt, status, la->side,
                                                                    side_sms, false, &tPd) != cudaSuccess)
                return GPTQ_ERR_CUDA;
            ++launches;
        }
        if (cudaEventRecord(la->done[k & 3], la->side) != cudaSuccess) return GPTQ_ERR_CUDA;
        // inverse stream: finish row k of L^-1, then pass panel k on to the rows below
        if (k > 0) {
            XFinSched xf{X, ldx, static_cast<int>(kb), kw};
            if (g3::launch<XFinSched, false, true, kChainStore>(tX, tXmn, xf, k, status, la->inv, inv_sms,
                                                                false, &tXd) !=
                cudaSuccess)
                return GPTQ_ERR_CUDA;
            ++launches;
        }
        if (m > 0) {
            BUpdSched bu{X, ldx, di, static_cast<int>(kb), mt};
            const int bt = mt * (k + 1);
            if (g3::launch<BUpdSched, false, true, g3::kEpiReduce>(tP, tXmn, bu, bt, status, la->inv,
                                                                   inv_sms, k > 0, &tXd) != cudaSuccess)
                return GPTQ_ERR_CUDA;
            ++launches;
        }
    }
    if (cudaEventRecord(la->side_end, la->side) != cudaSuccess ||
        cudaEventRecord(la->inv_end, la->inv) != cudaSuccess ||
        cudaStreamWaitEvent(stream, la->side_end, 0) != cudaSuccess ||
        cudaStreamWaitEvent(stream, la->inv_end, 0) != cudaSuccess)
        return GPTQ_ERR_CUDA;
    dim3 grid(static_cast<unsigned>((d / 4 + 255) / 256 < 4 ? (d / 4 + 255) / 256 : 4),
              static_cast<unsigned>(d));
    flip_kernel<<<grid, 256, 0, stream>>>(X, ldx, U, d);
    count_launches(launches + 1);
    return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ERR_CUDA;
}

}  // namespace gptq
