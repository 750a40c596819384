// Stage 1: H += 2 X^T X on the 5th-generation tensor cores.
//
// "GPTQ (GPT Quantization)", section "Fondation theorique : OBQ" defines
// H = 2 X^T X over the calibration inputs X (n tokens x d channels), and the
// pseudo-code ("Algorithme complet", step 1) computes it before anything
// else.  H is symmetric, so only tiles that touch the lower triangle are
// computed.
//
// Design (sm_100a):
//  * Each CTA owns one 256 x 256 block of D = X[:, m-block]^T X[:, n-block]
//    as two 128 x 256 halves (rows m0..m0+127 and m0+128..m0+255), each a
//    tcgen05.mma kind::f16 with bf16 operands and an fp32 accumulator in
//    tensor memory (2 x 256 of the 512 columns).  The two halves share the
//    n-block's operand B, so a 64-token stage brings 512 channels
//    (64 KB) for 2 x 128 x 256 x 64 multiply-adds, against 768 channels for
//    two unrelated 128 x 256 tiles: a third less L2-to-SM operand traffic,
//    which is what bounds the main loop (the same ~15.6 TB/s of operands at
//    1.54 and 1.97 GHz SM clocks with unrelated tiles).  On a diagonal block
//    (m-block = n-block) both halves' A is B itself: only B is loaded.
//  * Both operands are slices of the row-major X, so both are MN-major in
//    shared memory: a TMA box of 64 channels (128 bytes) x 64 tokens with the
//    128-byte swizzle is exactly one column of canonical SW128 MN-major atoms.
//  * All CTAs sweep the tokens in lockstep, so each token slice of X is
//    fetched from HBM once and served to every CTA from L2.
//  * Warp roles: warp 0 issues TMA, warp 1 owns TMEM and issues the MMAs,
//    warps 2..9 drain the accumulators (TMEM -> registers -> H), two warps
//    per TMEM lane quarter, each with half of the columns (twice the H loads
//    in flight while the tensor cores wait for the drain).
//  * The epilogue stores D[m][n] into H[n][m]: for a fixed n the 32 lanes of
//    a warp hold 32 consecutive m, so every store is one coalesced 128-byte
//    line.  Blocks have m-block <= n-block, so the written entries cover H's
//    lower triangle.
//  * Tokens are taken in chunks of 32,768: each chunk's partial block is
//    added into H by the epilogue (fp32, round to nearest), which bounds the
//    bias of the tensor cores' long fp32 accumulation.
//  * No atomics: every H entry has exactly one owner, so the result is
//    deterministic.  Every wait is bounded (GPTQ_ERR_TIMEOUT).
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"

namespace gptq {
namespace {

constexpr int BM = 128;                         // rows per MMA (one half of a block)
constexpr int BN = 256;                         // block width (and height: two halves)
constexpr int BK = 64;
constexpr int kStages = 3;
constexpr int kBox = 64;                        // channels per TMA box (128 bytes)
constexpr int kBoxBytes = kBox * BK * 2;        // 8 KB
constexpr int kABytes = BM * BK * 2;            // 16 KB per half
constexpr int kBBytes = BN * BK * 2;            // 32 KB
constexpr int kStageBytes = kBBytes + 2 * kABytes;  // 64 KB: B, then A of both halves
constexpr int kThreads = 320;   // TMA, MMA, 8 epilogue warps (two per TMEM lane quarter)
constexpr int kTmemCols = 512;
// Tokens accumulated in TMEM before the partial block is added into H.  The
// tensor cores' fp32 accumulation loses about 2^-25 of the running sum per
// accumulate step, with a consistent sign, so the bias grows with the number
// of steps (measured ~1.4e-3 relative over 262,144 tokens in one run);
// draining every 32,768 tokens (512 steps of 64 tokens) keeps it near 6e-5
// (full-size H rows within 1.8e-4 of a float64 sum; 16,384-token drains gave
// 8e-5 and cost 3-5 % more time) and the drains themselves are ordinary
// round-to-nearest fp32 adds.
constexpr int kChunkIters = 32768 / BK;
constexpr int kSmemBytes = kStages * kStageBytes + 1024 + 256;
constexpr uint32_t kIdesc = instr_desc(/*bf16*/ 1, /*A MN*/ 1, /*B MN*/ 1, BM, BN);

struct Barriers {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t acc_full;
    uint64_t acc_empty;
    uint64_t drain;
    uint64_t never;  // the timeout probe's barrier: nothing arrives on it
    uint32_t tmem_base;
    int abort;
};

// Block order.  Blocks are (pi, nj) in 256-channel units with pi <= nj.  They
// are enumerated in super-blocks of kSuperP row blocks x kSuperN column
// blocks (column super-blocks outer, row super-blocks inner; inside one, nj
// outer and pi inner), so that each wave of grid consecutive blocks touches
// few columns of X: a wave reads X[:, its channels] for every token, and
// compact waves keep the number of passes over X low at large d (about 11
// at d = 28672, against one per wave, 43, in an n-block-major order whose
// waves span every row block); d <= 4096 is one wave either way.
constexpr int kSuperP = 4;   // 1024 rows of H
constexpr int kSuperN = 16;  // 4096 columns of H

__device__ __forceinline__ int blocks_in_column(int nj, int plo, int phi) {
    const int top = min(phi, nj + 1);
    return top > plo ? top - plo : 0;
}

__device__ __forceinline__ void block_coords(int t, int NT, int& pi, int& nj) {
    for (int J0 = 0; J0 < NT; J0 += kSuperN) {
        const int J1 = min(NT, J0 + kSuperN);
        for (int P0 = 0; P0 < J1; P0 += kSuperP) {
            const int P1 = min(NT, P0 + kSuperP);
            int cnt = 0;
            for (int n = J0; n < J1; ++n) cnt += blocks_in_column(n, P0, P1);
            if (t < cnt) {
                for (nj = J0; nj < J1; ++nj) {
                    const int c = blocks_in_column(nj, P0, P1);
                    if (t < c) {
                        pi = P0 + t;
                        return;
                    }
                    t -= c;
                }
            }
            t -= cnt;
        }
    }
    pi = 0;
    nj = 0;
}

__global__ void __launch_bounds__(kThreads, 1)
    hessian_syrk_tcgen05(const __grid_constant__ CUtensorMap tmap_x, float* __restrict__ H,
                         int64_t ldh, int d, int n, int num_blocks, int32_t* status,
                         uint64_t probe_ns) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    Barriers* bars = reinterpret_cast<Barriers*>(smem + kStages * kStageBytes);
    volatile int* abort = &bars->abort;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int NT = (d + BN - 1) / BN;
    const int KB = (n + BK - 1) / BK;
    const int G = gridDim.x;
    const int nchunk = (KB + kChunkIters - 1) / kChunkIters;
    // a wave = (one block, one token chunk); the accumulators are drained
    // into H after every wave
    const int waves = ((num_blocks + G - 1) / G) * nchunk;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->empty[s], 1);
        }
        mbar_init(&bars->acc_full, 1);
        mbar_init(&bars->acc_empty, 256);
        mbar_init(&bars->drain, 1);
        mbar_init(&bars->never, 1);
        bars->abort = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmap_x);
    }
    if (warp == 1) {
        tmem_alloc(&bars->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t it = 0;
            for (int w = 0; w < waves && !*abort; ++w) {
                const int t = blockIdx.x + (w / nchunk) * G;
                if (t >= num_blocks) break;
                const int k0 = (w % nchunk) * kChunkIters;
                const int k1 = min(KB, k0 + kChunkIters);
                int pi, nj;
                block_coords(t, NT, pi, nj);
                const int m0 = pi * BN, n0 = nj * BN;
                const bool diag = pi == nj;
                const int halves = (m0 + BM < d) ? 2 : 1;
                const uint32_t bytes = kBBytes + (diag ? 0 : halves * kABytes);
                for (int k = k0; k < k1 && !*abort; ++k) {
                    const uint32_t st = it % kStages;
                    const uint32_t ph = (it / kStages) & 1u;
                    if (!mbar_wait(&bars->empty[st], ph ^ 1u, abort)) break;
                    uint8_t* b = smem + st * kStageBytes;
                    mbar_arrive_expect_tx(&bars->full[st], bytes);
                    const int tok = k * BK;
#pragma unroll
                    for (int c = 0; c < BN / kBox; ++c)
                        tma_load_2d(b + c * kBoxBytes, &tmap_x, &bars->full[st], n0 + c * kBox, tok);
                    if (!diag) {
                        for (int h = 0; h < halves; ++h)
#pragma unroll
                            for (int c = 0; c < BM / kBox; ++c)
                                tma_load_2d(b + kBBytes + h * kABytes + c * kBoxBytes, &tmap_x,
                                            &bars->full[st], m0 + h * BM + c * kBox, tok);
                    }
                    ++it;
                }
            }
            // Never leave with copies in flight: wait for the last issued
            // stages to land (bounded even when aborting).
            const uint32_t last = it < (uint32_t)kStages ? it : (uint32_t)kStages;
            volatile int no_abort = 0;
            for (uint32_t j = 0; j < last; ++j) {
                const uint32_t i2 = it - 1 - j;
                if (!mbar_wait(&bars->full[i2 % kStages], (i2 / kStages) & 1u, &no_abort)) {
                    *abort = 1;
                    break;
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            uint32_t it = 0;
            wait_probe(&bars->never, probe_ns, abort);
            for (int w = 0; w < waves && !*abort; ++w) {
                const int t = blockIdx.x + (w / nchunk) * G;
                if (t >= num_blocks) break;
                const int k0 = (w % nchunk) * kChunkIters;
                const int k1 = min(KB, k0 + kChunkIters);
                int pi, nj;
                block_coords(t, NT, pi, nj);
                const bool diag = pi == nj;
                const int halves = (pi * BN + BM < d) ? 2 : 1;
                if (!mbar_wait(&bars->acc_empty, (w & 1) ^ 1, abort)) break;
                tc_fence_after();
                bool ok = true;
                for (int k = k0; k < k1; ++k) {
                    const uint32_t st = it % kStages;
                    const uint32_t ph = (it / kStages) & 1u;
                    if (!mbar_wait(&bars->full[st], ph, abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t b = smem_u32(smem + st * kStageBytes);
                    for (int h = 0; h < halves; ++h) {
                        // a diagonal block's rows are its own columns: A is
                        // half h of B (two of its four boxes)
                        const uint32_t a = diag ? b + h * 2 * kBoxBytes : b + kBBytes + h * kABytes;
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk) {
                            // 16 tokens = two 8-row swizzle atoms (2 x 1024 B)
                            const uint64_t ad = smem_desc(a + kk * 2048, kBoxBytes, 1024, 2);
                            const uint64_t bd = smem_desc(b + kk * 2048, kBoxBytes, 1024, 2);
                            mma_f16_ss(tmem + h * BN, ad, bd, kIdesc, (k > k0 || kk > 0) ? 1u : 0u);
                        }
                    }
                    mma_commit(&bars->empty[st]);
                    ++it;
                }
                if (!ok) break;
                mma_commit(&bars->acc_full);
            }
            // Drain: every MMA issued by this thread has finished before the
            // tensor memory is released.
            mma_commit(&bars->drain);
            volatile int no_abort = 0;
            if (!mbar_wait(&bars->drain, 0, &no_abort)) *abort = 1;
        }
    } else {
        // ------------------------------------------------ epilogue warps 2..9
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        const int half = (warp - 2) >> 2;  // which 128 of each accumulator's 256 columns it drains
        for (int w = 0; w < waves && !*abort; ++w) {
            const int t = blockIdx.x + (w / nchunk) * G;
            if (t >= num_blocks) break;
            if (!mbar_wait(&bars->acc_full, w & 1, abort)) break;
            tc_fence_after();
            int pi, nj;
            block_coords(t, NT, pi, nj);
            const int halves = (pi * BN + BM < d) ? 2 : 1;
            for (int h = 0; h < halves; ++h) {
                const int m = pi * BN + h * BM + q * 32 + lane;
                const int nb = nj * BN;
#pragma unroll 1
                for (int cc = half * (BN / 64); cc < (half + 1) * (BN / 64); ++cc) {
                    float v[32];
                    tmem_ld32(tmem + (static_cast<uint32_t>(q * 32) << 16) + h * BN + cc * 32, v);
                    if (m < d) {
                        // all 32 loads in flight before any store (the
                        // compiler cannot prove the addresses distinct)
                        float hv[32];
                        float* base = H + static_cast<int64_t>(nb + cc * 32) * ldh + m;
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            hv[j] = (nb + cc * 32 + j < d) ? base[static_cast<int64_t>(j) * ldh] : 0.f;
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (nb + cc * 32 + j < d)
                                base[static_cast<int64_t>(j) * ldh] = fmaf(2.0f, v[j], hv[j]);
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&bars->acc_empty);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, kTmemCols);
    if (threadIdx.x == 0 && bars->abort) report(status, GPTQ_ERR_TIMEOUT);
}

}  // namespace

int hessian_num_tiles(int64_t d) {
    const int NT = static_cast<int>((d + BN - 1) / BN);
    return NT * (NT + 1) / 2;
}

gptq_status launch_hessian(const uint16_t* X, int64_t n, int64_t d, int64_t ldx, float* H,
                           int64_t ldh, int32_t* status, cudaStream_t stream) {
    if (cudaFuncSetAttribute(hessian_syrk_tcgen05, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSmemBytes) != cudaSuccess)
        return GPTQ_ERR_CUDA;
    CUtensorMap tmap;
    if (!make_tmap_2d(&tmap, /*bf16=*/true, X, static_cast<uint64_t>(d), static_cast<uint64_t>(n),
                      static_cast<uint64_t>(ldx), kBox, BK, Swz::k128))
        return GPTQ_ERR_INVALID_ARG;
    const int T = hessian_num_tiles(d);
    const int sms = num_sms();
    const int grid = T < sms ? T : sms;
    hessian_syrk_tcgen05<<<grid, kThreads, kSmemBytes, stream>>>(
        tmap, H, ldh, static_cast<int>(d), static_cast<int>(n), T, status,
        take_wait_probe(kProbeHessian));
    count_launches(1);
    return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ERR_CUDA;
}

}  // namespace gptq
