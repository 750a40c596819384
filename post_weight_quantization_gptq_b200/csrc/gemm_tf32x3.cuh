// fp32-accurate GEMM tiles on the tcgen05 tensor cores ("3xTF32").
//
// D[128 x 128] = sum_k A[m][k] B[n][k] with fp32 operands split as
// x = hi + lo, and three kind::tf32 MMAs accumulate hi*hi + hi*lo + lo*hi
// into one fp32 TMEM accumulator.  kind::tf32 reads a 32-bit operand and
// ignores its 13 low mantissa bits (truncation, measured on sm_100a).  Two
// splits (see kSplitTrunc / kSplitRound below): hi as TMA delivered it and
// lo = x - trunc13(x) (one buffer written per operand, products within about
// 2^-20 of |a||b|, biased towards zero), or hi and lo both rounded to the
// nearest tf32 (two buffers written, products within about 3 2^-22 of |a||b|
// and unbiased), at tensor-core speed either way.  The truncating split can
// also be done ahead (kSplitPre): the lo parts then come from memory with the
// operands.
//
// Persistent: each CTA walks a static list of output tiles (tile, tile +
// grid, ...), the stage ring runs on across tiles and two TMEM accumulators
// let the epilogue of one tile overlap the loads and MMAs of the next.
// Operands arrive through TMA, K-major (a row's K
// values contiguous: box of 32 K x 128 rows, 128-byte swizzle) or MN-major
// (a K row's M/N values contiguous: four boxes of 32 x 32, 128-byte swizzle
// with 32-byte chunks).  Warp roles:
//   warp 0      TMA producer
//   warp 1      TMEM owner and MMA issuer
//   warps 2..9  split each stage's operands (write lo, and hi when rounding;
//               with four warps the split was measurably on the critical path:
//               the lazy update without it ran 9-13 % faster)
//   warps 10..13 drain the accumulator (tcgen05.ld gives one tile row per
//               lane).  Plain outputs receive the product, read-modify-write
//               outputs (kRmw) D -= AB^T.  Three forms:
//               staged (kEpiStaged): into sched.dst() rows, sched.ncols()
//               columns, 32 columns at a time through a padded shared-memory
//               stage, leaving as 4 rows x 128 contiguous bytes per warp
//               access (read-modify-write outputs load the destination
//               values in the same order while the tile's MMAs still run);
//               the form for destinations that cannot be a tensor map;
//               reduce (kEpiReduce, read-modify-write outputs): the warp
//               writes -AB^T for 32 x 32 elements into a shared-memory buffer
//               (128-byte swizzle) and one lane hands it to a TMA tensor
//               reduction (cp.reduce.async.bulk.tensor .add) into D: the
//               read-modify-write happens in L2, with no global loads or
//               stores from the SM; two buffers per warp alternate;
//               store (kEpiStore, plain outputs): the same with AB^T and a
//               TMA tensor store.  Both write whole boxes, clipped only at
//               the tensor map's extent.
// Every wait is bounded; on expiry GPTQ_ERR_TIMEOUT is recorded and the CTA
// winds down after its copies and MMAs have landed.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "kernels.h"

namespace gptq {
namespace g3 {

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int BK = 32;                        // K per stage: 128 bytes of fp32
constexpr int kStages = 3;
constexpr int kTileBytes = 128 * BK * 4;      // 16 KB
constexpr int kStageBytes = 4 * kTileBytes;   // A (as loaded), A lo, B (as loaded), B lo
constexpr int kThreads = 448;                 // TMA, MMA, 8 split warps, 4 epilogue warps
constexpr int kSplitThreads = 256;
constexpr int kEpiPitch = 36;                 // floats per staged row (16-byte groups of 8
                                              // consecutive rows fall in distinct banks)
constexpr int kEpiBytes = 4 * 32 * kEpiPitch * 4;  // one 32 x 32 stage per epilogue warp
constexpr int kSmemBytes = kStages * kStageBytes + 1024 + 256 + kEpiBytes;
constexpr int kRedBufBytes = 32 * 32 * 4;  // one 32 x 32 fp32 box
// drain forms (see the header comment)
constexpr int kEpiStaged = 1, kEpiReduce = 2, kEpiStore = 3;
// dynamic shared memory of a drain form: the reduce buffers (two per warp)
// start 1024 bytes after the stages, on the 128-byte swizzle's 1024-byte period
template <int Epi>
constexpr int smem_bytes() {
    return Epi >= kEpiReduce ? kStages * kStageBytes + 1024 + 1024 + 8 * kRedBufBytes : kSmemBytes;
}
constexpr uint32_t kTmemCols = 256;           // two 128-column accumulators

// One output tile: rows m0.. of A, rows n0.. of B, K from ka0 (A) / kb0 (B),
// nk stages of 32.  nk <= 0 skips the tile.
struct Job {
    int m0, n0, ka0, kb0, nk;
};

struct Bars {
    uint64_t full[kStages];
    uint64_t conv[kStages];
    uint64_t empty[kStages];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t drain;
    uint64_t never;  // the timeout probe's barrier: nothing arrives on it
    uint32_t tmem;
    int abort;
};

// x minus the part of it a kind::tf32 MMA sees (exact: both share x's exponent)
__device__ __forceinline__ float tf32_rest(float x) {
    return x - __uint_as_float(__float_as_uint(x) & 0xffffe000u);
}

// x rounded to the nearest tf32 value (ties away from zero): adding half of
// the 13 dropped bits' range to the bit pattern carries into the kept
// mantissa (and, at the top of a binade, into the exponent) exactly when the
// dropped part is at least half a tf32 ulp.  Finite inputs only.
__device__ __forceinline__ float tf32_round(float x) {
    return __uint_as_float((__float_as_uint(x) + 0x1000u) & 0xffffe000u);
}
__device__ __forceinline__ float4 tf32_round4(float4 v) {
    return make_float4(tf32_round(v.x), tf32_round(v.y), tf32_round(v.z), tf32_round(v.w));
}
__device__ __forceinline__ float4 sub4(float4 a, float4 b) {
    return make_float4(a.x - b.x, a.y - b.y, a.z - b.z, a.w - b.w);
}

// Operand splits.  kSplitTrunc: hi is the value as loaded (the MMA truncates
// it), lo = the truncated-off remainder, which the MMA truncates in turn:
// only lo is written, but every product loses up to ~2^-20 of |ab|, always
// towards zero, so long sums drift one way.  kSplitRound: hi = x rounded to
// the nearest tf32, lo = the (exact) remainder rounded to the nearest tf32,
// both written: x - hi - lo is within 2^-22 |x| and of either sign, so a
// product's error (that, the two roundings and the dropped lo lo term) stays
// within ~3 2^-22 |ab| and long sums do not drift.
// kSplitPre: the truncating split done ahead of the GEMM: both operands' lo
// parts sit in memory of their own (the same values kSplitTrunc computes) and
// arrive by TMA with the operands; no split work between a stage's arrival and
// its MMAs.
constexpr int kSplitTrunc = 0, kSplitRound = 1, kSplitPre = 2;



template <bool MN>
__device__ __forceinline__ void load_operand(uint8_t* dst, const CUtensorMap* map, uint64_t* bar,
                                             int row0, int k) {
    if (MN) {
#pragma unroll
        for (int c = 0; c < 4; ++c) tma_load_2d(dst + c * 4096, map, bar, row0 + 32 * c, k);
    } else {
        tma_load_2d(dst, map, bar, k, row0);
    }
}

// Descriptor of K-step kk (8 tf32 values of K) inside a 32-wide stage.
//  K-major: 128-byte swizzle, 8-row atoms (SBO 1024), 32 bytes of K per step.
//  MN-major: 32-bit MN-major operands use the 128-byte swizzle with 32-byte
//  chunks (layout type 1): 4-row atoms of 512 bytes (SBO), 32-element MN
//  chunks 4 KB apart (LBO), 8 K-rows = 1024 bytes per step.
template <bool MN>
__device__ __forceinline__ uint64_t operand_desc(uint32_t base, int kk) {
    if (MN) return smem_desc(base + kk * 1024, 4096, 512, 1);
    return smem_desc(base + kk * 32, 16, 1024, 2);
}


template <class Sched, bool A_MN, bool B_MN, int Epi, int Split>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tf32x3_kernel(const __grid_constant__ CUtensorMap tma, const __grid_constant__ CUtensorMap tmb,
                       const __grid_constant__ CUtensorMap tmd, const __grid_constant__ CUtensorMap tmal,
                       const __grid_constant__ CUtensorMap tmbl, const Sched sched, int tiles,
                       int32_t* status, uint64_t probe_ns) {
    constexpr uint32_t kIdesc = instr_desc(/*tf32*/ 2, A_MN ? 1 : 0, B_MN ? 1 : 0, BM, BN);

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    Bars* bars = reinterpret_cast<Bars*>(smem + kStages * kStageBytes);
    volatile int* abort = &bars->abort;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    pdl_trigger();

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->conv[s], kSplitThreads);
            mbar_init(&bars->empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars->acc_full[s], 1);
            mbar_init(&bars->acc_empty[s], 128);
        }
        mbar_init(&bars->drain, 1);
        mbar_init(&bars->never, 1);
        bars->abort = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tma);
        tma_prefetch_desc(&tmb);
        if constexpr (Epi >= kEpiReduce) tma_prefetch_desc(&tmd);
        if constexpr (Split == kSplitPre) {
            tma_prefetch_desc(&tmal);
            tma_prefetch_desc(&tmbl);
        }
    }
    if (warp == 1) {
        tmem_alloc(&bars->tmem, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem;
    pdl_wait();  // set-up above touched no global memory

    if (warp == 0) {
        // ---------------------------------------------------- TMA producer
        if (lane == 0) {
            int it = 0;
            for (int t = blockIdx.x; t < tiles && !*abort; t += gridDim.x) {
                const Job job = sched.job(t);
                for (int s = 0; s < job.nk && !*abort; ++s, ++it) {
                    const int st = it % kStages;
                    const uint32_t ph = (it / kStages) & 1;
                    if (!mbar_wait(&bars->empty[st], ph ^ 1u, abort)) break;
                    uint8_t* a = smem + st * kStageBytes;
                    mbar_arrive_expect_tx(&bars->full[st], (Split == kSplitPre ? 4 : 2) * kTileBytes);
                    load_operand<A_MN>(a, &tma, &bars->full[st], job.m0, job.ka0 + s * BK);
                    load_operand<B_MN>(a + 2 * kTileBytes, &tmb, &bars->full[st], job.n0,
                                       job.kb0 + s * BK);
                    if constexpr (Split == kSplitPre) {
                        load_operand<A_MN>(a + kTileBytes, &tmal, &bars->full[st], job.m0,
                                           job.ka0 + s * BK);
                        load_operand<B_MN>(a + 3 * kTileBytes, &tmbl, &bars->full[st], job.n0,
                                           job.kb0 + s * BK);
                    }
                }
            }
            // never leave with copies in flight (bounded even when aborting)
            volatile int no_abort = 0;
            const int last = it < kStages ? it : kStages;
            for (int j = 0; j < last; ++j) {
                const int i2 = it - 1 - j;
                if (!mbar_wait(&bars->full[i2 % kStages], (i2 / kStages) & 1, &no_abort)) {
                    *abort = 1;
                    break;
                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------- MMA issuer
        if (lane == 0) {
            int it = 0, lt = 0;
            bool ok = wait_probe(&bars->never, probe_ns, abort);
            for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
                const Job job = sched.job(t);
                if (job.nk <= 0) continue;
                const int slot = lt & 1;
                const uint32_t use = static_cast<uint32_t>(lt >> 1);
                if (!mbar_wait(&bars->acc_empty[slot], (use & 1u) ^ 1u, abort)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t acc = tmem + slot * BN;
                for (int s = 0; s < job.nk; ++s, ++it) {
                    const int st = it % kStages;
                    const uint32_t ph = (it / kStages) & 1;
                    if (!mbar_wait(Split == kSplitPre ? &bars->full[st] : &bars->conv[st], ph, abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a = smem_u32(smem + st * kStageBytes);
                    const uint32_t alo = a + kTileBytes, b = a + 2 * kTileBytes, blo = a + 3 * kTileBytes;
#pragma unroll
                    for (int kk = 0; kk < BK / 8; ++kk) {
                        const uint64_t ah = operand_desc<A_MN>(a, kk), al = operand_desc<A_MN>(alo, kk);
                        const uint64_t bh = operand_desc<B_MN>(b, kk), bl = operand_desc<B_MN>(blo, kk);
                        mma_tf32_ss(acc, ah, bh, kIdesc, (s > 0 || kk > 0) ? 1u : 0u);
                        mma_tf32_ss(acc, ah, bl, kIdesc, 1u);
                        mma_tf32_ss(acc, al, bh, kIdesc, 1u);
                    }
                    mma_commit(&bars->empty[st]);
                }
                if (!ok) break;
                mma_commit(&bars->acc_full[slot]);
                ++lt;
            }
            mma_commit(&bars->drain);
            volatile int no_abort = 0;
            if (!mbar_wait(&bars->drain, 0, &no_abort)) *abort = 1;
        }
    } else if (warp < 10) {
        // ---------------------------------------------------- split into hi / lo
        if constexpr (Split == kSplitPre) {
            // the lo parts arrive with the operands: nothing to do
        } else {
            const int t0 = threadIdx.x - 64;
            int it = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
                const Job job = sched.job(t);
                for (int s = 0; s < job.nk; ++s, ++it) {
                    const int st = it % kStages;
                    const uint32_t ph = (it / kStages) & 1;
                    if (!mbar_wait(&bars->full[st], ph, abort)) {
                        ok = false;
                        break;
                    }
                    float4* a = reinterpret_cast<float4*>(smem + st * kStageBytes);
                    float4* alo = a + kTileBytes / 16;
                    float4* b = a + 2 * (kTileBytes / 16);
                    float4* blo = a + 3 * (kTileBytes / 16);
#pragma unroll 4
                    for (int i = t0; i < kTileBytes / 16; i += kSplitThreads) {
                        const float4 x = a[i], y = b[i];
                        if constexpr (Split == kSplitRound) {
                            const float4 xh = tf32_round4(x), yh = tf32_round4(y);
                            a[i] = xh;
                            b[i] = yh;
                            alo[i] = tf32_round4(sub4(x, xh));
                            blo[i] = tf32_round4(sub4(y, yh));
                        } else {
                            alo[i] = make_float4(tf32_rest(x.x), tf32_rest(x.y), tf32_rest(x.z), tf32_rest(x.w));
                            blo[i] = make_float4(tf32_rest(y.x), tf32_rest(y.y), tf32_rest(y.z), tf32_rest(y.w));
                        }
                    }
                    fence_async_smem();
                    mbar_arrive(&bars->conv[st]);
                }
            }
        }
    } else {
        // ---------------------------------------------------- epilogue
        const int q = warp & 3;  // TMEM lane quarter of this warp: tile rows 32 q ..
        const uint32_t stage = smem_u32(smem + kStages * kStageBytes + 256) + q * 32 * kEpiPitch * 4;
        const int rsub = lane >> 3;     // row within each group of 4 rows
        const int c4 = 4 * (lane & 7);  // this lane's first column within a chunk
        int lt = 0;
        for (int t = blockIdx.x; t < tiles; t += gridDim.x) {
            const Job job = sched.job(t);
            if (job.nk <= 0) continue;
            const int slot = lt & 1;
            const uint32_t use = static_cast<uint32_t>(lt >> 1);
            if constexpr (Epi >= kEpiReduce) {
                static_assert(Sched::kRmw == (Epi == kEpiReduce),
                              "reduce serves read-modify-write outputs, store plain ones");
                constexpr float sgn = Epi == kEpiReduce ? -1.f : 1.f;
                if (!mbar_wait(&bars->acc_full[slot], use & 1u, abort)) break;
                tc_fence_after();
                const uint32_t rbase = smem_u32(smem + kStages * kStageBytes + 1024) + q * 2 * kRedBufBytes;
#pragma unroll
                for (int cc = 0; cc < BN / 32; ++cc) {
                    const uint32_t buf = rbase + (cc & 1) * kRedBufBytes;
                    // the reduction that last read this buffer (two chunks ago) is done reading
                    if (lane == 0) bulk_wait_read_but1();
                    __syncwarp();
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        float v[16];
                        tmem_ld16(tmem + (static_cast<uint32_t>(q * 32) << 16) + slot * BN + cc * 32 + h * 16,
                                  v);
                        // row `lane` of the box, 16-byte chunk 4 h + j at its 128-byte-swizzle slot
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            sts128(buf + lane * 128 + ((((4 * h + j) ^ (lane & 7))) << 4),
                                   make_float4(sgn * v[4 * j], sgn * v[4 * j + 1], sgn * v[4 * j + 2],
                                               sgn * v[4 * j + 3]));
                    }
                    fence_async_smem();  // the writes above, before the async proxy reads them
                    __syncwarp();
                    if (lane == 0) {
                        if constexpr (Epi == kEpiReduce)
                            tma_reduce_add_2d(&tmd, buf, job.n0 + 32 * cc, job.m0 + 32 * q);
                        else
                            tma_store_2d(&tmd, buf, job.n0 + 32 * cc, job.m0 + 32 * q);
                        bulk_commit();
                    }
                }
                tc_fence_before();
                mbar_arrive(&bars->acc_empty[slot]);
                ++lt;
                continue;
            }
            // read-modify-write: this lane's destination values (rows
            // 32 q + 4 i + rsub, columns 32 cc + c4 ..) when the whole row
            // segment may be read: chunks 0 and 1 are loaded before the
            // accumulator is ready, chunk cc + 2 once chunk cc is written
            float4 old[2][8];
            bool pre = false;
            auto fetch = [&](int cc, float4 (&o)[8]) {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float* d = sched.dst(job, 32 * q + 4 * i + rsub);
                    const float* p = d != nullptr ? d + 32 * cc + c4 : nullptr;
                    o[i] = (p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15) == 0)
                               ? *reinterpret_cast<const float4*>(p)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
                }
            };
            if constexpr (Sched::kRmw) {
                pre = sched.nreadable(job) == BN;
                if (pre) {
                    fetch(0, old[0]);
                    fetch(1, old[1]);
                }
            }
            if (!mbar_wait(&bars->acc_full[slot], use & 1u, abort)) break;
            tc_fence_after();
#pragma unroll
            for (int cc = 0; cc < BN / 32; ++cc) {
                // the chunk into the stage, one tile row per lane
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    float v[16];
                    tmem_ld16(tmem + (static_cast<uint32_t>(q * 32) << 16) + slot * BN + cc * 32 + h * 16,
                              v);
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        sts128(stage + (lane * kEpiPitch + h * 16 + 4 * j) * 4,
                               make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]));
                }
                __syncwarp();
                // and out, 8 lanes per row: 4 columns each, 4 rows per access
                float4 st[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) st[i] = lds128(stage + ((4 * i + rsub) * kEpiPitch + c4) * 4);
                __syncwarp();  // every lane has read the stage: the next chunk may rewrite it
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int row = 32 * q + 4 * i + rsub;
                    float* d = sched.dst(job, row);
                    const int col = 32 * cc + c4;
                    const int n = d != nullptr ? sched.ncols(job, row) - col : 0;
                    if (n > 0) {
                        const float4 a = st[i];
                        float* p = d + col;
                        const bool vec = n >= 4 && (reinterpret_cast<uintptr_t>(p) & 15) == 0;
                        float4 out = a;
                        if constexpr (Sched::kRmw) {
                            float4 o;
                            if (pre && vec) {
                                o = old[cc & 1][i];
                            } else {
                                o.x = p[0];
                                o.y = n > 1 ? p[1] : 0.f;
                                o.z = n > 2 ? p[2] : 0.f;
                                o.w = n > 3 ? p[3] : 0.f;
                            }
                            out = make_float4(o.x - a.x, o.y - a.y, o.z - a.z, o.w - a.w);
                        }
                        if (vec) {
                            *reinterpret_cast<float4*>(p) = out;
                        } else {
                            p[0] = out.x;
                            if (n > 1) p[1] = out.y;
                            if (n > 2) p[2] = out.z;
                            if (n > 3) p[3] = out.w;
                        }
                    }
                }
                if constexpr (Sched::kRmw) {
                    if (pre && cc + 2 < BN / 32) fetch(cc + 2, old[cc & 1]);
                }
            }
            tc_fence_before();
            mbar_arrive(&bars->acc_empty[slot]);
            ++lt;
        }
        // reductions issued by this warp have completed (reads and writes)
        if constexpr (Epi >= kEpiReduce) {
            if (lane == 0) bulk_wait_all();
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, kTmemCols);
    if (threadIdx.x == 0 && bars->abort) report(status, GPTQ_ERR_TIMEOUT);
}

// pdl: launched with programmatic serialization (see launch_kernel).
// td: the destination's tensor map (box 32 x 32 fp32, 128-byte swizzle) for
// the reduce drain; unused by the other forms.
// tal, tbl: the lo parts' tensor maps (same boxes as ta, tb) for kSplitPre;
// unused by the other splits.
template <class Sched, bool A_MN, bool B_MN, int Epi, int Split = kSplitRound>
inline cudaError_t launch(const CUtensorMap& ta, const CUtensorMap& tb, const Sched& sched,
                          int tiles, int32_t* status, cudaStream_t stream, int sms,
                          bool pdl = false, const CUtensorMap* td = nullptr,
                          const CUtensorMap* tal = nullptr, const CUtensorMap* tbl = nullptr) {
    auto kern = gemm_tf32x3_kernel<Sched, A_MN, B_MN, Epi, Split>;
    if (Epi >= kEpiReduce && td == nullptr) return cudaErrorInvalidValue;
    if (Split == kSplitPre && (tal == nullptr || tbl == nullptr)) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         smem_bytes<Epi>());
    if (e != cudaSuccess) return e;
    if (tiles <= 0) return cudaSuccess;
    const int grid = tiles < sms ? tiles : sms;
    return launch_kernel(pdl, kern, dim3(grid), dim3(kThreads), smem_bytes<Epi>(), stream, ta, tb,
                         td != nullptr ? *td : tb, tal != nullptr ? *tal : ta,
                         tbl != nullptr ? *tbl : tb, sched, tiles, status,
                         take_wait_probe(kProbeGemm));
}

}  // namespace g3
}  // namespace gptq
