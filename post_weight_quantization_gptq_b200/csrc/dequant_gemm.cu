// Using the quantized layer, many-token (prefill) form: Y = X W_hat^T on the
// 5th-generation tensor cores.
//
// "GPTQ (GPT Quantization)", "Limitations" (items 1-2): the quantization is
// weight-only -- activations stay at 16 bits -- and the integer weights are
// dequantized to 16 bits before each product.  Here each CTA dequantizes a
// 256-row slice of the packed layer into bf16 tiles in shared memory, stage by
// stage, and the tensor cores multiply them with the (act-order gathered) bf16
// activations:
//   W_hat[n][k] = bf16( fp32(s[k/g][n]) * (q[n][k] - z[k/g][n]) )   (fp32 product,
//                 rounded to nearest-even bf16)
//   Y[t][n]     = sum_k Xq[t][k] W_hat[n][k]     (exact bf16 products, fp32 sums)
// with Xq[t][k] = X[t][perm[k]] (quantization order; gathered into the
// workspace when perm is given).
//
// CTA tile: 256 tokens x 256 layer outputs, K in stages of 64.  Warp roles:
//   warp 0      TMA: the stage's activations (256 x 64 bf16, 128-byte swizzle)
//   warp 10     TMA: the stage's packed words (256 rows x 64 codes), several
//               stages ahead in a ring of their own
//   warp 1      TMEM owner (512 columns: two 128-token accumulators of 256
//               fp32 columns) and MMA issuer: per stage, 2 x 4 MMAs
//               kind::f16 M=128 N=256 K=16, both operands K-major
//   warps 2..9  dequantize: thread n turns row n's 64 codes of the stage into
//               bf16 and writes them, 16 bytes at a time, in the 128-byte
//               swizzled K-major layout the MMA reads (three rotating
//               buffers, two at 8 bits); after the K loop they drain the
//               accumulators
// Every wait is bounded (GPTQ_ERR_TIMEOUT, as in the other tensor-core kernels).
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"

namespace gptq {
namespace {

constexpr int TM = 256;                       // tokens per CTA tile
constexpr int TN = 256;                       // layer outputs per CTA tile (MMA N)
constexpr int BK = 64;                        // k per stage: 128 bytes of bf16
constexpr int kAStages = 3;                   // activation tiles in flight
constexpr int kABytes = TM * BK * 2;          // 32 KB
constexpr int kBBytes = TN * BK * 2;          // 32 KB (one dequantized bf16 tile)
// Per code width: the packed words of a stage (TN rows x 64 codes), how many
// such stages are in flight (their own ring, released by the dequantization
// as soon as it has read them, so they arrive well before they are needed:
// when they shared the activations' stages, released only by the MMAs, a
// stage's words could not be loaded before the MMAs two stages back had
// finished) and the number of bf16 tiles the dequantization rotates through
// (three let it run two stages ahead of the MMAs).  Shared memory: the
// activation ring, the bf16 tiles, then the packed ring.
template <int BITS>
struct Geom {
    static constexpr int kPacked = TN * BK * BITS / 8;
    static constexpr int kPStages = BITS == 8 ? 3 : BITS == 4 ? 4 : 6;
    static constexpr int kBBufs = BITS == 8 ? 2 : 3;
    static constexpr int kSmemBytes =
        kAStages * kABytes + kBBufs * kBBytes + kPStages * kPacked + 1024 + 256;
};
constexpr int kMaxBBufs = 3;
constexpr int kMaxPStages = 6;
constexpr int kThreads = 352;  // TMA (activations), MMA, 8 dequantization warps, TMA (packed)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kIdesc = instr_desc(/*bf16*/ 1, /*A K-major*/ 0, /*B K-major*/ 0, 128, TN);

struct Bars {
    uint64_t afull[kAStages];     // TMA: activations landed
    uint64_t aempty[kAStages];    // MMA: activations consumed
    uint64_t pfull[kMaxPStages];  // TMA: packed words landed
    uint64_t pempty[kMaxPStages]; // dequantization: packed words read (256 arrivals)
    uint64_t bfull[kMaxBBufs];   // dequant warps: bf16 tile written (256 arrivals)
    uint64_t bempty[kMaxBBufs];  // MMA: bf16 tile consumed
    uint64_t acc_full;        // MMA: every product of the tile done
    uint64_t drain;
    uint32_t tmem;
    int abort;
};

// Pairs of fp32 values in one 64-bit register, operated on by the packed
// f32x2 instructions of sm_100 (one instruction, two IEEE round-to-nearest
// results: the same values as two scalar operations).
__device__ __forceinline__ uint64_t pk2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

// x rounded to the nearest bf16 (ties to even), as an fp32 whose low 16 bits
// are zero, on the fp32 pipe: Veltkamp's split with the factor 2^16 + 1,
// c = x (2^16 + 1), hi = c - (c - x), keeps the 8 leading significant bits of
// x rounded to nearest-even (|x| < 2^111); checked against the integer
// rounding rule on random values and exact ties.  It needs each step rounded
// on its own: the scalar intrinsics below are never fused into an fma,
// whereas the packed f32x2 form of the same steps was (its product merged
// into the subtraction after it, which turned the rounding into truncation:
// a one-ulp bf16 error that the parity test caught).  The conversion
// instruction runs on the narrow conversion pipe, which the dequantization
// saturated (ncu: 102 % of its peak); this form does not use it.
__device__ __forceinline__ uint32_t bf16_bits(float x) {
    const float c = __fmul_rn(x, 65537.f);
    return __float_as_uint(__fsub_rn(c, __fsub_rn(c, x)));
}
// both values of a pair as one bf16x2 word (the low value in the low half)
__device__ __forceinline__ uint32_t bf16x2_rne(uint64_t v) {
    float lo, hi;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
    return __byte_perm(bf16_bits(lo), bf16_bits(hi), 0x7632);
}

// The eight codes of chunk c (codes 8c .. 8c+7 of the stage's row) as the
// floats 2^23 + q: each code's bits land in the mantissa of 2^23 (a byte
// permute against the exponent byte 0x4B where a code fills its own byte;
// no int-to-float conversion).
template <int BITS>
__device__ __forceinline__ void chunk_codes(const uint32_t* w, int c, float (&f)[8]) {
    constexpr uint32_t kMagic = 0x4B000000u;
    if constexpr (BITS == 4) {
        const uint32_t x = w[c];
        const uint32_t ev = x & 0x0F0F0F0Fu;          // codes 0, 2, 4, 6 in bytes 0..3
        const uint32_t od = (x >> 4) & 0x0F0F0F0Fu;   // codes 1, 3, 5, 7
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            f[2 * b] = __uint_as_float(__byte_perm(ev, kMagic, 0x7440 + b));
            f[2 * b + 1] = __uint_as_float(__byte_perm(od, kMagic, 0x7440 + b));
        }
    } else if constexpr (BITS == 8) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
            f[i] = __uint_as_float(__byte_perm(w[2 * c + (i >> 2)], kMagic, 0x7440 + (i & 3)));
    } else {
        const uint32_t h = w[c >> 1] >> (16 * (c & 1));
#pragma unroll
        for (int i = 0; i < 8; ++i) f[i] = __uint_as_float(((h >> (2 * i)) & 3u) | kMagic);
    }
}

// prmt.b32 in its default mode: each selector nibble picks one of the 8
// bytes of (a, b); with the nibble's top bit set the picked byte's sign bit
// fills the result byte (0x00 or 0xFF).
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

// The 16 dequantized weights a 4-bit row group can take, bf16(s (q - z)) for
// q = 0..15 with the same arithmetic as the direct path, as byte tables: lo[j]
// holds the low bytes of entries 4j .. 4j+3, hi[j] their high bytes.
__device__ __forceinline__ void build_table4(float s, float z, uint32_t (&lo)[4], uint32_t (&hi)[4]) {
    const uint64_t s2 = pk2(s, s), z2 = pk2(z, z);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        uint32_t r[4];
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            const float q0 = static_cast<float>(4 * j + 2 * p);
            const uint64_t v = mul2(sub2(pk2(q0, q0 + 1.f), z2), s2);  // q - z exact, one rounding
            float a, b;
            asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
            r[2 * p] = bf16_bits(a);        // bf16 in the high half
            r[2 * p + 1] = bf16_bits(b);
        }
        const uint32_t u01 = __byte_perm(r[0], r[1], 0x7362);  // lo0 lo1 hi0 hi1
        const uint32_t u23 = __byte_perm(r[2], r[3], 0x7362);
        lo[j] = __byte_perm(u01, u23, 0x5410);
        hi[j] = __byte_perm(u01, u23, 0x7632);
    }
}

// The bf16 weights of the eight 4-bit codes of x (code i in bits 4i..4i+3) as
// four bf16x2 words, by table look-up: a byte permute selects each code's
// entry among 8 by its low three bits, in the tables' first and second
// halves, and its fourth bit picks the half.
__device__ __forceinline__ void lookup8(uint32_t x, const uint32_t (&lo)[4], const uint32_t (&hi)[4],
                                        uint32_t (&o)[4]) {
    const uint32_t xs = x << 4;  // a code's fourth bit at the top of a byte, even codes
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const uint32_t sel = (x >> (16 * h)) & 0x7777u;
        // 0xFF in byte i where code 4h + i is 8 or more (odd codes' fourth bit
        // is already the top of a byte of x)
        const uint32_t m = prmt(xs, x, h == 0 ? 0xD9C8u : 0xFBEAu);
        const uint32_t la = prmt(lo[0], lo[1], sel), lb = prmt(lo[2], lo[3], sel);
        const uint32_t ha = prmt(hi[0], hi[1], sel), hb = prmt(hi[2], hi[3], sel);
        const uint32_t L = (la & ~m) | (lb & m), H = (ha & ~m) | (hb & m);
        o[2 * h] = __byte_perm(L, H, 0x5140);      // codes 4h, 4h + 1
        o[2 * h + 1] = __byte_perm(L, H, 0x7362);  // codes 4h + 2, 4h + 3
    }
}

// kAligned: the group size is a multiple of the stage's 64 codes, so groups
// change only between stages.
template <int BITS, bool kAligned>
__global__ void __launch_bounds__(kThreads, 1)
    dequant_gemm_kernel(const __grid_constant__ CUtensorMap tma, const __grid_constant__ CUtensorMap tmp,
                        const float* __restrict__ scales, const int32_t* __restrict__ zeros,
                        float* __restrict__ Y, int64_t ldy, int n_tok, int d_row, int K, int g,
                        int32_t* status) {
    constexpr int kCpw = 32 / BITS;               // codes per packed word
    constexpr int kWords = BK / kCpw;             // words per row per stage
    constexpr int kRowBytes = kWords * 4;         // packed bytes per row per stage
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    constexpr int kBBufs = Geom<BITS>::kBBufs;
    constexpr int kPStages = Geom<BITS>::kPStages;
    constexpr int kPacked = Geom<BITS>::kPacked;
    uint8_t* bbuf = smem + kAStages * kABytes;     // the bf16 tiles, 1024-aligned
    uint8_t* pbuf = bbuf + kBBufs * kBBytes;       // the packed ring
    Bars* bars = reinterpret_cast<Bars*>(pbuf + kPStages * kPacked);
    volatile int* abort = &bars->abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * TN, t0 = blockIdx.y * TM;
    const int nk = K / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kAStages; ++s) {
            mbar_init(&bars->afull[s], 1);
            mbar_init(&bars->aempty[s], 1);
        }
        for (int s = 0; s < kPStages; ++s) {
            mbar_init(&bars->pfull[s], 1);
            mbar_init(&bars->pempty[s], 256);
        }
        for (int b = 0; b < kBBufs; ++b) {
            mbar_init(&bars->bfull[b], 256);
            mbar_init(&bars->bempty[b], 1);
        }
        mbar_init(&bars->acc_full, 1);
        mbar_init(&bars->drain, 1);
        bars->abort = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tma);
        tma_prefetch_desc(&tmp);
    }
    if (warp == 1) {
        tmem_alloc(&bars->tmem, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem;

    if (warp == 0 || warp == 10) {
        // ------------------------------------------------ TMA producers: warp 0
        // the activations (ring released by the MMAs), warp 10 the packed
        // words (ring released by the dequantization)
        if (lane == 0) {
            const bool act = warp == 0;
            const int depth = act ? kAStages : kPStages;
            uint64_t* fullb = act ? bars->afull : bars->pfull;
            uint64_t* emptyb = act ? bars->aempty : bars->pempty;
            int it = 0;
            for (; it < nk && !*abort; ++it) {
                const int st = it % depth;
                const uint32_t ph = (it / depth) & 1u;
                if (!mbar_wait(&emptyb[st], ph ^ 1u, abort)) break;
                if (act) {
                    mbar_arrive_expect_tx(&fullb[st], kABytes);
                    tma_load_2d(smem + st * kABytes, &tma, &fullb[st], it * BK, t0);
                } else {
                    mbar_arrive_expect_tx(&fullb[st], TN * kRowBytes);
                    tma_load_2d(pbuf + st * kPacked, &tmp, &fullb[st], it * kWords, n0);
                }
            }
            // never leave with copies in flight (bounded even when aborting)
            volatile int no_abort = 0;
            const int last = it < depth ? it : depth;
            for (int j = 0; j < last; ++j) {
                const int i2 = it - 1 - j;
                if (!mbar_wait(&fullb[i2 % depth], (i2 / depth) & 1u, &no_abort)) {
                    *abort = 1;
                    break;
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            bool ok = true;
            for (int it = 0; it < nk && ok; ++it) {
                const int st = it % kAStages, b = it % kBBufs;
                if (!mbar_wait(&bars->afull[st], (it / kAStages) & 1u, abort) ||
                    !mbar_wait(&bars->bfull[b], (it / kBBufs) & 1u, abort)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t a = smem_u32(smem + st * kABytes);
                const uint32_t bt = smem_u32(bbuf + b * kBBytes);
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)
                        mma_f16_ss(tmem + h * TN, smem_desc(a + h * (kABytes / 2) + kk * 32, 16, 1024, 2),
                                   smem_desc(bt + kk * 32, 16, 1024, 2), kIdesc,
                                   (it > 0 || kk > 0) ? 1u : 0u);
                mma_commit(&bars->aempty[st]);
                mma_commit(&bars->bempty[b]);
            }
            if (ok) mma_commit(&bars->acc_full);
            mma_commit(&bars->drain);
            volatile int no_abort = 0;
            if (!mbar_wait(&bars->drain, 0, &no_abort)) *abort = 1;
        }
    } else {
        // ------------------------------------------------ dequantize
        const int n = threadIdx.x - 64;  // row of the tile, 0..255
        const int ng = n0 + n;
        const bool live = ng < d_row;
        const int groups = (K + g - 1) / g;
        // the current group's scale and zero point, and the next group's,
        // loaded one group ahead so that no chunk waits on global memory;
        // the group starts are tracked by addition (no integer division in
        // the loop: its reciprocal runs on the narrow conversion pipe)
        int cur_g = -1, next_start = 0;
        float s = 0.f, z = 0.f, s_nx = 0.f, z_nx = 0.f;
        auto fetch = [&](int gi, float& sv, float& zv) {
            if (live && gi < groups) {
                sv = __ldg(scales + static_cast<int64_t>(gi) * d_row + ng);
                zv = static_cast<float>(__ldg(zeros + static_cast<int64_t>(gi) * d_row + ng));
            }
        };
        fetch(0, s_nx, z_nx);
        // 4-bit codes with groups of whole stages: a table of the group's 16
        // weights, built once per group (about 90 instructions, against about
        // 8 per code computed directly)
        constexpr bool kTable = BITS == 4 && kAligned;
        uint64_t s2 = 0, off2 = 0;
        uint32_t tlo[4] = {0, 0, 0, 0}, thi[4] = {0, 0, 0, 0};
        auto advance = [&]() {
            ++cur_g;
            next_start += g;
            s = s_nx;
            z = z_nx;
            fetch(cur_g + 1, s_nx, z_nx);
            if constexpr (kTable) {
                build_table4(s, z, tlo, thi);
            } else {
                s2 = pk2(s, s);
                // subtracting 2^23 + z from 2^23 + q leaves q - z exactly
                const float off = 8388608.f + z;
                off2 = pk2(off, off);
            }
        };
        bool ok = true;
        for (int it = 0; it < nk; ++it) {
            const int ps = it % kPStages, b = it % kBBufs;
            if (!mbar_wait(&bars->pfull[ps], (it / kPStages) & 1u, abort) ||
                !mbar_wait(&bars->bempty[b], ((it / kBBufs) & 1u) ^ 1u, abort)) {
                ok = false;
                break;
            }
            const uint32_t* words =
                reinterpret_cast<const uint32_t*>(pbuf + ps * kPacked + n * kRowBytes);
            uint32_t w[kWords];
#pragma unroll
            for (int q = 0; q < kWords / 4; ++q) {
                const uint4 v = reinterpret_cast<const uint4*>(words)[q];
                w[4 * q] = v.x; w[4 * q + 1] = v.y; w[4 * q + 2] = v.z; w[4 * q + 3] = v.w;
            }
            const uint32_t row = smem_u32(bbuf + b * kBBytes) + n * 128;
            if constexpr (kAligned) {
                if (it * BK >= next_start) advance();
            }
            // 8 codes (one 16-byte chunk of bf16) at a time
#pragma unroll
            for (int c = 0; c < BK / 8; ++c) {
                if constexpr (!kAligned) {
                    // g is a multiple of 8: a chunk lies inside one group
                    if (it * BK + 8 * c >= next_start) advance();
                }
                uint32_t o[4];
                if constexpr (kTable) {
                    lookup8(w[c], tlo, thi, o);
                } else {
                    float f[8];
                    chunk_codes<BITS>(w, c, f);
#pragma unroll
                    for (int p = 0; p < 4; ++p)
                        o[p] = bf16x2_rne(mul2(sub2(pk2(f[2 * p], f[2 * p + 1]), off2), s2));
                }
                sts128_u(row + ((c ^ (n & 7)) << 4), make_uint4(o[0], o[1], o[2], o[3]));
            }
            fence_async_smem();
            mbar_arrive(&bars->bfull[b]);
            // every word read from the slot has been used (so its load has
            // completed) before the slot may be refilled; released right after
            // the loads were issued, 8-bit rows (four-way bank conflicts, longer
            // loads) read words of the next refill
            mbar_arrive(&bars->pempty[ps]);
        }
        // ------------------------------------------------ drain: TMEM -> Y
        if (ok && mbar_wait(&bars->acc_full, 0, abort)) {
            tc_fence_after();
            const int q = warp & 3;           // TMEM lane quarter of this warp
            const int h = (warp - 2) >> 2;    // accumulator (token half)
            const int t = t0 + h * 128 + 32 * q + lane;
            float* yrow = Y + static_cast<int64_t>(t) * ldy;
#pragma unroll 1
            for (int c = 0; c < TN / 32; ++c) {
                float v[32];
                tmem_ld32(tmem + (static_cast<uint32_t>(32 * q) << 16) + h * TN + c * 32, v);
                const int nb = n0 + 32 * c;
                if (t < n_tok) {
                    if (nb + 32 <= d_row && (reinterpret_cast<uintptr_t>(yrow + nb) & 15) == 0) {
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            *reinterpret_cast<float4*>(yrow + nb + 4 * j) =
                                make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (nb + j < d_row) yrow[nb + j] = v[j];
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, kTmemCols);
    if (threadIdx.x == 0 && bars->abort) report(status, GPTQ_ERR_TIMEOUT);
}

// Xq[t][k] = X[t][perm[k]] (bf16, row pitch K); perm entries outside [0, K)
// are read as k.
// Xq[t][k] = X[t][perm[k]] (bf16 bits, quantization order), one token row per
// CTA at a time.  The row is first copied into shared memory with 16-byte
// loads when X's rows allow it (kStaged), so that HBM sees it read once and
// in order whatever the permutation; the permuted row leaves in 16-byte
// stores of 8 values (K is a multiple of 64 and Xq's rows are contiguous).
// Rows too wide for shared memory read their values through L1 instead.
constexpr int kGatherThreads = 256;
constexpr int kGatherSmemMax = 160 * 1024;

template <bool kStaged, bool kVecLoad>
__global__ void __launch_bounds__(kGatherThreads)
gather_bf16_kernel(const uint16_t* __restrict__ X, int64_t ldx, int64_t n_tok, int K,
                   const int32_t* __restrict__ perm, uint16_t* __restrict__ Xq) {
    extern __shared__ __align__(16) uint16_t row_s[];
    const int chunks = K / 8;
    for (int64_t t = blockIdx.x; t < n_tok; t += gridDim.x) {
        const uint16_t* xr = X + t * ldx;
        if constexpr (kStaged) {
            if constexpr (kVecLoad) {
                const uint4* src = reinterpret_cast<const uint4*>(xr);
                for (int c = threadIdx.x; c < chunks; c += kGatherThreads)
                    reinterpret_cast<uint4*>(row_s)[c] = __ldg(src + c);
            } else {
                for (int k = threadIdx.x; k < K; k += kGatherThreads) row_s[k] = xr[k];
            }
            __syncthreads();
        }
        uint4* dst = reinterpret_cast<uint4*>(Xq + t * static_cast<int64_t>(K));
        for (int c = threadIdx.x; c < chunks; c += kGatherThreads) {
            uint32_t v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int k = c * 8 + i;
                int col = perm != nullptr ? __ldg(perm + k) : k;
                if (col < 0 || col >= K) col = k;
                v[i] = kStaged ? row_s[col] : __ldg(xr + col);
            }
            dst[c] = make_uint4(v[0] | (v[1] << 16), v[2] | (v[3] << 16), v[4] | (v[5] << 16),
                                v[6] | (v[7] << 16));
        }
        if constexpr (kStaged) __syncthreads();  // the row buffer is refilled next
    }
}

// The same gather for aligned rows that fit, pipelined: the permutation is
// staged once per CTA in shared memory as 16-bit indices, and each CTA copies
// its next token row into the second of two row buffers (cp.async, 16 bytes
// per copy, no registers) while it gathers the current one, so HBM streams
// rows in and out while the shared-memory gathers run.  The first form read
// perm through L2 for every value, one dependent read after another.
constexpr int kPipeThreads = 512;

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)),
                 "l"(gsrc)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_older() {
    asm volatile("cp.async.wait_group 1;" ::: "memory");
}

__global__ void __launch_bounds__(kPipeThreads)
gather_bf16_piped_kernel(const uint16_t* __restrict__ X, int64_t ldx, int64_t n_tok, int K,
                         const int32_t* __restrict__ perm, uint16_t* __restrict__ Xq) {
    extern __shared__ __align__(16) uint16_t gs[];
    uint16_t* idx = gs;            // [K] source column of each position
    uint16_t* rows = gs + K;       // [2][K] token rows
    const int chunks = K / 8;
    for (int k = threadIdx.x; k < K; k += kPipeThreads) {
        int col = perm != nullptr ? perm[k] : k;
        if (col < 0 || col >= K) col = k;
        idx[k] = static_cast<uint16_t>(col);
    }
    auto fetch = [&](int64_t t, int buf) {
        if (t < n_tok) {
            const uint16_t* xr = X + t * ldx;
            uint16_t* dst = rows + buf * K;
            for (int c = threadIdx.x; c < chunks; c += kPipeThreads)
                cp_async16(dst + 8 * c, xr + 8 * c);
        }
        cp_async_commit();  // an empty group past the last row keeps the count
    };
    int buf = 0;
    fetch(blockIdx.x, 0);
    for (int64_t t = blockIdx.x; t < n_tok; t += gridDim.x) {
        fetch(t + gridDim.x, buf ^ 1);
        cp_async_wait_older();  // this thread's copies of row t have landed
        __syncthreads();        // ... and everyone's (and idx is written)
        const uint16_t* row = rows + buf * K;
        uint4* dst = reinterpret_cast<uint4*>(Xq + t * static_cast<int64_t>(K));
        for (int c = threadIdx.x; c < chunks; c += kPipeThreads) {
            const uint4 ix = reinterpret_cast<const uint4*>(idx)[c];
            const uint32_t iw[4] = {ix.x, ix.y, ix.z, ix.w};
            uint32_t o[4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
                o[j] = static_cast<uint32_t>(row[iw[j] & 0xFFFFu]) |
                       (static_cast<uint32_t>(row[iw[j] >> 16]) << 16);
            dst[c] = make_uint4(o[0], o[1], o[2], o[3]);
        }
        __syncthreads();  // row buffer `buf` is refilled two rows later
        buf ^= 1;
    }
    asm volatile("cp.async.wait_all;" ::: "memory");  // no copy outlives the CTA
}

cudaError_t launch_gather(const uint16_t* X, int64_t ldx, int64_t n_tok, int K,
                          const int32_t* perm, uint16_t* Xq, cudaStream_t stream) {
    const size_t smem = static_cast<size_t>(K) * 2;
    const bool vec = (ldx % 8) == 0 && (reinterpret_cast<uintptr_t>(X) & 15) == 0;
    const size_t piped = 3 * smem;  // indices and two rows
    if (vec && piped <= 227 * 1024 && K <= 65536) {
        auto kern = gather_bf16_piped_kernel;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(piped));
        if (e != cudaSuccess) return e;
        const int grid = static_cast<int>(n_tok < num_sms() ? n_tok : num_sms());
        kern<<<grid, kPipeThreads, piped, stream>>>(X, ldx, n_tok, K, perm, Xq);
        return cudaGetLastError();
    }
    if (smem > kGatherSmemMax) {
        const int grid = static_cast<int>(n_tok < 8 * num_sms() ? n_tok : 8 * num_sms());
        gather_bf16_kernel<false, false><<<grid, kGatherThreads, 0, stream>>>(X, ldx, n_tok, K,
                                                                              perm, Xq);
        return cudaGetLastError();
    }
    auto kern = vec ? gather_bf16_kernel<true, true> : gather_bf16_kernel<true, false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kGatherThreads, smem);
    if (e != cudaSuccess) return e;
    const int64_t resident = static_cast<int64_t>(per_sm > 0 ? per_sm : 1) * num_sms();
    const int grid = static_cast<int>(n_tok < resident ? n_tok : resident);
    kern<<<grid, kGatherThreads, smem, stream>>>(X, ldx, n_tok, K, perm, Xq);
    return cudaGetLastError();
}

template <int BITS>
cudaError_t launch_bits(const CUtensorMap& ta, const CUtensorMap& tp, const float* scales,
                        const int32_t* zeros, float* Y, int64_t ldy, int n_tok, int d_row, int K,
                        int g, int32_t* status, cudaStream_t stream) {
    auto kern = (g % BK == 0) ? dequant_gemm_kernel<BITS, true> : dequant_gemm_kernel<BITS, false>;
    constexpr int kSmemBytes = Geom<BITS>::kSmemBytes;
    static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    const dim3 grid((d_row + TN - 1) / TN, (n_tok + TM - 1) / TM);
    kern<<<grid, kThreads, kSmemBytes, stream>>>(ta, tp, scales, zeros, Y, ldy, n_tok, d_row, K, g,
                                                 status);
    return cudaGetLastError();
}

}  // namespace

size_t dequant_gemm_workspace_bytes(int64_t n_tok, int64_t d_col) {
    return ((static_cast<size_t>(n_tok) * d_col * 2 + 255) / 256) * 256;
}

gptq_status launch_dequant_gemm(const uint16_t* X, int64_t n_tok, int64_t d_col, int64_t ldx,
                                const uint32_t* packed, const float* scales, const int32_t* zeros,
                                const int32_t* perm, int64_t d_row, int bits, int group, float* Y,
                                int64_t ldy, int32_t* status, void* ws, cudaStream_t stream) {
    const int K = static_cast<int>(d_col);
    const int g = (group == -1 || group > K) ? K : group;
    const uint16_t* A = X;
    int64_t lda = ldx;
    int64_t launches = 1;
    if (perm != nullptr || (ldx % 8) != 0 || (reinterpret_cast<uintptr_t>(X) & 15) != 0) {
        uint16_t* Xq = static_cast<uint16_t*>(ws);
        if (launch_gather(X, ldx, n_tok, K, perm, Xq, stream) != cudaSuccess)
            return GPTQ_ERR_CUDA;
        A = Xq;
        lda = d_col;
        ++launches;
    }
    CUtensorMap ta, tp;
    const int64_t P = d_col * bits / 32;  // packed words per row
    // the packed words move as raw 32-bit elements (the map's fp32 type only
    // sizes them; nothing converts)
    if (!make_tmap_2d(&ta, true, A, d_col, n_tok, lda, BK, TM, Swz::k128) ||
        !make_tmap_2d(&tp, false, packed, P, d_row, P, BK * bits / 32, TN, Swz::kNone))
        return GPTQ_ERR_INVALID_ARG;
    cudaError_t e;
    const int nt = static_cast<int>(n_tok), nr = static_cast<int>(d_row);
    switch (bits) {
        case 2: e = launch_bits<2>(ta, tp, scales, zeros, Y, ldy, nt, nr, K, g, status, stream); break;
        case 4: e = launch_bits<4>(ta, tp, scales, zeros, Y, ldy, nt, nr, K, g, status, stream); break;
        case 8: e = launch_bits<8>(ta, tp, scales, zeros, Y, ldy, nt, nr, K, g, status, stream); break;
        default: return GPTQ_ERR_UNSUPPORTED;
    }
    if (e != cudaSuccess) return GPTQ_ERR_CUDA;
    count_launches(launches);
    return GPTQ_OK;
}

}  // namespace gptq
