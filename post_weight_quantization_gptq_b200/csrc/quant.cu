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
// the group's current min / max (range widened to contain 0, or the group's
// own range with the pure min-max option).
//
// Kernels:
//  permute_rows_kernel  W[:, k] <- W[:, perm[k]] (0 for dead columns), in place
//  block_quant_kernel   one 128-column block: row-parallel, 8 lanes per row,
//                       the block's U in shared memory, the column loop
//                       sequential with one shuffle per column
//  lazy update          W[:, c1:] -= Err * U[c0:c1, c1:] on the tensor cores
//                       (3xTF32 tcgen05 GEMM, fp32-accurate)
#include <cmath>
#include <tuple>
#include <type_traits>
#include <vector>

#include "common.cuh"
#include "gemm_tf32x3.cuh"
#include "kernels.h"

namespace gptq {
namespace {

constexpr int kBlock = 128;       // columns per block (the only supported block size)
// Warps per column-walk CTA (kWarpsSmall rows * 4 each at 8 lanes per row).
// Four (16 rows) while the layer's CTAs fit on the GPU at once (three per SM
// by shared memory: up to 7104 rows); seven (28 rows) beyond, so that larger
// layers still walk a block in one wave (measured at 8192 x 8192:
// quantize_layer 5.25 -> 4.51 ms; at 4096 rows seven warps are 4 % slower
// than four).
constexpr int kWarpsSmall = 4, kWarpsLarge = 7;
// Lanes per row of the column walk (each owns 32 / kWalkLanes columns of every
// 32-column chunk).  8 lanes: 4096 rows give ~7 warps per SM.  4 lanes halve
// the per-column work replicated on every lane of a row (quantizing the
// current column, the shuffles) for twice the feedback FMAs per lane, but
// leave one warp per SM sub-partition: measured slower (quantize_layer 1.287
// against 1.207 ms at 4096 x 4096, 5.31 against 5.08 ms at 4096 x 11008,
// interleaved A/B, identical codes).
constexpr int kWalkLanes = 8;
template <int L, int NW>
struct WalkShape {
    static_assert(NW * 32 >= kBlock, "block_quant_kernel: a thread per column of the U block");
    static constexpr int kCols = 32 / L;            // columns per lane per chunk
    static constexpr int kRowsPerWarp = 32 / L;
    static constexpr int kRowsPerCta = kRowsPerWarp * NW;
};

// ------------------------------------------------------------------------
// A perm entry outside [0, d) (the caller passed something other than
// gptq_prepare_hinv's output) is reported as GPTQ_ERR_INVALID_ARG and read as
// the column's own index, so no access leaves the row.
__global__ void permute_rows_kernel(float* __restrict__ W, int64_t r, int64_t d, int64_t ldw,
                                    const int32_t* __restrict__ perm,
                                    const uint8_t* __restrict__ dead, int32_t* status) {
    extern __shared__ float rowbuf[];
    pdl_trigger();
    for (int64_t row = blockIdx.x; row < r; row += gridDim.x) {
        float* w = W + row * ldw;
        for (int64_t k = threadIdx.x; k < d; k += blockDim.x) rowbuf[k] = w[k];
        __syncthreads();
        for (int64_t k = threadIdx.x; k < d; k += blockDim.x) {
            int64_t src = perm[k];
            if (src < 0 || src >= d) {
                if (row == blockIdx.x) report(status, GPTQ_ERR_INVALID_ARG);
                src = k;
            }
            w[k] = dead[src] ? 0.f : rowbuf[src];
        }
        __syncthreads();
    }
}

// U's lo parts for the lazy update's pre-split operand: U_lo = U - trunc13(U)
// elementwise, from the diagonal's 4-column group to the end of each row (U is
// d x d, contiguous; the update reads only rows of U right of their diagonal
// block, so the rest of U_lo is left unwritten).  Rows along grid y, four
// columns per thread (d is a multiple of 4).
__global__ void u_lo_kernel(const float* __restrict__ U, int64_t d, float* __restrict__ U_lo) {
    for (int64_t i = blockIdx.y; i < d; i += gridDim.y) {
        const float4* src = reinterpret_cast<const float4*>(U + i * d);
        float4* dst = reinterpret_cast<float4*>(U_lo + i * d);
        for (int64_t q = (i >> 2) + blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
             q < d / 4; q += static_cast<int64_t>(gridDim.x) * blockDim.x) {
            const float4 u = src[q];
            dst[q] = make_float4(g3::tf32_rest(u.x), g3::tf32_rest(u.y), g3::tf32_rest(u.z),
                                 g3::tf32_rest(u.w));
        }
    }
}

// Register layout: the block's 128 columns form four 32-column chunks; in
// every chunk lane l of a row's L-lane group owns the C = 32 / L columns
// C l .. C l + C - 1, so the lanes of a row read one 128-byte row segment of
// the U block per C / 4 vector loads without bank conflicts.  A lane keeps the
// chunk being quantized in cur[C] and the later chunks in nxt[3 C]; after each
// chunk the window rotates, so every register index below is a compile-time
// constant while the chunk loop stays rolled (the code fits the instruction
// cache).
//
// The column being quantized is held by every lane of the group (wcur): a
// lane derives columns j+1 and j+2 from values shuffled from their owners two
// steps earlier, applying the same FMAs the owners apply (so the copies are
// bit-identical to the owners' registers).  The shuffle then has a whole step
// to land, and the column-to-column chain is FMA -> quantize -> FMA.
struct GroupParams {
    float s, inv_s, zf, hi;  // scale, 1/scale, zero point, maxq - zero point
};

// Scale / zero point of the group [c0 + j, c0 + j + g) of this row from its
// current weights: the group's columns in this block (cur: chunk m, nxt:
// chunks m+1..3) plus, for groups wider than the block, the later columns in
// W (which already hold every earlier block's feedback).  Default: range
// widened to contain 0.  pure: the group's own [min, max] (the zero point may
// fall outside [0, maxq]); a constant group, or one whose real zero point
// lies more than 2^20 levels away (w / s then has an fp32 ulp of 1/16 level
// or more), takes the widened range.  An all-zero group gets the range
// [-1, 1] (zero point exactly 2^(bits-1)).
template <int L, int C = 32 / L>
__device__ __forceinline__ GroupParams group_params(const float (&cur)[C], const float (&nxt)[3 * C],
                                                    int m, int jj, int l, int g, int bw,
                                                    const float* __restrict__ wrow, int64_t c0,
                                                    int64_t d, bool live, int bits, bool pure,
                                                    const uint8_t* __restrict__ dead_mask) {
    const int j = 32 * m + jj;
    float lo = pure ? INFINITY : 0.f, hi = pure ? -INFINITY : 0.f;
#pragma unroll
    for (int i = 0; i < C; ++i) {
        const int c = 32 * m + C * l + i;
        if (c >= j && c < j + g && c < bw) {
            lo = fminf(lo, cur[i]);
            hi = fmaxf(hi, cur[i]);
        }
    }
#pragma unroll
    for (int s = 0; s < 3; ++s)
#pragma unroll
        for (int i = 0; i < C; ++i) {
            const int c = 32 * (m + 1 + s) + C * l + i;
            if (m + 1 + s < 4 && c < j + g && c < bw) {
                lo = fminf(lo, nxt[C * s + i]);
                hi = fmaxf(hi, nxt[C * s + i]);
            }
        }
    const int64_t gend = (c0 + j + g < d) ? c0 + j + g : d;
    if (live && gend > c0 + bw) {
        for (int64_t c = c0 + bw + l; c < gend; c += L) {
            const float v = (dead_mask != nullptr && dead_mask[c]) ? 0.f : wrow[c];
            lo = fminf(lo, v);
            hi = fmaxf(hi, v);
        }
    }
#pragma unroll
    for (int o = 1; o < L; o <<= 1) {
        lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
        hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    const float maxq = static_cast<float>((1 << bits) - 1);
    if (pure) {
        bool widen = !(hi > lo);
        if (!widen) widen = fabsf(lo / ((hi - lo) / maxq)) > 1048576.f;
        if (widen) {
            lo = fminf(lo, 0.f);
            hi = fmaxf(hi, 0.f);
        }
    }
    GroupParams p;
    if (hi == lo) {
        p.s = 2.f / maxq;
        p.zf = static_cast<float>(1 << (bits - 1));
    } else {
        p.s = (hi - lo) / maxq;
        p.zf = rintf(-lo / p.s);
    }
    p.inv_s = 1.f / p.s;
    p.hi = maxq - p.zf;
    return p;
}

// Value of column 32 m + k (3 <= k < 35) of this row, as held by its owner
// lane: the current chunk for k < 32, the next one after; ii = k mod C is a
// compile-time register index.
template <int C>
__device__ __forceinline__ float owner_value(int k, int ii, const float (&cur)[C],
                                             const float (&nxt)[3 * C], int gbase) {
    const float v = (k < 32) ? cur[ii] : nxt[ii];
    return __shfl_sync(0xffffffffu, v, gbase + ((k & 31) / C));
}

// Round half to even of |x| <= 2^22 by adding and removing 1.5 * 2^23 (its
// ulp is 1, so the first add rounds x to an integer under the IEEE
// round-to-nearest-even mode; both adds are explicit _rn, never contracted).
__device__ __forceinline__ float round_even(float x) {
    return __fadd_rn(__fadd_rn(x, 12582912.f), -12582912.f);
}

template <int L,               // lanes per row
          int NW,              // warps per CTA
          bool kSmallGroup,  // group_size < 32: groups start inside a chunk
          bool kFull>        // a full 128-column block (no column guard)
__global__ void __launch_bounds__(NW * 32, 1)
    block_quant_kernel(const __grid_constant__ CUtensorMap tmu, float* __restrict__ W, int64_t r,
                       int64_t d, int64_t ldw, int64_t c0, int bw, int bits, int g, int pure,
                       uint8_t* __restrict__ codes, float* __restrict__ scales,
                       int32_t* __restrict__ zeros, float* __restrict__ err_out,
                       float* __restrict__ err_lo_out, int64_t err_ld,
                       const uint8_t* __restrict__ dead_mask, int32_t* status) {
    // err_lo_out (may be null): each error's part below tf32 precision, the
    // lo operand of the lazy update's truncating 3xTF32 split, stored beside
    // the errors so that the update need not split them
    constexpr int C = WalkShape<L, NW>::kCols;
    constexpr int C4 = C / 4;  // float4s per lane per chunk
    extern __shared__ uint8_t smem_raw[];
    float* smem = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
    float* Us = smem;                      // [kBlock][kBlock]: U's diagonal block, strict upper part kept
    float* dinv = smem + kBlock * kBlock;  // 1 / U_jj
    __shared__ __align__(8) uint64_t bar;
    __shared__ int ok;
    const int tid = threadIdx.x;
    pdl_trigger();
    // U is an input of the whole call that none of its kernels writes, so
    // its diagonal block is fetched and prepared before waiting for the
    // previous kernel (which may still be updating W)
    if (tid == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
        mbar_arrive_expect_tx(&bar, kBlock * kBlock * 4);
        tma_load_2d(Us, &tmu, &bar, static_cast<int>(c0), static_cast<int>(c0));
        volatile int no_abort = 0;
        ok = mbar_wait(&bar, 0, &no_abort) ? 1 : 0;
        if (!ok) report(status, GPTQ_ERR_TIMEOUT);
    }
    __syncthreads();
    if (!ok) return;
    // 1 / U_jj (thread j), then the block is cleared at and below its
    // diagonal, float4 by float4 spread over all threads
    const float ujj = tid < kBlock ? Us[tid * kBlock + tid] : 1.f;
    __syncthreads();
    for (int q = tid; q < kBlock * kBlock / 4; q += NW * 32) {
        const int i = q >> 5, c = (q & 31) * 4;
        if (c > i) continue;
        float* u4 = Us + i * kBlock + c;
        if (c + 3 <= i) {
            *reinterpret_cast<float4*>(u4) = make_float4(0.f, 0.f, 0.f, 0.f);
        } else {
            for (int t = 0; c + t <= i; ++t) u4[t] = 0.f;
        }
    }
    if (tid < kBlock) dinv[tid] = (tid < bw) ? 1.f / ujj : 0.f;
    pdl_wait();

    const int lane = tid & 31;
    const int l = lane % L;
    const int gbase = lane - l;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * WalkShape<L, NW>::kRowsPerCta +
                        (tid >> 5) * WalkShape<L, NW>::kRowsPerWarp + lane / L;
    const bool live = row < r;
    float* wrow = W + (live ? row : 0) * ldw;
    // float4 access to W needs 16-byte aligned rows (base and pitch); a
    // lane's C codes go out as one C-byte store when codes' rows allow it
    const bool vec = (ldw & 3) == 0 && bw == kBlock && (reinterpret_cast<uintptr_t>(W) & 15) == 0;
    const bool vec_codes = vec && (d % C) == 0 && (reinterpret_cast<uintptr_t>(codes) % C) == 0;

    // the row's slice of the block (in flight while the U block arrives)
    float cur[C], nxt[3 * C];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        float v[C];
        if (live && vec) {
#pragma unroll
            for (int q = 0; q < C4; ++q) {
                const float4 t = *reinterpret_cast<const float4*>(wrow + c0 + 32 * m + C * l + 4 * q);
                v[4 * q] = t.x; v[4 * q + 1] = t.y; v[4 * q + 2] = t.z; v[4 * q + 3] = t.w;
            }
        } else {
#pragma unroll
            for (int i = 0; i < C; ++i) {
                const int c = 32 * m + C * l + i;
                v[i] = (live && c < bw) ? wrow[c0 + c] : 0.f;
            }
        }
#pragma unroll
        for (int i = 0; i < C; ++i) {
            // columns whose H diagonal is 0 quantize zero weights (in the
            // permuted form the permutation pass has zeroed them already)
            if (dead_mask != nullptr && 32 * m + C * l + i < bw && dead_mask[c0 + 32 * m + C * l + i])
                v[i] = 0.f;
            if (m == 0) cur[i] = v[i];
            else nxt[C * (m - 1) + i] = v[i];
        }
    }
    GroupParams gp{1.f, 1.f, 0.f, 0.f};
    if (live && (c0 % g) != 0) {
        // this block continues a group opened by an earlier block (group
        // size > block): take that group's scale and zero point
        const int64_t grp = c0 / g;
        gp.s = scales[grp * r + row];
        gp.zf = static_cast<float>(zeros[grp * r + row]);
        gp.inv_s = 1.f / gp.s;
        gp.hi = static_cast<float>((1 << bits) - 1) - gp.zf;
    }

    __syncthreads();  // the prepared U block and 1 / U_jj

    // columns 0, 1, 2 for every lane of the group; afterwards, at the start of
    // step j: wcur = column j (final), t1 = column j+1 after the feedback of
    // columns < j, t2 = column j+2 after the feedback of columns < j
    float wcur = __shfl_sync(0xffffffffu, cur[0], gbase);
    float t1 = __shfl_sync(0xffffffffu, cur[1], gbase);
    float t2 = __shfl_sync(0xffffffffu, cur[2], gbase);

    // one 32-column chunk; m is a compile-time constant in each of the four
    // instantiations, so the feedback into the later chunks (nxt) is exactly
    // the live part: 3, 2, 1, 0 chunks
    auto walk_chunk = [&](auto mc) {
        constexpr int m = decltype(mc)::value;
        if (!kSmallGroup && ((c0 + 32 * m) % g) == 0) {
            gp = group_params<L>(cur, nxt, m, 0, l, g, bw, wrow, c0, d, live, bits, pure != 0,
                                 dead_mask);
            if (live && l == 0) {
                const int64_t grp = (c0 + 32 * m) / g;
                scales[grp * r + row] = gp.s;
                zeros[grp * r + row] = static_cast<int32_t>(gp.zf);
            }
        }
        float ev[C];
        uint32_t qv[C];
#pragma unroll
        for (int i = 0; i < C; ++i) {
            ev[i] = 0.f;
            qv[i] = 0u;
        }
        // L rolled steps (one per owner lane) of C unrolled columns: register
        // indices stay compile-time while the loop body stays small
#pragma unroll 1
        for (int jo = 0; jo < L; ++jo) {
#pragma unroll
            for (int ii = 0; ii < C; ++ii) {
                const int jj = C * jo + ii;
                const int j = 32 * m + jj;
                if (kFull || j < bw) {
                    if (kSmallGroup && ((c0 + j) % g) == 0) {
                        gp = group_params<L>(cur, nxt, m, jj, l, g, bw, wrow, c0, d, live, bits,
                                             pure != 0, dead_mask);
                        if (live && l == 0) {
                            const int64_t grp = (c0 + j) / g;
                            scales[grp * r + row] = gp.s;
                            zeros[grp * r + row] = static_cast<int32_t>(gp.zf);
                        }
                    }
                    const float* urow = Us + j * kBlock;
                    const float dj = dinv[j];
                    const float u1 = urow[(j + 1) & (kBlock - 1)];
                    const float u2 = urow[(j + 2) & (kBlock - 1)];
                    // q = clamp(rint(w / s) + z, 0, maxq) = rint(clamp(w / s, -z, maxq - z)) + z
                    // (z and maxq are integers); e = (w - s (q - z)) / U_jj
                    const float cq = round_even(fminf(fmaxf(wcur * gp.inv_s, -gp.zf), gp.hi));
                    const float e = fmaf(-(gp.s * dj), cq, wcur * dj);
                    const bool mine = l == jo;
                    qv[ii] = mine ? static_cast<uint32_t>(cq + gp.zf) : qv[ii];
                    ev[ii] = mine ? e : ev[ii];
                    // columns j+1 and j+2 for every lane: the owners' own updates, replicated
                    wcur = fmaf(-e, u1, t1);
                    t1 = fmaf(-e, u2, t2);
                    // feedback into this block's later columns (U row j is zero
                    // at and left of the diagonal, so earlier columns are untouched)
                    const float4* urow4 = reinterpret_cast<const float4*>(urow);
#pragma unroll
                    for (int q = 0; q < C4; ++q) {
                        const float4 u = urow4[8 * m + C4 * l + q];
                        cur[4 * q + 0] = fmaf(-e, u.x, cur[4 * q + 0]);
                        cur[4 * q + 1] = fmaf(-e, u.y, cur[4 * q + 1]);
                        cur[4 * q + 2] = fmaf(-e, u.z, cur[4 * q + 2]);
                        cur[4 * q + 3] = fmaf(-e, u.w, cur[4 * q + 3]);
                    }
#pragma unroll
                    for (int s = 0; s < 3 - m; ++s)
#pragma unroll
                        for (int q = 0; q < C4; ++q) {
                            const float4 u = urow4[8 * (m + 1 + s) + C4 * l + q];
                            nxt[C * s + 4 * q + 0] = fmaf(-e, u.x, nxt[C * s + 4 * q + 0]);
                            nxt[C * s + 4 * q + 1] = fmaf(-e, u.y, nxt[C * s + 4 * q + 1]);
                            nxt[C * s + 4 * q + 2] = fmaf(-e, u.z, nxt[C * s + 4 * q + 2]);
                            nxt[C * s + 4 * q + 3] = fmaf(-e, u.w, nxt[C * s + 4 * q + 3]);
                        }
                    // column j+3 as of this step (used one step later)
                    t2 = owner_value<C>(jj + 3, (ii + 3) % C, cur, nxt, gbase);
                }
            }
        }
        // chunk m done: pre-quantization weights, scaled errors, codes
        if (live) {
            const int cb = 32 * m + C * l;
#pragma unroll
            for (int q = 0; q < C4; ++q)
                *reinterpret_cast<float4*>(err_out + row * err_ld + cb + 4 * q) =
                    make_float4(ev[4 * q], ev[4 * q + 1], ev[4 * q + 2], ev[4 * q + 3]);
            if (err_lo_out != nullptr) {
#pragma unroll
                for (int q = 0; q < C4; ++q)
                    *reinterpret_cast<float4*>(err_lo_out + row * err_ld + cb + 4 * q) =
                        make_float4(g3::tf32_rest(ev[4 * q]), g3::tf32_rest(ev[4 * q + 1]),
                                    g3::tf32_rest(ev[4 * q + 2]), g3::tf32_rest(ev[4 * q + 3]));
            }
            if (vec) {
#pragma unroll
                for (int q = 0; q < C4; ++q)
                    *reinterpret_cast<float4*>(wrow + c0 + cb + 4 * q) =
                        make_float4(cur[4 * q], cur[4 * q + 1], cur[4 * q + 2], cur[4 * q + 3]);
            }
            if (vec_codes) {
                uint32_t word[C4];
#pragma unroll
                for (int q = 0; q < C4; ++q)
                    word[q] = qv[4 * q] | (qv[4 * q + 1] << 8) | (qv[4 * q + 2] << 16) |
                              (qv[4 * q + 3] << 24);
                if constexpr (C4 == 2)
                    *reinterpret_cast<uint2*>(codes + row * d + c0 + cb) = make_uint2(word[0], word[1]);
                else
                    *reinterpret_cast<uint32_t*>(codes + row * d + c0 + cb) = word[0];
            }
#pragma unroll
            for (int i = 0; i < C; ++i) {
                const int c = cb + i;
                if (c < bw) {
                    if (!vec) wrow[c0 + c] = cur[i];
                    if (!vec_codes) codes[row * d + c0 + c] = static_cast<uint8_t>(qv[i]);
                }
            }
        }
        // rotate the window
#pragma unroll
        for (int i = 0; i < C; ++i) {
            cur[i] = nxt[i];
            nxt[i] = nxt[C + i];
            nxt[C + i] = nxt[2 * C + i];
            nxt[2 * C + i] = 0.f;
        }
    };
    walk_chunk(std::integral_constant<int, 0>{});
    if (kFull || bw > 32) walk_chunk(std::integral_constant<int, 1>{});
    if (kFull || bw > 64) walk_chunk(std::integral_constant<int, 2>{});
    if (kFull || bw > 96) walk_chunk(std::integral_constant<int, 3>{});
}

// ------------------------------------------------------------------------
// Lazy update of the columns [c1, c1 + n) from the errors of the columns
// [k0, k0 + klen):  W[:, c1:] -= Err[:, k0:k0+klen] U[k0:k0+klen, c1:]
// as 128 x 128 output tiles of the 3xTF32 GEMM: A = Err (K-major, held in the
// error buffer from column ke), B = U's rows (MN-major).
struct LazySched {
    static constexpr bool kRmw = true;
    float* W;
    int64_t ldw;
    int r, d, c1, mt, ke, k0, nk;
    __device__ g3::Job job(int t) const {
        return {128 * (t % mt), c1 + 128 * (t / mt), ke, k0, nk};
    }
    __device__ float* dst(const g3::Job& jb, int row) const {
        const int rr = jb.m0 + row;
        return rr < r ? W + static_cast<int64_t>(rr) * ldw + jb.n0 : nullptr;
    }
    __device__ int ncols(const g3::Job& jb, int) const {
        return d - jb.n0 < g3::BN ? d - jb.n0 : g3::BN;
    }
    __device__ int nreadable(const g3::Job& jb) const { return ncols(jb, 0); }
};

}  // namespace

namespace {

constexpr int kMaxDefer = 8;  // blocks whose errors the lazy update may defer

int64_t num_blocks(int64_t d_col) { return (d_col + kBlock - 1) / kBlock; }

// Host model of the deferred schedule (see launch_quantize): applied[b] =
// the number of leading blocks whose feedback block b has received.  Checks
// that every block, and every later block its group reads when the group
// starts there, is complete when it is quantized.
bool schedule_valid(int nb, int defer, int g_blocks) {
    std::vector<int> applied(nb, 0);
    bool ok = true;
    auto gemm = [&](int a, int c, int e) {
        for (int b = c; b < e; ++b) {
            ok = ok && applied[b] == a;
            applied[b] = c;
        }
    };
    auto quant = [&](int b) {
        ok = ok && applied[b] == b;
        if (g_blocks > 1 && b % g_blocks == 0)
            for (int x = b + 1; x < nb && x < b + g_blocks; ++x) ok = ok && applied[x] == b;
    };
    // recursion on [lo, hi): quantize [lo, mid), update [mid, hi), quantize [mid, hi)
    for (int s0 = 0; s0 < nb; s0 += defer) {
        const int s1 = s0 + defer < nb ? s0 + defer : nb;
        std::vector<std::tuple<int, int, int>> stack{{s0, s1, 0}};
        while (!stack.empty()) {
            auto [lo, hi, state] = stack.back();
            stack.pop_back();
            if (hi - lo == 1) {
                quant(lo);
                continue;
            }
            int half = 1;
            while (2 * half < hi - lo) half *= 2;
            const int mid = lo + half;
            if (state == 0) {
                stack.push_back({lo, hi, 1});
                stack.push_back({lo, mid, 0});
            } else {
                gemm(lo, mid, hi);
                stack.push_back({mid, hi, 0});
            }
        }
        if (s1 < nb) gemm(s0, s1, nb);
    }
    return ok;
}

}  // namespace

namespace {
size_t round256(size_t x) { return (x + 255) / 256 * 256; }

// Workspace layout of the column walk: the deferred errors (d_row x 128 per
// block of the run), then -- for the pre-split lazy update -- the errors' lo
// parts in the same layout and U's lo parts (d_col x d_col).
struct QuantWs {
    size_t err, err_lo, u_lo, total;
};
QuantWs quant_ws(int64_t d_row, int64_t d_col, int defer) {
    QuantWs w;
    const size_t e = round256(static_cast<size_t>(d_row) * kBlock * defer * sizeof(float));
    w.err = 0;
    w.err_lo = e;
    w.u_lo = 2 * e;
    w.total = 2 * e + round256(static_cast<size_t>(d_col) * d_col * sizeof(float));
    return w;
}
}  // namespace

size_t quant_workspace_bytes(int64_t d_row, int64_t d_col, int block) {
    (void)block;
    const int64_t nb = num_blocks(d_col);
    const int defer = static_cast<int>(nb < kMaxDefer ? nb : kMaxDefer);
    return quant_ws(d_row, d_col, defer).total;
}

size_t quant_min_workspace_bytes(int64_t d_row, int block) {
    return ((static_cast<size_t>(d_row) * block * sizeof(float) + 255) / 256) * 256;
}

// The column walk.  Blocks of 128 columns are quantized in order; the lazy
// update of the pages' batched form is deferred and regrouped so that most of
// its arithmetic runs as long-K products: within a run of up to kMaxDefer
// blocks (as many as the workspace holds), blocks [lo, hi) are handled as
// [lo, mid) -> W[:, mid:hi] -= Err[:, lo:mid] U[lo:mid, mid:hi] -> [mid, hi),
// recursively; after the run, one product applies its errors to every later
// column.  Every block still receives the feedback of every earlier block
// before it is quantized (the same sums, in another order).  Groups wider than
// a block must find their later columns complete when the group starts; the
// host checks the schedule and shortens the runs (down to the per-block
// form) when a group size does not fit it.
gptq_status launch_quantize(float* W, int64_t d_row, int64_t d_col, int64_t ldw, const float* U,
                            const int32_t* perm, const uint8_t* dead, int desc_act, int bits,
                            int group, int block, int pure_minmax, uint8_t* codes, float* scales,
                            int32_t* zeros, int32_t* status, void* ws, size_t ws_bytes,
                            cudaStream_t stream) {
    if (block != kBlock) return GPTQ_ERR_UNSUPPORTED;
    const int pure = pure_minmax != 0 ? 1 : 0;
    const int g = (group == -1 || group > d_col) ? static_cast<int>(d_col) : group;
    const int nb = static_cast<int>(num_blocks(d_col));
    const int defer_max = nb < kMaxDefer ? nb : kMaxDefer;
    // the lazy update reads pre-split operands when the workspace holds the
    // full layout (and W's rows can be a tensor map: the fallback drain keeps
    // the in-kernel split); the lo parts are the values the in-kernel split
    // would compute, so the results are the same bit for bit either way
    const QuantWs full = quant_ws(d_row, d_col, defer_max);
    // the lazy update adds -Err U into W through TMA reductions when W's rows
    // can be a tensor map (16-byte aligned base and row pitch); else it
    // drains through shared memory and plain loads and stores
    CUtensorMap tW;
    const bool w_tma = (reinterpret_cast<uintptr_t>(W) & 15) == 0 && (ldw % 4) == 0 &&
                       make_tmap_2d(&tW, false, W, d_col, d_row, ldw, 32, 32, Swz::k128);
    const bool pre = ws_bytes >= full.total && w_tma;
    int defer = defer_max;
    while (!pre && defer > 1 && static_cast<size_t>(d_row) * kBlock * defer * sizeof(float) > ws_bytes)
        defer /= 2;
    const int g_blocks = g > kBlock ? (g + kBlock - 1) / kBlock : 1;
    while (defer > 1 && !schedule_valid(nb, defer, g_blocks)) defer /= 2;
    float* err = static_cast<float*>(ws);
    float* err_lo = pre ? reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + full.err_lo) : nullptr;
    float* u_lo = pre ? reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + full.u_lo) : nullptr;
    const int64_t err_ld = static_cast<int64_t>(defer) * kBlock;

    // With act-order the columns are permuted (and dead ones zeroed) in one
    // pass; without it the permutation is the identity and the column walk
    // zeroes dead columns as it loads them.
    const bool permuted = desc_act != 0;
    if (permuted) {
        const size_t row_smem = static_cast<size_t>(d_col) * sizeof(float);
        if (cudaFuncSetAttribute(permute_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(row_smem)) != cudaSuccess)
            return GPTQ_ERR_CUDA;
        const int prow_grid = static_cast<int>(d_row < 4 * num_sms() ? d_row : 4 * num_sms());
        permute_rows_kernel<<<prow_grid, 256, row_smem, stream>>>(W, d_row, d_col, ldw, perm, dead,
                                                                   status);
    }
    const uint8_t* dead_mask = permuted ? nullptr : dead;

    CUtensorMap tU, tUmn, tErr, tUlo, tErrLo;
    if (!make_tmap_2d(&tU, false, U, d_col, d_col, d_col, kBlock, kBlock, Swz::kNone) ||
        !make_tmap_2d(&tUmn, false, U, d_col, d_col, d_col, 32, 32, Swz::k128Atom32) ||
        !make_tmap_2d(&tErr, false, err, err_ld, d_row, err_ld, 32, 128, Swz::k128))
        return GPTQ_ERR_INVALID_ARG;
    if (pre && (!make_tmap_2d(&tUlo, false, u_lo, d_col, d_col, d_col, 32, 32, Swz::k128Atom32) ||
                !make_tmap_2d(&tErrLo, false, err_lo, err_ld, d_row, err_ld, 32, 128, Swz::k128)))
        return GPTQ_ERR_INVALID_ARG;
    const size_t q_smem = (kBlock * kBlock + kBlock) * sizeof(float) + 1024;
    const bool small_group = g < 32;
    constexpr int Lw = kWalkLanes;
    auto set_smem = [&](auto kern) {
        return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    static_cast<int>(q_smem)) == cudaSuccess;
    };
    const auto q4f = small_group ? block_quant_kernel<Lw, kWarpsSmall, true, true>
                                 : block_quant_kernel<Lw, kWarpsSmall, false, true>;
    const auto q4p = small_group ? block_quant_kernel<Lw, kWarpsSmall, true, false>
                                 : block_quant_kernel<Lw, kWarpsSmall, false, false>;
    const auto q7f = small_group ? block_quant_kernel<Lw, kWarpsLarge, true, true>
                                 : block_quant_kernel<Lw, kWarpsLarge, false, true>;
    const auto q7p = small_group ? block_quant_kernel<Lw, kWarpsLarge, true, false>
                                 : block_quant_kernel<Lw, kWarpsLarge, false, false>;
    if (!set_smem(q4f) || !set_smem(q4p) || !set_smem(q7f) || !set_smem(q7p)) return GPTQ_ERR_CUDA;
    // four warps per CTA when all the layer's CTAs are resident at once
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, q4f, kWarpsSmall * 32, q_smem) !=
        cudaSuccess)
        return GPTQ_ERR_CUDA;
    constexpr int kRows4 = WalkShape<Lw, kWarpsSmall>::kRowsPerCta;
    constexpr int kRows7 = WalkShape<Lw, kWarpsLarge>::kRowsPerCta;
    const bool four = (d_row + kRows4 - 1) / kRows4 <= static_cast<int64_t>(per_sm) * num_sms();
    const auto qfull = four ? q4f : q7f;
    const auto qpart = four ? q4p : q7p;
    const int qthreads = (four ? kWarpsSmall : kWarpsLarge) * 32;
    const int qrows = four ? kRows4 : kRows7;
    const unsigned qgrid = static_cast<unsigned>((d_row + qrows - 1) / qrows);
    const int mt = static_cast<int>((d_row + 127) / 128);
    const int sms = num_sms();
    int64_t launches = permuted ? 1 : 0;
    if (pre) {
        const unsigned gx = static_cast<unsigned>((d_col / 4 + 255) / 256 < 8 ? (d_col / 4 + 255) / 256 : 8);
        const unsigned gy = static_cast<unsigned>(d_col < 65535 ? d_col : 65535);
        u_lo_kernel<<<dim3(gx, gy), 256, 0, stream>>>(U, d_col, u_lo);
        ++launches;
    }
    int run0 = 0;  // first block of the current run (its errors sit at column 0 of err)

    auto quantize_block = [&](int b) -> bool {
        const int64_t c0 = static_cast<int64_t>(b) * kBlock;
        const int bw = static_cast<int>((d_col - c0 < kBlock) ? d_col - c0 : kBlock);
        ++launches;
        // programmatic (early) launch after a kernel of this call only: the
        // kernel fetches U before waiting, and the work before this call may
        // still be writing U
        const int64_t eoff = static_cast<int64_t>(b - run0) * kBlock;
        return launch_kernel(b > 0 || permuted || pre, bw == kBlock ? qfull : qpart, dim3(qgrid),
                             dim3(qthreads), q_smem, stream, tU, W, d_row, d_col, ldw, c0, bw,
                             bits, g, pure, codes, scales, zeros, err + eoff,
                             pre ? err_lo + eoff : nullptr, err_ld, dead_mask,
                             status) == cudaSuccess;
    };
    // W[:, blocks [c, e)) -= Err[:, blocks [a, c)) U[blocks [a, c), blocks [c, e))
    auto update = [&](int a, int c, int e) -> bool {
        const int64_t c1 = static_cast<int64_t>(c) * kBlock;
        const int64_t cend = static_cast<int64_t>(e) * kBlock < d_col ? static_cast<int64_t>(e) * kBlock
                                                                    : d_col;
        const int nt = static_cast<int>((cend - c1 + 127) / 128);
        LazySched ls{W, ldw, static_cast<int>(d_row), static_cast<int>(cend), static_cast<int>(c1), mt,
                     (a - run0) * kBlock, a * kBlock, (c - a) * (kBlock / 32)};
        ++launches;
        // truncating split: the walk given the same U matches the float64
        // loop as closely with it as with the rounding split, which costs the
        // split warps a second store per operand
        // (pre-split: the same truncating split, read from the workspace)
        if (pre)
            return g3::launch<LazySched, false, true, g3::kEpiReduce, g3::kSplitPre>(
                       tErr, tUmn, ls, mt * nt, status, stream, sms, true, &tW, &tErrLo, &tUlo) ==
                   cudaSuccess;
        return (w_tma ? g3::launch<LazySched, false, true, g3::kEpiReduce, g3::kSplitTrunc>(
                            tErr, tUmn, ls, mt * nt, status, stream, sms, true, &tW)
                      : g3::launch<LazySched, false, true, g3::kEpiStaged, g3::kSplitTrunc>(
                            tErr, tUmn, ls, mt * nt, status, stream, sms, true)) == cudaSuccess;
    };
    // blocks [lo, hi) of the current run, complete w.r.t. every block < lo
    std::vector<std::tuple<int, int, int>> stack;
    for (run0 = 0; run0 < nb; run0 += defer) {
        const int run1 = run0 + defer < nb ? run0 + defer : nb;
        stack.assign(1, {run0, run1, 0});
        while (!stack.empty()) {
            auto [lo, hi, state] = stack.back();
            stack.pop_back();
            if (hi - lo == 1) {
                if (!quantize_block(lo)) return GPTQ_ERR_CUDA;
                continue;
            }
            int half = 1;
            while (2 * half < hi - lo) half *= 2;
            const int mid = lo + half;
            if (state == 0) {
                stack.push_back({lo, hi, 1});
                stack.push_back({lo, mid, 0});
            } else {
                if (!update(lo, mid, hi)) return GPTQ_ERR_CUDA;
                stack.push_back({mid, hi, 0});
            }
        }
        if (run1 < nb && !update(run0, run1, nb)) return GPTQ_ERR_CUDA;
    }
    count_launches(launches);
    return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ERR_CUDA;
}

}  // namespace gptq
