// Stage 2a: dead columns, damping and act-order.
//
// "GPTQ (GPT Quantization)", pseudo-code step 1 adds lambda I to H for
// stability; the AutoGPTQ guide ("Quantizar seu proprio modelo") sets
// damp_percent = 0.01, read here as lambda = damp * mean(diag H).  desc_act
// ("Quantification avec AutoGPTQ": True = order by importance) quantizes the
// columns by descending diag(H).  A column whose diagonal is exactly 0 (an
// input channel that never fires) gets H_ii = 1 and zero weights.
//
// The output is the working matrix of the Cholesky stage, already flipped:
//   P[a][b] = Hd[q[a]][q[b]],  q[a] = perm[d-1-a],
// where Hd is the dead-fixed, damped H.  Only P's lower triangle is written.
#include "common.cuh"
#include "kernels.h"

namespace gptq {
namespace {

struct PrepScratch {
    double lambda;
    float pad[2];
};

// diag -> keys (dead columns count as 1), dead mask, lambda (fp64 sum).  A
// diagonal that is not finite (NaN or infinite: the calibration data held a
// non-finite value) makes H unusable: it is reported as not positive
// definite, and the act-order ranking below still yields a permutation.
__global__ void __launch_bounds__(1024)
    diag_kernel(const float* __restrict__ H, int64_t d, int64_t ldh, float damp,
                float* __restrict__ keys, uint8_t* __restrict__ dead, PrepScratch* scratch,
                int32_t* status) {
    __shared__ double part[32];
    double acc = 0.0;
    bool finite = true;
    for (int64_t i = threadIdx.x; i < d; i += blockDim.x) {
        const float h = H[i * ldh + i];
        const bool is_dead = (h == 0.f);
        const float k = is_dead ? 1.f : h;
        finite = finite && isfinite(h);
        keys[i] = k;
        dead[i] = is_dead ? 1 : 0;
        acc += static_cast<double>(k);
    }
    if (!finite) report(status, GPTQ_ERR_NOT_PD);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x < 32) {
        double v = (threadIdx.x < (blockDim.x >> 5)) ? part[threadIdx.x] : 0.0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (threadIdx.x == 0) scratch->lambda = static_cast<double>(damp) * v / static_cast<double>(d);
    }
}

// Sort key of a float as an unsigned integer whose order is the float order
// (negative values: all bits flipped; others: the sign bit set), with every
// NaN mapped to 0, below all of them.  Integers compare totally, so the ranks
// below are a permutation whatever the keys hold; NaN keys rank last, after
// every number, in index order (as a stable sort of -diag puts them).
__device__ __forceinline__ uint32_t order_key(float x) {
    const uint32_t b = __float_as_uint(x);
    if (isnan(x)) return 0u;
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Stable descending rank of every key: rank_i = #{j : k_j > k_i} +
// #{j < i : k_j == k_i}; perm[rank_i] = i.  O(d^2) comparisons, exact.
__global__ void __launch_bounds__(256)
    rank_kernel(const float* __restrict__ keys, int64_t d, int32_t* __restrict__ perm) {
    __shared__ uint32_t tile[1024];
    const int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
    const uint32_t ki = (i < d) ? order_key(keys[i]) : 0u;
    int rank = 0;  // d < 2^31
    for (int64_t j0 = 0; j0 < d; j0 += 1024) {
        __syncthreads();
        for (int t = threadIdx.x; t < 1024; t += blockDim.x)
            tile[t] = (j0 + t < d) ? order_key(keys[j0 + t]) : 0u;
        __syncthreads();
        const int64_t jn = (d - j0 < 1024) ? d - j0 : 1024;
        for (int t = 0; t < jn; ++t) {
            const uint32_t kj = tile[t];
            rank += (kj > ki) || (kj == ki && j0 + t < i);
        }
    }
    if (i < d) perm[rank] = static_cast<int32_t>(i);
}

__global__ void iota_kernel(int32_t* __restrict__ perm, int64_t d) {
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < d;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x)
        perm[i] = static_cast<int32_t>(i);
}

// P[a][b] for the lower triangle, 32 x 32 tiles through shared memory so that
// both the reads of H's lower triangle and the writes of P are coalesced
// when the permutation is the identity; 32 x 8 threads, four rows each.
__global__ void __launch_bounds__(256)
    gather_kernel(const float* __restrict__ H, int64_t d, int64_t ldh,
                  const int32_t* __restrict__ perm, const float* __restrict__ keys,
                  const PrepScratch* __restrict__ scratch, float* __restrict__ P) {
    __shared__ float tile[32][33];
    const int64_t a0 = static_cast<int64_t>(blockIdx.y) * 32;
    const int64_t b0 = static_cast<int64_t>(blockIdx.x) * 32;
    if (b0 > a0 + 31) return;  // strictly upper tile
    const int tx = threadIdx.x, ty = threadIdx.y;
    const float lam = static_cast<float>(scratch->lambda);
    // load: element (a = a0 + tx, b = b0 + y)
    const int64_t a = a0 + tx;
    const int64_t qa = a < d ? perm[d - 1 - a] : 0;
#pragma unroll
    for (int y = ty; y < 32; y += 8) {
        const int64_t b = b0 + y;
        float v = 0.f;
        if (a < d && b < d) {
            const int64_t qb = perm[d - 1 - b];
            if (qa == qb) {
                v = keys[qa] + lam;
            } else {
                const int64_t r = qa > qb ? qa : qb, c = qa > qb ? qb : qa;
                v = H[r * ldh + c];
            }
        }
        tile[y][tx] = v;
    }
    __syncthreads();
    // store: P[a0 + y][b0 + tx] = element (a0 + y, b0 + tx) = tile[tx][y]
#pragma unroll
    for (int y = ty; y < 32; y += 8) {
        const int64_t ar = a0 + y, b = b0 + tx;
        if (ar < d && b < d && b <= ar) P[ar * d + b] = tile[tx][y];
    }
}

}  // namespace

size_t prep_workspace_bytes(int64_t d) {
    return ((sizeof(PrepScratch) + 255) / 256) * 256 + ((static_cast<size_t>(d) * 4 + 255) / 256) * 256;
}

gptq_status launch_prep(const float* H, int64_t d, int64_t ldh, float damp, int desc_act,
                        float* P, int32_t* perm, uint8_t* dead, int32_t* status, void* ws,
                        cudaStream_t stream) {
    uint8_t* base = static_cast<uint8_t*>(ws);
    PrepScratch* scratch = reinterpret_cast<PrepScratch*>(base);
    float* keys = reinterpret_cast<float*>(base + ((sizeof(PrepScratch) + 255) / 256) * 256);
    diag_kernel<<<1, 1024, 0, stream>>>(H, d, ldh, damp, keys, dead, scratch, status);
    if (desc_act) {
        rank_kernel<<<static_cast<unsigned>((d + 255) / 256), 256, 0, stream>>>(keys, d, perm);
    } else {
        iota_kernel<<<static_cast<unsigned>((d + 255) / 256), 256, 0, stream>>>(perm, d);
    }
    const unsigned nt = static_cast<unsigned>((d + 31) / 32);
    gather_kernel<<<dim3(nt, nt), dim3(32, 8), 0, stream>>>(H, d, ldh, perm, keys, scratch, P);
    count_launches(3);
    return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ERR_CUDA;
}

}  // namespace gptq
