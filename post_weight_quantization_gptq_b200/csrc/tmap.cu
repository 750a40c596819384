// Host helper: 2-D TMA tensor maps (cuTensorMapEncodeTiled through the
// runtime's driver entry point, so the library needs no -lcuda).
#include <cuda.h>

#include "kernels.h"

namespace gptq {
namespace {

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                 const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                 const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                 CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// Looked up once per process (a function-local static is initialized by one
// thread while concurrent callers wait); nullptr if the driver lacks it.
EncodeTiled encoder() {
    static const EncodeTiled fn = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<EncodeTiled>(p);
        return static_cast<EncodeTiled>(nullptr);
    }();
    return fn;
}

}  // namespace

bool make_tmap_2d(CUtensorMap* map, bool bf16, const void* base, uint64_t inner, uint64_t outer,
                  uint64_t ld_elems, uint32_t box_inner, uint32_t box_outer, Swz swizzle) {
    EncodeTiled enc = encoder();
    if (enc == nullptr) return false;
    const uint64_t esz = bf16 ? 2 : 4;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {ld_elems * esz};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    return enc(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
               const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               swizzle == Swz::k128 ? CU_TENSOR_MAP_SWIZZLE_128B
               : swizzle == Swz::k128Atom32 ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B
                                            : CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace gptq
