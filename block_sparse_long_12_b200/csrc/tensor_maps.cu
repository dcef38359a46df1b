// Host-side TMA tensor-map encoding through the driver entry point (no
// link-time dependency on libcuda).
#include <cudaTypedefs.h>

#include "msa_internal.h"

namespace msa {

namespace {
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (fn == nullptr) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}
}  // namespace

bool encode_2d(CUtensorMap *map, CUtensorMapDataType dt, void *base, unsigned long long inner,
               unsigned long long rows, unsigned long long row_stride_bytes, unsigned box_x, unsigned box_y,
               CUtensorMapSwizzle swizzle) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
    if (enc == nullptr) return false;
    const cuuint64_t dim[2] = {inner, rows};
    const cuuint64_t stride[1] = {row_stride_bytes};
    const cuuint32_t box[2] = {box_x, box_y};
    const cuuint32_t ones[2] = {1, 1};
    return enc(map, dt, 2, base, dim, stride, box, ones, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_3d(CUtensorMap *map, CUtensorMapDataType dt, void *base, const unsigned long long dims[3],
               const unsigned long long strides_bytes[2], const unsigned box[3], CUtensorMapSwizzle swizzle) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
    if (enc == nullptr) return false;
    const cuuint64_t dim[3] = {dims[0], dims[1], dims[2]};
    const cuuint64_t stride[2] = {strides_bytes[0], strides_bytes[1]};
    const cuuint32_t bx[3] = {box[0], box[1], box[2]};
    const cuuint32_t ones[3] = {1, 1, 1};
    return enc(map, dt, 3, base, dim, stride, bx, ones, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace msa
