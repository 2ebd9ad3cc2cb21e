// Host side of the TMA helpers: tensor-map encoding through the driver.
#include "tma.cuh"

namespace slstm {

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
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

bool make_map_f32_3d(CUtensorMap *map, const void *base, uint64_t n0, uint64_t n1, uint64_t n2, uint64_t ld1,
                     uint64_t ld2, uint32_t b0, uint32_t b1)
{
    auto fn = tensor_map_encoder();
    if (fn == nullptr) return false;
    cuuint64_t dims[3] = {n0, n1, n2};
    cuuint64_t strides[2] = {ld1 * 4, ld2 * 4};
    cuuint32_t box[3] = {b0, b1, 1u};
    cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void *>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool make_map_f32_4d(CUtensorMap *map, const void *base, uint64_t n0, uint64_t n1, uint64_t n2, uint64_t n3,
                     uint64_t ld1, uint64_t ld2, uint64_t ld3, uint32_t b0, uint32_t b2)
{
    auto fn = tensor_map_encoder();
    if (fn == nullptr) return false;
    cuuint64_t dims[4] = {n0, n1, n2, n3};
    cuuint64_t strides[3] = {ld1 * 4, ld2 * 4, ld3 * 4};
    cuuint32_t box[4] = {b0, 1u, b2, 1u};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<void *>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace slstm
