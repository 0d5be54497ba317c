// Host helper: TMA tensor maps over row-major bf16, fp32 or byte tensors. The driver's
// encoder is fetched once through the runtime's entry-point query (no link-time libcuda).
#include "hlta_internal.cuh"

#include <cudaTypedefs.h>
#include <mutex>

namespace hlta {
namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

// the driver's tensor-map encoder (looked up once)
PFN_cuTensorMapEncodeTiled_v12000 encoder()
{
    std::call_once(g_encode_once, [] {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = (PFN_cuTensorMapEncodeTiled_v12000)fn;
    });
    return g_encode;
}

}  // namespace

static cudaError_t encode_2d(CUtensorMap *map, CUtensorMapDataType dt, uint32_t elem,
                             const void *base, uint64_t rows, uint64_t cols, uint32_t box_cols,
                             uint32_t box_rows, bool swizzle128)
{
    if (!encoder()) return cudaErrorNotSupported;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * elem};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE,
                          swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t make_tmap_2d_bf16(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols,
                              uint32_t box_cols, uint32_t box_rows, bool swizzle128)
{
    return encode_2d(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, rows, cols, box_cols,
                     box_rows, swizzle128);
}

cudaError_t make_tmap_2d_f32(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols,
                             uint32_t box_cols, uint32_t box_rows, bool swizzle128)
{
    return encode_2d(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, base, rows, cols, box_cols,
                     box_rows, swizzle128);
}

cudaError_t make_tmap_2d_u8(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols,
                            uint32_t box_cols, uint32_t box_rows)
{
    return encode_2d(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, base, rows, cols, box_cols, box_rows,
                     true);
}

}  // namespace hlta
