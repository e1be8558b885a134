// gdn_tc_host.cu -- host-side tensor-map encoding for the TMA tensor copies.
#include <cudaTypedefs.h>

#include "gdn_tc.cuh"

namespace gdn {
namespace tc {
namespace {

// cuTensorMapEncodeTiled, looked up once per process: the runtime API hands out the driver's
// function, so the library has no link-time dependency on libcuda.
cudaError_t encoder(PFN_cuTensorMapEncodeTiled_v12000* out) {
    static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    if (!encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
        if (e != cudaSuccess) return e;
        if (q != cudaDriverEntryPointSuccess || !fn) return cudaErrorNotSupported;
        encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    *out = encode;
    return cudaSuccess;
}

}  // namespace

cudaError_t encode_tmap_f32_sw128(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                                  uint32_t box_rows) {
    PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    cudaError_t e = encoder(&encode);
    if (e != cudaSuccess) return e;
    if (cols % 32 != 0 || box_rows == 0 || box_rows > 256) return cudaErrorInvalidValue;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * sizeof(float)};
    const cuuint32_t box[2] = {32, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides,
                              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t encode_tmap_tokens(CUtensorMap* map, const void* base, bool bf16, uint64_t d, uint64_t heads,
                               uint64_t T, uint64_t B, uint32_t box_tokens) {
    PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    cudaError_t e = encoder(&encode);
    if (e != cudaSuccess) return e;
    const uint64_t es = bf16 ? 2 : 4;
    if ((d * es) % 16 != 0 || d == 0 || d > 256 || box_tokens == 0 || box_tokens > 256) return cudaErrorInvalidValue;
    const cuuint64_t dims[4] = {d, heads, T, B};
    const cuuint64_t strides[3] = {d * es, heads * d * es, T * heads * d * es};
    const cuuint32_t box[4] = {(cuuint32_t)d, 1, box_tokens, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUresult r =
        encode(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4,
               const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace tc
}  // namespace gdn
