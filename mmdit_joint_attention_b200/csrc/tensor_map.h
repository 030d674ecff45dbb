// Host side of the TMA tensor maps used by the attention kernels: the driver's
// cuTensorMapEncodeTiled, fetched once through the runtime's entry-point query
// (no link against libcuda), and the map shapes the kernels use.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

namespace mmdit {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// [B, N, H, 128] bf16 tensor read in boxes of `rows` tokens x 64 head-dim
// elements (128 bytes, 128-byte swizzle) of one head of one sample.  Tokens
// past N read as zero.
inline bool encode_tokens(CUtensorMap* m, const void* base, int B, int N, int H, int rows) {
    const cuuint64_t dims[4] = {128, (cuuint64_t)H, (cuuint64_t)N, (cuuint64_t)B};
    const cuuint64_t strides[3] = {128 * 2, (cuuint64_t)H * 128 * 2,
                                   (cuuint64_t)N * H * 128 * 2};
    const cuuint32_t box[4] = {64, 1, (cuuint32_t)rows, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims,
                             strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// [B, rows, H, 128] fp32 accumulator, written by reduce-adds of boxes of 32
// rows x 32 head-dim elements (128 bytes, no swizzle) of one head of one
// sample.  Rows past `rows` are not written.
inline bool encode_acc_f32(CUtensorMap* m, void* base, int B, int rows, int H) {
    const cuuint64_t dims[4] = {128, (cuuint64_t)H, (cuuint64_t)rows, (cuuint64_t)B};
    const cuuint64_t strides[3] = {128 * 4, (cuuint64_t)H * 128 * 4,
                                   (cuuint64_t)rows * H * 128 * 4};
    const cuuint32_t box[4] = {32, 1, 32, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, base, dims, strides, box,
                             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                             CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace mmdit
