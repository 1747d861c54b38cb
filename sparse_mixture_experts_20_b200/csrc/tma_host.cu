// Host helpers shared by the tensor-core kernels: TMA tensor-map encoding
// (through the driver entry point, so the library needs no link against
// libcuda) and the SM count of the current device.
#include <cuda.h>
#include <cudaTypedefs.h>
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

CUtensorMapDataType dtype_of(int elem) {
    return elem == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                     : (elem == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8);
}

}  // namespace

// 2D map over (rows, K) row-major with box (128 bytes of K, box_rows rows),
// 128-byte swizzle, out-of-range elements read as zero.
bool encode_tma_2d(void* map, const void* base, int rows, int K, int elem, int box_rows) {
    auto fn = get_encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * elem};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / elem), static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    return fn(static_cast<CUtensorMap*>(map), dtype_of(elem), 2, const_cast<void*>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3D map over (n_mats, N, K) with box (128 bytes of K, box_rows of N, 1).
bool encode_tma_3d(void* map, const void* base, int n_mats, int N, int K, int elem, int box_rows) {
    auto fn = get_encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(n_mats)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(K) * elem, static_cast<cuuint64_t>(N) * K * elem};
    cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / elem), static_cast<cuuint32_t>(box_rows), 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(static_cast<CUtensorMap*>(map), dtype_of(elem), 3, const_cast<void*>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2D map over (rows, cols) row-major for TMA stores of boxes of 64 bytes x
// box_rows rows (box_cols * elem == 64) in the 64-byte swizzled layout.
bool encode_tma_2d_store64(void* map, const void* base, int rows, int cols, int elem, int box_rows) {
    auto fn = get_encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * elem};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(64 / elem), static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    return fn(static_cast<CUtensorMap*>(map), dtype_of(elem), 2, const_cast<void*>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int device_sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
    return n;
}

}  // namespace moe
