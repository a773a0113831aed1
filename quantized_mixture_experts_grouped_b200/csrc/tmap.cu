// Host-side tensor-map construction for the packed weight banks (layout "MW4T v2": 512-byte
// chunks of 8 rows x 128 K, the chunks of one row group contiguous over K). The grouped GEMM and
// the batched decode kernel load whole 128 x 128 tiles, which in this layout are 16 chunks spaced
// one row group apart; a tensor map with a (128 words, 1 K group, 16 row groups) box fetches such a
// tile in one copy of sixteen 512-byte lines.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"

namespace moe {
namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    const cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
    if (e == cudaSuccess && q == cudaDriverEntryPointSuccess) fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

int encode3(void* map, CUtensorMapDataType type, const void* base, const cuuint64_t (&dims)[3],
            const cuuint64_t (&strides)[2], const cuuint32_t (&box)[3], const char* what) {
  auto fn = encode_fn();
  if (!fn) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(static_cast<CUtensorMap*>(map), type, 3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled (%s) failed (%d)", what, (int)r);
  return MOE_OK;
}

}  // namespace

int make_chunk_code_map(void* map, const void* base, int N, int K, int slots) {
  const int G = K / kGroup;
  const cuuint64_t dims[3] = {kChunkBytes / 4, (cuuint64_t)G, (cuuint64_t)(N / kRowGroup) * (cuuint64_t)slots};
  const cuuint64_t strides[2] = {kChunkBytes, (cuuint64_t)G * kChunkBytes};
  const cuuint32_t box[3] = {kChunkBytes / 4, 1, kRowBlock / kRowGroup};
  return encode3(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, base, dims, strides, box, "weight codes");
}

int make_chunk_scale_map(void* map, const void* base, int N, int K, int slots) {
  const int G = K / kGroup;
  const cuuint64_t dims[3] = {kRowGroup, (cuuint64_t)G, (cuuint64_t)(N / kRowGroup) * (cuuint64_t)slots};
  const cuuint64_t strides[2] = {kRowGroup * 2, (cuuint64_t)G * kRowGroup * 2};
  const cuuint32_t box[3] = {kRowGroup, 1, kRowBlock / kRowGroup};
  return encode3(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, base, dims, strides, box, "weight scales");
}

}  // namespace moe
