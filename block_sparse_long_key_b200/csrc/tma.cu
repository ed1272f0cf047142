// Host side of the TMA loads: tensor maps over [rows, d] bf16 tables (Q or
// dO viewed as T*H_q rows of d values, or the block centroids), boxes of 64
// elements (128 bytes) by `box_rows` rows with the 128-byte swizzle (one row
// high for the tile::gather4 row gathers); and over the [T, h_kv, d] key and
// value tensors, boxes of 64 channels x one head x a key block's tokens.
// The driver entry point is looked up once through the runtime.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "launch.h"

namespace moba {
namespace {

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encode_fn() {
  static std::once_flag once;
  static EncodeTiled fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiled>(p);
  });
  return fn;
}

}  // namespace

cudaError_t make_row_map(CUtensorMap* map, const void* base, unsigned long long nrows, int d, int box_rows) {
  EncodeTiled fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  if ((reinterpret_cast<uintptr_t>(base) & 15) != 0 || nrows == 0) return cudaErrorInvalidValue;
  const cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)nrows};
  const cuuint64_t strides[1] = {(cuuint64_t)d * 2};  // bytes between rows
  if (box_rows < 1 || box_rows > 256) return cudaErrorInvalidValue;
  const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t make_kv_map(CUtensorMap* map, const void* base, int total_tokens, int h_kv, int d, int box_tokens) {
  EncodeTiled fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  if ((reinterpret_cast<uintptr_t>(base) & 15) != 0 || total_tokens <= 0) return cudaErrorInvalidValue;
  if (box_tokens < 1 || box_tokens > 256) return cudaErrorInvalidValue;
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)h_kv, (cuuint64_t)total_tokens};
  const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)h_kv * d * 2};  // bytes
  const cuuint32_t box[3] = {64, 1, (cuuint32_t)box_tokens};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace moba
