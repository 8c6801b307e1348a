// Host-side TMA descriptor encoding shared by the tensor-core kernels.
#include <cudaTypedefs.h>

#include "vda_internal.cuh"

namespace vda {
namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

}  // namespace

bool make_bf16_rows_map(CUtensorMap* m, const void* ptr, int rows, int items, int box_rows) {
  auto fn = encode_fn();
  if (!fn || rows < 1 || items < 1 || box_rows < 1 || box_rows > 256) return false;
  cuuint64_t dims[3] = {128, (cuuint64_t)rows, (cuuint64_t)items};
  cuuint64_t strides[2] = {128 * 2, (cuuint64_t)rows * 128 * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tok_map(CUtensorMap* m, const void* ptr, int layout, int B, int H, int T, int rows, int box_rows) {
  auto fn = encode_fn();
  if (!fn || B < 1 || H < 1 || T < 1 || rows < 1 || box_rows < 1 || box_rows > 256) return false;
  const cuuint64_t row = 128 * 2;   // one token's 128 features, bytes
  cuuint64_t dims[5], strides[4];
  cuuint32_t box[5];
  // [B][H][T][rows][128]: the 3-D map (c, r, unit).
  if (layout == 0) return make_bf16_rows_map(m, ptr, rows, B * H * T, box_rows);
  // [B][T][rows][H][128]: dims (c, h, r, t, b).
  {
    const cuuint64_t d[5] = {128, (cuuint64_t)H, (cuuint64_t)rows, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t s[4] = {row, row * H, row * H * rows, row * H * rows * T};
    const cuuint32_t b[5] = {64, 1, (cuuint32_t)box_rows, 1, 1};
    for (int i = 0; i < 5; ++i) dims[i] = d[i], box[i] = b[i];
    for (int i = 0; i < 4; ++i) strides[i] = s[i];
  }
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_f32_rows_map(CUtensorMap* m, const void* ptr, long long rows, int box_rows) {
  auto fn = encode_fn();
  if (!fn || rows < 1 || box_rows < 1 || box_rows > 256) return false;
  cuuint64_t dims[2] = {128, (cuuint64_t)rows};
  cuuint64_t strides[1] = {128 * 4};
  cuuint32_t box[2] = {32, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace vda
