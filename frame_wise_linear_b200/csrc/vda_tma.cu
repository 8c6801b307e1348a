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

bool make_bf16_box_map(CUtensorMap* m, const void* ptr, int rows, int items, int box_cols, int box_rows,
                       int swizzle_bytes) {
  auto fn = encode_fn();
  if (!fn || rows < 1 || items < 1 || box_rows < 1 || box_rows > 256) return false;
  if (box_cols * 2 != swizzle_bytes || (swizzle_bytes != 32 && swizzle_bytes != 64 && swizzle_bytes != 128))
    return false;   // one box row spans the swizzle exactly
  const CUtensorMapSwizzle sw = swizzle_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                      : CU_TENSOR_MAP_SWIZZLE_32B;
  cuuint64_t dims[3] = {128, (cuuint64_t)rows, (cuuint64_t)items};
  cuuint64_t strides[2] = {128 * 2, (cuuint64_t)rows * 128 * 2};
  cuuint32_t box[3] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_bf16_2d_map(CUtensorMap* m, const void* ptr, long long rows, long long cols, int box_cols, int box_rows) {
  auto fn = encode_fn();
  if (!fn || rows < 1 || cols < 1 || box_rows < 1 || box_rows > 256 || box_cols * 2 != 128) return false;
  if ((cols * 2) % 16) return false;   // row stride: a multiple of 16 bytes
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tok_map(CUtensorMap* m, const void* ptr, int layout, int B, int H, int T, int rows, int box_rows,
                  int elem_bytes, int box_bytes) {
  auto fn = encode_fn();
  if (!fn || B < 1 || H < 1 || T < 1 || rows < 1 || box_rows < 1 || box_rows > 256) return false;
  if (elem_bytes != 1 && elem_bytes != 2) return false;
  // A box row is box_bytes (128 by default: 64 bf16 or 128 e4m3 features),
  // with the swizzle of that span.
  if (box_bytes != 32 && box_bytes != 64 && box_bytes != 128) return false;
  const CUtensorMapSwizzle sw = box_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                : box_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                  : CU_TENSOR_MAP_SWIZZLE_32B;
  const CUtensorMapDataType dt = elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  const cuuint64_t row = 128 * (cuuint64_t)elem_bytes;   // one token's 128 features, bytes
  const cuuint32_t inner = box_bytes / elem_bytes;        // features per box row
  cuuint64_t dims[5], strides[4];
  cuuint32_t box[5];
  int rank;
  if (layout == 0) {
    // [B][H][T][rows][128]: the 3-D map (c, r, unit).
    rank = 3;
    const cuuint64_t d[3] = {128, (cuuint64_t)rows, (cuuint64_t)B * H * T};
    const cuuint64_t s[2] = {row, row * rows};
    const cuuint32_t b[3] = {inner, (cuuint32_t)box_rows, 1};
    for (int i = 0; i < 3; ++i) dims[i] = d[i], box[i] = b[i];
    for (int i = 0; i < 2; ++i) strides[i] = s[i];
  } else {
    // [B][T][rows][H][128]: dims (c, h, r, t, b).
    rank = 5;
    const cuuint64_t d[5] = {128, (cuuint64_t)H, (cuuint64_t)rows, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t s[4] = {row, row * H, row * H * rows, row * H * rows * T};
    const cuuint32_t b[5] = {inner, 1, (cuuint32_t)box_rows, 1, 1};
    for (int i = 0; i < 5; ++i) dims[i] = d[i], box[i] = b[i];
    for (int i = 0; i < 4; ++i) strides[i] = s[i];
  }
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return fn(m, dt, rank, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
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
