// Tensor maps (TMA descriptors) over the projected-query / projected-key
// tensors and over K/V caches, shared by the prefill kernels.
#include <cudaTypedefs.h>

#include "launch.h"

namespace rtp {

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// Tensor map over a [B, H, R, D] bf16 view (D = 16 or 128), box of `box_rows`
// rows x `box_cols` columns.  Strides of size-1 dims are replaced by dense ones
// (the encoder wants them to be multiples of 16 bytes even where unused).
static bool make_map(CUtensorMap* map, const View4& v, int64_t B, int64_t H, int64_t R, int64_t D, int box_rows,
                     int box_cols, CUtensorMapSwizzle swz) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)R, (cuuint64_t)H, (cuuint64_t)B};
  cuuint64_t st1 = (cuuint64_t)v.sn * 2, st2 = (cuuint64_t)v.sh * 2, st3 = (cuuint64_t)v.sb * 2;
  if (R <= 1) st1 = (cuuint64_t)D * 2;
  if (H <= 1) st2 = st1 * (cuuint64_t)(R > 0 ? R : 1);
  if (B <= 1) st3 = st2 * (cuuint64_t)(H > 0 ? H : 1);
  cuuint64_t strides[3] = {st1, st2, st3};
  cuuint32_t box[4] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(v.data), dims, strides, box,
                        estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_idx_map(CUtensorMap* map, const View4& v, int64_t B, int64_t H, int64_t R, int box_rows) {
  return make_map(map, v, B, H, R, kIdxDim, box_rows, kIdxDim, CU_TENSOR_MAP_SWIZZLE_32B);
}

bool make_row_map(CUtensorMap* map, const View4& v, int64_t B, int64_t H, int64_t R, int box_rows) {
  // 128-byte swizzle: the box is 64 bf16 columns (128 bytes) wide, so a
  // 128-column row is fetched as two boxes (column halves)
  return make_map(map, v, B, H, R, kHeadDim, box_rows, 64, CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace rtp
