// wall_tma.cu -- TMA tensor maps for the tensor-core kernels.
#include <cuda.h>

#include "wall_internal.h"

namespace wall {

namespace {
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}
}  // namespace

// A [rows, heads, dim] bf16 array viewed as the 3-D tensor (dim, heads, rows);
// one box is 64 elements (128 B, 128-byte swizzle) x 1 head x box_rows rows.
bool make_tile_map(CUtensorMap* m, const void* base, long rows, int heads, int dim,
                   int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rows <= 0 || dim % 64 != 0) return false;
  cuuint64_t gdim[3] = {(cuuint64_t)dim, (cuuint64_t)heads, (cuuint64_t)rows};
  cuuint64_t gstride[2] = {(cuuint64_t)dim * 2, (cuuint64_t)dim * heads * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)box_rows};
  cuuint32_t estride[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), gdim, gstride,
                  box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// A [B, Tcap, heads, dim] bf16 cache of which the first T rows of every batch
// row are read, viewed as the 4-D tensor (dim, heads, T, B) with batch rows
// Tcap rows apart; rows at or past T read as zeros.  Box as above.
bool make_cache_map(CUtensorMap* m, const void* base, int B, int T, int Tcap, int heads, int dim,
                    int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || B <= 0 || T <= 0 || Tcap < T || dim % 64 != 0) return false;
  cuuint64_t gdim[4] = {(cuuint64_t)dim, (cuuint64_t)heads, (cuuint64_t)T, (cuuint64_t)B};
  cuuint64_t gstride[3] = {(cuuint64_t)dim * 2, (cuuint64_t)dim * heads * 2,
                           (cuuint64_t)Tcap * heads * dim * 2};
  cuuint32_t box[4] = {64, 1, (cuuint32_t)box_rows, 1};
  cuuint32_t estride[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), gdim, gstride,
                  box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// A [rows, 128] bf16 array of stored 128 x 128 tiles viewed as the 2-D tensor
// (128, rows).  Loads: one box is 64 columns (128 B, 128-byte swizzle) x
// box_rows rows.  Stores: 32 columns (64 B, 64-byte swizzle) x box_rows.
bool make_rows128_map(CUtensorMap* m, const void* base, long rows, int box_rows, int box_cols) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rows <= 0 || (box_cols != 32 && box_cols != 64)) return false;
  cuuint64_t gdim[2] = {128, (cuuint64_t)rows};
  cuuint64_t gstride[1] = {256};
  cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  cuuint32_t estride[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), gdim, gstride,
                  box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  box_cols == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace wall
