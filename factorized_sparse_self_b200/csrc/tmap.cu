// TMA tensor-map encoding for the three row orders of a [B*H, T, d] tensor.
// cuTensorMapEncodeTiled is reached through cudaGetDriverEntryPoint, so the
// library needs no link against the driver library.
#include <cuda.h>

#include "launch.h"

namespace st {
namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

}  // namespace

bool make_view_maps(CUtensorMap out[3], const void* base, bool is_f32, const Geom& g, int BH,
                    int d) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const CUtensorMapDataType dt =
      is_f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const cuuint64_t es = is_f32 ? 4 : 2;
  const cuuint32_t inner = is_f32 ? 32 : 64;
  const cuuint64_t row = (cuuint64_t)d * es;
  void* gp = const_cast<void*>(base);
  const cuuint32_t one[4] = {1, 1, 1, 1};
  {
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)g.T, (cuuint64_t)BH};
    cuuint64_t str[2] = {row, (cuuint64_t)g.T * row};
    cuuint32_t box[3] = {inner, (cuuint32_t)kTile, 1};
    if (enc(&out[VIEW_NAT], dt, 3, gp, dims, str, box, one, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  }
  out[VIEW_SUM] = out[VIEW_NAT];
  out[VIEW_CLS] = out[VIEW_NAT];
  if (g.P > 0) {
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)g.l, (cuuint64_t)(g.T / g.l), (cuuint64_t)BH};
    cuuint64_t str[3] = {row, (cuuint64_t)g.l * row, (cuuint64_t)g.T * row};
    cuuint32_t box[4] = {inner, 1, (cuuint32_t)kTile, 1};
    if (enc(&out[VIEW_CLS], dt, 4, gp, dims, str, box, one, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
    if (g.nsum > 0) {
      cuuint32_t sbox[4] = {inner, (cuuint32_t)g.c, (cuuint32_t)(kTile / g.c), 1};
      if (enc(&out[VIEW_SUM], dt, 4, gp, dims, str, sbox, one, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return false;
    }
  }
  return true;
}

}  // namespace st
