// TMA tensor-map encoding for the three row orders of a [B*H, T, d] tensor.
// cuTensorMapEncodeTiled is reached through cudaGetDriverEntryPoint, so the
// library needs no link against the driver library. Encoded maps are cached
// per (address, shape): calls that reuse their buffers (training loops,
// benchmarks) skip the encoding.
#include <cuda.h>

#include <cstring>
#include <mutex>

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

bool encode_views(CUtensorMap out[3], const void* base, int elem, const Geom& g, int BH, int d) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const bool is_f32 = (elem == ELEM_F32);
  const CUtensorMapDataType dt = is_f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                 : elem == ELEM_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                    : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
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
    // packed short classes (cpt > 1) move one class of P rows per box
    cuuint32_t box[4] = {inner, 1, (cuuint32_t)(g.cpt > 1 ? g.P : kTile), 1};
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

// The summary rows of one natural 128-row tile of an fp32 [B*H, T, d]
// accumulator (fixed pattern, l dividing 128 or 128 dividing l): the box is 32
// columns by c rows by max(1, 128 / l) l-blocks, i.e. the last c rows of each
// block the tile covers, packed block after block.
bool encode_summary_rows(CUtensorMap* out, const void* base, const Geom& g, int BH, int d) {
  EncodeTiledFn enc = encode_fn();
  if (!enc || g.nsum == 0) return false;
  const cuuint64_t row = (cuuint64_t)d * 4;
  const cuuint32_t one[4] = {1, 1, 1, 1};
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)g.l, (cuuint64_t)(g.T / g.l), (cuuint64_t)BH};
  cuuint64_t str[3] = {row, (cuuint64_t)g.l * row, (cuuint64_t)g.T * row};
  const int bpt = g.l < kTile ? kTile / g.l : 1;
  cuuint32_t box[4] = {32, (cuuint32_t)g.c, (cuuint32_t)bpt, 1};
  return enc(out, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<void*>(base), dims, str, box,
             one, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

struct Key {
  const void* base;
  int what;  // 0: the three views, 1: the summary-rows map (in maps[0])
  int elem, T, l, c, P, nsum, BH, d;
  bool operator==(const Key& o) const { return std::memcmp(this, &o, sizeof(Key)) == 0; }
};

struct Entry {
  Key key;
  CUtensorMap maps[3];
  uint64_t stamp;
  bool valid;
};

constexpr int kCacheSize = 64;
Entry g_cache[kCacheSize];
uint64_t g_clock = 0;
std::mutex g_cache_mu;

bool cached_maps(CUtensorMap* out, int n, int what, const void* base, int elem, const Geom& g,
                 int BH, int d) {
  Key key;
  std::memset(&key, 0, sizeof(key));
  key.base = base;
  key.what = what;
  key.elem = elem;
  key.T = g.T;
  key.l = g.l;
  key.c = g.c;
  key.P = g.P;
  key.nsum = g.nsum;
  key.BH = BH;
  key.d = d;
  std::lock_guard<std::mutex> lk(g_cache_mu);
  int victim = -1;
  for (int e = 0; e < kCacheSize; ++e) {
    if (g_cache[e].valid && g_cache[e].key == key) {
      g_cache[e].stamp = ++g_clock;
      std::memcpy(out, g_cache[e].maps, n * sizeof(CUtensorMap));
      return true;
    }
    // the first free slot, else the least recently used one
    if (victim < 0 || (g_cache[victim].valid &&
                       (!g_cache[e].valid || g_cache[e].stamp < g_cache[victim].stamp)))
      victim = e;
  }
  const bool ok = what == 0 ? encode_views(out, base, elem, g, BH, d)
                            : encode_summary_rows(out, base, g, BH, d);
  if (!ok) return false;
  g_cache[victim].key = key;
  std::memcpy(g_cache[victim].maps, out, n * sizeof(CUtensorMap));
  g_cache[victim].stamp = ++g_clock;
  g_cache[victim].valid = true;
  return true;
}

}  // namespace

bool make_view_maps(CUtensorMap out[3], const void* base, int elem, const Geom& g, int BH,
                    int d) {
  return cached_maps(out, 3, 0, base, elem, g, BH, d);
}

bool make_summary_rows_map(CUtensorMap* out, const void* base, const Geom& g, int BH, int d) {
  return cached_maps(out, 1, 1, base, ELEM_F32, g, BH, d);
}

int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev < 0 || dev >= 64) return 148;
  if (!cached[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

}  // namespace st
