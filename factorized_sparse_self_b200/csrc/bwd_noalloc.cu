// st_sparse_attn_bwd_noalloc: the backward pass without a caller workspace.
//
// The regular backward needs device scratch (the fp32 dQ/dK/dV accumulators
// and D), which its caller allocates and passes in. Some callers cannot do
// that: a plugin whose host application owns every device allocation, or a
// latency-critical path that may not call cudaMalloc and has nowhere to keep
// a workspace between calls. For them this entry point uses a fixed scratch
// array in the library's own device memory instead.
//
// The array is a file-scope __device__ variable: it is created on a device
// when the library's device code is loaded there and held until the process
// exits. Under CUDA's default lazy loading that is the first call of this
// entry point on the device (its cudaGetSymbolAddress); with
// CUDA_MODULE_LOADING=EAGER it is when the process creates its context on
// each device, whether or not this entry point is ever called. Host code
// cannot use the array's name as a device address (in host code it is only a
// host-side stand-in), so the device address is looked up with
// cudaGetSymbolAddress once per device, on the first call made on that
// device, with that device current.
#include <cuda_runtime.h>

#include <mutex>

#include "launch.h"

namespace {

constexpr size_t kScratchBytes = size_t(64) << 20;  // 64 MiB per device

static __device__ __align__(256) unsigned char g_bwd_scratch[kScratchBytes];

constexpr int kMaxDev = 64;
void* g_scratch_ptr[kMaxDev] = {nullptr};
std::mutex g_scratch_mu;

// Device address of g_bwd_scratch on the current device (looked up once).
st_status scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return ST_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_bwd_scratch) != cudaSuccess || !p) return ST_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return ST_OK;
}

}  // namespace

extern "C" {

st_status st_sparse_attn_bwd_noalloc(const st_layout* layout, st_dtype dtype, int32_t B, int32_t H,
                                     int32_t T, int32_t d, float scale, const void* q,
                                     const void* k, const void* v, const void* o,
                                     const float* lse, const void* dout, void* dq, void* dk,
                                     void* dv, void* stream) {
  size_t need = 0;
  st_status s = st_sparse_attn_bwd_workspace(layout, dtype, B, H, T, d, &need);
  if (s != ST_OK) return s;
  if (need > kScratchBytes) return ST_ERR_WORKSPACE;
  // the layout's device must be current before the array is looked up (and,
  // under lazy loading, created) on it
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return ST_ERR_CUDA;
  if (!layout->on_device || dev != layout->device) return ST_ERR_INVALID;
  void* scratch = nullptr;
  s = scratch_address(&scratch);
  if (s != ST_OK) return s;
  // The backward zeroes the accumulators and overwrites D itself, so the
  // previous call's contents of the scratch never leak into this one.
  return st_sparse_attn_bwd(layout, dtype, B, H, T, d, scale, q, k, v, o, lse, dout, dq, dk, dv,
                            scratch, kScratchBytes, stream);
}

}  // extern "C"
