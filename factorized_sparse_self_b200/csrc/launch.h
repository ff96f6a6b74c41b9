// Host-side launch entry points of the kernels (internal; CUDA files only).
#pragma once

#include <cuda_runtime.h>

#include <algorithm>

#include "st_internal.h"

namespace st {

struct Call {
  const st_layout* L;
  int dtype;  // st_dtype
  int B, H, d;
  int h0 = 0, hn = 0;  // heads h0 .. h0+hn-1 of the H in the tensors
  float scale;
  int nclasses;     // head classes of the layout
  int* status;      // device status word
  uint64_t wait_ns; // bound of every on-device wait
  cudaStream_t stream;
  // Benchmark events recorded right before the first and right after the
  // last attention launch of the call (null when timing is off).
  cudaEvent_t ev_begin = nullptr, ev_end = nullptr;
};

inline void record_begin(const Call& c) {
  if (c.ev_begin) cudaEventRecord(c.ev_begin, c.stream);
}
inline void record_end(const Call& c) {
  if (c.ev_end) cudaEventRecord(c.ev_end, c.stream);
}

// Multiprocessor count of the current device (queried once per device).
int sm_count();

// Exact fp32 path (CUDA cores): float32 tensors, d = 32 or 64.
cudaError_t simt_fwd(const Call& c, const void* q, const void* k, const void* v, void* o,
                     float* lse);
cudaError_t simt_bwd(const Call& c, const void* q, const void* k, const void* v,
                     const float* lse, const void* dout, const float* D, float* dq_acc,
                     float* dk_acc, float* dv_acc);

// fp32 backward prologue: D_i = dout_i . O_i (and zeroes acc_elems floats).
cudaError_t bwd_prologue(const Call& c, const void* o, const void* dout, float* D, float* acc,
                         size_t acc_elems);

// 16-bit backward, around the tensor-core kernel: bwd_prep writes D for every
// row, zeroes the fp32 accumulator rows that collect several contributions
// and the work counter the tensor-core kernel claims its units from, and
// writes the largest |dout| of each of its *nslots blocks into slots;
// bwd_finish rounds the accumulated rows into dq, dk, dv (scale applied to dQ
// and dK, the inverse of the dout scale to dV). Rows that a single backward
// unit produces, and rows nobody writes (zero-filled), are written by the
// tensor-core kernel itself.
cudaError_t bwd_prep(const Call& c, const void* o, const void* dout, float* D, float* dq_acc,
                     float* dk_acc, float* dv_acc, int* sched_counter, float* slots,
                     int* nslots);
cudaError_t bwd_finish(const Call& c, const float* dq_acc, const float* dk_acc,
                       const float* dv_acc, const float* slots, int nslots, void* dq, void* dk,
                       void* dv);

// Tensor-core path (tcgen05 + TMA): bf16, d = 64.
cudaError_t tc_fwd(const Call& c, const void* q, const void* k, const void* v, void* o,
                   float* lse, int force_timeout);
cudaError_t tc_bwd(const Call& c, const void* q, const void* k, const void* v,
                   const float* lse, const void* dout, const float* D, float* dq_acc,
                   float* dk_acc, float* dv_acc, void* dq, void* dk, void* dv,
                   int* sched_counter, const float* slots, int nslots);

}  // namespace st

#include <cuda.h>

namespace st {

// Units per item: the most heads of one class among the selected heads, times B.
inline int heads_per_class(const Call& c) {
  if (c.nclasses == 1) return c.B * c.hn;
  int most = 0;
  for (int p = 0; p < 2; ++p) {
    const int first = c.h0 + ((p - c.h0) & 1);
    const int end = c.h0 + c.hn;
    most = std::max(most, first < end ? (end - 1 - first) / 2 + 1 : 0);
  }
  return c.B * most;
}

inline Heads heads_of(const Call& c) {
  Heads h;
  h.B = c.B;
  h.H = c.H;
  h.h0 = c.h0;
  h.hn = c.hn;
  h.nclasses = c.nclasses;
  for (int p = 0; p < 2; ++p) {
    const int first = c.h0 + ((p - c.h0) & 1);
    const int end = c.h0 + c.hn;
    h.first[p] = first;
    h.per[p] = first < end ? (end - 1 - first) / 2 + 1 : 0;
    h.fper[p] = make_fastdiv(h.per[p]);
  }
  h.fhn = make_fastdiv(c.hn);
  h.fnh = make_fastdiv(heads_per_class(c));
  return h;
}

// Element types of tensor maps.
enum Elem : int { ELEM_BF16 = 0, ELEM_F16 = 1, ELEM_F32 = 2 };

// Encodes the natural (3-D), summary and residue-class (4-D) TMA views of a
// [B*H, T, d] tensor: 16-bit elements with 64-element boxes, or fp32 with
// 32-element boxes; 128-byte swizzle; 128-row boxes (in a layout that packs
// short residue classes, Geom::cpt > 1, the class view's box is one class of
// P rows). Views the layout lacks get a copy of the natural map (never used).
// Returns false if the driver rejects one.
bool make_view_maps(CUtensorMap out[3], const void* base, int elem, const Geom& g, int BH,
                    int d);

// Encodes the summary rows of one natural 128-row tile of an fp32 [B*H, T, d]
// tensor (the fixed pattern's last c rows of each l-block the tile covers,
// l dividing 128 or 128 dividing l): a 4-D map over (d, l, T / l, B*H) with a
// 32 x c x max(1, 128 / l) box, 128-byte swizzle. False when the layout has
// no summary view or the driver rejects it.
bool make_summary_rows_map(CUtensorMap* out, const void* base, const Geom& g, int BH, int d);

// Element type of a call's 16-bit tensors.
inline int elem16(const Call& c) { return c.dtype == ST_F16 ? ELEM_F16 : ELEM_BF16; }

}  // namespace st
