// Exact-fp32 path on CUDA cores, plus the backward prologue (fp32) and the
// prep / finish kernels around the bf16 tensor-core backward.
//
// The fp32 kernels walk the same schedule as the tensor-core kernels (work
// items of 128-row query or key tiles, each with its live tiles) and test
// membership with the segment rules on PARTIAL tiles. They exist for float32
// inputs, whose tolerance leaves no room for reduced-precision tensor-core
// arithmetic; one thread owns one query (forward, dQ) or one key (dK, dV).
//
// Attention over an allowed set and its normalisation: "Sparse Transformer"
// milestone page (nlp-lineage), "The notation"; llm-arch-kb section 2,
// "Sparse attention as an unnormalized form". Backward with the attention
// matrix recomputed from LSE: milestone page, "Recomputation".
#include <math.h>

#include <algorithm>

#include "device_common.cuh"
#include "launch.h"

namespace st {
namespace {

constexpr int kThreads = 128;

template <int D>
__device__ __forceinline__ float dot_smem(const float* a, const float* b) {
  float s = 0.f;
#pragma unroll
  for (int x = 0; x < D; ++x) s = fmaf(a[x], b[x], s);
  return s;
}

// smem: Ks[128][D+1], Vs[128][D+1], jpos[128]
template <class E, int D>
__global__ void __launch_bounds__(kThreads)
simt_fwd_kernel(Geom g, const FwdItem* __restrict__ items, const KeyEnt* __restrict__ keys,
                Heads hs, float scale, const E* __restrict__ q,
                const E* __restrict__ k, const E* __restrict__ v, E* __restrict__ o,
                float* __restrict__ lse) {
  extern __shared__ float sm[];
  float* Ks = sm;
  float* Vs = Ks + kTile * (D + 1);
  int* jpos = reinterpret_cast<int*>(Vs + kTile * (D + 1));
  const FwdItem it = items[blockIdx.y];
  const int bh = head_of(blockIdx.x, it.hclass, hs);
  if (bh < 0) return;
  const size_t base = (size_t)bh * g.T * D;
  const int tid = threadIdx.x;
  const int i = view_pos(g, it.qview, it.qtile, tid);
  float qr[D], acc[D];
#pragma unroll
  for (int x = 0; x < D; ++x) {
    qr[x] = (i >= 0) ? to_f32(q[base + (size_t)i * D + x]) * scale : 0.f;
    acc[x] = 0.f;
  }
  float m = -INFINITY, lsum = 0.f;
  for (int e = it.kbeg; e < it.kend; ++e) {
    const KeyEnt ke = keys[e];
    __syncthreads();
    for (int idx = tid; idx < kTile * D; idx += kThreads) {
      int r = idx / D, x = idx - r * D;
      int j = view_pos(g, ke.kview, ke.ktile, r);
      Ks[r * (D + 1) + x] = (j >= 0) ? to_f32(k[base + (size_t)j * D + x]) : 0.f;
      Vs[r * (D + 1) + x] = (j >= 0) ? to_f32(v[base + (size_t)j * D + x]) : 0.f;
    }
    jpos[tid] = view_pos(g, ke.kview, ke.ktile, tid);
    __syncthreads();
    if (i < 0) continue;
    for (int r = 0; r < kTile; ++r) {
      const int j = jpos[r];
      if (j < 0) continue;
      if (ke.flag != TILE_FULL && !rule_live(g, ke.rule, i, j)) continue;
      const float s = dot_smem<D>(qr, Ks + r * (D + 1));
      if (s > m) {
        const float corr = expf(m - s);
        lsum *= corr;
#pragma unroll
        for (int x = 0; x < D; ++x) acc[x] *= corr;
        m = s;
      }
      const float p = expf(s - m);
      lsum += p;
      const float* vr = Vs + r * (D + 1);
#pragma unroll
      for (int x = 0; x < D; ++x) acc[x] = fmaf(p, vr[x], acc[x]);
    }
  }
  if (i < 0) return;
  float L = (lsum > 0.f) ? m + logf(lsum) : -INFINITY;
  float w_cur = (lsum > 0.f) ? 1.f / lsum : 0.f;
  float w_prev = 0.f;
  const size_t orow = base + (size_t)i * D;
  if (it.merge) {
    const float Lp = lse[(size_t)bh * g.T + i];
    const float mx = fmaxf(Lp, L);
    if (mx == -INFINITY) {
      L = -INFINITY;
      w_cur = 0.f;
    } else {
      const float ep = expf(Lp - mx), ec = expf(L - mx);
      const float Ln = mx + logf(ep + ec);
      w_prev = expf(Lp - Ln);
      w_cur *= expf(L - Ln);
      L = Ln;
    }
  }
#pragma unroll
  for (int x = 0; x < D; ++x) {
    float val = acc[x] * w_cur;
    if (it.merge) val = fmaf(w_prev, to_f32(o[orow + x]), val);
    o[orow + x] = from_f32<E>(val);
  }
  lse[(size_t)bh * g.T + i] = L;
}

// Key-major dK, dV. smem: Ks, Vs (own rows), Qs, dOs [128][D+1]; lses, Ds, ipos [128].
template <class E, int D>
__global__ void __launch_bounds__(kThreads)
simt_bwd_kv_kernel(Geom g, const BwdItem* __restrict__ items, const QEnt* __restrict__ qents,
                   Heads hs, float scale, const E* __restrict__ q,
                   const E* __restrict__ k, const E* __restrict__ v, const float* __restrict__ lse,
                   const E* __restrict__ dout, const float* __restrict__ Dv,
                   float* __restrict__ dk_acc, float* __restrict__ dv_acc) {
  extern __shared__ float sm[];
  float* Ks = sm;
  float* Vs = Ks + kTile * (D + 1);
  float* Qs = Vs + kTile * (D + 1);
  float* dOs = Qs + kTile * (D + 1);
  float* lses = dOs + kTile * (D + 1);
  float* Ds = lses + kTile;
  int* ipos = reinterpret_cast<int*>(Ds + kTile);
  const BwdItem it = items[blockIdx.y];
  const int bh = head_of(blockIdx.x, it.hclass, hs);
  if (bh < 0) return;
  const size_t base = (size_t)bh * g.T * D;
  const size_t rbase = (size_t)bh * g.T;
  const int tid = threadIdx.x;
  const int j = view_pos(g, it.kview, it.ktile, tid);
  float* kr = Ks + tid * (D + 1);
  float* vr = Vs + tid * (D + 1);
  float dk[D], dv[D];
#pragma unroll
  for (int x = 0; x < D; ++x) {
    kr[x] = (j >= 0) ? to_f32(k[base + (size_t)j * D + x]) : 0.f;
    vr[x] = (j >= 0) ? to_f32(v[base + (size_t)j * D + x]) : 0.f;
    dk[x] = 0.f;
    dv[x] = 0.f;
  }
  for (int e = it.qbeg; e < it.qend; ++e) {
    const QEnt qe = qents[e];
    __syncthreads();
    for (int idx = tid; idx < kTile * D; idx += kThreads) {
      int r = idx / D, x = idx - r * D;
      int ii = view_pos(g, it.qview, qe.qtile, r);
      Qs[r * (D + 1) + x] = (ii >= 0) ? to_f32(q[base + (size_t)ii * D + x]) : 0.f;
      dOs[r * (D + 1) + x] = (ii >= 0) ? to_f32(dout[base + (size_t)ii * D + x]) : 0.f;
    }
    {
      int ii = view_pos(g, it.qview, qe.qtile, tid);
      ipos[tid] = ii;
      lses[tid] = (ii >= 0) ? lse[rbase + ii] : 0.f;
      Ds[tid] = (ii >= 0) ? Dv[rbase + ii] : 0.f;
    }
    __syncthreads();
    if (j < 0) continue;
    for (int r = 0; r < kTile; ++r) {
      const int ii = ipos[r];
      if (ii < 0) continue;
      if (qe.flag != TILE_FULL && !rule_live(g, it.rule, ii, j)) continue;
      const float* qr = Qs + r * (D + 1);
      const float* dor = dOs + r * (D + 1);
      const float s = scale * dot_smem<D>(qr, kr);
      const float p = expf(s - lses[r]);
      const float dp = dot_smem<D>(dor, vr);
      const float ds = p * (dp - Ds[r]) * scale;
#pragma unroll
      for (int x = 0; x < D; ++x) {
        dv[x] = fmaf(p, dor[x], dv[x]);
        dk[x] = fmaf(ds, qr[x], dk[x]);
      }
    }
  }
  if (j < 0) return;
#pragma unroll
  for (int x = 0; x < D; ++x) {
    atomicAdd(dk_acc + base + (size_t)j * D + x, dk[x]);
    atomicAdd(dv_acc + base + (size_t)j * D + x, dv[x]);
  }
}

// Query-major dQ over the forward schedule. smem: Ks, Vs [128][D+1], own Q and
// dO rows [128][D+1], jpos [128].
template <class E, int D>
__global__ void __launch_bounds__(kThreads)
simt_bwd_q_kernel(Geom g, const FwdItem* __restrict__ items, const KeyEnt* __restrict__ keys,
                  Heads hs, float scale, const E* __restrict__ q,
                  const E* __restrict__ k, const E* __restrict__ v,
                  const float* __restrict__ lse, const E* __restrict__ dout,
                  const float* __restrict__ Dv, float* __restrict__ dq_acc) {
  extern __shared__ float sm[];
  float* Ks = sm;
  float* Vs = Ks + kTile * (D + 1);
  float* Qo = Vs + kTile * (D + 1);
  float* dOo = Qo + kTile * (D + 1);
  int* jpos = reinterpret_cast<int*>(dOo + kTile * (D + 1));
  const FwdItem it = items[blockIdx.y];
  if (it.kbeg == it.kend) return;
  const int bh = head_of(blockIdx.x, it.hclass, hs);
  if (bh < 0) return;
  const size_t base = (size_t)bh * g.T * D;
  const int tid = threadIdx.x;
  const int i = view_pos(g, it.qview, it.qtile, tid);
  float* qr = Qo + tid * (D + 1);
  float* dor = dOo + tid * (D + 1);
  float dq[D];
#pragma unroll
  for (int x = 0; x < D; ++x) {
    qr[x] = (i >= 0) ? to_f32(q[base + (size_t)i * D + x]) : 0.f;
    dor[x] = (i >= 0) ? to_f32(dout[base + (size_t)i * D + x]) : 0.f;
    dq[x] = 0.f;
  }
  const float Li = (i >= 0) ? lse[(size_t)bh * g.T + i] : 0.f;
  const float Di = (i >= 0) ? Dv[(size_t)bh * g.T + i] : 0.f;
  for (int e = it.kbeg; e < it.kend; ++e) {
    const KeyEnt ke = keys[e];
    __syncthreads();
    for (int idx = tid; idx < kTile * D; idx += kThreads) {
      int r = idx / D, x = idx - r * D;
      int j = view_pos(g, ke.kview, ke.ktile, r);
      Ks[r * (D + 1) + x] = (j >= 0) ? to_f32(k[base + (size_t)j * D + x]) : 0.f;
      Vs[r * (D + 1) + x] = (j >= 0) ? to_f32(v[base + (size_t)j * D + x]) : 0.f;
    }
    jpos[tid] = view_pos(g, ke.kview, ke.ktile, tid);
    __syncthreads();
    if (i < 0) continue;
    for (int r = 0; r < kTile; ++r) {
      const int j = jpos[r];
      if (j < 0) continue;
      if (ke.flag != TILE_FULL && !rule_live(g, ke.rule, i, j)) continue;
      const float* kr = Ks + r * (D + 1);
      const float s = scale * dot_smem<D>(qr, kr);
      const float p = expf(s - Li);
      const float dp = dot_smem<D>(dor, Vs + r * (D + 1));
      const float ds = p * (dp - Di);
#pragma unroll
      for (int x = 0; x < D; ++x) dq[x] = fmaf(ds, kr[x], dq[x]);
    }
  }
  if (i < 0) return;
#pragma unroll
  for (int x = 0; x < D; ++x) atomicAdd(dq_acc + base + (size_t)i * D + x, dq[x] * scale);
}

// One warp per row: D_i = sum_x dout_ix * o_ix; then the accumulators are zeroed.
template <class E>
__global__ void prologue_kernel(const E* __restrict__ o, const E* __restrict__ dout,
                                float* __restrict__ Dv, size_t rows, int d,
                                float4* __restrict__ acc, size_t acc_vec) {
  const int lane = threadIdx.x & 31;
  const size_t warp = (blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 5;
  const size_t nwarps = (gridDim.x * (size_t)blockDim.x) >> 5;
  for (size_t r = warp; r < rows; r += nwarps) {
    float s = 0.f;
    for (int x = lane; x < d; x += 32) s = fmaf(to_f32(dout[r * d + x]), to_f32(o[r * d + x]), s);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0) Dv[r] = s;
  }
  const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
  for (size_t t = blockIdx.x * (size_t)blockDim.x + threadIdx.x; t < acc_vec;
       t += gridDim.x * (size_t)blockDim.x)
    acc[t] = z;
}

// Segments of the accumulated rows, per head class: [hc][0] dQ rows,
// [hc][1] dK / dV rows (see RowSeg).
struct SegSet {
  const RowSeg* segs[2][2];
  int32_t n[2][2];
};

// Segment list k of head class hc, picked without dynamic indexing of the
// parameter (which would copy it to local memory).
__device__ __forceinline__ const RowSeg* segs_of(const SegSet& ss, int hc, int k, int& n) {
  if (hc) {
    n = k ? ss.n[1][1] : ss.n[1][0];
    return k ? ss.segs[1][1] : ss.segs[1][0];
  }
  n = k ? ss.n[0][1] : ss.n[0][0];
  return k ? ss.segs[0][1] : ss.segs[0][0];
}

SegSet seg_set_of(const st_layout* L) {
  SegSet r;
  for (int hc = 0; hc < 2; ++hc)
    for (int k = 0; k < 2; ++k) {
      r.segs[hc][k] = (const RowSeg*)L->dev.segs[hc][k];
      r.n[hc][k] = L->dev.n_segs[hc][k];
    }
  return r;
}

// Flat head index of the y-th selected head (heads h0 .. h0+hn-1 of every
// batch entry).
__device__ __forceinline__ int sel_head(int y, const Heads& hs) {
  const int b = fdiv(y, hs.fhn);
  return b * hs.H + hs.h0 + (y - b * hs.hn);
}

// Dot product of eight 16-bit values (fp16 if F16, else bf16), in fp32.
template <bool F16>
__device__ __forceinline__ float dot8(const uint4& a, const uint4& b) {
  const uint32_t* x = reinterpret_cast<const uint32_t*>(&a);
  const uint32_t* y = reinterpret_cast<const uint32_t*>(&b);
  float s = 0.f;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    float2 u, v;
    if constexpr (F16) {
      u = __half22float2(*reinterpret_cast<const __half2*>(&x[k]));
      v = __half22float2(*reinterpret_cast<const __half2*>(&y[k]));
    } else {
      u = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&x[k]));
      v = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&y[k]));
    }
    s = fmaf(u.x, v.x, s);
    s = fmaf(u.y, v.y, s);
  }
  return s;
}

// Largest |x| of eight bf16 values, as a bf16 bit pattern (the magnitude
// bits of a bf16 order like the values for every non-NaN input).
__device__ __forceinline__ uint32_t absmax8_bf16(const uint4& a) {
  const uint32_t m = 0x7fff7fffu;
  const uint32_t x = __vmaxu2(__vmaxu2(a.x & m, a.y & m), __vmaxu2(a.z & m, a.w & m));
  return max(x & 0xffffu, x >> 16);
}

// Backward prologue of the 16-bit path (rows of d = 64 16-bit values, 128
// bytes). Its work comes in items of one warp, dealt round robin: for every
// selected head, D_i = dout_i . O_i of its rows in blocks of 16, then its
// accumulated dQ row segments and dK / dV row segments, zeroed. Each item is
// one contiguous run of memory with all of a lane's loads in flight at once
// (8 of 16 bytes for D), so the kernel streams. Also zeroes the backward
// kernel's work counter and (bf16) writes the largest |dout| the block read
// into slots[blockIdx.x], from which the backward kernel takes the
// power-of-two scale of its fp16 copy of dout.
// Rows of a D item per group of eight lanes (items of 16 rows: more, smaller
// items balance the warps better than 32-row ones did at T = 12288).
constexpr int kDU = 4;

template <bool F16>
__global__ void __launch_bounds__(256, 3)
bwd_prep_kernel(const uint4* __restrict__ o, const uint4* __restrict__ dout,
                float* __restrict__ Dv, int T, Heads hs, SegSet ss, int maxq, int maxk,
                float4* __restrict__ dq_acc, float4* __restrict__ dk_acc,
                float4* __restrict__ dv_acc, int* __restrict__ sched_counter,
                float* __restrict__ slots) {
  if (blockIdx.x == 0 && threadIdx.x == 0) *sched_counter = 0;
  const int lane = threadIdx.x & 31, sub = lane & 7;
  constexpr int kDRows = 4 * kDU;  // rows of one D item
  const int rblocks = T / kDRows;  // T is a multiple of 128
  const int per_head = rblocks + maxq + maxk;
  const long long items = (long long)hs.B * hs.hn * per_head;
  const int nw = (int)((gridDim.x * blockDim.x) >> 5);
  const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
  uint32_t amax = 0;  // bf16 bits of the largest |dout| this thread read
  for (long long w = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; w < items; w += nw) {
    const int y = (int)(w / per_head);
    const int k = (int)(w - (long long)y * per_head);
    const int bh = sel_head(y, hs);
    const size_t rb = (size_t)bh * T;
    if (k < rblocks) {
      // rows kDRows k .. kDRows (k+1) - 1: eight lanes per row (one 16-byte
      // chunk each), rows (lane >> 3) + 4u for u < kDU
      const size_t r0 = rb + kDRows * (size_t)k;
      uint4 a[kDU], b[kDU];
#pragma unroll
      for (int u = 0; u < kDU; ++u) {
        const size_t at = (r0 + (lane >> 3) + 4 * u) * 8 + sub;
        a[u] = __ldg(o + at);
        b[u] = __ldg(dout + at);
      }
#pragma unroll
      for (int u = 0; u < kDU; ++u) {
        if constexpr (!F16) amax = max(amax, absmax8_bf16(b[u]));
        float sacc = dot8<F16>(a[u], b[u]);
        sacc += __shfl_xor_sync(0xffffffffu, sacc, 4);
        sacc += __shfl_xor_sync(0xffffffffu, sacc, 2);
        sacc += __shfl_xor_sync(0xffffffffu, sacc, 1);
        if (sub == 0) Dv[r0 + (lane >> 3) + 4 * u] = sacc;
      }
    } else {
      const int kk = k - rblocks;
      const int isk = kk >= maxq ? 1 : 0;
      int n;
      const RowSeg* sg = segs_of(ss, class_of(bh, hs), isk, n);
      const int si = isk ? kk - maxq : kk;
      if (si >= n) continue;
      const RowSeg seg = sg[si];
      const size_t e0 = (rb + seg.start) * 16;  // float4 index of the segment's first row
      const int ne = seg.len * 16;
      if (isk) {
        for (int x = lane; x < ne; x += 32) {
          dk_acc[e0 + x] = z4;
          dv_acc[e0 + x] = z4;
        }
      } else {
        for (int x = lane; x < ne; x += 32) dq_acc[e0 + x] = z4;
      }
    }
  }
  // the block's largest |dout|: warp, then block (bf16 bits widen to fp32 bits)
  __shared__ uint32_t wmax[32];
  amax = __reduce_max_sync(0xffffffffu, amax);
  if (lane == 0) wmax[threadIdx.x >> 5] = amax;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t m = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) m = max(m, wmax[w]);
    slots[blockIdx.x] = __uint_as_float(m << 16);
  }
}

template <bool F16>
__device__ __forceinline__ uint32_t round2(float lo, float hi) {
  if constexpr (F16) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
  } else {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
  }
}

template <bool F16>
__device__ __forceinline__ uint4 round8f(const float4& a, const float4& b, float s) {
  return make_uint4(round2<F16>(a.x * s, a.y * s), round2<F16>(a.z * s, a.w * s),
                    round2<F16>(b.x * s, b.y * s), round2<F16>(b.z * s, b.w * s));
}

// Rounds the accumulated rows into the 16-bit outputs: items of one warp,
// one row segment of one selected head each (dQ segments first, then dK / dV
// segments), with a lane's 16 loads of 16 bytes in flight at once. dQ and dK
// take the softmax scale; dV partials carry the factor 2^e of the backward's
// fp16 dout (from the prologue's slots; nslots = 0 means e = 0).
// One row segment of an accumulator rounded into a 16-bit output, by one
// warp: float4 pair p (eight elements, one 16-byte output) for p = lane +
// 32 i, all loads in flight before the first store.
template <bool F16>
__device__ __forceinline__ void round_seg(const float4* __restrict__ acc, uint4* __restrict__ out,
                                          size_t p0, int np, float sc, int lane) {
  float4 a[8], b[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int p = lane + 32 * i;
    a[i] = b[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (p < np) {
      a[i] = __ldg(acc + 2 * (p0 + p));
      b[i] = __ldg(acc + 2 * (p0 + p) + 1);
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i)
    if (lane + 32 * i < np) out[p0 + lane + 32 * i] = round8f<F16>(a[i], b[i], sc);
}

template <bool F16>
__global__ void __launch_bounds__(256, 2)
bwd_finish_kernel(const float4* __restrict__ dq_acc, const float4* __restrict__ dk_acc,
                  const float4* __restrict__ dv_acc, int T, Heads hs, SegSet ss, int maxq,
                  int maxk, float scale, const float* __restrict__ slots, int nslots,
                  uint4* __restrict__ dq, uint4* __restrict__ dk, uint4* __restrict__ dv) {
  __shared__ float bmax[32];
  float m = 0.f;
  for (int x = threadIdx.x; x < nslots; x += blockDim.x) m = fmaxf(m, __ldg(slots + x));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  if ((threadIdx.x & 31) == 0) bmax[threadIdx.x >> 5] = m;
  __syncthreads();
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, bmax[w]);
  const float dv_scale = pow2f(-dout_exp(m));
  const int lane = threadIdx.x & 31;
  const int per_head = maxq + maxk;
  const long long items = (long long)hs.B * hs.hn * per_head;
  const int nw = (int)((gridDim.x * blockDim.x) >> 5);
  for (long long w = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; w < items; w += nw) {
    const int y = (int)(w / per_head);
    const int k = (int)(w - (long long)y * per_head);
    const int bh = sel_head(y, hs);
    const int isk = k >= maxq ? 1 : 0;
    int n;
    const RowSeg* sg = segs_of(ss, class_of(bh, hs), isk, n);
    const int si = isk ? k - maxq : k;
    if (si >= n) continue;
    const RowSeg seg = sg[si];
    const size_t p0 = ((size_t)bh * T + seg.start) * 8;
    const int np = seg.len * 8;  // at most 256: eight per lane
    if (isk) {
      round_seg<F16>(dk_acc, dk, p0, np, scale, lane);
      round_seg<F16>(dv_acc, dv, p0, np, dv_scale, lane);
    } else {
      round_seg<F16>(dq_acc, dq, p0, np, scale, lane);
    }
  }
}

int grid_cap(size_t work, int per_block) {
  size_t b = (work + per_block - 1) / per_block;
  if (b > 148 * 16) b = 148 * 16;
  if (b < 1) b = 1;
  return (int)b;
}

template <class E, int D>
cudaError_t simt_fwd_t(const Call& c, const void* q, const void* k, const void* v, void* o,
                       float* lse) {
  const st_layout* L = c.L;
  size_t smem = sizeof(float) * 2 * kTile * (D + 1) + sizeof(int) * kTile;
  auto kern = simt_fwd_kernel<E, D>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
  if (err != cudaSuccess) return err;
  record_begin(c);
  for (int pass = 0; pass < L->n_passes; ++pass) {
    int n = L->dev.n_fwd_items[pass];
    if (n == 0) continue;
    dim3 grid(heads_per_class(c), n);
    kern<<<grid, kThreads, smem, c.stream>>>(
        L->geom, (const FwdItem*)L->dev.fwd_items[pass], (const KeyEnt*)L->dev.key_ents,
        heads_of(c), c.scale, (const E*)q, (const E*)k, (const E*)v, (E*)o, lse);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  record_end(c);
  return cudaSuccess;
}

template <class E, int D>
cudaError_t simt_bwd_t(const Call& c, const void* q, const void* k, const void* v,
                       const float* lse, const void* dout, const float* Dv, float* dq_acc,
                       float* dk_acc, float* dv_acc) {
  const st_layout* L = c.L;
  size_t smem_kv = sizeof(float) * (4 * kTile * (D + 1) + 2 * kTile) + sizeof(int) * kTile;
  size_t smem_q = sizeof(float) * 4 * kTile * (D + 1) + sizeof(int) * kTile;
  auto kv = simt_bwd_kv_kernel<E, D>;
  auto kq = simt_bwd_q_kernel<E, D>;
  cudaError_t err =
      cudaFuncSetAttribute(kv, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_kv);
  if (err != cudaSuccess) return err;
  err = cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_q);
  if (err != cudaSuccess) return err;
  record_begin(c);
  if (L->dev.n_bwd_items > 0) {
    dim3 grid(heads_per_class(c), L->dev.n_bwd_items);
    kv<<<grid, kThreads, smem_kv, c.stream>>>(
        L->geom, (const BwdItem*)L->dev.bwd_items, (const QEnt*)L->dev.q_ents,
        heads_of(c), c.scale, (const E*)q, (const E*)k, (const E*)v, lse, (const E*)dout, Dv,
        dk_acc, dv_acc);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  for (int pass = 0; pass < L->n_passes; ++pass) {
    int n = L->dev.n_fwd_items[pass];
    if (n == 0) continue;
    dim3 grid(heads_per_class(c), n);
    kq<<<grid, kThreads, smem_q, c.stream>>>(
        L->geom, (const FwdItem*)L->dev.fwd_items[pass], (const KeyEnt*)L->dev.key_ents,
        heads_of(c), c.scale, (const E*)q, (const E*)k, (const E*)v, lse, (const E*)dout,
        Dv, dq_acc);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  record_end(c);
  return cudaSuccess;
}

}  // namespace

cudaError_t simt_fwd(const Call& c, const void* q, const void* k, const void* v, void* o,
                     float* lse) {
  if (c.dtype == ST_F32) {
    if (c.d == 32) return simt_fwd_t<float, 32>(c, q, k, v, o, lse);
    if (c.d == 64) return simt_fwd_t<float, 64>(c, q, k, v, o, lse);
  }
  return cudaErrorInvalidValue;
}

cudaError_t simt_bwd(const Call& c, const void* q, const void* k, const void* v,
                     const float* lse, const void* dout, const float* Dv, float* dq_acc,
                     float* dk_acc, float* dv_acc) {
  if (c.dtype == ST_F32) {
    if (c.d == 32)
      return simt_bwd_t<float, 32>(c, q, k, v, lse, dout, Dv, dq_acc, dk_acc, dv_acc);
    if (c.d == 64)
      return simt_bwd_t<float, 64>(c, q, k, v, lse, dout, Dv, dq_acc, dk_acc, dv_acc);
  }
  return cudaErrorInvalidValue;
}

cudaError_t bwd_prologue(const Call& c, const void* o, const void* dout, float* Dv, float* acc,
                         size_t acc_elems) {
  size_t rows = (size_t)c.B * c.H * c.L->geom.T;
  int threads = 256;
  int blocks = grid_cap(rows * 32 > acc_elems / 4 ? rows * 32 : acc_elems / 4, threads);
  if (c.dtype != ST_F32) return cudaErrorInvalidValue;  // 16-bit calls use bwd_prep
  prologue_kernel<float><<<blocks, threads, 0, c.stream>>>(
      (const float*)o, (const float*)dout, Dv, rows, c.d, (float4*)acc, acc_elems / 4);
  return cudaGetLastError();
}

// Largest segment counts over the head classes: dQ rows, dK / dV rows.
void max_segs(const st_layout* L, int& maxq, int& maxk) {
  maxq = maxk = 0;
  for (int hc = 0; hc < (int)L->hcs.size(); ++hc) {
    maxq = std::max(maxq, L->dev.n_segs[hc][0]);
    maxk = std::max(maxk, L->dev.n_segs[hc][1]);
  }
}

// Blocks of 8 warps for `items` warp items, at most `cap`.
int warp_grid(long long items, int cap) {
  return (int)std::max<long long>(1, std::min<long long>((items + 7) / 8, cap));
}

cudaError_t bwd_prep(const Call& c, const void* o, const void* dout, float* Dv, float* dq_acc,
                     float* dk_acc, float* dv_acc, int* sched_counter, float* slots,
                     int* nslots) {
  const int T = c.L->geom.T;
  int maxq, maxk;
  max_segs(c.L, maxq, maxk);
  const long long items = (long long)c.B * c.hn * (T / (4 * kDU) + maxq + maxk);
  const int grid = warp_grid(items, std::min(kDoutSlots, sm_count() * 3));
  *nslots = grid;
  auto kern = (c.dtype == ST_F16) ? bwd_prep_kernel<true> : bwd_prep_kernel<false>;
  kern<<<grid, 256, 0, c.stream>>>((const uint4*)o, (const uint4*)dout, Dv, T, heads_of(c),
                                   seg_set_of(c.L), maxq, maxk, (float4*)dq_acc,
                                   (float4*)dk_acc, (float4*)dv_acc, sched_counter, slots);
  return cudaGetLastError();
}

cudaError_t bwd_finish(const Call& c, const float* dq_acc, const float* dk_acc,
                       const float* dv_acc, const float* slots, int nslots, void* dq, void* dk,
                       void* dv) {
  const st_layout* L = c.L;
  int maxq, maxk;
  max_segs(L, maxq, maxk);
  if (maxq + maxk == 0) return cudaSuccess;  // every row was written directly
  const long long items = (long long)c.B * c.hn * (maxq + maxk);
  const int grid = warp_grid(items, sm_count() * 2);
  auto kern = (c.dtype == ST_F16) ? bwd_finish_kernel<true> : bwd_finish_kernel<false>;
  kern<<<grid, 256, 0, c.stream>>>(
      (const float4*)dq_acc, (const float4*)dk_acc, (const float4*)dv_acc, L->geom.T,
      heads_of(c), seg_set_of(L), maxq, maxk, c.scale, slots, c.dtype == ST_F16 ? 0 : nslots,
      (uint4*)dq, (uint4*)dk, (uint4*)dv);
  return cudaGetLastError();
}

}  // namespace st
