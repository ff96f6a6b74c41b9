// Device helpers shared by every kernel of the library: view-row mapping,
// the membership rules of the segments, and the device status word.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "st_internal.h"

namespace st {

// floor(n / d) for 0 <= n < 2^31, with f = make_fastdiv(d).
__device__ __forceinline__ int fdiv(int n, FastDiv f) {
  const uint32_t t = __umulhi(f.m, (uint32_t)n);
  return (int)((t + (uint32_t)n) >> f.s);
}

// Natural position of row k of tile `tile` in view v; -1 for padding rows.
__device__ __forceinline__ int view_pos(const Geom& g, int v, int tile, int k) {
  if (v == VIEW_NAT) {
    int t = tile * kTile + k;
    return t < g.T ? t : -1;
  }
  if (v == VIEW_SUM) {
    int s = tile * kTile + k;
    if (s >= g.nsum) return -1;
    const int q = fdiv(s, g.fc);
    return q * g.l + (g.l - g.c) + (s - q * g.c);
  }
  // class view: view row y = r * cw + p
  const int y = tile * kTile + k;
  const int r = fdiv(y, g.fcw), p = y - r * g.cw;
  if (p >= g.P || r >= g.l) return -1;
  return p * g.l + r;
}

// Membership of the pair (i, j), natural positions, in a segment rule. The
// rules restate the index sets: strided window / stride, fixed block /
// summary positions ("Sparse Transformer", llm-arch-kb, section 2).
__device__ __forceinline__ bool rule_live(const Geom& g, int rule, int i, int j) {
  if (i < 0 || j < 0 || j > i) return false;
  const int l = g.l, c = g.c;
  switch (rule) {
    case RULE_CAUSAL:
      return true;
    case RULE_BAND:
      return j >= i - l;
    case RULE_BLOCK:
      return j / l == i / l;
    case RULE_STRIDE:
      return (i - j) % l == 0;
    case RULE_STRIDE_FAR:
      return (i - j) % l == 0 && i - j >= 2 * l;
    case RULE_SUMMARY:
      return j % l >= l - c;
    case RULE_SUMMARY_EARLIER:
      return j % l >= l - c && j / l < i / l;
    default:
      return false;
  }
}

// Head index bh = b*H + h of grid column x for a head class: split mode puts
// even heads in class 0 and odd heads in class 1. Returns -1 past the end.
// Flat index of the x-th head of class hclass among the heads h0 .. h0+hn-1
// of a [B, H, T, d] tensor, or -1 past the end. Split layouts give class p
// the heads of parity p (global head index, so a head range keeps each head's
// set); merged layouts have one class.
__device__ __forceinline__ int head_of(int x, int hclass, const Heads& hs) {
  if (hs.nclasses == 1) {
    if (x >= hs.B * hs.hn) return -1;
    const int b = fdiv(x, hs.fhn);
    return b * hs.H + hs.h0 + (x - b * hs.hn);
  }
  const int per = hclass ? hs.per[1] : hs.per[0];
  if (per == 0 || x >= hs.B * per) return -1;
  const int b = fdiv(x, hclass ? hs.fper[1] : hs.fper[0]);
  return b * hs.H + (hclass ? hs.first[1] : hs.first[0]) + 2 * (x - b * per);
}

// Head class of flat head index bh (0 for merged layouts).
__device__ __forceinline__ int class_of(int bh, const Heads& hs) {
  return hs.nclasses == 2 ? ((bh % hs.H) & 1) : 0;
}

// The backward pass of the 16-bit path forms dV from P and dout rounded to
// fp16 (three more significant bits for P than bf16 gives). dout enters that
// product as dout * 2^e, with e chosen from m = max |dout| so that
// m * 2^e lies in [2^13, 2^14): far from fp16 overflow, and every bf16 value
// within 2^27 of m keeps all its bits. e = 0 for m = 0 (or not finite).
__device__ __forceinline__ int dout_exp(float m) {
  if (!(m > 0.f) || !(m < INFINITY)) return 0;
  const int E = (int)((__float_as_uint(m) >> 23) & 0xffu);  // m in [2^(E-127), 2^(E-126))
  return max(-100, min(100, 140 - E));
}
// 2^e for -126 <= e <= 127.
__device__ __forceinline__ float pow2f(int e) { return __uint_as_float((uint32_t)(127 + e) << 23); }

__device__ __forceinline__ void set_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <class T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) {
  return x;
}
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

}  // namespace st
