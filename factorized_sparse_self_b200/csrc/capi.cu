// C ABI of libsparse_transformer_attn.so: argument checks, layout upload and
// export, and the forward / backward call sequences. See
// include/sparse_transformer_attn.h for the contract of every entry point.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "launch.h"

using namespace st;

namespace {

constexpr uint64_t kDefaultWaitNs = 2000000000ull;
// Process-wide, read by every later launch from any host thread.
std::atomic<uint64_t> g_wait_ns{kDefaultWaitNs};
std::atomic<int> g_force_timeout{0};

constexpr int kMaxDevices = 64;
int* g_status[kMaxDevices] = {nullptr};
std::mutex g_mu;

// Device status word of the current device (allocated on first use, which
// is always inside st_pattern_layout, never inside fwd/bwd).
int* status_word(int dev, bool create) {
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_status[dev] && create) {
    int* p = nullptr;
    if (cudaMalloc(&p, sizeof(int)) != cudaSuccess) return nullptr;
    if (cudaMemset(p, 0, sizeof(int)) != cudaSuccess) {
      cudaFree(p);
      return nullptr;
    }
    g_status[dev] = p;
  }
  return g_status[dev];
}

template <class T>
cudaError_t upload(void** dst, const std::vector<T>& src, cudaStream_t s) {
  *dst = nullptr;
  size_t bytes = std::max<size_t>(sizeof(T), src.size() * sizeof(T));
  cudaError_t e = cudaMalloc(dst, bytes);
  if (e != cudaSuccess) return e;
  if (!src.empty()) e = cudaMemcpyAsync(*dst, src.data(), src.size() * sizeof(T),
                                        cudaMemcpyHostToDevice, s);
  return e;
}

void free_device(st_layout* L) {
  if (!L->on_device) return;
  int prev = -1;
  cudaGetDevice(&prev);
  cudaSetDevice(L->device);
  for (int p = 0; p < 2; ++p) cudaFree(L->dev.fwd_items[p]);
  cudaFree(L->dev.key_ents);
  cudaFree(L->dev.bwd_items);
  for (int f = 1; f < 3; ++f) cudaFree(L->dev.bwd_split[f]);
  cudaFree(L->dev.sched_slots);
  cudaFree(L->dev.q_ents);
  for (int hc = 0; hc < 2; ++hc) {
    for (int k = 0; k < N_ROWLISTS; ++k) cudaFree(L->dev.rows[hc][k]);
    for (int k = 0; k < 2; ++k) cudaFree(L->dev.segs[hc][k]);
  }
  if (prev >= 0) cudaSetDevice(prev);
  L->on_device = false;
}

bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Common checks of fwd / bwd. Returns ST_OK and fills the call on success.
st_status prepare(const st_layout* L, st_dtype dtype, int32_t B, int32_t H, int32_t h0, int32_t hn,
                  int32_t T, int32_t d, float scale, void* stream, Call& c) {
  if (!L || !L->on_device) return ST_ERR_INVALID;
  if (dtype != ST_F32 && dtype != ST_BF16 && dtype != ST_F16) return ST_ERR_INVALID;
  if (B < 1 || H < 1 || d < 1 || T != L->geom.T) return ST_ERR_INVALID;
  if (h0 < 0 || hn < 1 || (int64_t)h0 + hn > H) return ST_ERR_INVALID;
  if ((int64_t)B * H > (1 << 30) || (int64_t)B * H * T * d > (int64_t)1 << 40) return ST_ERR_INVALID;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return ST_ERR_CUDA;
  if (dev != L->device) return ST_ERR_INVALID;
  if (dtype == ST_F32) {
    if (d != 32 && d != 64) return ST_ERR_UNSUPPORTED;
  } else {
    if (d != 64) return ST_ERR_UNSUPPORTED;
    if (T % kTile != 0 || !L->tc_ok) return ST_ERR_UNSUPPORTED;
  }
  int nclasses = (int)L->hcs.size();
  if ((int64_t)B * hn > 2147483647 / 2) return ST_ERR_UNSUPPORTED;
  for (int p = 0; p < L->n_passes; ++p)
    if (L->dev.n_fwd_items[p] > 65535) return ST_ERR_UNSUPPORTED;
  if (L->dev.n_bwd_items > 65535) return ST_ERR_UNSUPPORTED;
  c.L = L;
  c.dtype = dtype;
  c.B = B;
  c.H = H;
  c.h0 = h0;
  c.hn = hn;
  c.d = d;
  c.scale = (scale > 0.f) ? scale : 1.0f / sqrtf((float)d);
  c.nclasses = nclasses;
  c.status = status_word(dev, false);
  c.wait_ns = g_wait_ns.load();
  c.stream = reinterpret_cast<cudaStream_t>(stream);
  if (!c.status) return ST_ERR_CUDA;
  return ST_OK;
}

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

// Benchmark instrumentation (st_kernel_timing).
// Kernels with a pair of events: 0 forward attention launches, 1 backward
// main kernel, 2 backward prologue, 3 backward epilogue.
constexpr int kTimed = 4;
bool g_timing = false;
cudaEvent_t g_ev[kTimed][2] = {};
bool g_ev_used[kTimed] = {};

// Hands the benchmark events of `kernel` to a call (when timing is on).
void arm(Call& c, int kernel) {
  if (!g_timing) return;
  c.ev_begin = g_ev[kernel][0];
  c.ev_end = g_ev[kernel][1];
  g_ev_used[kernel] = true;
}

}  // namespace

extern "C" {

const char* st_version(void) { return "0.1.0"; }

const char* st_status_string(st_status s) {
  switch (s) {
    case ST_OK: return "ok";
    case ST_ERR_INVALID: return "invalid argument";
    case ST_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case ST_ERR_CUDA: return "CUDA error";
    case ST_ERR_DEVICE_TIMEOUT: return "on-device wait timed out";
    case ST_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

st_status st_pattern_layout_host(const st_pattern_desc* desc, st_layout** out) {
  if (!desc || !out) return ST_ERR_INVALID;
  *out = nullptr;
  st_layout* L = new (std::nothrow) st_layout();
  if (!L) return ST_ERR_INVALID;
  st_status s = build_layout(desc, L);
  if (s != ST_OK) {
    delete L;
    return s;
  }
  *out = L;
  return ST_OK;
}

st_status st_pattern_layout(const st_pattern_desc* desc, st_layout** out, void* stream) {
  st_layout* L = nullptr;
  st_status s = st_pattern_layout_host(desc, &L);
  if (s != ST_OK) return s;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || !status_word(dev, true)) {
    delete L;
    return ST_ERR_CUDA;
  }
  L->device = dev;
  L->on_device = true;
  cudaError_t e = cudaSuccess;
  for (int p = 0; p < 2 && e == cudaSuccess; ++p) {
    e = upload(&L->dev.fwd_items[p], L->fwd_items[p], cs);
    L->dev.n_fwd_items[p] = (int32_t)L->fwd_items[p].size();
  }
  if (e == cudaSuccess) e = upload(&L->dev.key_ents, L->key_ents, cs);
  if (e == cudaSuccess) e = upload(&L->dev.bwd_items, L->bwd_items, cs);
  if (e == cudaSuccess) e = upload(&L->dev.q_ents, L->q_ents, cs);
  L->dev.n_bwd_items = (int32_t)L->bwd_items.size();
  L->dev.bwd_split[0] = L->dev.bwd_items;
  L->dev.n_bwd_split[0] = L->dev.n_bwd_items;
  for (int f = 1; f < 3 && e == cudaSuccess; ++f) {
    e = upload(&L->dev.bwd_split[f], L->bwd_split[f - 1], cs);
    L->dev.n_bwd_split[f] = (int32_t)L->bwd_split[f - 1].size();
  }
  for (int f = 0; f < 3; ++f) {
    const std::vector<BwdItem>& v = f == 0 ? L->bwd_items : L->bwd_split[f - 1];
    L->dev.max_split_len[f] = v.empty() ? 0 : v.front().qend - v.front().qbeg;
  }
  L->dev.q_ents_total = (int64_t)L->q_ents.size();
  if (e == cudaSuccess)
    e = cudaMalloc(reinterpret_cast<void**>(&L->dev.sched_slots),
                   2 * kSchedSlots * sizeof(int32_t));
  if (e == cudaSuccess)
    e = cudaMemsetAsync(L->dev.sched_slots, 0, 2 * kSchedSlots * sizeof(int32_t), cs);
  for (int hc = 0; hc < (int)L->hcs.size() && e == cudaSuccess; ++hc)
    for (int k = 0; k < N_ROWLISTS && e == cudaSuccess; ++k) {
      e = upload(&L->dev.rows[hc][k], L->rows[hc][k], cs);
      L->dev.n_rows[hc][k] = (int32_t)L->rows[hc][k].size();
    }
  for (int hc = 0; hc < (int)L->hcs.size() && e == cudaSuccess; ++hc)
    for (int k = 0; k < 2 && e == cudaSuccess; ++k) {
      e = upload(&L->dev.segs[hc][k], L->segs[hc][k], cs);
      L->dev.n_segs[hc][k] = (int32_t)L->segs[hc][k].size();
    }
  if (e == cudaSuccess) e = cudaStreamSynchronize(cs);
  if (e != cudaSuccess) {
    free_device(L);
    delete L;
    return ST_ERR_CUDA;
  }
  *out = L;
  return ST_OK;
}

void st_layout_destroy(st_layout* L) {
  if (!L) return;
  free_device(L);
  delete L;
}

st_status st_layout_counts(const st_layout* L, int32_t* nhc, int32_t* nseg) {
  if (!L) return ST_ERR_INVALID;
  if (nhc) *nhc = (int32_t)L->hcs.size();
  if (nseg) *nseg = (int32_t)L->hcs[0].segs.size();
  return ST_OK;
}

st_status st_layout_segment_info(const st_layout* L, int32_t hc, int32_t seg, int32_t* qv,
                                 int32_t* kv, int32_t* rule) {
  if (!L || hc < 0 || hc >= (int32_t)L->hcs.size()) return ST_ERR_INVALID;
  const HeadClass& H = L->hcs[(size_t)hc];
  if (seg < 0 || seg >= (int32_t)H.segs.size()) return ST_ERR_INVALID;
  if (qv) *qv = H.segs[(size_t)seg].qview;
  if (kv) *kv = H.segs[(size_t)seg].kview;
  if (rule) *rule = H.segs[(size_t)seg].rule;
  return ST_OK;
}

st_status st_layout_nnz(const st_layout* L, int32_t hc, int64_t* nnz) {
  if (!L || !nnz || hc < 0 || hc >= (int32_t)L->hcs.size()) return ST_ERR_INVALID;
  *nnz = L->hcs[(size_t)hc].nnz;
  return ST_OK;
}

st_status st_layout_rows(const st_layout* L, int32_t hc, int32_t list, int32_t* rows,
                         int64_t* count) {
  if (!L || !count || hc < 0 || hc >= (int32_t)L->hcs.size() || list < 0 ||
      list >= N_ROWLISTS)
    return ST_ERR_INVALID;
  const std::vector<int32_t>& r = L->rows[hc][list];
  const int64_t cap = *count;
  *count = (int64_t)r.size();
  if (!rows) return ST_OK;
  if (cap < (int64_t)r.size()) return ST_ERR_WORKSPACE;
  if (!r.empty()) std::memcpy(rows, r.data(), sizeof(int32_t) * r.size());
  return ST_OK;
}

st_status st_layout_export(const st_layout* L, int32_t hc, int32_t seg, int32_t transpose,
                           int32_t* ptr, int32_t* idx, uint8_t* flags, int32_t* live,
                           int64_t* sizes) {
  if (!L || !sizes || hc < 0 || hc >= (int32_t)L->hcs.size()) return ST_ERR_INVALID;
  const HeadClass& H = L->hcs[(size_t)hc];
  if (seg < -1 || seg >= (int32_t)H.segs.size()) return ST_ERR_INVALID;
  std::vector<Tile> nat;
  const std::vector<Tile>* tiles;
  int32_t nq, nk;
  if (seg == -1) {
    natural_tiles(L, hc, nat);
    tiles = &nat;
    nq = nk = (L->geom.T + kTile - 1) / kTile;
  } else {
    tiles = &H.segs[(size_t)seg].tiles;
    nq = H.segs[(size_t)seg].nq;
    nk = H.segs[(size_t)seg].nk;
  }
  const int32_t nrows = transpose ? nk : nq;
  const int64_t cap_ptr = sizes[0], cap_idx = sizes[1];
  sizes[0] = nrows + 1;
  sizes[1] = (int64_t)tiles->size();
  if ((ptr && cap_ptr < nrows + 1) || ((idx || flags || live) && cap_idx < (int64_t)tiles->size()))
    return ST_ERR_WORKSPACE;
  std::vector<size_t> order(tiles->size());
  for (size_t t = 0; t < order.size(); ++t) order[t] = t;
  if (transpose)
    std::stable_sort(order.begin(), order.end(), [&](size_t a, size_t b) {
      const Tile &x = (*tiles)[a], &y = (*tiles)[b];
      return x.k != y.k ? x.k < y.k : x.q < y.q;
    });
  std::vector<int32_t> counts((size_t)nrows + 1, 0);
  for (size_t t = 0; t < order.size(); ++t) {
    const Tile& x = (*tiles)[order[t]];
    counts[(size_t)(transpose ? x.k : x.q) + 1] += 1;
    if (idx) idx[t] = transpose ? x.q : x.k;
    if (flags) flags[t] = x.flag;
    if (live) live[t] = x.live;
  }
  for (int32_t r = 0; r < nrows; ++r) counts[(size_t)r + 1] += counts[(size_t)r];
  if (ptr) std::memcpy(ptr, counts.data(), sizeof(int32_t) * counts.size());
  return ST_OK;
}

st_status st_sparse_attn_fwd(const st_layout* L, st_dtype dtype, int32_t B, int32_t H, int32_t T,
                             int32_t d, float scale, const void* q, const void* k, const void* v,
                             void* o, float* lse, void* stream) {
  return st_sparse_attn_fwd_heads(L, dtype, B, H, 0, H, T, d, scale, q, k, v, o, lse, stream);
}

st_status st_sparse_attn_fwd_heads(const st_layout* L, st_dtype dtype, int32_t B, int32_t H,
                                   int32_t h_begin, int32_t h_count, int32_t T, int32_t d,
                                   float scale, const void* q, const void* k, const void* v,
                                   void* o, float* lse, void* stream) {
  Call c;
  st_status s = prepare(L, dtype, B, H, h_begin, h_count, T, d, scale, stream, c);
  if (s != ST_OK) return s;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return ST_ERR_INVALID;
  cudaError_t e;
  arm(c, 0);
  if (dtype == ST_F32) {
    e = simt_fwd(c, q, k, v, o, lse);
  } else {
    e = tc_fwd(c, q, k, v, o, lse, g_force_timeout.exchange(0));
  }
  return e == cudaSuccess ? ST_OK : ST_ERR_CUDA;
}

st_status st_sparse_attn_bwd_workspace(const st_layout* L, st_dtype dtype, int32_t B, int32_t H,
                                       int32_t T, int32_t d, size_t* bytes) {
  if (!L || !bytes || B < 1 || H < 1 || d < 1 || T != L->geom.T) return ST_ERR_INVALID;
  if (dtype != ST_F32 && dtype != ST_BF16 && dtype != ST_F16) return ST_ERR_INVALID;
  const size_t rows = (size_t)B * H * T;
  size_t b = round256(rows * sizeof(float));  // D
  if (dtype != ST_F32) b += 3 * round256(rows * (size_t)d * sizeof(float)) + kMiscBytes;
  *bytes = b;
  return ST_OK;
}

st_status st_sparse_attn_bwd(const st_layout* L, st_dtype dtype, int32_t B, int32_t H, int32_t T,
                             int32_t d, float scale, const void* q, const void* k, const void* v,
                             const void* o, const float* lse, const void* dout, void* dq,
                             void* dk, void* dv, void* workspace, size_t ws_bytes, void* stream) {
  return st_sparse_attn_bwd_heads(L, dtype, B, H, 0, H, T, d, scale, q, k, v, o, lse, dout, dq,
                                  dk, dv, workspace, ws_bytes, stream);
}

st_status st_sparse_attn_bwd_heads(const st_layout* L, st_dtype dtype, int32_t B, int32_t H,
                                   int32_t h_begin, int32_t h_count, int32_t T, int32_t d,
                                   float scale, const void* q, const void* k, const void* v,
                                   const void* o, const float* lse, const void* dout, void* dq,
                                   void* dk, void* dv, void* workspace, size_t ws_bytes,
                                   void* stream) {
  Call c;
  st_status s = prepare(L, dtype, B, H, h_begin, h_count, T, d, scale, stream, c);
  if (s != ST_OK) return s;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
      !aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return ST_ERR_INVALID;
  size_t need = 0;
  st_sparse_attn_bwd_workspace(L, dtype, B, H, T, d, &need);
  if (!workspace || ws_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return ST_ERR_WORKSPACE;
  const size_t rows = (size_t)B * H * T;
  const size_t elems = rows * (size_t)d;
  float* Dv = reinterpret_cast<float*>(workspace);
  cudaError_t e;
  if (dtype == ST_F32) {
    // the selected heads of every batch: B rows of hn*T*d floats, H*T*d apart
    const size_t head = (size_t)T * d * sizeof(float);
    void* outs[3] = {dq, dk, dv};
    e = cudaSuccess;
    for (int x = 0; x < 3 && e == cudaSuccess; ++x)
      e = cudaMemset2DAsync(static_cast<char*>(outs[x]) + (size_t)c.h0 * head, (size_t)H * head, 0,
                            (size_t)c.hn * head, (size_t)B, c.stream);
    if (e == cudaSuccess) e = bwd_prologue(c, o, dout, Dv, nullptr, 0);
    Call cm = c;
    arm(cm, 1);
    if (e == cudaSuccess)
      e = simt_bwd(cm, q, k, v, lse, dout, Dv, (float*)dq, (float*)dk, (float*)dv);
  } else {
    float* acc = reinterpret_cast<float*>(reinterpret_cast<char*>(workspace) +
                                          round256(rows * sizeof(float)));
    const size_t stride = round256(elems * sizeof(float)) / sizeof(float);
    float* dq_acc = acc;
    float* dk_acc = acc + stride;
    float* dv_acc = acc + 2 * stride;
    int* counter = reinterpret_cast<int*>(dv_acc + stride);  // work counter of the kernel
    float* slots = reinterpret_cast<float*>(reinterpret_cast<char*>(counter) + 256);
    int nslots = 0;
    Call cp = c, cm = c, cf = c;
    arm(cp, 2);
    arm(cm, 1);
    arm(cf, 3);
    record_begin(cp);
    e = bwd_prep(c, o, dout, Dv, dq_acc, dk_acc, dv_acc, counter, slots, &nslots);
    record_end(cp);
    if (e == cudaSuccess)
      e = tc_bwd(cm, q, k, v, lse, dout, Dv, dq_acc, dk_acc, dv_acc, dq, dk, dv, counter, slots,
                 nslots);
    record_begin(cf);
    if (e == cudaSuccess) e = bwd_finish(c, dq_acc, dk_acc, dv_acc, slots, nslots, dq, dk, dv);
    record_end(cf);
  }
  return e == cudaSuccess ? ST_OK : ST_ERR_CUDA;
}

st_status st_last_device_status(void* stream) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return ST_ERR_CUDA;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return ST_ERR_CUDA;
  int* w = status_word(dev, false);
  if (!w) return ST_OK;
  int h = 0;
  if (cudaMemcpy(&h, w, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return ST_ERR_CUDA;
  if (h != 0 && cudaMemset(w, 0, sizeof(int)) != cudaSuccess) return ST_ERR_CUDA;
  return (st_status)h;
}

st_status st_layout_launches(const st_layout* L, st_dtype dtype, int32_t* fwd, int32_t* bwd) {
  if (!L || (dtype != ST_F32 && dtype != ST_BF16 && dtype != ST_F16)) return ST_ERR_INVALID;
  int32_t nf = 0;
  for (int p = 0; p < L->n_passes; ++p) nf += L->fwd_items[p].empty() ? 0 : 1;
  int32_t nb;
  if (dtype == ST_F32) {
    nb = 1 + (L->bwd_items.empty() ? 0 : 1) + nf;  // prologue, key-major kernel, dQ per pass
  } else {
    nb = 2 + (L->bwd_items.empty() ? 0 : 1);       // prep, main kernel, finish
  }
  if (fwd) *fwd = nf;
  if (bwd) *bwd = nb;
  return ST_OK;
}

st_status st_kernel_timing(int32_t enable) {
  if (enable) {
    for (int k = 0; k < kTimed; ++k)
      for (int w = 0; w < 2; ++w)
        if (!g_ev[k][w] && cudaEventCreate(&g_ev[k][w]) != cudaSuccess) return ST_ERR_CUDA;
    for (int k = 0; k < kTimed; ++k) g_ev_used[k] = false;
  }
  g_timing = enable != 0;
  return ST_OK;
}

st_status st_kernel_elapsed_ms(int32_t kernel, float* ms) {
  if (kernel < 0 || kernel >= kTimed || !ms || !g_ev[kernel][1] || !g_ev_used[kernel])
    return ST_ERR_INVALID;
  if (cudaEventSynchronize(g_ev[kernel][1]) != cudaSuccess) return ST_ERR_CUDA;
  if (cudaEventElapsedTime(ms, g_ev[kernel][0], g_ev[kernel][1]) != cudaSuccess)
    return ST_ERR_CUDA;
  return ST_OK;
}

st_status st_set_wait_limit(uint64_t ns, int32_t force_timeout) {
  g_wait_ns.store(ns ? ns : kDefaultWaitNs);
  g_force_timeout.store(force_timeout ? 1 : 0);
  return ST_OK;
}

}  // extern "C"
