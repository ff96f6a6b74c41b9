// Backward pass on the tensor cores (sm_100a), with the attention matrix
// recomputed from LSE rather than stored (milestone page "Sparse Transformer",
// nlp-lineage, "The idea", "Recomputation").
//
// Per live tile pair (key tile j held by the CTA, query tile i streamed):
//   S^T  = K Q^T                  (M=128 keys, N=128 queries, K=64)
//   dP^T = V dO^T
//   P^T  = exp(scale S^T - LSE_i) on the live pairs, 0 elsewhere
//   dS^T = P^T (dP^T - D_i),      D_i = dO_i . O_i (prologue kernel)
//   dV  += P^T dO                 (M=128, N=64, K=128; P^T read from TMEM),
//                                 in fp16: P^T rounded to fp16 and, for bf16
//                                 inputs, dO copied to fp16 in place (times a
//                                 power of two from the prologue's max |dO|)
//                                 once dP^T has read it
//   dK  += dS^T Q                 (dS^T from shared memory)
//   dQ_i = dS K
// dV and dK stay in TMEM for a whole work unit (a key tile, or a chunk of a
// long key column). A gradient tile whose rows no other unit (for dK, dV) or
// pair (for dQ) touches is scaled, rounded to bf16 and TMA-stored straight
// into the output; every other tile is TMA reduce-added into an fp32
// accumulator, which a later kernel scales and rounds. K and V are
// double-buffered across units.
//
// Persistent CTAs, one per SM. The producer warp claims work units (sorted
// longest first) from a global counter and publishes them to the other roles
// through a small shared-memory ring, so that every CTA takes the next unit
// when it is ready for one. Warpgroup roles:
//   warpgroups 0, 1  compute: thread = key row = TMEM lane for S^T / dP^T;
//                    warpgroup w owns query columns 64w .. 64w+63 of every
//                    tile, the dQ columns 32w .. 32w+31, and writes out dK
//                    (w = 0) or dV (w = 1) at the end of a unit;
//   warpgroup 2      warp 8 TMA producer (K, V per unit into two buffers; Q,
//                    dO per query tile into a 2-stage ring, with LSE and D by
//                    plain loads), warp 9 TMEM owner and MMA issuer, warp 10
//                    writer (TMA reduce-adds or stores of the staged dQ, dK,
//                    dV tiles, so that no compute warp waits on a bulk copy).
// The MMA warp issues S, dP of the next tile as soon as the compute warps hold
// the current tile's in registers, ahead of dV, dK, dQ of the current tile,
// so the exponentials overlap the tensor pipe. All waits are bounded.
#include <math.h>

#include <algorithm>

#include "launch.h"
#include "tc_common.cuh"

namespace st {
namespace {

using namespace tc;

constexpr int NS = 2;
constexpr int kSched = 6;                   // published work units in flight
constexpr int kTileBytes = kTile * 64 * 2;  // 128 x 64 bf16 = 16 KB
constexpr int kThreads = 384;
constexpr uint32_t kRegsCompute = 200, kRegsIssue = 104;  // launch: 168 per thread
static_assert(256 * kRegsCompute + 128 * kRegsIssue == kThreads * 168, "register split");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 320, kColDQ = 384;
constexpr uint32_t kColPT = 448;  // P^T as packed bf16 pairs, 64 columns
// packed fp32 summary rows of one column half (kv_direct == 2 units), staged
// in the dS^T buffer at the end of a unit: dK halves, then dV halves
constexpr int kSumBoxBytes = kMixedMaxRows * 128;
static_assert(4 * kSumBoxBytes <= 2 * kTileBytes, "summary-row boxes exceed the dS^T buffer");
constexpr float kLog2e = 1.4426950408889634f;

struct BwdMaps {
  CUtensorMap q[3], k[3], v[3], dout[3];  // bf16, indexed by View
  CUtensorMap dq[3], dk[3], dv[3];        // fp32 accumulators, 32-float boxes
  CUtensorMap dqo[3], dko[3], dvo[3];     // bf16 outputs (direct tiles)
  CUtensorMap dks, dvs;  // fp32 accumulators: the summary rows of a natural tile
};

// A published work unit: its index (n_units: no more work), head, item and
// query entries, so that no consuming role reads the schedule from global
// memory at a unit boundary.
struct SchedSlot {
  int u, bh;
  BwdItem it;
  QEnt q[kBwdChunk];
};

// Natural rows of each head class whose gradient no unit writes (zero),
// for dQ and for dK / dV.
struct ZeroRows {
  const int32_t* q[2];
  const int32_t* k[2];
  int32_t nq[2], nk[2];
};

struct SmemBwd {
  uint8_t k[2][kTileBytes];
  uint8_t v[2][kTileBytes];
  uint8_t q[NS][kTileBytes];
  uint8_t dout[NS][kTileBytes];
  uint8_t dst[2 * kTileBytes];   // dS^T (keys x queries), two 64-query K-blocks
  uint8_t stage[2 * kTileBytes]; // dQ tile: fp32 in two 32-column halves, or bf16
  uint8_t kvst[2 * kTileBytes];  // end of a unit: dK (fp32), or dK and dV (bf16 / fp16)
  float l2[NS][kTile];           // -LSE_i * log2(e) of the stage's query rows
  float dd[NS][kTile];           // -D_i
  uint64_t kv_full[2], kv_done[2], full[NS], empty[NS];
  uint64_t s_full, dp_full, sdp_free, ds_ready, pds_free, dq_full, dq_free, stg_full, stg_free;
  uint64_t acc_full, acc_free, out_full, dst_free, kvst_free, fin;
  uint64_t sched_full[kSched], sched_empty[kSched];
  SchedSlot slot[kSched];        // published units
  float bmax[8];                 // per compute warp: largest |dO| (start of the kernel)
  uint32_t tmem_base;
  int abort;
};

// PACKED: the layout packs short residue classes (Geom::cpt > 1); a separate
// instantiation, so that other layouts' kernels carry none of its code.
template <bool PACKED>
__device__ __forceinline__ void load_tile(void* dst, const CUtensorMap* maps, int view,
                                          const Geom& g, int tile, int bh, uint64_t* bar) {
  if (view == VIEW_NAT) {
    tma_load_3d(dst, &maps[VIEW_NAT], bar, 0, tile * kTile, bh);
  } else if (view == VIEW_SUM) {
    tma_load_4d(dst, &maps[VIEW_SUM], bar, 0, g.l - g.c, tile * g.sum_rows, bh);
  } else if (PACKED) {
    // packed short classes: one box of P rows per class, class after class
    // (classes past l are zero-filled)
    for (int k = 0; k < g.cpt; ++k)
      tma_load_4d(static_cast<uint8_t*>(dst) + k * g.P * 128, &maps[VIEW_CLS], bar, 0,
                  tile * g.cpt + k, 0, bh);
  } else {
    int r = fdiv(tile, g.fpt), pb = tile - r * g.ptiles;
    tma_load_4d(dst, &maps[VIEW_CLS], bar, 0, r, pb * kTile, bh);
  }
}

// Prefetches a tile into L2 (the actual load follows when a ring stage frees).
template <bool PACKED>
__device__ __forceinline__ void prefetch_tile(const CUtensorMap* maps, int view, const Geom& g,
                                              int tile, int bh) {
  if (view == VIEW_NAT) {
    tma_prefetch_3d(&maps[VIEW_NAT], 0, tile * kTile, bh);
  } else if (view == VIEW_SUM) {
    tma_prefetch_4d(&maps[VIEW_SUM], 0, g.l - g.c, tile * g.sum_rows, bh);
  } else if (PACKED) {
    for (int k = 0; k < g.cpt; ++k) tma_prefetch_4d(&maps[VIEW_CLS], 0, tile * g.cpt + k, 0, bh);
  } else {
    int r = fdiv(tile, g.fpt), pb = tile - r * g.ptiles;
    tma_prefetch_4d(&maps[VIEW_CLS], 0, r, pb * kTile, bh);
  }
}

// Reduce-adds one 32-column half h of a 128-row fp32 tile staged as two
// halves. (TMA copies issued by one thread are processed one after another,
// copies of different threads in parallel: the two halves go out from two
// lanes.)
template <bool PACKED>
__device__ __forceinline__ void reduce_half(const CUtensorMap* maps, int view, const Geom& g,
                                            int tile, int bh, const uint8_t* src, int h) {
  const uint8_t* s = src + h * kTileBytes;
  if (view == VIEW_NAT) {
    tma_reduce_add_3d(&maps[VIEW_NAT], s, h * 32, tile * kTile, bh);
  } else if (view == VIEW_SUM) {
    tma_reduce_add_4d(&maps[VIEW_SUM], s, h * 32, g.l - g.c, tile * g.sum_rows, bh);
  } else if (PACKED) {
    // packed short classes: one box per class (rows of classes past l are dropped)
    for (int k = 0; k < g.cpt; ++k)
      tma_reduce_add_4d(&maps[VIEW_CLS], s + k * g.P * 128, h * 32, tile * g.cpt + k, 0, bh);
  } else {
    int r = fdiv(tile, g.fpt), pb = tile - r * g.ptiles;
    tma_reduce_add_4d(&maps[VIEW_CLS], s, h * 32, r, pb * kTile, bh);
  }
}

// Reduce-adds column half h of the summary rows of natural key tile `tile`,
// staged packed (one 128-byte row per summary row, block after block) at src.
__device__ __forceinline__ void reduce_summary_rows(const CUtensorMap* map, const Geom& g,
                                                    int tile, int bh, const uint8_t* src,
                                                    int h) {
  tma_reduce_add_4d(map, src, h * 32, g.l - g.c, fdiv(tile * kTile, g.fl), bh);
}

// Stores a 128-row bf16 tile (coordinates are never negative).
template <bool PACKED>
__device__ __forceinline__ void store_tile(const CUtensorMap* maps, int view, const Geom& g,
                                           int tile, int bh, const uint8_t* src) {
  if (view == VIEW_NAT) {
    tma_store_3d(&maps[VIEW_NAT], src, 0, tile * kTile, bh);
  } else if (view == VIEW_SUM) {
    tma_store_4d(&maps[VIEW_SUM], src, 0, g.l - g.c, tile * g.sum_rows, bh);
  } else if (PACKED) {
    for (int k = 0; k < g.cpt; ++k)
      tma_store_4d(&maps[VIEW_CLS], src + k * g.P * 128, 0, tile * g.cpt + k, 0, bh);
  } else {
    int r = fdiv(tile, g.fpt), pb = tile - r * g.ptiles;
    tma_store_4d(&maps[VIEW_CLS], src, 0, r, pb * kTile, bh);
  }
}

// Eight fp32 values (bit patterns), times s, as four packed 16-bit pairs.
template <bool F16>
__device__ __forceinline__ void round8(const uint32_t* v, float s, uint32_t w[4]) {
#pragma unroll
  for (int x = 0; x < 4; ++x)
    w[x] = pack2<F16>(__uint_as_float(v[2 * x]) * s, __uint_as_float(v[2 * x + 1]) * s);
}

// Live query columns [lo, hi) of a query tile for the key at natural
// position j (segment rules restated as intervals over queries).
__device__ __forceinline__ void live_rows(const Geom& g, int kview, int qview, int rule,
                                          int qtile, int j, int& lo, int& hi) {
  if (j < 0) {
    lo = hi = 0;
    return;
  }
  const int l = g.l, c = g.c;
  const int jb = fdiv(j, g.fl);  // the key's block (its class row in the residue view)
  int a = 0, b = 0, base, lim;
  if (qview == VIEW_NAT) {
    base = qtile * kTile;
    lim = g.T;
    if (kview == VIEW_SUM) {
      a = (rule == RULE_SUMMARY) ? j : (jb + 1) * l;
      b = lim;
    } else {
      switch (rule) {
        case RULE_CAUSAL: a = j; b = lim; break;
        case RULE_BAND: a = j; b = j + l + 1; break;
        case RULE_BLOCK: a = j; b = (jb + 1) * l; break;
        case RULE_STRIDE: a = j; b = j + 1; break;                          // l >= T only
        case RULE_SUMMARY: a = j; b = (j - jb * l >= l - c) ? lim : j; break;  // l >= T only
        default: a = 0; b = 0; break;
      }
    }
  } else {
    // query tile column x holds view row qtile * 128 + x; the key's class r
    // starts at view row r * cw
    base = qtile * kTile - (j - jb * l) * g.cw;
    lim = g.P;
    a = (rule == RULE_STRIDE) ? jb : jb + 2;
    b = lim;
  }
  b = min(b, lim);
  lo = max(a - base, 0);
  hi = min(b - base, kTile);
  if (hi < lo) hi = lo;
}

struct Unit {
  BwdItem it;
  int bh;
};

// Unit order: item-major (every head of the longest item first), or, when
// the fp32 accumulator rows of all heads would not stay in L2, head-major
// (all items of one head, longest first, then the next head).
struct UnitOrder {
  int head_major, n_items;
  FastDiv fitems;
};

__device__ __forceinline__ Unit unit_of(const BwdItem* items, int u, int NH, const Heads& hs,
                                        const UnitOrder& uo) {
  Unit x;
  if (uo.head_major) {
    const int h = fdiv(u, uo.fitems);
    x.it = items[u - h * uo.n_items];
    x.bh = head_of(h, x.it.hclass, hs);
  } else {
    const int q = fdiv(u, hs.fnh);  // NH = the divisor of hs.fnh
    x.it = items[q];
    x.bh = head_of(u - q * NH, x.it.hclass, hs);
  }
  return x;
}

// F16: 16-bit element type, fp16 if true, else bf16. PACKED: see load_tile.
template <bool F16, bool PACKED>
__global__ void __launch_bounds__(kThreads, 1)
bwd_tc_kernel(const __grid_constant__ BwdMaps maps, Geom g, const BwdItem* __restrict__ items,
              int n_units, int NH, UnitOrder uo, const QEnt* __restrict__ qents, Heads hs,
              float scale, float scale_log2, const float* __restrict__ lse,
              const float* __restrict__ Dg, ZeroRows zr, uint4* __restrict__ dq_out,
              uint4* __restrict__ dk_out, uint4* __restrict__ dv_out, int* sched_counter,
              const float* __restrict__ dmax_slots, int nslots, int* status, uint64_t wait_ns) {
  // The shared-memory plan fills the 227 KB a CTA may hold, with no room to
  // realign: the swizzled tiles need the dynamic window at a 1024-byte
  // boundary (where it starts when the kernel has no static shared memory).
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {
    if (threadIdx.x == 0) set_status(status, ST_ERR_UNSUPPORTED);
    return;
  }
  SmemBwd& S = *reinterpret_cast<SmemBwd*>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort = &S.abort;

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&S.kv_full[b], 1);
      mbar_init(&S.kv_done[b], 1);
    }
    for (int s = 0; s < NS; ++s) {
      mbar_init(&S.full[s], 33);  // expect_tx arrive + 32 producer lanes
      mbar_init(&S.empty[s], 1);
    }
    mbar_init(&S.s_full, 1);
    mbar_init(&S.dp_full, 1);
    mbar_init(&S.sdp_free, 256);
    mbar_init(&S.ds_ready, 256);
    mbar_init(&S.pds_free, 1);
    mbar_init(&S.dq_full, 1);
    mbar_init(&S.dq_free, 256);
    mbar_init(&S.stg_full, 256);
    mbar_init(&S.stg_free, 1);
    mbar_init(&S.acc_full, 1);
    mbar_init(&S.acc_free, 256);
    mbar_init(&S.out_full, 256);
    mbar_init(&S.dst_free, 1);
    mbar_init(&S.kvst_free, 1);
    mbar_init(&S.fin, 1);
    for (int k = 0; k < kSched; ++k) {
      mbar_init(&S.sched_full[k], 1);
      mbar_init(&S.sched_empty[k], 10);  // MMA lane, reducer lane, 8 compute warps
    }
    S.abort = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(&S.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 11) {  // the tensor maps into the descriptor cache, one per lane
    const CUtensorMap* m = &maps.q[0];
    if (lane < (int)(sizeof(BwdMaps) / sizeof(CUtensorMap))) tma_prefetch_desc(m + lane);
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  auto fail = [&]() {
    *abort = 1;
    set_status(status, ST_ERR_DEVICE_TIMEOUT);
  };
  // Next published unit for a consuming role: its slot k. A role releases
  // the slot (one arrival per consuming warp) once it has finished the unit.
  int sk = 0;
  auto next_unit = [&](int& u, int& k) -> bool {
    k = sk % kSched;
    const bool w = mbar_wait(&S.sched_full[k], (sk / kSched) & 1, wait_ns, abort);
    if (!w) return false;
    u = *reinterpret_cast<volatile int*>(&S.slot[k].u);
    ++sk;
    return true;
  };

  if (warp >= 8) {
    regs_decrease<kRegsIssue>();
    if (warp == 8) {
      // ---------------- producer ----------------
      int full_last[NS] = {-1, -1};
      int kv_last = -1;
      bool ok = true;
      int gt = 0, n = 0, pub = 0;
      // The CTA's first unit is blockIdx.x (the longest units spread one per
      // CTA); later ones come from the counter, offset by the grid. Units
      // without a head of their class are skipped.
      // The first valid unit at or after u (n_units if none), decoded into y.
      auto valid = [&](int u, Unit& y) -> int {
        for (;;) {
          if (u >= n_units) return n_units;
          y = unit_of(items, u, NH, hs, uo);
          if (y.bh >= 0) return u;
          int t = 0;
          if (lane == 0) t = atomicAdd(sched_counter, 1);
          u = (int)gridDim.x + __shfl_sync(0xffffffffu, t, 0);
        }
      };
      auto publish = [&](int u, const Unit& x) -> bool {
        const int k = pub % kSched;
        const bool w = mbar_wait(&S.sched_empty[k], ((pub / kSched) & 1) ^ 1, wait_ns, abort);
        if (!__all_sync(0xffffffffu, w)) return false;
        SchedSlot& sl = S.slot[k];
        if (u < n_units) {
          if (lane < x.it.qend - x.it.qbeg) sl.q[lane] = qents[x.it.qbeg + lane];
          if (lane == 0) {
            sl.bh = x.bh;
            sl.it = x.it;
          }
        }
        if (lane == 0) sl.u = u;
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.sched_full[k]);
        ++pub;
        return true;
      };
      Unit x;
      int cur = valid(blockIdx.x, x);
      while (ok && cur < n_units) {
        ok = publish(cur, x);
        if (!ok) break;
        // the claim of the following unit goes out now; its answer is first
        // needed once this unit's K, V are on their way
        int ticket = 0;
        if (lane == 0) ticket = atomicAdd(sched_counter, 1);
        const int cnt = x.it.qend - x.it.qbeg;
        auto issue_q = [&](int e) -> bool {
          const int s = gt % NS;
          // schedule entries and the LSE / D rows are read before the wait for
          // the ring stage, so that their latency stays off the critical path
          const QEnt qe = qents[x.it.qbeg + e];
          const int pf = (e + 2 < cnt) ? qents[x.it.qbeg + e + 2].qtile : -1;
          float Lv[4], Dv[4];
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const int i = view_pos(g, x.it.qview, qe.qtile, lane + 32 * t);
            const size_t at = (size_t)x.bh * g.T + (i >= 0 ? i : 0);
            Lv[t] = __ldg(lse + at);
            Dv[t] = __ldg(Dg + at);
            if (i < 0) Lv[t] = Dv[t] = 0.f;
          }
          const bool w = mbar_wait(&S.empty[s], ((gt / NS) & 1) ^ 1, wait_ns, abort);
          if (!__all_sync(0xffffffffu, w)) return false;
          if (lane == 0) mbar_arrive_expect_tx(&S.full[s], 2 * kTileBytes);
          __syncwarp();
          // Q from lane 0, dO from lane 1; the L2 prefetches of the tile two
          // ahead from lanes 2, 3 (each thread's copies run one at a time)
          if (lane < 2)
            load_tile<PACKED>(lane ? S.dout[s] : S.q[s], lane ? maps.dout : maps.q, x.it.qview, g,
                      qe.qtile, x.bh, &S.full[s]);
          else if (lane < 4 && pf >= 0)
            prefetch_tile<PACKED>(lane == 3 ? maps.dout : maps.q, x.it.qview, g, pf, x.bh);
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const int row = lane + 32 * t;
            // rows with an empty set (LSE = -inf) have no live pair; 0 keeps
            // their masked exponents at -inf instead of -inf + inf
            S.l2[s][row] = (Lv[t] > -INFINITY) ? -Lv[t] * kLog2e : 0.f;
            S.dd[s][row] = -Dv[t];
          }
          mbar_arrive(&S.full[s]);
          full_last[s] = gt;
          ++gt;
          return true;
        };
        // K, V of a unit go into buffer n & 1 (n counts this CTA's units),
        // last read by unit n - 2. They are normally loaded one unit ahead,
        // below; only the CTA's first unit loads its own here.
        auto load_kv = [&](int m, const Unit& y) -> bool {
          const int kb = m & 1;
          const bool w = mbar_wait(&S.kv_done[kb], ((m >> 1) & 1) ^ 1, wait_ns, abort);
          if (!__all_sync(0xffffffffu, w)) return false;
          if (lane == 0) mbar_arrive_expect_tx(&S.kv_full[kb], 2 * kTileBytes);
          __syncwarp();
          if (lane < 2)  // K from lane 0, V from lane 1
            load_tile<PACKED>(lane ? S.v[kb] : S.k[kb], lane ? maps.v : maps.k, y.it.kview, g,
                      y.it.ktile, y.bh, &S.kv_full[kb]);
          kv_last = m;
          return true;
        };
        if (kv_last < n) ok = load_kv(n, x);
        if (!ok) break;
        // Q, dO of the unit's query tiles in order; the claimed next unit is
        // resolved after the first, and its K, V go out after the second (or
        // after the last, for shorter units), as soon as unit n - 1 has
        // released their buffer. One call site per loader keeps the warp's
        // code small.
        int nxt = n_units;
        Unit y;
        bool kv_next = false;
        for (int e = 0; ok; ++e) {
          if (e < cnt) ok = issue_q(e);
          if (!ok) break;
          if (e == 0) nxt = valid((int)gridDim.x + __shfl_sync(0xffffffffu, ticket, 0), y);
          const bool last = e + 1 >= cnt;
          if (!kv_next && (e == 1 || last)) {
            kv_next = true;
            if (nxt < n_units) ok = load_kv(n + 1, y);
          }
          if (last && kv_next) break;
        }
        ++n;
        cur = nxt;
        x = y;
      }
      if (ok) ok = publish(n_units, x);  // no more work
      if (!ok && lane == 0) fail();
      if (lane == 0) {
        // the last K / V loads of both buffers have landed before the exit
        // (these waits ignore the abort flag: the copies were issued and will land)
        for (int m = max(kv_last - 1, 0); m <= kv_last; ++m)
          if (!mbar_wait_drain(&S.kv_full[m & 1], (m >> 1) & 1, wait_ns)) fail();
        for (int s = 0; s < NS; ++s)
          if (full_last[s] >= 0 &&
              !mbar_wait_drain(&S.full[s], (full_last[s] / NS) & 1, wait_ns))
            fail();
      }
    } else if (warp == 9) {
      // ---------------- MMA issuer ----------------
      if (lane == 0) {
        const uint32_t idSS = idesc_16(128, 128, false, false, F16);
        const uint32_t idKM = idesc_16(128, 64, false, true, F16);  // A K-major, B MN-major
        const uint32_t idDV = idesc_16(128, 64, false, true, true);  // fp16 P^T and dO
        const uint32_t idMM = idesc_16(128, 64, true, true, F16);   // A MN-major, B MN-major
        const uint32_t ds_addr = smem_u32(S.dst);
        const uint64_t dsk = sdesc(ds_addr, 16, 1024);          // dS^T, K-major (dK)
        const uint64_t dsm = sdesc(ds_addr, kTileBytes, 1024);  // dS^T read MN-major (dQ)
        uint64_t kd = 0, vd = 0, kdm = 0;  // this unit's K, V tiles
        bool ok = true;
        int gt = 0, n = 0;
        auto issue_s_dp = [&](int t) -> bool {
          const int s = t % NS;
          if (!mbar_wait(&S.full[s], (t / NS) & 1, wait_ns, abort)) return false;
          tc_fence_after();
          const uint64_t qd = sdesc(smem_u32(S.q[s]), 16, 1024);
          const uint64_t od = sdesc(smem_u32(S.dout[s]), 16, 1024);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss(tmem + kColS, sdesc_at(kd, kk * 32), sdesc_at(qd, kk * 32), idSS, kk > 0);
          mma_commit(&S.s_full);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss(tmem + kColDP, sdesc_at(vd, kk * 32), sdesc_at(od, kk * 32), idSS, kk > 0);
          mma_commit(&S.dp_full);
          return true;
        };
        for (;;) {
          int u = 0, sl = 0;
          if (!next_unit(u, sl)) {
            ok = false;
            break;
          }
          if (u >= n_units) break;
          const int cnt = S.slot[sl].it.qend - S.slot[sl].it.qbeg;
          const int kb = n & 1;
          kd = sdesc(smem_u32(S.k[kb]), 16, 1024);
          vd = sdesc(smem_u32(S.v[kb]), 16, 1024);
          kdm = sdesc(smem_u32(S.k[kb]), 16384, 1024);
          ok = mbar_wait(&S.kv_full[kb], (n >> 1) & 1, wait_ns, abort);
          // e = -1 issues S^T, dP^T of the unit's first tile; tile e issues
          // those of tile e + 1 as soon as the compute warps hold tile e's in
          // registers (one issue site)
          for (int e = -1; ok && e < cnt; gt += (e >= 0), ++e) {
            if (e + 1 < cnt) {
              if (e >= 0 && !mbar_wait(&S.sdp_free, gt & 1, wait_ns, abort)) {
                ok = false;
                break;
              }
              if (!issue_s_dp(e < 0 ? gt : gt + 1)) {
                ok = false;
                break;
              }
            }
            if (e < 0) continue;
            const int s = gt % NS;
            if (!mbar_wait(&S.ds_ready, gt & 1, wait_ns, abort)) {
              ok = false;
              break;
            }
            tc_fence_after();
            if (e == 0 && !mbar_wait(&S.acc_free, (n & 1) ^ 1, wait_ns, abort)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t qdm = sdesc(smem_u32(S.q[s]), 16384, 1024);
            const uint64_t odm = sdesc(smem_u32(S.dout[s]), 16384, 1024);
            // dV += P^T dO (P^T from TMEM), dK += dS^T Q: K = 128 queries in 8
            // steps of 16, the two accumulation chains interleaved
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t acc = (e > 0 || kk > 0) ? 1u : 0u;
              mma_ts(tmem + kColDV, tmem + kColPT + kk * 8, sdesc_at(odm, kk * 2048),
                     idDV, acc);
              mma_ss(tmem + kColDK,
                     sdesc_at(dsk, (kk >> 2) * kTileBytes + (kk & 3) * 32),
                     sdesc_at(qdm, kk * 2048), idKM, acc);
            }
            mma_commit(&S.empty[s]);  // Q, dO of this stage are no longer read
            if (gt > 0 && !mbar_wait(&S.dq_free, (gt - 1) & 1, wait_ns, abort)) {
              ok = false;
              break;
            }
            tc_fence_after();
            // dQ = dS K   (A = dS^T read MN-major, K = 128 keys)
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_ss(tmem + kColDQ, sdesc_at(dsm, kk * 2048), sdesc_at(kdm, kk * 2048), idMM,
                     kk > 0 ? 1u : 0u);
            mma_commit(&S.dq_full);
            mma_commit(&S.pds_free);
          }
          if (!ok) break;
          mbar_arrive(&S.sched_empty[sl]);
          mma_commit(&S.kv_done[n & 1]);
          mma_commit(&S.acc_full);
          ++n;
        }
        if (!ok) fail();
        // every MMA issued has completed before TMEM is freed
        mma_commit(&S.fin);
        if (!mbar_wait_drain(&S.fin, 0, wait_ns)) fail();
      }
    } else if (warp == 10) {
      // ---------------- writer: TMA stores / reduce-adds of the staged tiles ----------------
      // Every copy goes out from a lane of its own, so that they run in parallel.
      bool ok = true;
      int gt = 0, n = 0;
      int pv = 0, ptile = 0, pbh = 0, pdirect = 0;  // query tile of tile gt - 1
      auto reduce_dq = [&](int t) -> bool {
        const bool w = mbar_wait(&S.stg_full, t & 1, wait_ns, abort);
        if (!__all_sync(0xffffffffu, w)) return false;
        if (pdirect) {
          if (lane == 0) store_tile<PACKED>(maps.dqo, pv, g, ptile, pbh, S.stage);
        } else if (lane < 2) {
          reduce_half<PACKED>(maps.dq, pv, g, ptile, pbh, S.stage, lane);
        }
        if (lane < 2) {
          bulk_commit();
          bulk_wait_read_all();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.stg_free);
        return true;
      };
      for (;;) {
        int u = 0, sl = 0;
        const bool got = next_unit(u, sl);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        const bool end = u >= n_units;
        Unit x;
        x.it = S.slot[sl].it;
        x.bh = S.slot[sl].bh;
        // the dQ of each tile goes out while the next is computed; the end of
        // the work is one more step that only sends the last tile's (one call
        // site)
        const int cnt = end ? 1 : x.it.qend - x.it.qbeg;
        for (int e = 0; ok && e < cnt; ++e, ++gt) {
          if (gt > 0 && !reduce_dq(gt - 1)) {
            ok = false;
            break;
          }
          if (end) break;
          const QEnt qe = S.slot[sl].q[e];
          pv = x.it.qview;
          ptile = qe.qtile;
          pdirect = qe.q_direct;
          pbh = x.bh;
        }
        if (!ok || end) break;
        const bool w = mbar_wait(&S.out_full, n & 1, wait_ns, abort);
        if (!__all_sync(0xffffffffu, w)) {
          ok = false;
          break;
        }
        if (x.it.kv_direct) {  // both 16-bit tiles in kvst
          if (lane < 2) {
            store_tile<PACKED>(lane ? maps.dvo : maps.dko, x.it.kview, g, x.it.ktile, x.bh,
                       S.kvst + lane * kTileBytes);
            bulk_commit();
          } else if (x.it.kv_direct == 2 && lane < 6) {
            // the packed fp32 summary rows in dst: dK halves, then dV halves
            const int q = lane - 2;
            reduce_summary_rows(q < 2 ? &maps.dks : &maps.dvs, g, x.it.ktile, x.bh,
                                S.dst + q * kSumBoxBytes, q & 1);
            bulk_commit();
            bulk_wait_read_all();
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&S.dst_free);
        } else {  // lanes 0, 1: dV halves (in dst), read first; lanes 2, 3: dK halves
          if (lane < 4) {
            reduce_half<PACKED>(lane < 2 ? maps.dv : maps.dk, x.it.kview, g, x.it.ktile, x.bh,
                        lane < 2 ? S.dst : S.kvst, lane & 1);
            bulk_commit();
          }
          if (lane < 2) bulk_wait_read_all();
          __syncwarp();
          if (lane == 0) mbar_arrive(&S.dst_free);
        }
        if (lane < 4) bulk_wait_read_all();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&S.kvst_free);
          mbar_arrive(&S.sched_empty[sl]);
        }
        ++n;
      }
      if (!ok && lane == 0) fail();
      bulk_wait_all();
    } else if (warp == 11) {
      // ---------------- zero-fill of the rows no unit writes ----------------
      // (their gradient is zero), in the background of the other roles. Work
      // items of 128 listed rows of one head are spread over the CTAs; eight
      // lanes cover a 128-byte row, four rows per step.
      const uint4 z = make_uint4(0u, 0u, 0u, 0u);
      const int nheads = hs.B * hs.hn;
      for (int pass = 0; pass < 2; ++pass) {
        const int most = pass ? max(zr.nk[0], zr.nk[1]) : max(zr.nq[0], zr.nq[1]);
        const int chunks = (most + 127) / 128;
        const int items_total = nheads * chunks;
        for (int w = blockIdx.x; w < items_total; w += gridDim.x) {
          const int x = w / chunks, ck = w - x * chunks;
          const int xb = fdiv(x, hs.fhn);
          const int bh = xb * hs.H + hs.h0 + (x - xb * hs.hn);
          const int hc = class_of(bh, hs);
          const int n = pass ? (hc ? zr.nk[1] : zr.nk[0]) : (hc ? zr.nq[1] : zr.nq[0]);
          const int32_t* rows = pass ? (hc ? zr.k[1] : zr.k[0]) : (hc ? zr.q[1] : zr.q[0]);
          const int r1 = min(n, ck * 128 + 128);
          uint4* base0 = (pass ? dk_out : dq_out) + (size_t)bh * g.T * 8 + (lane & 7);
          uint4* base1 = dv_out + (size_t)bh * g.T * 8 + (lane & 7);
          for (int r = ck * 128 + (lane >> 3); r < r1; r += 4) {
            const size_t at = (size_t)rows[r] * 8;
            base0[at] = z;
            if (pass) base1[at] = z;
          }
        }
      }
    }
  } else {
    regs_increase<kRegsCompute>();
    // ---------------- compute warpgroups ----------------
    const int wg = warp >> 2;                    // query-column half of this warpgroup
    const int lg = warp & 3;
    const int row = lg * 32 + lane;              // key row (S^T, dP^T) / query row (dQ)
    const uint32_t tl = (uint32_t)(lg * 32) << 16;
    bool ok = true;
    const uint32_t ds_addr = smem_u32(S.dst);
    const uint32_t st_addr = smem_u32(S.stage);
    int gt = 0, n = 0;
    int pend_direct = 0;  // q_direct of the tile whose dQ is pending
    // dV is formed in fp16: for bf16 inputs dO is copied to fp16 times 2^e
    // (e from the largest |dO|, over the prologue's per-block maxima), and the
    // dV tile is scaled back by 2^-e when it is written
    float do_scale = 1.f, dv_scale = 1.f;
    if constexpr (!F16) {
      float m = 0.f;
      for (int x = threadIdx.x; x < nslots; x += 256) m = fmaxf(m, __ldg(dmax_slots + x));
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
      if (lane == 0) S.bmax[warp] = m;
      named_sync(1, 256);
#pragma unroll
      for (int w2 = 0; w2 < 8; ++w2) m = fmaxf(m, S.bmax[w2]);
      const int e = dout_exp(m);
      do_scale = pow2f(e);
      dv_scale = pow2f(-e);
    }

    // dQ of tile t: TMEM -> registers -> staging (fp32 for the reduce-add, or
    // scaled bf16 for the direct store)
    auto drain_dq = [&](int t, int direct) -> bool {
      bool w = mbar_wait(&S.dq_full, t & 1, wait_ns, abort);
      if (!__all_sync(0xffffffffu, w)) return false;
      tc_fence_after();
      uint32_t dq[32];
      tmem_ld32(tmem + tl + kColDQ + wg * 32, dq);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&S.dq_free);
      w = mbar_wait(&S.stg_free, (t & 1) ^ 1, wait_ns, abort);
      if (!__all_sync(0xffffffffu, w)) return false;
      if (direct) {
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t o4[4];
          round8<F16>(dq + ch * 8, scale, o4);
          st_shared_v4(st_addr + swz128(row, wg * 4 + ch), o4[0], o4[1], o4[2], o4[3]);
        }
      } else {
#pragma unroll
        for (int ch = 0; ch < 8; ++ch)
          st_shared_v4(st_addr + wg * kTileBytes + swz128(row, ch), dq[ch * 4 + 0],
                       dq[ch * 4 + 1], dq[ch * 4 + 2], dq[ch * 4 + 3]);
      }
      fence_async_smem();
      mbar_arrive(&S.stg_full);
      return true;
    };

    for (;;) {
      int u = 0, sl = 0;
      const bool got = next_unit(u, sl);
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      if (u >= n_units) break;
      Unit x;
      x.it = S.slot[sl].it;
      x.bh = S.slot[sl].bh;
      const BwdItem& it = x.it;
      const int cnt = it.qend - it.qbeg;
      const int j = view_pos(g, it.kview, it.ktile, row);
      for (int e = 0; e < cnt; ++e, ++gt) {
        const int s = gt % NS;
        const QEnt qe = S.slot[sl].q[e];
        bool w = mbar_wait(&S.s_full, gt & 1, wait_ns, abort);
        w = w && mbar_wait(&S.dp_full, gt & 1, wait_ns, abort);
        w = w && mbar_wait(&S.full[s], (gt / NS) & 1, wait_ns, abort);
        if (!__all_sync(0xffffffffu, w)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const bool full = (qe.flag == TILE_FULL);
        int lo = 0, hi = kTile;
        if (!full) live_rows(g, it.kview, it.qview, it.rule, qe.qtile, j, lo, hi);
        float sv[64], dp[64];
        tmem_ld32(tmem + tl + kColS + wg * 64, reinterpret_cast<uint32_t*>(sv));
        tmem_ld32(tmem + tl + kColS + wg * 64 + 32, reinterpret_cast<uint32_t*>(sv) + 32);
        tmem_ld32(tmem + tl + kColDP + wg * 64, reinterpret_cast<uint32_t*>(dp));
        tmem_ld32(tmem + tl + kColDP + wg * 64 + 32, reinterpret_cast<uint32_t*>(dp) + 32);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&S.sdp_free);  // S^T, dP^T of this tile may now be overwritten
        if constexpr (!F16) {
          // dP^T has read this stage's dO: turn it into the fp16 operand of dV
          // (each thread converts 4 of the 1024 16-byte chunks; the swizzle
          // moves whole chunks, so the element order inside them is kept)
          const uint32_t da = smem_u32(S.dout[s]);
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            const uint32_t at = da + (uint32_t)(threadIdx.x + 256 * x) * 16u;
            uint32_t w4[4];
            ld_shared_v4(at, w4[0], w4[1], w4[2], w4[3]);
#pragma unroll
            for (int y = 0; y < 4; ++y) {
              float lo, hi;
              fmul2(lo, hi, __uint_as_float(w4[y] << 16), __uint_as_float(w4[y] & 0xffff0000u),
                    do_scale, do_scale);
              w4[y] = pack2<true>(lo, hi);
            }
            st_shared_v4(at, w4[0], w4[1], w4[2], w4[3]);
          }
        }
        if (!full) mask_cols<2>(sv, wg * 64, lo, hi);
        const float* l2 = S.l2[s] + wg * 64;
        const float* dd = S.dd[s] + wg * 64;
        // P^T and dS^T of the whole row slice in registers first: the tensor
        // core may still be reading the previous tile's from shared memory
        uint32_t pw[8][4], dw[8][4];
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const float4 la = *reinterpret_cast<const float4*>(l2 + ch * 8);
          const float4 lb = *reinterpret_cast<const float4*>(l2 + ch * 8 + 4);
          const float4 da = *reinterpret_cast<const float4*>(dd + ch * 8);
          const float4 db = *reinterpret_cast<const float4*>(dd + ch * 8 + 4);
          const float lv[8] = {la.x, la.y, la.z, la.w, lb.x, lb.y, lb.z, lb.w};
          const float dv8[8] = {da.x, da.y, da.z, da.w, db.x, db.y, db.z, db.w};
#pragma unroll
          for (int x2 = 0; x2 < 4; ++x2) {
            const int xk = ch * 8 + x2 * 2;
            float a0, a1;
            ffma2(a0, a1, sv[xk], sv[xk + 1], scale_log2, scale_log2, lv[2 * x2],
                  lv[2 * x2 + 1]);
            const float p0 = fast_exp2(a0), p1 = fast_exp2(a1);
            float t0, t1, q0, q1;
            fadd2(t0, t1, dp[xk], dp[xk + 1], dv8[2 * x2], dv8[2 * x2 + 1]);
            fmul2(q0, q1, p0, p1, t0, t1);
            pw[ch][x2] = pack2<true>(p0, p1);
            dw[ch][x2] = pack2<F16>(q0, q1);
          }
        }
        // the previous tile's dV, dK, dQ products are done with P^T, dS^T; at
        // the start of a unit the writer has also read the previous unit's
        // fp32 dV staging, which sits in the dS^T buffer
        w = true;
        if (gt > 0) w = mbar_wait(&S.pds_free, (gt - 1) & 1, wait_ns, abort);
        if (e == 0 && n > 0) w = w && mbar_wait(&S.dst_free, (n - 1) & 1, wait_ns, abort);
        if (!__all_sync(0xffffffffu, w)) {
          ok = false;
          break;
        }
        tc_fence_after();
        tmem_st32(tmem + tl + kColPT + wg * 32, &pw[0][0]);
#pragma unroll
        for (int ch = 0; ch < 8; ++ch)
          st_shared_v4(ds_addr + wg * kTileBytes + swz128(row, ch), dw[ch][0], dw[ch][1],
                       dw[ch][2], dw[ch][3]);
        tmem_wait_st();
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(&S.ds_ready);
        if (gt > 0 && !drain_dq(gt - 1, pend_direct)) {
          ok = false;
          break;
        }
        pend_direct = qe.q_direct;
      }
      if (!ok) break;
      // ---- end of unit: dK (warpgroup 0) or dV (warpgroup 1) out of TMEM ----
      bool w = mbar_wait(&S.acc_full, n & 1, wait_ns, abort);
      if (!__all_sync(0xffffffffu, w)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t r[64];
      tmem_ld32(tmem + tl + (wg ? kColDV : kColDK), r);
      tmem_ld32(tmem + tl + (wg ? kColDV : kColDK) + 32, r + 32);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&S.acc_free);
      // stage for the writer warp: 16-bit dK and dV both in kvst; fp32 dK in
      // kvst and fp32 dV in the dS^T buffer (free: every product of the unit
      // has completed). kvst must have been read for the previous unit.
      if (n > 0) {
        w = mbar_wait(&S.kvst_free, (n - 1) & 1, wait_ns, abort);
        if (!__all_sync(0xffffffffu, w)) {
          ok = false;
          break;
        }
      }
      const uint32_t kv_addr = smem_u32(S.kvst);
      const uint32_t dst =
          it.kv_direct ? kv_addr + (wg ? kTileBytes : 0) : (wg ? ds_addr : kv_addr);
      if (it.kv_direct) {
        const float sc = wg ? dv_scale : scale;  // dK carries the softmax scale
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          uint32_t o4[4];
          round8<F16>(r + ch * 8, sc, o4);
          st_shared_v4(dst + swz128(row, ch), o4[0], o4[1], o4[2], o4[3]);
        }
        if (it.kv_direct == 2 && j >= 0) {
          // a summary row also goes out unscaled in fp32, packed: row
          // (offset in its block - (l - c)) + c (block - the tile's first block)
          const int jb = fdiv(j, g.fl), o = j - jb * g.l;
          if (o >= g.l - g.c) {
            const int rr = (o - (g.l - g.c)) + g.c * (jb - fdiv(it.ktile * kTile, g.fl));
            const uint32_t sb = ds_addr + wg * 2 * kSumBoxBytes;
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
              for (int ch = 0; ch < 8; ++ch)
                st_shared_v4(sb + h * kSumBoxBytes + swz128(rr, ch), r[h * 32 + ch * 4 + 0],
                             r[h * 32 + ch * 4 + 1], r[h * 32 + ch * 4 + 2],
                             r[h * 32 + ch * 4 + 3]);
          }
        }
      } else {
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int ch = 0; ch < 8; ++ch)
            st_shared_v4(dst + h * kTileBytes + swz128(row, ch), r[h * 32 + ch * 4 + 0],
                         r[h * 32 + ch * 4 + 1], r[h * 32 + ch * 4 + 2],
                         r[h * 32 + ch * 4 + 3]);
      }
      fence_async_smem();
      mbar_arrive(&S.out_full);
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.sched_empty[sl]);  // this warp is done with the slot
      ++n;
    }
    if (ok && gt > 0 && !drain_dq(gt - 1, pend_direct)) ok = false;
    if (!ok) fail();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

namespace {

template <bool F16>
cudaError_t tc_bwd_t(const Call& c, const void* q, const void* k, const void* v,
                     const float* lse, const void* dout, const float* D, float* dq_acc,
                     float* dk_acc, float* dv_acc, void* dq, void* dk, void* dv,
                     int* sched_counter, const float* slots, int nslots) {
  const st_layout* L = c.L;
  const int BH = c.B * c.H;
  if (L->dev.n_bwd_items == 0) return cudaSuccess;
  BwdMaps maps;
  const int el = F16 ? ELEM_F16 : ELEM_BF16;
  if (!make_view_maps(maps.q, q, el, L->geom, BH, c.d) ||
      !make_view_maps(maps.k, k, el, L->geom, BH, c.d) ||
      !make_view_maps(maps.v, v, el, L->geom, BH, c.d) ||
      !make_view_maps(maps.dout, dout, el, L->geom, BH, c.d) ||
      !make_view_maps(maps.dq, dq_acc, ELEM_F32, L->geom, BH, c.d) ||
      !make_view_maps(maps.dk, dk_acc, ELEM_F32, L->geom, BH, c.d) ||
      !make_view_maps(maps.dv, dv_acc, ELEM_F32, L->geom, BH, c.d) ||
      !make_view_maps(maps.dqo, dq, el, L->geom, BH, c.d) ||
      !make_view_maps(maps.dko, dk, el, L->geom, BH, c.d) ||
      !make_view_maps(maps.dvo, dv, el, L->geom, BH, c.d))
    return cudaErrorInvalidValue;
  if (L->summary_rows) {
    if (!make_summary_rows_map(&maps.dks, dk_acc, L->geom, BH, c.d) ||
        !make_summary_rows_map(&maps.dvs, dv_acc, L->geom, BH, c.d))
      return cudaErrorInvalidValue;
  } else {
    maps.dks = maps.dk[VIEW_NAT];  // never used
    maps.dvs = maps.dv[VIEW_NAT];
  }
  const size_t smem = sizeof(SmemBwd);
  static_assert(sizeof(SmemBwd) <= 227 * 1024, "shared memory plan exceeds a CTA's 227 KB");
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  cudaError_t err = cudaSuccess;
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    err = cudaFuncSetAttribute(bwd_tc_kernel<F16, false>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err == cudaSuccess)
      err = cudaFuncSetAttribute(bwd_tc_kernel<F16, true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  const int sms = sm_count();
  const int NH = heads_per_class(c);
  // Cut accumulating items finer while the longest unit would exceed a CTA's
  // share of all tile pairs (few units per CTA: the tail would be one long
  // unit). Finer cuts cost fp32 reduce-adds, so they are taken only then
  // (measured: cutting at half a share made the fixed split T=4096 backward
  // 7% slower).
  const double share = (double)L->dev.q_ents_total * NH / sms;
  int f = 0;
  while (f < 2 && L->dev.max_split_len[f] > share) ++f;
  const long long units = (long long)L->dev.n_bwd_split[f] * NH;
  if (units > 0x7fffffff) return cudaErrorInvalidValue;
  // fp32 accumulator rows all heads reduce into: head-major order when they
  // exceed about the L2 (126 MB), so that one head's rows stay resident
  double acc_bytes = 0.0;
  for (int hc = 0; hc < (int)L->hcs.size(); ++hc)
    acc_bytes += (double)(L->dev.n_rows[hc][ROWS_Q_ACC] + 2.0 * L->dev.n_rows[hc][ROWS_K_ACC]) *
                 c.d * 4.0 * NH;
  UnitOrder uo;
  uo.head_major = acc_bytes > 128.0 * (1 << 20) ? 1 : 0;
  uo.n_items = L->dev.n_bwd_split[f];
  uo.fitems = make_fastdiv(uo.n_items);
  const int grid = (int)std::min<long long>(units, sms);
  ZeroRows zr;
  for (int hc = 0; hc < 2; ++hc) {
    zr.q[hc] = (const int32_t*)L->dev.rows[hc][ROWS_Q_ZERO];
    zr.k[hc] = (const int32_t*)L->dev.rows[hc][ROWS_K_ZERO];
    zr.nq[hc] = L->dev.n_rows[hc][ROWS_Q_ZERO];
    zr.nk[hc] = L->dev.n_rows[hc][ROWS_K_ZERO];
  }
  record_begin(c);
  auto kernel = L->geom.cpt > 1 ? bwd_tc_kernel<F16, true> : bwd_tc_kernel<F16, false>;
  kernel<<<grid, kThreads, smem, c.stream>>>(
      maps, L->geom, (const BwdItem*)L->dev.bwd_split[f], (int)units, NH, uo,
      (const QEnt*)L->dev.q_ents, heads_of(c), c.scale, c.scale * kLog2e, lse, D,
      zr, (uint4*)dq, (uint4*)dk, (uint4*)dv, sched_counter, slots, F16 ? 0 : nslots,
      c.status, c.wait_ns);
  err = cudaGetLastError();
  record_end(c);
  return err;
}

}  // namespace

cudaError_t tc_bwd(const Call& c, const void* q, const void* k, const void* v, const float* lse,
                   const void* dout, const float* D, float* dq_acc, float* dk_acc,
                   float* dv_acc, void* dq, void* dk, void* dv, int* sched_counter,
                   const float* slots, int nslots) {
  return c.dtype == ST_F16 ? tc_bwd_t<true>(c, q, k, v, lse, dout, D, dq_acc, dk_acc, dv_acc,
                                            dq, dk, dv, sched_counter, slots, nslots)
                           : tc_bwd_t<false>(c, q, k, v, lse, dout, D, dq_acc, dk_acc, dv_acc,
                                             dq, dk, dv, sched_counter, slots, nslots);
}

}  // namespace st
